"""Pins for the CPU oracle: each check ties the oracle to something other than
itself (closed forms, brute force, invariants the pages fix, library routines
for special cases), chosen so that a dropped term, a wrong sign or index, or a
transposed operand fails at least one of them.  CPU only."""
import json
import math
import os

import numpy as np
import pytest

import oracle
from mixture_experts_layer_shifted_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- generator
def test_philox_known_answers():
    # Known-answer vectors of Philox4x32-10 (Random123 distribution, kat_vectors).
    cases = [
        ((0, 0, 0, 0), (0, 0), (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
        ((0xffffffff,) * 4, (0xffffffff, 0xffffffff), (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
        ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
         (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
    ]
    for c, k, want in cases:
        got = synth.philox4x32_10(*c, *k)
        assert tuple(int(v) for v in got) == want


def test_generator_recipes():
    v = synth.normal_f32(np.arange(200000, dtype=np.uint64), synth.TID_X, 0, 1.0)
    assert abs(v.mean()) < 0.01 and abs(v.var() - 1.0) < 0.01
    assert v.min() >= -6.0 and v.max() <= 6.0
    # the Irwin-Hall value is exact: z * 65536 is an integer
    assert np.all((v * 65536.0) == np.round(v * 65536.0))
    u = synth.uniform_f32(np.arange(100000, dtype=np.uint64), synth.TID_BIAS, 0, -0.2, 0.2)
    assert u.min() > -0.2 and u.max() < 0.2 and abs(u.mean()) < 0.005
    # bf16 rounding: nearest-even on hand-made bit patterns
    f = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5], dtype=np.float32)
    got = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(f))
    assert got.tolist() == [1.0, 1.0, 1.0 + 4 * 2 ** -8, 1.0, -2.5]
    o = synth.zipf_logit_offsets(16)
    assert sorted(np.round(np.exp(-o / 1.1)).astype(int).tolist()) == list(range(1, 17))


# ---------------------------------------------------------------- exp
def test_zexp_accuracy_and_special_values():
    assert oracle.zexp(0.0) == 1.0
    assert oracle.zexp(-200.0) == 0.0
    xs = np.concatenate([np.linspace(-86.0, 0.0, 20011), -np.logspace(-8, 1.9, 4001)]).astype(np.float32)
    worst = 0.0
    for x in xs:
        z = oracle.zexp(float(x))
        ref = math.exp(float(x))
        worst = max(worst, abs(z - ref) / float(np.spacing(np.float32(ref))))
    assert worst <= 2.0, worst
    # at fp32 inputs next to n ln 2 the result is 2**n times exp of the input's rounding error
    for n in range(-100, 1):
        x = np.float32(n * math.log(2))
        want = 2.0 ** n * math.exp(float(x) - n * math.log(2))
        assert oracle.zexp(x) == pytest.approx(want, rel=2.5e-7)


# ---------------------------------------------------------------- router
def test_router_logits_against_library_matmul():
    x = synth.normal((7, 33), synth.TID_X, 3, 1.0, "bf16")
    wr = synth.normal((5, 33), synth.TID_WR, 3, 0.5, "bf16")
    off = np.array([0.0, 1.0, -2.0, 0.5, 0.25], np.float32)
    got = oracle.router_logits(x, wr, off)
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ synth.bf16_bits_to_f32(wr).astype(np.float64).T + off
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # operand order matters: a transposed weight would change the shape or values
    assert got.shape == (7, 5)


def test_softmax_closed_forms():
    l = np.array([[0.3, -1.2], [5.0, 5.0], [1000.0, 999.0]])
    s = oracle.softmax(l)
    assert s[0, 0] == pytest.approx(1.0 / (1.0 + math.exp(-1.5)), rel=1e-15)
    assert s[1, 0] == s[1, 1] == 0.5
    assert s[2, 0] == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    r = _rng(1).normal(size=(9, 24))
    s = oracle.softmax(r)
    np.testing.assert_allclose(s.sum(1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(oracle.softmax(r + 7.0), s, rtol=1e-13)  # shift invariance
    np.testing.assert_allclose(s[:, 3] / s[:, 5], np.exp(r[:, 3] - r[:, 5]), rtol=1e-12)


# ---------------------------------------------------------------- top-k
def test_topk_brute_force_tiny_config():
    # tiny layer shape: E = 16 FFN + 8 zero experts, k = 4, bias ~ U(-0.1, 0.1)
    T, E, k = 12, 24, 4
    s = oracle.softmax(_rng(2).normal(size=(T, E)))
    b = _rng(3).uniform(-0.1, 0.1, size=E)
    idx, gate, margin = oracle.topk(s, b, k, scale=1.0)
    for t in range(T):
        v = s[t] + b
        assert list(idx[t]) == oracle.brute_force_topk(v, k)
        np.testing.assert_array_equal(gate[t], s[t, idx[t]])
        assert margin[t] > 0


def test_topk_ties_and_order():
    s = np.array([[0.1, 0.3, 0.3, 0.2, 0.1]])
    idx, gate, margin = oracle.topk(s, None, 3)
    assert idx[0].tolist() == [1, 2, 3]
    assert margin[0] == pytest.approx(0.1)
    idx, _, margin = oracle.topk(s, None, 4)
    assert idx[0].tolist() == [1, 2, 3, 0]  # tie between experts 0 and 4 goes to 0
    assert margin[0] == 0.0
    # bias reorders selection, gate stays the unbiased score times the scale
    b = np.array([0.0, 0.0, 0.0, 0.0, 0.5])
    idx, gate, _ = oracle.topk(s, b, 2, scale=2.5)
    assert idx[0].tolist() == [4, 1]
    assert gate[0].tolist() == [2.5 * 0.1, 2.5 * 0.3]


def test_topk_nan_scores_rank_below_every_number():
    """A biased score that is not a number ranks as -inf: the numbers are chosen
    first, in the usual order, then the NaN experts by ascending id; every pick is
    a distinct valid id.  Reduces to the finite case with those scores at -1e300."""
    T, E, k = 6, 24, 6
    s = oracle.softmax(_rng(21).normal(size=(T, E)))
    b = _rng(22).uniform(-0.1, 0.1, size=E)
    b[[3, 7, 8]] = np.nan
    idx, gate, _ = oracle.topk(s, b, k)
    b_fin = b.copy()
    b_fin[[3, 7, 8]] = -1e300
    ref, _, _ = oracle.topk(s, b_fin, k)
    np.testing.assert_array_equal(idx, ref)
    # more NaN experts than finite ones left: the remaining picks are the lowest NaN ids
    b2 = np.full(E, np.nan)
    b2[[10, 20]] = 0.0
    idx2, gate2, _ = oracle.topk(s, b2, 5)
    for t in range(T):
        first = sorted([10, 20], key=lambda e: (-s[t, e], e))
        assert idx2[t].tolist() == first + [0, 1, 2]
        np.testing.assert_array_equal(gate2[t], s[t, idx2[t]])


def test_replica_nan_and_inf_logits_pick_valid_distinct_experts():
    """fp32 replica on rows that are not all finite: a NaN logit is skipped by the
    max and gets weight zexp(NaN) = 0, so the row equals the same row with that
    logit at -inf; a +inf logit makes every score NaN and the picks are experts
    0..k-1 in order; an all -inf row likewise; a NaN bias ranks its expert last."""
    E, k = 24, 4
    l = _rng(23).normal(size=(6, E)).astype(np.float32)
    l[1, 5] = np.nan
    l[5, 0] = np.nan
    l[2, 9] = np.inf
    l[3, :] = -np.inf
    l[4, :] = np.nan
    bias = _rng(24).uniform(-0.1, 0.1, size=E).astype(np.float32)
    idx, gate, sc = oracle.route_replica_f32(l, bias, k, 1.0, want_scores=True)
    ref_row = l[1].copy()
    ref_row[5] = -np.inf
    i1, g1, s1 = oracle.route_replica_f32(ref_row[None], bias, k, 1.0, want_scores=True)
    np.testing.assert_array_equal(idx[1], i1[0])
    np.testing.assert_array_equal(sc[1].view(np.uint32), s1[0].view(np.uint32))
    assert sc[1, 5] == 0.0 and np.isfinite(sc[1]).all()
    ref_row = l[5].copy()
    ref_row[0] = -np.inf
    i5, _, s5 = oracle.route_replica_f32(ref_row[None], bias, k, 1.0, want_scores=True)
    np.testing.assert_array_equal(idx[5], i5[0])
    np.testing.assert_array_equal(sc[5].view(np.uint32), s5[0].view(np.uint32))
    for t in (2, 3, 4):
        assert np.isnan(sc[t]).all()
        assert idx[t].tolist() == [0, 1, 2, 3]
        assert np.isnan(gate[t]).all()
    b_nan = bias.copy()
    b_nan[[0, 1]] = np.nan
    i_nan, _, _ = oracle.route_replica_f32(l[:1], b_nan, k, 1.0)
    assert 0 not in i_nan[0] and 1 not in i_nan[0]
    for t in range(6):
        assert len(set(idx[t].tolist())) == k and idx[t].min() >= 0 and idx[t].max() < E


def test_topk_unbiased_equals_topk_of_logits():
    l = _rng(4).normal(size=(20, 24))
    idx, _, _ = oracle.topk(oracle.softmax(l), None, 6)
    ref = np.argsort(-l, axis=1, kind="stable")[:, :6]
    np.testing.assert_array_equal(idx, ref)


def test_bias_changes_selection_never_gates():
    T, E, k = 64, 24, 4
    s = oracle.softmax(_rng(5).normal(size=(T, E)))
    b = _rng(6).uniform(-0.1, 0.1, size=E)
    i0, g0, _ = oracle.topk(s, None, k, 1.5)
    i1, g1, _ = oracle.topk(s, b, k, 1.5)
    assert (i0 != i1).any()  # the bias does change selection here
    for t in range(T):
        for j in range(k):
            assert g1[t, j] == 1.5 * s[t, i1[t, j]]
        common = set(i0[t]) & set(i1[t])
        for e in common:
            assert g0[t, list(i0[t]).index(e)] == g1[t, list(i1[t]).index(e)]


def test_raising_zero_bias_never_lowers_zero_picks():
    T, N, Z, k = 128, 16, 8, 4
    s = oracle.softmax(_rng(7).normal(size=(T, N + Z)))
    prev = -1
    for beta in [0.0, 0.01, 0.03, 0.1, 0.3, 1.0]:
        b = np.concatenate([np.zeros(N), np.full(Z, beta)])
        idx, _, _ = oracle.topk(s, b, k)
        zero_picks = int((idx >= N).sum())
        assert zero_picks >= prev
        prev = zero_picks
        ffn_per_token = (idx < N).sum(1)
        assert ffn_per_token.min() >= 0 and ffn_per_token.max() <= k
    assert prev == T * min(k, Z)


def test_replica_matches_fp64_routing_away_from_ties():
    T, E, k = 256, 96, 8
    l = _rng(8).normal(size=(T, E)).astype(np.float32) * 3
    b = _rng(9).uniform(-0.2, 0.2, size=E).astype(np.float32)
    i32, g32, s32 = oracle.route_replica_f32(l, b, k, 1.0, want_scores=True)
    s64 = oracle.softmax(l.astype(np.float64))
    np.testing.assert_allclose(s32, s64, rtol=4e-6, atol=1e-30)
    i64, g64, margin = oracle.topk(s64, b.astype(np.float64), k)
    ok = margin > 1e-5
    assert ok.mean() > 0.9
    np.testing.assert_array_equal(i32[ok], i64[ok])
    np.testing.assert_allclose(g32, s32[np.arange(T)[:, None], i32], rtol=0)
    # the 32-way summation rule gives a sum of exactly 1 +- a few ulp
    np.testing.assert_allclose(s32.astype(np.float64).sum(1), 1.0, atol=5e-6)



def test_replica_ties_go_to_the_lower_index():
    """Equal logits give bit-equal fp32 scores, so the replica's tie rule decides:
    the lower expert index first, as in the fp64 rule."""
    l = np.array([[1.0, 2.0, 2.0, 0.0, 2.0, 1.0]], np.float32)
    idx, gate, s = oracle.route_replica_f32(l, None, 4, 1.0, want_scores=True)
    assert s[0, 1] == s[0, 2] == s[0, 4] and s[0, 0] == s[0, 5]
    assert idx[0].tolist() == [1, 2, 4, 0]
    b = np.array([0.0, 0.0, 0.0, 0.0, 0.0, 0.0], np.float32)
    assert oracle.route_replica_f32(l, b, 4, 1.0)[0][0].tolist() == [1, 2, 4, 0]
    ref = oracle.brute_force_topk(s[0].astype(np.float64), 4)
    assert sorted(ref) == sorted(idx[0].tolist())


def test_replica_is_shift_invariant_bit_for_bit():
    """The rule subtracts the largest logit before the exponential.  On logits on a
    2^-10 grid, adding 128 (or 1024) is exact in fp32 and so is the subtraction, so
    the scores, indices and gates must come out bit-identical, and finite."""
    rng = _rng(31)
    l = (np.round(rng.uniform(-8, 8, size=(64, 96)) * 1024) / 1024).astype(np.float32)
    b = rng.uniform(-0.01, 0.01, size=96).astype(np.float32)
    i0, g0, s0 = oracle.route_replica_f32(l, b, 8, 1.0, want_scores=True)
    for c in (128.0, 1024.0):
        lc = (l + np.float32(c)).astype(np.float32)
        assert np.array_equal(lc - np.float32(c), l)   # the shift is exact
        i1, g1, s1 = oracle.route_replica_f32(lc, b, 8, 1.0, want_scores=True)
        assert np.isfinite(s1).all()
        np.testing.assert_array_equal(s1.view(np.uint32), s0.view(np.uint32))
        np.testing.assert_array_equal(i1, i0)
        np.testing.assert_array_equal(g1.view(np.uint32), g0.view(np.uint32))


# ---------------------------------------------------------------- integer stage
def test_integer_stage_against_stable_sort():
    T, N, Z, k = 300, 16, 8, 4
    s = oracle.softmax(_rng(10).normal(size=(T, N + Z)))
    idx, _, _ = oracle.topk(s, None, k)
    counts, offsets, perm, pos = oracle.integer_stage(idx, N, N + Z)
    assert counts.sum() == T * k
    np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=N + Z))
    assert offsets[0] == 0 and np.all(np.diff(offsets) >= 0) and offsets[N] == (idx < N).sum()
    flat = idx.ravel()
    pairs = np.nonzero(flat < N)[0]
    key = flat[pairs].astype(np.int64) * (T * k) + pairs
    ref = pairs[np.argsort(key, kind="stable")]
    np.testing.assert_array_equal(perm, ref)
    assert len(set(perm.tolist())) == len(perm)  # bijection onto the FFN pairs
    pf = pos.ravel()
    assert np.all(pf[flat >= N] == -1)
    np.testing.assert_array_equal(perm[pf[flat < N]], np.nonzero(flat < N)[0])


# ---------------------------------------------------------------- expert math
def _silu(z):
    return z / (1.0 + math.exp(-z))


def test_ffn_scalar_closed_form():
    for xg, wg, wu, wd in [(1.5, 0.7, -2.0, 0.3), (-0.4, 2.0, 1.0, -1.5)]:
        x = np.array([[xg]], np.float32)
        got = oracle.ffn(x, np.array([[wg]], np.float32), np.array([[wu]], np.float32), np.array([[wd]], np.float32))
        a, b, c, xv = (float(np.float32(v)) for v in (wg, wu, wd, xg))
        assert got[0, 0] == pytest.approx(c * _silu(a * xv) * (b * xv), rel=1e-15)


def test_ffn_against_library_matmul():
    d, inter, n = 40, 24, 5
    x = synth.normal((n, d), 11, 0, 1.0)
    wg = synth.normal((inter, d), 12, 0, 0.2)
    wu = synth.normal((inter, d), 13, 0, 0.2)
    wd = synth.normal((d, inter), 14, 0, 0.2)
    got = oracle.ffn(x, wg, wu, wd)
    x64 = x.astype(np.float64)
    g = x64 @ wg.astype(np.float64).T
    u = x64 @ wu.astype(np.float64).T
    ref = (g / (1.0 + np.exp(-g)) * u) @ wd.astype(np.float64).T
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)
    # gate and up are not interchangeable: swapping them changes the result
    assert not np.allclose(oracle.ffn(x, wu, wg, wd), got)


def _tiny_layer(seed=0, T=16, d=32, N=6, Z=3, inter=8, k=3):
    x = synth.normal((T, d), synth.TID_X, seed, 1.0)
    wg = synth.normal((N, inter, d), synth.TID_WG, seed, 0.2)
    wu = synth.normal((N, inter, d), synth.TID_WU, seed, 0.2)
    wd = synth.normal((N, d, inter), synth.TID_WD, seed, 0.2)
    return x, wg, wu, wd


def test_layer_dense_masked_formulation():
    T, d, N, Z, inter, k = 16, 32, 6, 3, 8, 3
    x, wg, wu, wd = _tiny_layer(T=T, d=d, N=N, Z=Z, inter=inter, k=k)
    s = oracle.softmax(_rng(12).normal(size=(T, N + Z)))
    idx, gate, _ = oracle.topk(s, None, k, 0.75)
    y = oracle.layer(x, idx, gate, N, wg, wu, wd)
    # dense: every FFN expert on every token, then a gate mask
    F = np.stack([oracle.ffn(x, wg[e], wu[e], wd[e]) for e in range(N)], 1)  # [T, N, d]
    G = np.zeros((T, N + Z))
    np.put_along_axis(G, idx.astype(np.int64), gate, 1)
    ref = np.einsum("te,ted->td", G[:, :N], F) + G[:, N:].sum(1, keepdims=True) * x.astype(np.float64)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)
    # the per-expert fetch path gives the same numbers
    y2 = oracle.layer_outputs(x, idx, gate, N, lambda e: (wg[e], wu[e], wd[e]))
    np.testing.assert_allclose(y2, y, rtol=1e-12, atol=1e-14)



def test_layer_outputs_bf16_rows_and_quantized_expert_flags():
    """The per-expert fetch path on bf16 bit patterns equals the same path on the
    fp32 values they encode; with fp8 / fp4 it runs the FP8 expert on weights
    quantized per [128,128], or the MXFP4 expert on weights quantized per [1,32]."""
    T, d, N, Z, inter, k = 12, 128, 4, 2, 128, 3
    x, wg, wu, wd = _tiny_layer(T=T, d=d, N=N, Z=Z, inter=inter, k=k)
    s = oracle.softmax(_rng(17).normal(size=(T, N + Z)))
    idx, gate, _ = oracle.topk(s, None, k, 1.25)
    bits = synth.f32_to_bf16_bits(x)
    xb = synth.bf16_bits_to_f32(bits)
    fetch = lambda e: (wg[e], wu[e], wd[e])  # noqa: E731
    np.testing.assert_array_equal(oracle.layer_outputs(bits, idx, gate, N, fetch),
                                  oracle.layer_outputs(xb, idx, gate, N, fetch))
    np.testing.assert_allclose(oracle.layer_outputs(xb, idx, gate, N, fetch), oracle.layer(xb, idx, gate, N, wg, wu, wd),
                               rtol=1e-12, atol=1e-14)   # the same sum, added in another order

    def fp8_expert(e, rows):
        q = [oracle.quantize_blocks(w, 128) for w in fetch(e)]
        return oracle.ffn_fp8(rows, [c for c, _ in q], [s_ for _, s_ in q])

    def fp4_expert(e, rows):
        q = [oracle.quantize_mx4(w) for w in fetch(e)]
        return oracle.ffn_fp4(rows, [c for c, _ in q], [s_ for _, s_ in q])

    y8 = oracle.layer_outputs(bits, idx, gate, N, fetch, fp8=True)
    np.testing.assert_array_equal(y8, oracle.layer_outputs(bits, idx, gate, N, None, expert_fn=fp8_expert))
    y4 = oracle.layer_outputs(bits, idx, gate, N, fetch, fp4=True)
    np.testing.assert_array_equal(y4, oracle.layer_outputs(bits, idx, gate, N, None, expert_fn=fp4_expert))
    y = oracle.layer_outputs(bits, idx, gate, N, fetch)
    assert not np.array_equal(y8, y) and not np.array_equal(y4, y) and not np.array_equal(y8, y4)


def test_layer_identical_experts_closed_form():
    T, d, N, Z, inter, k = 10, 16, 4, 4, 8, 4
    x, wg, wu, wd = _tiny_layer(T=T, d=d, N=N, Z=Z, inter=inter, k=k)
    wg[:] = wg[0]
    wu[:] = wu[0]
    wd[:] = wd[0]
    s = oracle.softmax(_rng(13).normal(size=(T, N + Z)))
    idx, gate, _ = oracle.topk(s, None, k)
    y = oracle.layer(x, idx, gate, N, wg, wu, wd)
    F = oracle.ffn(x, wg[0], wu[0], wd[0])
    gf = np.where(idx < N, gate, 0).sum(1, keepdims=True)
    gz = np.where(idx >= N, gate, 0).sum(1, keepdims=True)
    np.testing.assert_allclose(y, gf * F + gz * x.astype(np.float64), rtol=1e-12, atol=1e-14)


def test_zero_only_tokens_return_weighted_input_exactly():
    T, d, N, Z, k = 8, 16, 4, 4, 3
    x, wg, wu, wd = _tiny_layer(T=T, d=d, N=N, Z=Z, inter=8, k=k)
    s = oracle.softmax(_rng(14).normal(size=(T, N + Z)))
    b = np.concatenate([np.zeros(N), np.full(Z, 0.5)])  # +0.5 on zero experts: every pick is a zero expert
    idx, gate, _ = oracle.topk(s, b, k)
    assert np.all(idx >= N)
    y = oracle.layer(x, idx, gate, N, wg, wu, wd)
    zsum = np.zeros(T)
    for j in range(k):
        zsum += gate[:, j]
    np.testing.assert_array_equal(y, zsum[:, None] * x.astype(np.float64))


def test_all_experts_chosen_when_k_equals_E():
    T, d, N, Z, inter = 6, 16, 3, 2, 8
    x, wg, wu, wd = _tiny_layer(T=T, d=d, N=N, Z=Z, inter=inter, k=N + Z)
    s = oracle.softmax(_rng(15).normal(size=(T, N + Z)))
    idx, gate, margin = oracle.topk(s, None, N + Z)
    assert np.all(np.sort(idx, 1) == np.arange(N + Z))
    assert np.all(np.isinf(margin))
    y = oracle.layer(x, idx, gate, N, wg, wu, wd)
    ref = sum(s[:, e:e + 1] * oracle.ffn(x, wg[e], wu[e], wd[e]) for e in range(N)) + \
        s[:, N:].sum(1, keepdims=True) * x.astype(np.float64)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- controller
def test_update_bias_hand_worked_step():
    N, Z, k = 2, 1, 2
    counts = np.array([3, 1, 4], np.int64)  # 4 tokens x k=2 = 8 picks
    tokens = np.array([4], np.int64)
    b0 = np.array([0.0, 0.1, -0.1], np.float32)
    st = oracle.new_controller_state(b0)
    kp, ki, kd, decay, K = 0.5, 0.25, 2.0, 0.5, 1.5
    oracle.update_bias(counts, tokens, N, Z, k, (kp, ki, kd, decay, K), b0, st)
    eta = 0.5
    tau = [K / N, K / N, (k - K) / Z]
    load = [3 / 4, 1 / 4, 4 / 4]
    for i in range(3):
        e = tau[i] - load[i]
        integ = eta * e
        want = kp * eta * e + ki * integ + kd * eta * (e - 0.0) + float(b0[i])
        assert st["bias"][i] == pytest.approx(want, abs=2e-7)
        assert st["integ"][i] == pytest.approx(integ, abs=1e-7)
        assert st["eprev"][i] == pytest.approx(e, abs=1e-7)
    assert st["eta"][0] == 0.5
    assert counts.tolist() == [0, 0, 0] and tokens[0] == 0
    # errors sum to zero: sum(load) == sum(tau) == k
    assert abs(float(st["eprev"].astype(np.float64).sum())) < 1e-6
    # an underloaded expert gains bias, an overloaded one loses it
    assert st["bias"][1] > b0[1] and st["bias"][2] < b0[2]



def test_update_bias_second_step_uses_the_previous_error():
    """Two hand-worked steps, so the derivative term sees a non-zero previous error
    and the integral term carries the first step's value."""
    N, Z, k = 2, 1, 2
    b0 = np.array([0.0, 0.1, -0.1], np.float32)
    st = oracle.new_controller_state(b0)
    kp, ki, kd, decay, K = 0.5, 0.25, 2.0, 0.5, 1.5
    tau = [K / N, K / N, (k - K) / Z]
    steps = [[3, 1, 4], [1, 4, 3]]       # 4 tokens x k = 2 picks each step
    eta, integ, eprev = 1.0, [0.0] * 3, [0.0] * 3
    for c in steps:
        counts = np.array(c, np.int64)
        tokens = np.array([4], np.int64)
        oracle.update_bias(counts, tokens, N, Z, k, (kp, ki, kd, decay, K), b0, st)
        eta *= decay
        for i in range(3):
            e = tau[i] - c[i] / 4
            integ[i] += eta * e
            want = kp * eta * e + ki * integ[i] + kd * eta * (e - eprev[i]) + float(b0[i])
            assert st["bias"][i] == pytest.approx(want, abs=2e-7), (c, i)
            eprev[i] = e
    # the second step's derivative term is kd * eta * (e2 - e1), not its sum
    assert eprev[0] != 0.0 and abs(kd * 0.25 * (eprev[0] - 0.0)) > 1e-3


def test_update_bias_fixed_point_and_incremental_form():
    N, Z, k = 4, 4, 4
    b0 = np.full(N + Z, 0.01, np.float32)
    st = oracle.new_controller_state(b0)
    # loads exactly on target (K = 2): FFN 2/4 = 0.5 per expert, zero 2/4 = 0.5
    for _ in range(3):
        counts = np.full(N + Z, 8, np.int64)
        tokens = np.array([16], np.int64)
        oracle.update_bias(counts, tokens, N, Z, k, (0.0, 0.1, 0.0, 1.0, 2.0), b0, st)
    np.testing.assert_array_equal(st["bias"], b0)
    # kp = kd = 0: the positional form equals incremental b += ki * eta * e
    st = oracle.new_controller_state(b0)
    ref = b0.astype(np.float64).copy()
    eta = 1.0
    rng = _rng(16)
    for _ in range(5):
        c = rng.multinomial(64, [1 / 8] * 8).astype(np.int64)
        tokens = np.array([16], np.int64)
        load = c / 16.0
        eta *= 0.9
        tau = np.array([2 / 4] * 4 + [2 / 4] * 4)
        ref += 0.1 * eta * (tau - load)
        oracle.update_bias(c, tokens, N, Z, k, (0.0, 0.1, 0.0, 0.9, 2.0), b0, st)
    np.testing.assert_allclose(st["bias"], ref, atol=2e-6)
    assert st["eta"][0] == pytest.approx(0.9 ** 5, rel=1e-6)
    # nothing accumulated: no change at all
    before = st["bias"].copy()
    oracle.update_bias(np.zeros(8, np.int64), np.zeros(1, np.int64), N, Z, k, (1, 1, 1, 1, 2.0), b0, st)
    np.testing.assert_array_equal(st["bias"], before)


def test_controller_moves_ffn_share_towards_target():
    # closed loop on the oracle alone: router + top-k + counts + controller
    T, N, Z, k = 512, 16, 8, 4
    rng = _rng(17)
    l = rng.normal(size=(T, N + Z)) * 0.5
    s = oracle.softmax(l)
    b0 = np.zeros(N + Z, np.float32)
    st = oracle.new_controller_state(b0)
    K = 3.0
    first = None
    for step in range(30):
        idx, _, _ = oracle.topk(s, st["bias"].astype(np.float64), k)
        ffn = float((idx < N).sum()) / T
        first = ffn if first is None else first
        c = np.bincount(idx.ravel(), minlength=N + Z).astype(np.int64)
        oracle.update_bias(c, np.array([T], np.int64), N, Z, k, (0.0, 0.05, 0.0, 1.0, K), b0, st)
    assert abs(ffn - K) < abs(first - K)


# ---------------------------------------------------------------- the pages' layer shape
def test_page_layer_shape_is_consistent():
    cfg = json.load(open(os.path.join(GOLDEN, "longcat_flash_layer.json")))
    per_layer = cfg["n_ffn"] * 3 * cfg["hidden"] * cfg["expert_inter"]
    total = per_layer * cfg["layers"]
    # the FFN experts alone are ~97% of the stated 560B parameters
    assert 0.9 * cfg["total_params_billion"] * 1e9 < total < cfg["total_params_billion"] * 1e9
    # uniform routing over 512 + 256 experts picks k * N / E = 8 FFN experts per token,
    # inside the range the thread reports for realised experts per token
    expect = cfg["top_k"] * cfg["n_ffn"] / (cfg["n_ffn"] + cfg["n_zero"])
    lo, hi = min(cfg["realised_ffn_per_token"].values()), max(cfg["realised_ffn_per_token"].values())
    assert lo <= expect <= hi


# ---------------------------------------------------------------- block-scaled FP8 (oracle only)

def test_e4m3_decode_all_codes_against_torch():
    import torch
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy().astype(np.float64)
    got = np.array([oracle.e4m3_decode(c) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x38] == 1.0 and np.isnan(got[0x7F])


def test_e4m3_encode_against_torch():
    """Round to nearest even on exact values, midpoints (ties) and random values in [-448, 448]."""
    import torch
    exact = np.array([oracle.e4m3_decode(c) for c in range(256)])
    exact = np.unique(exact[~np.isnan(exact)])
    mids = (exact[1:] + exact[:-1]) / 2.0
    rng = np.random.default_rng(11)
    rnd = rng.uniform(-1, 1, 20000) * np.exp2(rng.integers(-12, 9, 20000))
    vals = np.concatenate([exact, mids, rnd, [-0.0, 448.0, -448.0, 2.0 ** -10, 3 * 2.0 ** -10]]).astype(np.float32)
    vals = vals[np.abs(vals) <= 448.0]
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(v) for v in vals], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(vals[i]), int(got[i]), int(ref[i])) for i in bad[:5]]
    # saturation beyond the largest finite value
    assert oracle.e4m3_encode(1e6) == 0x7E and oracle.e4m3_encode(-500.0) == 0xFE


def test_e8m0_scale_is_the_smallest_sufficient_power_of_two():
    rng = np.random.default_rng(12)
    amax = (rng.uniform(0.5, 1.0, 5000) * np.exp2(rng.integers(-100, 100, 5000))).astype(np.float32)
    for a in amax:
        c = oracle.e8m0_scale(float(a))
        assert 0 < c < 254
        s = 2.0 ** (c - 127)
        assert a / s <= 448.0 < a / (s / 2), (a, c)
    assert oracle.e8m0_scale(0.0) == 127
    assert oracle.e8m0_scale(448.0) == 127 and oracle.e8m0_scale(np.nextafter(np.float32(448), np.float32(1e9))) == 128
    assert oracle.e8m0_scale(1.75 * 2.0 ** 20) == 127 + 12 and oracle.e8m0_scale(2.0 ** 21) == 127 + 13
    assert oracle.e8m0_scale(2.0 ** -140) == 0      # clamped: the block quantizes to zeros and small codes
    assert oracle.e8m0_scale(3e38) == 127 + 120


@pytest.mark.parametrize("block_rows,rows", [(1, 7), (128, 300)])
def test_quantize_blocks_error_bound_and_structure(block_rows, rows):
    rng = np.random.default_rng(13)
    cols = 384
    x = (rng.standard_normal((rows, cols)) * np.exp2(rng.integers(-6, 6, (rows, 1)))).astype(np.float32)
    codes, scales = oracle.quantize_blocks(x, block_rows)
    assert scales.shape == ((rows + block_rows - 1) // block_rows, cols // 128)
    deq = oracle.dequantize_blocks(codes, scales, block_rows)
    s = np.ldexp(1.0, np.repeat(np.repeat(scales.astype(np.int64) - 127, block_rows, 0)[:rows], 128, 1))
    v = x.astype(np.float64) / s                         # exact scaled values
    assert np.abs(v).max() <= 448.0
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -6)))
    spacing = np.exp2(e - 3)                             # 2^-9 below the smallest normal
    assert np.all(np.abs(v - deq / s) <= spacing / 2)
    # each block's scale is minimal: its largest scaled value exceeds 224
    for rb in range(scales.shape[0]):
        for cb in range(scales.shape[1]):
            blk = np.abs(v[rb * block_rows:(rb + 1) * block_rows, cb * 128:(cb + 1) * 128])
            assert blk.max() > 224.0


def test_ffn_fp8_lossless_closed_form():
    """One token, one active hidden unit, every value exactly representable after
    quantization: g = 64 (silu(64) rounds to 64 in fp32), u = 1, so y = 64 * W_d[:, 0]
    exactly.  Swapping gate and up would give silu(1) * 64 instead."""
    d = inter = 128
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 1.0
    wg = np.zeros((inter, d), np.float32)
    wu = np.zeros((inter, d), np.float32)
    wg[0, 0], wu[0, 0] = 64.0, 1.0
    wd = np.zeros((d, inter), np.float32)
    wd[:, 0] = ((np.arange(d) % 8) - 4) * 0.25
    q = [oracle.quantize_blocks(w, 128) for w in (wg, wu, wd)]
    for (c, s_), w in zip(q, (wg, wu, wd)):
        assert np.array_equal(oracle.dequantize_blocks(c, s_, 128), w)   # lossless
    y = oracle.ffn_fp8(x, [c for c, _ in q], [s_ for _, s_ in q])
    assert np.array_equal(y[0], 64.0 * wd[:, 0].astype(np.float64))
    y_swapped = oracle.ffn_fp8(x, [q[1][0], q[0][0], q[2][0]], [q[1][1], q[0][1], q[2][1]])
    assert not np.allclose(y_swapped, y)



def test_ffn_fp8_quantizes_h_per_block():
    """Two active hidden units with exact operands: h = silu(64) * 7 = 448 sets the
    [1,128] block's scale to 2^0, and h = silu(48) * 6.5 = 312 lies between the E4M3
    values 288 and 320, so it must reach the down projection as 320:
    y = 448 W_d[:, 0] + 320 W_d[:, 1] exactly (312 would mean H was not quantized)."""
    d = inter = 128
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 1.0
    wg = np.zeros((inter, d), np.float32)
    wu = np.zeros((inter, d), np.float32)
    wg[0, 0], wu[0, 0] = 64.0, 7.0
    wg[1, 0], wu[1, 0] = 48.0, 6.5
    wd = np.zeros((d, inter), np.float32)
    wd[:, 0] = ((np.arange(d) % 8) - 4) * 0.25
    wd[:, 1] = ((np.arange(d) % 5) - 2) * 0.5
    q = [oracle.quantize_blocks(w, 128) for w in (wg, wu, wd)]
    for (c, s_), w in zip(q, (wg, wu, wd)):
        assert np.array_equal(oracle.dequantize_blocks(c, s_, 128), w)   # lossless
    y = oracle.ffn_fp8(x, [c for c, _ in q], [s_ for _, s_ in q])
    want = 448.0 * wd[:, 0].astype(np.float64) + 320.0 * wd[:, 1].astype(np.float64)
    assert np.array_equal(y[0], want)
    assert not np.array_equal(y[0], 448.0 * wd[:, 0].astype(np.float64) + 312.0 * wd[:, 1].astype(np.float64))



def _blocky(rng, rows, cols, block_rows, block_cols, std=1.0):
    """Normal values whose blocks have different magnitudes (factors 1/4 .. 8), so
    that neighbouring quantization blocks get different scales."""
    a = rng.normal(size=(rows, cols)) * std
    f = np.array([1.0, 8.0, 0.25, 2.0])
    for rb in range(0, rows, block_rows):
        for cb in range(0, cols, block_cols):
            a[rb:rb + block_rows, cb:cb + block_cols] *= f[(rb // block_rows + 2 * (cb // block_cols)) % 4]
    return a.astype(np.float32)


def test_ffn_fp8_equals_matmuls_on_the_quantized_operands():
    """The FP8 expert restated with library matmuls over the operands as the pinned
    quantizer leaves them: x per [1,128], the weights per [128,128], and H = silu(g) u
    rounded to fp32 then quantized per [1,128].  Each block has its own scale."""
    rng = _rng(41)
    n, d, inter = 6, 256, 384
    x = _blocky(rng, n, d, 1, 128)
    wg, wu = _blocky(rng, inter, d, 128, 128, 0.05), _blocky(rng, inter, d, 128, 128, 0.05)
    wd = _blocky(rng, d, inter, 128, 128, 0.05)
    q = [oracle.quantize_blocks(m, 128) for m in (wg, wu, wd)]
    Wg, Wu, Wd = (oracle.dequantize_blocks(c, s_, 128) for c, s_ in q)
    assert len(np.unique(q[0][1])) > 1                   # the blocks' scales differ
    y = oracle.ffn_fp8(x, [c for c, _ in q], [s_ for _, s_ in q])
    xq = oracle.dequantize_blocks(*oracle.quantize_blocks(x, 1), 1)
    g, u = xq @ Wg.T, xq @ Wu.T
    h32 = (g / (1.0 + np.exp(-g)) * u).astype(np.float32)
    want = oracle.dequantize_blocks(*oracle.quantize_blocks(h32, 1), 1) @ Wd.T
    np.testing.assert_allclose(y, want, rtol=1e-10, atol=1e-12 * np.abs(want).max())


def test_ffn_fp8_is_close_to_the_unquantized_expert():
    """The quantization error of the method on random data: a few percent of a row's
    largest output, far below the difference a wrong operand or scale would make."""
    rng = np.random.default_rng(14)
    d, inter = 256, 384
    x = rng.standard_normal((4, d)).astype(np.float32)
    wg, wu = (rng.standard_normal((inter, d)) * 0.06).astype(np.float32), (rng.standard_normal((inter, d)) * 0.06).astype(np.float32)
    wd = (rng.standard_normal((d, inter)) * 0.05).astype(np.float32)
    q = [oracle.quantize_blocks(w, 128) for w in (wg, wu, wd)]
    y8 = oracle.ffn_fp8(x, [c for c, _ in q], [s_ for _, s_ in q])
    y = oracle.ffn(x, wg, wu, wd)
    rel = np.abs(y8 - y).max(axis=1) / np.abs(y).max(axis=1)
    assert rel.max() < 0.08, rel
    assert rel.max() > 1e-4          # it is a lossy path


# ---------------------------------------------------------------- W4A4 (MXFP4, oracle only)

# E2M1 magnitudes of the OCP Microscaling Formats (MX) v1.0 specification (FP4 E2M1 element).
E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_is_the_mx_value_set():
    got = [oracle.e2m1_decode(c) for c in range(16)]
    assert got[:8] == E2M1_VALUES
    assert [-v for v in got[8:]] == E2M1_VALUES and np.signbit(got[8])
    assert all(oracle.e2m1_encode(got[c]) == c for c in range(16))   # round trip


def test_e2m1_encode_against_brute_force():
    """Nearest representable magnitude, ties to the even code (mantissa bit 0), saturating at 6."""
    mags = np.array(E2M1_VALUES)
    rng = np.random.default_rng(21)
    vals = np.concatenate([np.arange(-7.0, 7.0, 1 / 64), (mags[1:] + mags[:-1]) / 2, rng.uniform(-8, 8, 3000)])
    for v in vals.astype(np.float32):
        a = min(abs(float(v)), 6.0)
        dist = np.abs(mags - a)
        best = np.flatnonzero(dist == dist.min())
        code = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        want = code | (8 if np.signbit(v) else 0)
        assert oracle.e2m1_encode(v) == want, (float(v), oracle.e2m1_encode(v), want)


def test_mx4_scale_is_the_smallest_sufficient_power_of_two():
    rng = np.random.default_rng(22)
    amax = (rng.uniform(0.5, 1.0, 3000) * np.exp2(rng.integers(-100, 100, 3000))).astype(np.float32)
    for a in amax:
        c = oracle.mx4_scale(float(a))
        s = 2.0 ** (c - 127)
        assert a / s <= 6.0 < a / (s / 2), (a, c)
    assert oracle.mx4_scale(0.0) == 127 and oracle.mx4_scale(6.0) == 127 and oracle.mx4_scale(1.0) == 125
    assert oracle.mx4_scale(np.nextafter(np.float32(6), np.float32(10))) == 128


def test_quantize_mx4_bound_and_packing():
    rng = np.random.default_rng(23)
    x = (rng.standard_normal((5, 96)) * np.exp2(rng.integers(-8, 8, (5, 1)))).astype(np.float32)
    codes, scales = oracle.quantize_mx4(x)
    assert codes.shape == (5, 48) and scales.shape == (5, 3)
    deq = oracle.dequantize_mx4(codes, scales)
    s = np.ldexp(1.0, np.repeat(scales.astype(np.int64) - 127, 32, 1))
    v = x.astype(np.float64) / s
    assert np.abs(v).max() <= 6.0
    spacing = np.where(np.abs(v) < 1.0, 0.5, np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 1.0))) - 1))
    assert np.all(np.abs(v - deq / s) <= spacing / 2)
    # even element in the low nibble
    y = np.zeros((1, 32), np.float32)
    y[0, :2] = [6.0, 1.0]
    c, sc = oracle.quantize_mx4(y)
    assert sc[0, 0] == 127 and c[0, 0] == (0x7 | (0x2 << 4))


def test_ffn_fp4_lossless_closed_form():
    """As the FP8 closed form: g = 64, u = 1 on one active unit, every value exactly
    representable after MXFP4 quantization, so y = 64 * W_d[:, 0] exactly."""
    d = inter = 64
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 1.0
    wg = np.zeros((inter, d), np.float32)
    wu = np.zeros((inter, d), np.float32)
    wg[0, 0], wu[0, 0] = 64.0, 1.0
    wd = np.zeros((d, inter), np.float32)
    wd[:, 0] = ((np.arange(d) % 8) - 4) * 0.25
    q = [oracle.quantize_mx4(w) for w in (wg, wu, wd)]
    for (c, s_), w in zip(q, (wg, wu, wd)):
        assert np.array_equal(oracle.dequantize_mx4(c, s_), w)
    y = oracle.ffn_fp4(x, [c for c, _ in q], [s_ for _, s_ in q])
    assert np.array_equal(y[0], 64.0 * wd[:, 0].astype(np.float64))
    y_swapped = oracle.ffn_fp4(x, [q[1][0], q[0][0], q[2][0]], [q[1][1], q[0][1], q[2][1]])
    assert not np.allclose(y_swapped, y)



def test_ffn_fp4_quantizes_h_per_block():
    """The MXFP4 counterpart: h = silu(64) * 6 = 384 sets the [1,32] block's scale to
    2^6 (384 = 6 * 64), and h = silu(48) * 6 = 288 = 4.5 * 64 lies between the E2M1
    values 4 and 6, so it reaches the down projection as 4 * 64 = 256."""
    d = inter = 64
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 1.0
    wg = np.zeros((inter, d), np.float32)
    wu = np.zeros((inter, d), np.float32)
    wg[0, 0], wu[0, 0] = 64.0, 6.0
    wg[1, 0], wu[1, 0] = 48.0, 6.0
    wd = np.zeros((d, inter), np.float32)
    wd[:, 0] = np.resize([1.0, -1.0, 0.5, -0.5], d)
    wd[:, 1] = np.resize([0.5, 1.0, -1.0, 0.0], d)
    q = [oracle.quantize_mx4(w) for w in (wg, wu, wd)]
    for (c, s_), w in zip(q, (wg, wu, wd)):
        assert np.array_equal(oracle.dequantize_mx4(c, s_), w)   # lossless
    y = oracle.ffn_fp4(x, [c for c, _ in q], [s_ for _, s_ in q])
    want = 384.0 * wd[:, 0].astype(np.float64) + 256.0 * wd[:, 1].astype(np.float64)
    assert np.array_equal(y[0], want)



def test_ffn_fp4_equals_matmuls_on_the_quantized_operands():
    """The MXFP4 expert restated the same way: every operand row quantized per [1,32],
    H rounded to fp32 then quantized per [1,32]."""
    rng = _rng(42)
    n, d, inter = 6, 128, 192
    x = _blocky(rng, n, d, 1, 32)
    wg, wu = _blocky(rng, inter, d, 1, 32, 0.05), _blocky(rng, inter, d, 1, 32, 0.05)
    wd = _blocky(rng, d, inter, 1, 32, 0.05)
    q = [oracle.quantize_mx4(m) for m in (wg, wu, wd)]
    Wg, Wu, Wd = (oracle.dequantize_mx4(c, s_) for c, s_ in q)
    y = oracle.ffn_fp4(x, [c for c, _ in q], [s_ for _, s_ in q])
    xq = oracle.dequantize_mx4(*oracle.quantize_mx4(x))
    g, u = xq @ Wg.T, xq @ Wu.T
    h32 = (g / (1.0 + np.exp(-g)) * u).astype(np.float32)
    want = oracle.dequantize_mx4(*oracle.quantize_mx4(h32)) @ Wd.T
    np.testing.assert_allclose(y, want, rtol=1e-10, atol=1e-12 * np.abs(want).max())


def test_ffn_fp4_is_close_to_the_unquantized_expert():
    rng = np.random.default_rng(24)
    d, inter = 256, 384
    x = rng.standard_normal((4, d)).astype(np.float32)
    wg, wu = (rng.standard_normal((inter, d)) * 0.06).astype(np.float32), (rng.standard_normal((inter, d)) * 0.06).astype(np.float32)
    wd = (rng.standard_normal((d, inter)) * 0.05).astype(np.float32)
    q = [oracle.quantize_mx4(w) for w in (wg, wu, wd)]
    y4 = oracle.ffn_fp4(x, [c for c, _ in q], [s_ for _, s_ in q])
    y = oracle.ffn(x, wg, wu, wd)
    rel = np.abs(y4 - y).max(axis=1) / np.abs(y).max(axis=1)
    assert 1e-3 < rel.max() < 0.35, rel


# ---------------------------------------------------------------- W4A4 as NVFP4
def _e4m3_round_up(t):
    """The smallest finite E4M3 value >= t, through torch's float8 conversion (a library
    routine: round to nearest, then one code up if that fell below t)."""
    import torch
    t = np.float32(t)
    v = torch.tensor([t], dtype=torch.float32).to(torch.float8_e4m3fn)
    code = int(v.view(torch.uint8).item())
    if float(v.to(torch.float32).item()) < t:
        code += 1
    return min(code, 0x7E)


def test_nv4_scale_against_library_e4m3_rounding():
    """The block scale is the smallest UE4M3 value s with amax <= 6 s g, decided in fp32
    (t = fl32(amax / fl32(6 g))): the same as rounding t up through torch's float8 E4M3."""
    rng = np.random.default_rng(61)
    amax = (rng.uniform(0.5, 1.0, 2000) * np.exp2(rng.integers(-12, 12, 2000))).astype(np.float32)
    gs = np.concatenate([np.ones(1000, np.float32), (rng.uniform(0.5, 1, 1000) * 2.0 ** -8).astype(np.float32)])
    for a, g in zip(amax, gs):
        t = np.float32(a) / (np.float32(6.0) * np.float32(g))
        want = 0x7E if t > 448 else _e4m3_round_up(t)
        assert oracle.nv4_scale(float(a), float(g)) == want, (a, g)
        s = oracle.e4m3_decode(want)
        if t <= 448:
            assert a <= 6 * s * g * (1 + 2 ** -20)          # no saturation
    assert oracle.nv4_scale(0.0, 1.0) == 0x38                   # an all-zero block: 1.0
    assert oracle.nv4_scale(6.0, 1.0) == 0x38 and oracle.e4m3_decode(0x38) == 1.0
    assert oracle.nv4_scale(1e9, 1.0) == 0x7E                   # saturates at 448


def test_nv4_global_makes_the_largest_block_scale_448():
    rng = np.random.default_rng(62)
    for std in (0.006, 0.5, 30.0):
        w = (rng.standard_normal((8, 64)) * std).astype(np.float32)
        c, s_, g = oracle.quantize_weight_nv4(w)
        assert g == np.float32(np.abs(w).max()) / np.float32(2688.0)
        assert s_.max() == 0x7E                                  # the block holding the matrix amax
        assert oracle.e4m3_decode(int(s_.max())) == 448.0
    assert oracle.nv4_global(0.0) == 1.0


def test_quantize_nv4_bound_and_packing():
    rng = np.random.default_rng(63)
    x = (rng.standard_normal((5, 96)) * np.exp2(rng.integers(-4, 4, (5, 1)))).astype(np.float32)
    for g in (1.0, 2.0 ** -6):
        codes, scales = oracle.quantize_nv4(x, g)
        assert codes.shape == (5, 48) and scales.shape == (5, 6)
        deq = oracle.dequantize_nv4(codes, scales, g)
        s = np.repeat(np.array([oracle.e4m3_decode(int(c)) for c in scales.ravel()]).reshape(scales.shape), 16, 1) * g
        v = x.astype(np.float64) / s
        assert np.abs(v).max() <= 6.0 * (1 + 2 ** -20)
        spacing = np.where(np.abs(v) < 1.0, 0.5, np.exp2(np.floor(np.log2(np.maximum(np.abs(v), 1.0))) - 1))
        assert np.all(np.abs(v - deq / s) <= spacing / 2 * (1 + 2 ** -20) + 2 ** -20)
    y = np.zeros((1, 16), np.float32)
    y[0, :2] = [6.0, 1.0]                                        # scale 1.0: codes 6 -> 0x7, 1 -> 0x2
    c, sc = oracle.quantize_nv4(y)
    assert sc[0, 0] == 0x38 and c[0, 0] == (0x7 | (0x2 << 4))


def test_ffn_nv4_lossless_closed_form():
    """Values that quantize exactly at tensor scale 1.  A 6 in each block sets its scale
    to 1.0 (x = [6, 0..]; W_g row 0 = [4, 6, 0..]; W_u row 0 = [1, 6, 0..]; every W_d row
    = [v, 6, 0..] with v an E2M1 value), so g = 24, u = 6 and h = silu(24) * 6 rounds to
    144 in fp32; h's block holds 144 alone, its scale 24 is an E4M3 value and its code 6.
    Then y = 144 * W_d[:, 0] exactly, and a tensor scale on W_d multiplies y."""
    d = inter = 64
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 6.0
    wg = np.zeros((inter, d), np.float32)
    wu = np.zeros((inter, d), np.float32)
    wg[0, :2] = [4.0, 6.0]
    wu[0, :2] = [1.0, 6.0]
    wd = np.zeros((d, inter), np.float32)
    wd[:, 0] = np.resize([6.0, -3.0, 1.5, -0.5, 0.0, 4.0, -2.0, 1.0], d)
    wd[:, 1] = 6.0
    q = [oracle.quantize_nv4(w, 1.0) for w in (wg, wu, wd)]
    for (c, s_), w in zip(q, (wg, wu, wd)):
        assert np.array_equal(oracle.dequantize_nv4(c, s_, 1.0), w)      # lossless
    codes, scales = [c for c, _ in q], [s_ for _, s_ in q]
    y = oracle.ffn_nv4(x, codes, scales, [1.0, 1.0, 1.0])
    assert np.array_equal(y[0], 144.0 * wd[:, 0].astype(np.float64))
    assert np.array_equal(oracle.ffn_nv4(x, codes, scales, [1.0, 1.0, 0.5])[0], 72.0 * wd[:, 0].astype(np.float64))


def test_ffn_nv4_equals_matmuls_on_the_quantized_operands():
    """The NVFP4 expert restated with library matmuls over the separately pinned
    quantizers: operand rows per [1,16] (x and H at g = 1, weights at their matrix
    scale), H rounded to fp32 first."""
    rng = _rng(64)
    n, d, inter = 6, 128, 192
    x = _blocky(rng, n, d, 1, 16)
    wg, wu = _blocky(rng, inter, d, 1, 16, 0.05), _blocky(rng, inter, d, 1, 16, 0.05)
    wd = _blocky(rng, d, inter, 1, 16, 0.05)
    q = [oracle.quantize_weight_nv4(m) for m in (wg, wu, wd)]
    Wg, Wu, Wd = (oracle.dequantize_nv4(c, s_, g) for c, s_, g in q)
    y = oracle.ffn_nv4(x, [c for c, _, _ in q], [s_ for _, s_, _ in q], [g for _, _, g in q])
    xq = oracle.dequantize_nv4(*oracle.quantize_nv4(x))
    g_, u = xq @ Wg.T, xq @ Wu.T
    h32 = (g_ / (1.0 + np.exp(-g_)) * u).astype(np.float32)
    want = oracle.dequantize_nv4(*oracle.quantize_nv4(h32)) @ Wd.T
    np.testing.assert_allclose(y, want, rtol=1e-9, atol=1e-12 * np.abs(want).max())


def test_ffn_nv4_is_close_to_the_unquantized_expert():
    rng = np.random.default_rng(65)
    d, inter = 256, 384
    x = rng.standard_normal((4, d)).astype(np.float32)
    wg = (rng.standard_normal((inter, d)) * 0.06).astype(np.float32)
    wu = (rng.standard_normal((inter, d)) * 0.06).astype(np.float32)
    wd = (rng.standard_normal((d, inter)) * 0.05).astype(np.float32)
    q = [oracle.quantize_weight_nv4(w) for w in (wg, wu, wd)]
    y4 = oracle.ffn_nv4(x, [c for c, _, _ in q], [s_ for _, s_, _ in q], [g for _, _, g in q])
    y = oracle.ffn(x, wg, wu, wd)
    rel = np.abs(y4 - y).max(axis=1) / np.abs(y).max(axis=1)
    assert 1e-3 < rel.max() < 0.45, rel


# ---------------------------------------------------------------- backward (oracle only)

def _tiny_fwd_loss(x, wr, wg, wu, wd, bias, dy, N, k, scale, offset):
    l = oracle.router_logits(x, wr, offset)
    s = oracle.softmax(l)
    idx, gate, _ = oracle.topk(s, bias, k, scale)
    y = oracle.layer(x, idx, gate, N, wg, wu, wd)
    return float((y * dy).sum()), idx, s


def test_backward_against_central_differences():
    """Every gradient of the fp64 backward (x, W_r, W_g, W_u, W_d) agrees with central
    differences of <dy, y(x, W)> on a tiny layer, the routing held by small steps
    (checked: the same experts are picked on both sides of every step)."""
    rng = np.random.default_rng(31)
    T, d, N, Z, k, inter, scale = 5, 16, 3, 2, 3, 8, 1.7
    E = N + Z
    x = rng.standard_normal((T, d)).astype(np.float32)
    wr = (rng.standard_normal((E, d)) * 0.4).astype(np.float32)
    wg = (rng.standard_normal((N, inter, d)) * 0.3).astype(np.float32)
    wu = (rng.standard_normal((N, inter, d)) * 0.3).astype(np.float32)
    wd = (rng.standard_normal((N, d, inter)) * 0.3).astype(np.float32)
    bias = rng.uniform(-0.05, 0.05, E)
    offset = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    dy = rng.standard_normal((T, d))
    params = {"x": x, "wr": wr, "wg": wg, "wu": wu, "wd": wd}
    L0, idx0, s0 = _tiny_fwd_loss(x, wr, wg, wu, wd, bias, dy, N, k, scale, offset)
    grads = dict(zip(params, oracle.layer_backward(x, idx0, s0, scale, dy, N, wr, wg, wu, wd)))
    checked = 0
    for name, arr in params.items():
        flat = arr.reshape(-1)
        for i in rng.choice(flat.size, size=min(12, flat.size), replace=False):
            v = float(flat[i])
            hp, hm = np.float32(v + 1e-2), np.float32(v - 1e-2)
            flat[i] = hp
            Lp, idxp, _ = _tiny_fwd_loss(params["x"], params["wr"], params["wg"], params["wu"], params["wd"], bias, dy,
                                         N, k, scale, offset)
            flat[i] = hm
            Lm, idxm, _ = _tiny_fwd_loss(params["x"], params["wr"], params["wg"], params["wu"], params["wd"], bias, dy,
                                         N, k, scale, offset)
            flat[i] = np.float32(v)
            if not (np.array_equal(idxp, idx0) and np.array_equal(idxm, idx0)):
                continue  # the step changed a selection; this coordinate is not differentiable here
            fd = (Lp - Lm) / (float(hp) - float(hm))
            an = float(grads[name].reshape(-1)[i])
            assert abs(fd - an) <= 2e-4 * max(1.0, abs(an)), (name, int(i), fd, an)
            checked += 1
    assert checked >= 50


def test_backward_bias_gets_no_gradient_and_zero_experts_pass_dy():
    """With only zero experts chosen the layer is y = (sum of their gates) x: dx = zsum dy
    plus the router term; the bias never appears in any gradient formula (it only
    selects), so moving it without changing the selection changes no gradient."""
    rng = np.random.default_rng(32)
    T, d, N, Z, k, inter = 3, 8, 2, 4, 2, 8
    E = N + Z
    x = rng.standard_normal((T, d)).astype(np.float32)
    wr = (rng.standard_normal((E, d)) * 0.3).astype(np.float32)
    wg = rng.standard_normal((N, inter, d)).astype(np.float32)
    wu = rng.standard_normal((N, inter, d)).astype(np.float32)
    wd = rng.standard_normal((N, d, inter)).astype(np.float32)
    bias = np.zeros(E)
    bias[N:] = 5.0   # every pick is a zero expert
    dy = rng.standard_normal((T, d))
    l = oracle.router_logits(x, wr)
    s = oracle.softmax(l)
    idx, gate, _ = oracle.topk(s, bias, k, 1.0)
    assert (idx >= N).all()
    g1 = oracle.layer_backward(x, idx, s, 1.0, dy, N, wr, wg, wu, wd)
    assert not g1[2].any() and not g1[3].any() and not g1[4].any()   # no FFN expert ran
    zsum = gate.sum(axis=1)
    dl_part = g1[0] - zsum[:, None] * dy
    # the remaining dx is the router's W_r^T dl, with dl = s * (ds - <s, ds>), ds_e = <dy, x> on picked e
    ds = np.zeros((T, E))
    for t in range(T):
        for j in range(k):
            ds[t, idx[t, j]] += float(dy[t] @ x[t].astype(np.float64))
    dl = s * (ds - (s * ds).sum(axis=1, keepdims=True))
    assert np.allclose(dl_part, dl @ wr.astype(np.float64), rtol=1e-12, atol=1e-12)
    bias2 = bias.copy()
    bias2[N:] = 7.0
    idx2, _, _ = oracle.topk(s, bias2, k, 1.0)
    assert np.array_equal(idx2, idx)
    g2 = oracle.layer_backward(x, idx2, s, 1.0, dy, N, wr, wg, wu, wd)
    assert all(np.array_equal(a_, b_) for a_, b_ in zip(g1, g2))
