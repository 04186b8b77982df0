"""GPU parity on the small workloads: the fp32 tiny layer and the bf16 small
layer, plus ragged shapes that exercise partial tiles, every stage compared
with the CPU oracle through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_shifted_b200 import configs, synth, zcmoe
from tests.gpu_harness import TOL, Run, row_rel_err

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS


@pytest.fixture(scope="module")
def tiny(cuda_ok):
    r = Run(W["tiny_f32"])
    r.forward()
    yield r
    r.close()


@pytest.fixture(scope="module")
def small(cuda_ok):
    r = Run(W["small_bf16"])
    r.forward()
    yield r
    r.close()


# ---------------------------------------------------------------- tiny fp32 (64 tokens, 16+8 experts, k=4)
def test_tiny_routing_bitexact(tiny):
    tiny.check_routing_bitexact()


def test_tiny_fp64_routing_and_logits(tiny):
    frac = tiny.check_logits_and_fp64_routing(np.arange(tiny.T))
    assert frac > 0.9


def test_tiny_expert_outputs_all_pairs(tiny):
    tiny.check_expert_outputs(range(tiny.P))


def test_tiny_layer_outputs_all_tokens(tiny):
    assert tiny.check_layer_outputs(np.arange(tiny.T)) <= TOL["f32"]


def test_tiny_layer_against_oracle_own_routing(tiny):
    # oracle end to end (its own fp64 logits and routing), tokens away from near-ties
    x = tiny.x_host()
    l = oracle.router_logits(x, tiny.router_host(), tiny.offset)
    idx, gate, margin = oracle.topk(oracle.softmax(l), tiny.bias.astype(np.float64), tiny.w.top_k)
    _, wg, wu, wd = (None,) + tuple(t.cpu().numpy() for t in tiny.weights[1:])
    ref = oracle.layer(x, idx, gate, tiny.w.n_ffn, wg, wu, wd)
    ok = margin >= 1e-5
    err = row_rel_err(tiny.y[ok], ref[ok])
    assert err.max() <= TOL["f32"]


def test_tiny_brute_force_selection(tiny):
    s = tiny.dbg["scores"].astype(np.float64)
    v = s + tiny.bias.astype(np.float64)
    for t in range(0, tiny.T, 8):
        # exact fp32 biased scores decide; the brute force sums them in fp64
        vv = (tiny.dbg["scores"][t] + tiny.bias).astype(np.float32)
        assert list(tiny.dbg["idx"][t]) == oracle.brute_force_topk(vv, tiny.w.top_k)
    assert v.shape == (tiny.T, tiny.w.E)


def test_tiny_determinism(tiny):
    y0 = tiny.y.copy()
    tiny.forward()
    np.testing.assert_array_equal(tiny.y, y0)


# ---------------------------------------------------------------- small bf16 (4096 tokens, 64+32 experts, k=8)
def test_small_routing_bitexact(small):
    small.check_routing_bitexact()


def test_small_fp64_routing_and_logits(small):
    rows = np.arange(0, small.T, 7)
    assert small.check_logits_and_fp64_routing(rows) > 0.5


def test_small_expert_outputs(small):
    rng = np.random.default_rng(0)
    pairs = rng.choice(small.P, size=min(small.P, 600), replace=False)
    # include the first and last row of several experts (tile edges)
    offs = small.dbg["offsets"]
    edges = [int(offs[e]) for e in range(0, small.w.n_ffn, 5) if offs[e + 1] > offs[e]]
    edges += [int(offs[e + 1]) - 1 for e in range(0, small.w.n_ffn, 5) if offs[e + 1] > offs[e]]
    small.check_expert_outputs(sorted(set(pairs.tolist()) | set(edges)))


def test_small_layer_outputs(small):
    rows = np.concatenate([np.arange(0, 64), np.arange(small.T - 64, small.T), np.arange(64, small.T, 97)])
    assert small.check_layer_outputs(rows) <= TOL["bf16"]


def test_small_determinism(small):
    y0 = small.y.copy()
    small.forward()
    np.testing.assert_array_equal(small.y, y0)


def test_small_bias_changes_selection_never_gates(small):
    r0 = Run(small.w, bias=np.zeros(small.w.E, np.float32), weights=small.weights, x=small.x)
    r0.forward()
    try:
        i1, g1, s = small.dbg["idx"], small.dbg["gate"], small.dbg["scores"]
        i0, g0 = r0.dbg["idx"], r0.dbg["gate"]
        assert (i0 != i1).any()
        np.testing.assert_array_equal(r0.dbg["scores"].view(np.uint32), s.view(np.uint32))
        rows = np.arange(small.T)[:, None]
        np.testing.assert_array_equal(g1.view(np.uint32), s[rows, i1].view(np.uint32))
        np.testing.assert_array_equal(g0.view(np.uint32), s[rows, i0].view(np.uint32))
    finally:
        r0.close()


def test_small_zero_only_tokens_return_weighted_input(small):
    b = np.zeros(small.w.E, np.float32)
    b[small.w.n_ffn:] = 0.5
    r = Run(small.w, bias=b, weights=small.weights, x=small.x)
    r.forward()
    try:
        r.check_routing_bitexact()
        assert np.all(r.dbg["idx"] >= small.w.n_ffn) and r.P == 0
        # y = bf16(fl32(sum of gates in slot order) * x), bit for bit
        z = np.zeros(r.T, np.float32)
        for j in range(r.w.top_k):
            z = (z + r.dbg["gate"][:, j]).astype(np.float32)
        x = synth.bf16_bits_to_f32(r.x_host())
        want = synth.f32_to_bf16_bits((z[:, None] * x).astype(np.float32))
        np.testing.assert_array_equal(r.y, want)
    finally:
        r.close()


# ---------------------------------------------------------------- ragged shapes and edge cases

@pytest.mark.parametrize("T,d,N,inter,Z,k", [
    (1, 256, 8, 128, 4, 3),          # one token
    (1000, 320, 40, 192, 24, 6),     # d and inter not multiples of the column tiles; ragged T
    (300, 512, 33, 64, 0, 5),        # no zero experts
    (257, 192, 4, 256, 60, 32),      # k = 32, most picks zero experts
    (2000, 256, 3, 128, 1, 2),       # > 256 tokens per expert: several token tiles
])
def test_ragged_bf16(cuda_ok, T, d, N, inter, Z, k):
    w = configs.Workload("ragged", T=T, d=d, n_ffn=N, inter=inter, n_zero=Z, top_k=k, dtype="bf16", w_std=0.05,
                         bias=("uniform", -0.05, 0.05), seed=3)
    r = Run(w, max_tokens=T + 5)
    try:
        r.forward()
        r.check_routing_bitexact()
        if r.P:
            r.check_expert_outputs(range(r.P))
        r.check_layer_outputs(np.arange(T))
    finally:
        r.close()


def test_ragged_f32(cuda_ok):
    w = configs.Workload("ragged32", T=77, d=192, n_ffn=10, inter=64, n_zero=6, top_k=5, dtype="f32", w_std=0.05,
                         bias=("uniform", -0.05, 0.05), seed=5)
    r = Run(w)
    try:
        r.forward()
        r.check_routing_bitexact()
        r.check_expert_outputs(range(r.P))
        r.check_layer_outputs(np.arange(r.T))
    finally:
        r.close()


def test_empty_batch_is_a_no_op(tiny):
    x = torch.empty((0, tiny.w.d), dtype=torch.float32, device="cuda")
    y = tiny.layer.forward(x)
    assert y.shape == (0, tiny.w.d)
    st = tiny.layer.state()
    assert st["tokens"] >= 0


def test_too_many_tokens_is_rejected(tiny):
    from mixture_experts_layer_shifted_b200.zcmoe import ZCMOE_ERANGE, ZcmoeError
    x = torch.zeros((tiny.layer.max_tokens + 1, tiny.w.d), dtype=torch.float32, device="cuda")
    with pytest.raises(ZcmoeError) as ei:
        tiny.layer.forward(x)
    assert ei.value.code == ZCMOE_ERANGE


def test_controller_step_bitexact(cuda_ok):
    w = W["small_bf16"]
    r = Run(w)
    try:
        st_o = oracle.new_controller_state(r.bias)
        gains = (0.3, 0.05, 0.2, 0.97, 5.0)
        for step in range(4):
            r.x = configs.device_tokens(w, step=step)
            r.forward(debug=False)
            s = r.layer.state()
            counts = s["counts"].copy()
            tokens = np.array([s["tokens"]], np.int64)
            assert tokens[0] == w.T
            oracle.update_bias(counts, tokens, w.n_ffn, w.n_zero, w.top_k, gains, r.bias, st_o)
            r.layer.update_bias(*gains[:4], target_ffn_per_token=gains[4])
            s2 = r.layer.state()
            np.testing.assert_array_equal(s2["bias"].view(np.uint32), st_o["bias"].view(np.uint32))
            assert s2["tokens"] == 0 and not s2["counts"].any()
            assert s2["eta"] == float(st_o["eta"][0])
    finally:
        r.close()



def test_controller_checkpoint_and_resume(cuda_ok):
    """A checkpoint of the whole controller state (bias, I, e_prev, eta and the counts
    accumulated since the last step), loaded into a fresh handle made with the same
    init_bias: both handles then take bit-identical steps, equal to the oracle's."""
    w = W["small_bf16"]
    gains = (0.3, 0.05, 0.2, 0.97, 5.0)
    a = Run(w)
    b = Run(w, weights=a.weights)
    try:
        st_o = oracle.new_controller_state(a.bias)
        for step in range(3):
            a.x = configs.device_tokens(w, step=step)
            a.forward(debug=False)
            s = a.layer.state()
            oracle.update_bias(s["counts"].copy(), np.array([s["tokens"]], np.int64), w.n_ffn, w.n_zero, w.top_k,
                               gains, a.bias, st_o)
            a.layer.update_bias(*gains[:4], target_ffn_per_token=gains[4])
        a.x = configs.device_tokens(w, step=3)
        a.forward(debug=False)                       # counts pending at the checkpoint
        ck = a.layer.controller_state()
        np.testing.assert_array_equal(ck["integ"].view(np.uint32), st_o["integ"].view(np.uint32))
        np.testing.assert_array_equal(ck["eprev"].view(np.uint32), st_o["eprev"].view(np.uint32))
        assert ck["tokens"][0] == w.T and ck["counts"].sum() == w.T * w.top_k
        b.layer.load_controller_state(ck)
        back = b.layer.controller_state()
        for key in ck:
            np.testing.assert_array_equal(back[key], ck[key])
        for step in range(4, 7):
            for r in (a, b):
                r.layer.update_bias(*gains[:4], target_ffn_per_token=gains[4])
                r.x = configs.device_tokens(w, step=step)
                r.forward(debug=False)
            sa, sb = a.layer.controller_state(), b.layer.controller_state()
            for key in sa:
                np.testing.assert_array_equal(sa[key], sb[key])
        with pytest.raises(zcmoe.ZcmoeError) as ei:   # negative counts are refused, nothing changed
            b.layer.load_controller_state(dict(ck, counts=-np.ones(w.E, np.int64)))
        assert ei.value.code == zcmoe.ZCMOE_EINVAL
        np.testing.assert_array_equal(b.layer.controller_state()["bias"], sb["bias"])
    finally:
        a.close()
        b.close()



def test_update_bias_refuses_gains_that_are_not_finite(small):
    """A NaN or infinite gain would poison the bias and every later routing decision:
    the step is refused on the host and the controller state stays as it was."""
    before = small.layer.controller_state()
    for bad in (dict(kp=float("nan")), dict(ki=float("inf")), dict(kd=-float("inf")), dict(decay=float("nan"))):
        gains = dict(dict(kp=0.0, ki=0.05, kd=0.0, decay=1.0), **bad)
        with pytest.raises(zcmoe.ZcmoeError) as ei:
            small.layer.update_bias(target_ffn_per_token=5.0, **gains)
        assert ei.value.code == zcmoe.ZCMOE_EINVAL
    after = small.layer.controller_state()
    for key in before:
        np.testing.assert_array_equal(after[key], before[key])


def test_counts_exchange_roundtrip(small):
    E = small.w.E
    buf = torch.empty(E + 1, dtype=torch.int64, device="cuda")
    small.layer.read_counts(buf)
    before = small.layer.state()
    doubled = buf * 2
    small.layer.write_counts(doubled)
    after = small.layer.state()
    np.testing.assert_array_equal(after["counts"], before["counts"] * 2)
    assert after["tokens"] == before["tokens"] * 2
    small.layer.write_counts(buf)


def test_forward_host_matches_device(small):
    xh = small.x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    small.layer.forward_host(xh, yh)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(yh.view(torch.int16).numpy().view(np.uint16), small.y)


@pytest.mark.parametrize("n", [1, 2, 5])
def test_forward_host_pipelined(small, n):
    """The pipelined host-buffer forward: each call's output, complete after the next call
    (or the flush), equals the device forward of its input; the stream is not synchronised
    between calls, and a plain zcmoe_forward_host call in between keeps the order."""
    xs = [configs.device_tokens(small.w, step=s) for s in range(10, 10 + n)]
    want = []
    for x in xs:
        want.append(small.layer.forward(x).view(torch.int16).cpu().numpy())
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty_like(x).pin_memory() for x in xh]
    for i, (a, b) in enumerate(zip(xh, yh)):
        small.layer.forward_host(a, b, pipelined=(i != 2))  # call 2 (if any) is the plain form
    small.layer.flush_host()
    torch.cuda.synchronize()
    for b, w in zip(yh, want):
        np.testing.assert_array_equal(b.view(torch.int16).numpy(), w)


def test_forward_host_back_to_back_calls(small):
    """Several host-buffer calls in flight (uploads double-buffered on the copy
    stream) each return their own input's output."""
    xs = [configs.device_tokens(small.w, step=s) for s in (5, 6, 7)]
    want = []
    for x in xs:
        y = small.layer.forward(x)
        torch.cuda.synchronize()
        want.append(y.view(torch.int16).cpu().numpy())
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty_like(x).pin_memory() for x in xh]
    for a, b in zip(xh, yh):
        small.layer.forward_host(a, b)
    torch.cuda.synchronize()
    for b, w in zip(yh, want):
        np.testing.assert_array_equal(b.view(torch.int16).numpy(), w)
