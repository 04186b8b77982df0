"""GPU parity at the limits zcmoe_create accepts, and on inputs that are not finite.

  * E = 1024 experts (32 per lane in the top-k kernel, one thread per expert in the
    scan kernel) with k = 32: routing bit-exact on every token, expert and layer
    outputs against the fp64 oracle;
  * T = 2^20 tokens, the largest batch a handle accepts, on a narrow layer:
    routing bit-exact on every token, layer outputs on sampled rows;
  * token rows holding NaN or infinite values: routing still follows the oracle's
    rule (a NaN biased score ranks as -inf), every pick is a valid distinct
    expert, the finite rows' outputs are unaffected, and no kernel gives up.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_shifted_b200 import configs
from tests.gpu_harness import Run

pytestmark = pytest.mark.gpu


def test_1024_experts_top32(cuda_ok):
    w = configs.Workload("e1024", T=4096, d=256, n_ffn=768, inter=128, n_zero=256, top_k=32, dtype="bf16",
                         w_std=0.05, bias=("uniform", -2e-4, 2e-4), seed=7)
    r = Run(w)
    try:
        r.forward()
        r.check_routing_bitexact()
        rng = np.random.default_rng(0)
        r.check_expert_outputs(sorted(rng.choice(r.P, size=min(r.P, 400), replace=False)))
        r.check_layer_outputs(np.sort(rng.choice(r.T, size=256, replace=False)))
        frac = r.check_logits_and_fp64_routing(np.arange(0, r.T, 16))
        assert frac > 0.5
    finally:
        r.close()


def test_largest_batch_2_pow_20_tokens(cuda_ok):
    T = 1 << 20
    w = configs.Workload("t2p20", T=T, d=256, n_ffn=64, inter=128, n_zero=32, top_k=8, dtype="bf16", w_std=0.05,
                         bias=("uniform", -0.02, 0.02), seed=9)
    r = Run(w, max_tokens=T)
    try:
        r.forward()
        r.check_routing_bitexact()
        rng = np.random.default_rng(1)
        rows = np.sort(np.concatenate([rng.choice(T, size=200, replace=False), np.arange(T - 56, T)]))
        r.check_layer_outputs(rows)
        pairs = np.sort(np.concatenate([rng.choice(r.P, size=200, replace=False), np.arange(r.P - 40, r.P)]))
        r.check_expert_outputs(pairs)
    finally:
        r.close()


def test_rows_that_are_not_finite(cuda_ok):
    w = configs.WORKLOADS["small_bf16"]
    T = 1000
    x = configs.device_tokens(w, T)
    bad = {0: float("nan"), 1: float("inf"), 2: -float("inf")}
    for t, v in bad.items():
        x[t, 5] = v
    x[3, :] = float("nan")
    r = Run(w, T=T, x=x)
    try:
        r.forward()  # also checks that no kernel gave up on a wait
        d = r.dbg
        idx, gate, scores = oracle.route_replica_f32(d["logits"], r.cur_bias, w.top_k, 1.0, want_scores=True)
        np.testing.assert_array_equal(d["idx"], idx)
        for got, ref in ((d["gate"], gate), (d["scores"], scores)):
            nan = np.isnan(ref)
            np.testing.assert_array_equal(np.isnan(got), nan)
            np.testing.assert_array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))
        counts, offsets, perm, pos = oracle.integer_stage(idx, w.n_ffn, w.E)
        np.testing.assert_array_equal(d["counts"], counts)
        np.testing.assert_array_equal(d["perm"][: r.P], perm)
        np.testing.assert_array_equal(d["pos"], pos)
        for t in range(T):
            assert len(set(d["idx"][t].tolist())) == w.top_k
        assert d["idx"].min() >= 0 and d["idx"].max() < w.E
        for t in (0, 3):  # every logit NaN: all scores NaN, picks are experts 0..k-1
            assert d["idx"][t].tolist() == list(range(w.top_k))
        good = np.arange(4, T)
        y = torch.from_numpy(r.y[good].view(np.int16)).view(torch.bfloat16).float().numpy()
        assert np.isfinite(y).all()
        r.check_layer_outputs(good[::7])
    finally:
        r.close()


def test_routing_with_many_exact_ties(cuda_ok):
    """Logits on a coarse grid (multiples of 1/2) and biases on a coarser one make many
    experts share the same biased score, at and around the k-th place: the picks must
    follow the oracle's rule (equal scores: the lower id first) bit for bit, whether
    the selection takes its sorted-candidates path or its one-pick-at-a-time path."""
    import ctypes
    from mixture_experts_layer_shifted_b200 import zcmoe as Z
    N, Zn, k, T = 512, 256, 12, 4096
    E = N + Zn
    rng = np.random.default_rng(13)
    l = (np.round(rng.normal(size=(T, E)) * 2.0) / 2.0).astype(np.float32)
    l[: T // 4] = np.round(l[: T // 4])          # coarser grid: more ties
    l[T // 4: T // 4 + 8] = 1.5                  # every expert tied
    bias = np.zeros(E, np.float32)
    bias[::7] = np.float32(2.0 ** -20)
    logits, b = torch.from_numpy(l).cuda(), torch.from_numpy(bias).cuda()
    out = {"idx": (T * k, torch.int32), "gate": (T * k, torch.float32), "counts": (E, torch.int32),
           "offsets": (N + 1, torch.int32), "perm": (T * k, torch.int32), "pos": (T * k, torch.int32)}
    out = {key: torch.full((n,), -7, dtype=dt, device="cuda") for key, (n, dt) in out.items()}
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    Z.zcmoe_route_noalloc(p(logits), p(b), T, N, Zn, k, 1.0, p(out["idx"]), p(out["gate"]), p(out["counts"]),
                          p(out["offsets"]), p(out["perm"]), p(out["pos"]))
    torch.cuda.synchronize()
    idx, gate, _ = oracle.route_replica_f32(l, bias, k, 1.0, want_scores=True)
    np.testing.assert_array_equal(out["idx"].cpu().numpy().reshape(T, k), idx)
    np.testing.assert_array_equal(out["gate"].cpu().numpy().reshape(T, k).view(np.uint32), gate.view(np.uint32))
    counts, offsets, perm, pos = oracle.integer_stage(idx, N, E)
    np.testing.assert_array_equal(out["counts"].cpu().numpy(), counts)
    np.testing.assert_array_equal(out["perm"].cpu().numpy()[: int(offsets[-1])], perm)
    np.testing.assert_array_equal(out["pos"].cpu().numpy().reshape(T, k), pos)
