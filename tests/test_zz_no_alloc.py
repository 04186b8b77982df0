"""The allocation-free routing entry point, zcmoe_route_noalloc.

It exists for callers that cannot call cudaMalloc (code inside a framework's
memory pool or a fixed memory budget, and latency-critical loops where an
allocation could synchronise the device).  Its scratch is a fixed device array
inside the library.  This file is collected last so that a run stopping at the
first failure has already run every other test; it also passes on its own in
a fresh process.

The checks:
  * the routing outputs of two back-to-back calls (the second one reusing the
    scratch the first one left behind) equal, bit for bit, what the regular
    zcmoe_forward computes for the same logits and bias, and that forward's
    routing is itself checked bit-exact against the oracle's fp32 replica;
  * at the largest T the scratch allows, the outputs equal the oracle's replica
    and integer stage; one block more is refused;
  * rows that are not all finite (NaN or infinite logits, NaN bias) still pick
    k distinct valid experts, as the oracle's rule says, and nothing is written
    out of bounds."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_shifted_b200 import configs
from mixture_experts_layer_shifted_b200 import zcmoe as Z
from tests.gpu_harness import Run

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _outputs(T, E, k, N):
    return {
        "idx": torch.full((T, k), -7, dtype=torch.int32, device="cuda"),
        "gate": torch.full((T, k), -7.0, dtype=torch.float32, device="cuda"),
        "counts": torch.full((E,), -7, dtype=torch.int32, device="cuda"),
        "offsets": torch.full((N + 1,), -7, dtype=torch.int32, device="cuda"),
        "perm": torch.full((T * k,), -7, dtype=torch.int32, device="cuda"),
        "pos": torch.full((T, k), -7, dtype=torch.int32, device="cuda"),
    }


def _route(logits, bias, T, N, Zn, k, out, scale=1.0):
    Z.zcmoe_route_noalloc(_p(logits), _p(bias), T, N, Zn, k, scale, _p(out["idx"]), _p(out["gate"]),
                          _p(out["counts"]), _p(out["offsets"]), _p(out["perm"]), _p(out["pos"]))
    torch.cuda.synchronize()
    return {key: v.cpu().numpy() for key, v in out.items()}


def _check_against_replica(got, logits_h, bias_h, N, E, k, scale=1.0):
    """Replica routing and integer stage on the same fp32 logits; NaN gates compare
    as NaN (their bit patterns are not part of the rule)."""
    idx, gate, _ = oracle.route_replica_f32(logits_h, bias_h, k, scale, want_scores=True)
    np.testing.assert_array_equal(got["idx"], idx)
    nan = np.isnan(gate)
    np.testing.assert_array_equal(np.isnan(got["gate"]), nan)
    np.testing.assert_array_equal(got["gate"][~nan].view(np.uint32), gate[~nan].view(np.uint32))
    counts, offsets, perm, pos = oracle.integer_stage(idx, N, E)
    np.testing.assert_array_equal(got["counts"], counts)
    np.testing.assert_array_equal(got["offsets"], offsets)
    P = int(offsets[-1])
    np.testing.assert_array_equal(got["perm"][:P], perm)
    np.testing.assert_array_equal(got["pos"], pos)


@pytest.mark.parametrize("name,T", [("small_bf16", None), ("prefill_probe", 3000)])
def test_noalloc_routing_matches_forward_twice(cuda_ok, name, T):
    w = configs.WORKLOADS[name]
    r = Run(w, T=T)
    try:
        r.forward()
        r.check_routing_bitexact()  # the forward compared with is itself checked against the oracle
        Tn, E, k, N = r.T, w.E, w.top_k, w.n_ffn
        logits = torch.from_numpy(r.dbg["logits"]).cuda()
        bias = torch.from_numpy(r.cur_bias).cuda()
        for call in range(2):
            got = _route(logits, bias, Tn, N, w.n_zero, k, _outputs(Tn, E, k, N))
            np.testing.assert_array_equal(got["idx"], r.dbg["idx"])
            np.testing.assert_array_equal(got["gate"].view(np.uint32), r.dbg["gate"].view(np.uint32))
            np.testing.assert_array_equal(got["counts"], r.dbg["counts"])
            np.testing.assert_array_equal(got["offsets"], r.dbg["offsets"])
            P = int(r.dbg["offsets"][-1])
            np.testing.assert_array_equal(got["perm"][:P], r.dbg["perm"][:P])
            np.testing.assert_array_equal(got["pos"], r.dbg["pos"])
    finally:
        r.close()


def test_noalloc_at_its_largest_T_matches_the_oracle(cuda_ok):
    """E = 768 (512 FFN + 256 zero experts, top-12): T = 86,528 is the largest T whose
    routing scratch fits the fixed 1 MiB array; every output equals the replica."""
    N, Zn, k = 512, 256, 12
    E = N + Zn
    T = 86_528
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    logits = torch.randn((T, E), generator=g, device="cuda", dtype=torch.float32)
    bias = (torch.rand((E,), generator=g, device="cuda", dtype=torch.float32) - 0.5) * 2e-3
    for call in range(2):
        got = _route(logits, bias, T, N, Zn, k, _outputs(T, E, k, N))
        _check_against_replica(got, logits.cpu().numpy(), bias.cpu().numpy(), N, E, k)
    with pytest.raises(Z.ZcmoeError) as ei:
        _route(logits, bias, T + 1, N, Zn, k, _outputs(8, E, k, N))
    assert ei.value.code == Z.ZCMOE_ERANGE and "86528" in Z.zcmoe_last_error()


def test_noalloc_rows_that_are_not_finite(cuda_ok):
    """NaN and infinite logits and NaN biases: every row still selects k distinct valid
    experts (a NaN biased score ranks as -inf, the lowest id first among equals), the
    same as the oracle's replica, and the integer stage stays within its buffers."""
    N, Zn, k = 16, 8, 4
    E = N + Zn
    T = 300
    rng = np.random.default_rng(12)
    l = rng.normal(size=(T, E)).astype(np.float32)
    l[0, :] = np.nan
    l[1, 3] = np.inf
    l[2, :] = -np.inf
    l[3, 7] = np.nan
    l[4, 0] = -np.inf
    l[5, :] = np.inf
    l[6, 10:] = np.nan
    bias = rng.uniform(-0.1, 0.1, size=E).astype(np.float32)
    bias[[2, 17]] = np.nan
    logits = torch.from_numpy(l).cuda()
    b = torch.from_numpy(bias).cuda()
    for call in range(2):
        got = _route(logits, b, T, N, Zn, k, _outputs(T, E, k, N))
        _check_against_replica(got, l, bias, N, E, k)
        for t in range(T):
            row = got["idx"][t]
            assert len(set(row.tolist())) == k and row.min() >= 0 and row.max() < E
        assert int(got["counts"].sum()) == T * k


def test_noalloc_refuses_a_scale_that_is_not_finite(cuda_ok):
    dummy = torch.zeros(64, dtype=torch.int32, device="cuda")
    for bad in (float("nan"), float("inf")):
        with pytest.raises(Z.ZcmoeError) as ei:
            Z.zcmoe_route_noalloc(_p(dummy), _p(dummy), 8, 16, 8, 4, bad, *([_p(dummy)] * 6))
        assert ei.value.code == Z.ZCMOE_EINVAL


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_ok):
    E, k, N = 768, 12, 512
    T = 100_000  # needs ~1.2 MB of routing scratch; the fixed array holds 1 MiB
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(Z.ZcmoeError) as ei:
        Z.zcmoe_route_noalloc(_p(dummy), _p(dummy), T, N, E - N, k, 1.0, *([_p(dummy)] * 6))
    assert ei.value.code == Z.ZCMOE_ERANGE
    assert "scratch" in Z.zcmoe_last_error()
