"""GPU parity of the W4A4 experts in NVFP4 (ZCMOE_NVFP4 layers: E2M1 codes, one UE4M3
scale per 16 elements, one fp32 scale per expert weight matrix; zcmoe_quantize_nv4)
through the C ABI.

A LongCat-Flash news page (gate.com post) reports W4A4 serving without naming the
format; NVFP4 is the second reading, beside MXFP4.

Tolerances (from the arithmetic):
  * quantizer: bit-exact codes, block scales and tensor scales (every decision is
    taken in fp32 on the same values on both sides);
  * routing: bit-exact (the router is unchanged);
  * expert and layer outputs vs the NVFP4 oracle: max over rows of
    ||err||_inf / ||ref||_inf <= 2e-2 and median row <= 4e-3 -- a product of two
    E2M1 codes and two UE4M3 scales has at most 12 significant bits, so the MMA's
    products are exact in fp32; what remains is fp32 accumulation, one fp32
    rounding per tensor scale, the two bf16 roundings of Y and y (2 * 2^-9), and the
    rare silu(g)*u element on the other side of an E2M1 or UE4M3 rounding boundary.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_shifted_b200 import configs, zcmoe
from tests.gpu_harness import TOL, Run, row_rel_err, to_host_bits

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS
MEDIAN_TOL = 4e-3  # two bf16 roundings (Y, y): 2 * 2^-9


def _inputs(dtype, rows, cols):
    g = torch.Generator(device="cuda").manual_seed(rows * 7 + cols)
    x = torch.randn((rows, cols), generator=g, device="cuda", dtype=torch.float32)
    x *= torch.exp2(torch.randint(-12, 12, (rows, 1), generator=g, device="cuda").float())
    x[0, :16] = 0.0                      # an all-zero block
    x[0, 16:32] = 1e-39                  # a subnormal-only block
    x[0, 32] = 6.0                       # a block whose maximum is 6 * 1.0 exactly
    x[0, 48:64] = 2688.0                 # a block at the largest scale (448) under g = 1
    x[0, 64:80] = 5000.0                 # beyond it: saturates
    return x.to(dtype)


def _compare(got_c, got_s, ref_c, ref_s):
    assert np.array_equal(got_s, ref_s), np.argwhere(got_s != ref_s)[:5]
    bad = np.argwhere(got_c != ref_c)
    assert bad.size == 0, [(int(r), int(c), int(got_c[r, c]), int(ref_c[r, c])) for r, c in bad[:5]]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,cols", [(1, 256), (77, 512), (300, 768)])
@pytest.mark.parametrize("g", [1.0, 0.0123])
def test_quantizer_nv4_bitexact_given_scale(cuda_ok, dtype, rows, cols, g):
    x = _inputs(dtype, rows, cols)
    codes, scales, gout = zcmoe.quantize_nv4(x, global_scale=g)
    torch.cuda.synchronize()
    ref_c, ref_s = oracle.quantize_nv4(to_host_bits(x), np.float32(g))
    _compare(codes.cpu().numpy(), scales.cpu().numpy(), ref_c, ref_s)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,cols", [(1, 256), (300, 768), (2048, 1024)])
def test_quantizer_nv4_bitexact_derived_scale(cuda_ok, dtype, rows, cols):
    """global_scale 0: the weight rule, g = fl32(amax / 2688), then blocks under it."""
    x = _inputs(dtype, rows, cols)
    codes, scales, gout = zcmoe.quantize_nv4(x, global_scale=0.0)
    torch.cuda.synchronize()
    host = to_host_bits(x)
    ref_c, ref_s, ref_g = oracle.quantize_weight_nv4(host)
    assert np.float32(gout.item()).view(np.uint32) == np.float32(ref_g).view(np.uint32)
    _compare(codes.cpu().numpy(), scales.cpu().numpy(), ref_c, ref_s)


def test_quantizer_nv4_all_zero_tensor(cuda_ok):
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    codes, scales, gout = zcmoe.quantize_nv4(x, global_scale=0.0)
    torch.cuda.synchronize()
    assert gout.item() == 1.0
    assert (codes == 0).all() and (scales == 0x38).all()


def test_quantizer_nv4_rejects_bad_scale(cuda_ok):
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    for bad in (-1.0, float("nan"), float("inf")):
        with pytest.raises(zcmoe.ZcmoeError) as ei:
            zcmoe.quantize_nv4(x, global_scale=bad)
        assert ei.value.code == zcmoe.ZCMOE_EINVAL


def _check(r, pairs, rows):
    if r.P:
        assert r.check_expert_outputs(pairs) <= TOL["nvfp4"]
    r.check_layer_outputs(rows)


def _median_layer_err(r, rows):
    idx = r.dbg["idx"][rows]
    gate = r.dbg["gate"][rows].astype(np.float64)
    ref = oracle.layer_outputs(r.x_host(rows), idx, gate, r.w.n_ffn, r.expert_weights, nv4=True)
    err = row_rel_err(r.y[rows], ref)
    return float(np.median(err)), float(err.max())


def test_nvfp4_layer_small(cuda_ok):
    r = Run(W["small_nvfp4"])
    try:
        r.forward()
        r.check_routing_bitexact()
        rng = np.random.default_rng(1)
        pairs = np.unique(np.concatenate([[0, r.P - 1], rng.integers(0, r.P, 150)]))
        rows = np.unique(np.concatenate([[0, r.T - 1], rng.integers(0, r.T, 40)]))
        _check(r, pairs, rows)
        med, worst = _median_layer_err(r, rows)
        assert med <= MEDIAN_TOL and worst <= TOL["nvfp4"], (med, worst)
    finally:
        r.close()


@pytest.mark.parametrize("T,d,N,inter,Z,k", [
    (1, 512, 8, 256, 4, 3),        # one token
    (333, 512, 5, 256, 3, 4),      # ragged T
    (2000, 512, 3, 256, 1, 2),     # several row blocks per expert, partial last block
    (300, 1024, 9, 768, 0, 5),     # no zero experts; inter not a multiple of 512
])
def test_nvfp4_layer_ragged(cuda_ok, T, d, N, inter, Z, k):
    w = configs.Workload("ragged_nvfp4", T=T, d=d, n_ffn=N, inter=inter, n_zero=Z, top_k=k, dtype="nvfp4",
                         w_std=0.05, bias=("uniform", -0.05, 0.05), seed=3)
    r = Run(w, max_tokens=T + 5)
    try:
        r.forward()
        r.check_routing_bitexact()
        _check(r, range(r.P), np.arange(T))
        med, _ = _median_layer_err(r, np.arange(T))
        assert med <= MEDIAN_TOL, med
    finally:
        r.close()


def test_nvfp4_layer_prefill_full_size_sampled(cuda_ok):
    r = Run(W["prefill_560b_nvfp4"])
    try:
        r.forward()
        r.check_routing_bitexact()
        rng = np.random.default_rng(2)
        pairs = np.unique(np.concatenate([[0, r.P - 1], rng.integers(0, r.P, 24)]))
        rows = np.unique(np.concatenate([[0, r.T - 1], rng.integers(0, r.T, 6)]))
        _check(r, pairs, rows)
    finally:
        r.close()


def test_nvfp4_layer_decode_full_size(cuda_ok):
    r = Run(W["decode_560b_nvfp4"])
    try:
        r.forward()
        r.check_routing_bitexact()
        rng = np.random.default_rng(3)
        _check(r, np.unique(rng.integers(0, r.P, 30)), np.arange(0, r.T, 16))
    finally:
        r.close()


def test_nvfp4_against_bf16_and_mxfp4_layers(cuda_ok):
    """The quantization error of W4A4 NVFP4 on the same weights and tokens as the bf16
    layer: bounded and really 4-bit (the oracle's closeness pin gives the scale of it).
    The MXFP4 layer's error on the same inputs is printed beside it."""
    rb = Run(W["small_bf16"])
    try:
        rn = Run(W["small_nvfp4"], weights=rb.weights, x=rb.x)
        r4 = Run(W["small_fp4"], weights=rb.weights, x=rb.x)
        try:
            for r in (rb, rn, r4):
                r.forward()
            assert np.array_equal(rb.dbg["idx"], rn.dbg["idx"])

            def f64(y):
                return (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)

            yb = f64(rb.y)
            rel_n = np.abs(f64(rn.y) - yb).max(axis=1) / np.abs(yb).max(axis=1)
            rel_4 = np.abs(f64(r4.y) - yb).max(axis=1) / np.abs(yb).max(axis=1)
            print(f"median row error vs bf16: nvfp4 {np.median(rel_n):.4f}, mxfp4 {np.median(rel_4):.4f}")
            assert rel_n.max() < 0.5 and np.median(rel_n) < 0.25, (rel_n.max(), np.median(rel_n))
            assert np.median(rel_n) > 1e-2  # it really quantizes to 4 bits
        finally:
            rn.close()
            r4.close()
    finally:
        rb.close()
