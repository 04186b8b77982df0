"""GPU parity of the block-scaled FP8 experts (ZCMOE_FP8 layers, zcmoe_quantize_e4m3)
through the C ABI.

LongCat-Flash technical summary (zhangjingwei.cn), 六 推理與部署 定制內核 "量化":
DeepSeek-V3's fine-grained blocks, one scale per [1,128] of activations and per
[128,128] of weights.

Tolerances (from the arithmetic):
  * quantizer: bit-exact codes and scales (every decision is taken on exact
    values: the block maximum of the inputs and a power-of-two rescaling);
  * routing: bit-exact as for bf16 layers (the router is unchanged);
  * expert and layer outputs vs the FP8 oracle (same quantization rules, fp64
    arithmetic on the dequantized operands): max over rows of
    ||err||_inf / ||ref||_inf <= 2e-2, and the median row <= 4e-3.  The FP8
    products are exact in fp32; what remains are the two bf16 roundings the path
    keeps (expert output Y and layer output y, each <= 2^-9 of a row's largest
    value, 3.9e-3 together), fp32 accumulation, and the rare silu(g)*u element
    whose fp32 value falls on the other side of an E4M3 rounding boundary than the
    oracle's (one code step, a fraction of a percent of the row).
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


# ---------------------------------------------------------------- quantizer

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("block_rows,rows,cols", [(1, 1, 128), (1, 77, 384), (128, 128, 256), (128, 300, 640)])
def test_quantizer_bitexact(cuda_ok, dtype, block_rows, rows, cols):
    g = torch.Generator(device="cuda").manual_seed(rows * 7 + cols)
    x = torch.randn((rows, cols), generator=g, device="cuda", dtype=torch.float32)
    # rows spanning many binades, a zero block, a subnormal-only block
    x *= torch.exp2(torch.randint(-20, 20, (rows, 1), generator=g, device="cuda").float())
    x[0, :128] = 0.0
    if rows > 1:
        x[1, 128:256] = 1e-39
    x = x.to(dtype)
    codes, scales = zcmoe.quantize_e4m3(x, block_rows)
    torch.cuda.synchronize()
    ref_c, ref_s = oracle.quantize_blocks(to_host_bits(x), block_rows)
    assert np.array_equal(scales.cpu().numpy(), ref_s)
    got_c = codes.cpu().numpy()
    bad = np.argwhere(got_c != ref_c)
    assert bad.size == 0, [(int(r), int(c), int(got_c[r, c]), int(ref_c[r, c])) for r, c in bad[:5]]


def test_quantizer_rejects_bad_arguments(cuda_ok):
    x = torch.zeros((4, 100), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(zcmoe.ZcmoeError) as ei:
        zcmoe.quantize_e4m3(x, 1)
    assert ei.value.code == zcmoe.ZCMOE_EINVAL
    y = torch.zeros((4, 128), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(zcmoe.ZcmoeError):
        zcmoe.quantize_e4m3(y, 64)


# ---------------------------------------------------------------- FP8 layers

def _check(r, pairs, rows):
    tol = TOL["fp8"]
    if r.P:
        byexp_err = r.check_expert_outputs(pairs)
        assert byexp_err <= tol
    r.check_layer_outputs(rows)


def _median_layer_err(r, rows):
    idx = r.dbg["idx"][rows]
    gate = r.dbg["gate"][rows].astype(np.float64)
    ref = oracle.layer_outputs(r.x_host(rows), idx, gate, r.w.n_ffn, r.expert_weights, fp8=True)
    err = row_rel_err(r.y[rows], ref)
    return float(np.median(err)), float(err.max())


def test_fp8_layer_small(cuda_ok):
    r = Run(W["small_fp8"])
    try:
        r.forward()
        r.check_routing_bitexact()
        rng = np.random.default_rng(1)
        pairs = np.unique(np.concatenate([[0, r.P - 1], rng.integers(0, r.P, 150)]))
        rows = np.unique(np.concatenate([[0, r.T - 1], rng.integers(0, r.T, 40)]))
        _check(r, pairs, rows)
        med, worst = _median_layer_err(r, rows)
        assert med <= MEDIAN_TOL and worst <= TOL["fp8"], (med, worst)
    finally:
        r.close()


@pytest.mark.parametrize("T,d,N,inter,Z,k", [
    (1, 512, 8, 128, 4, 3),        # one token
    (333, 512, 5, 256, 3, 4),      # ragged T, a few experts
    (2000, 512, 3, 128, 1, 2),     # > 128 pairs per expert: several row blocks, partial last block
    (300, 1024, 9, 384, 0, 5),     # no zero experts; inter not a multiple of 512
])
def test_fp8_layer_ragged(cuda_ok, T, d, N, inter, Z, k):
    w = configs.Workload("ragged_fp8", T=T, d=d, n_ffn=N, inter=inter, n_zero=Z, top_k=k, dtype="fp8", w_std=0.05,
                         bias=("uniform", -0.05, 0.05), seed=3)
    r = Run(w, max_tokens=T + 5)
    try:
        r.forward()
        r.check_routing_bitexact()
        _check(r, range(r.P), np.arange(T))
        med, worst = _median_layer_err(r, np.arange(T))
        assert med <= MEDIAN_TOL, med
    finally:
        r.close()


def test_fp8_layer_prefill_full_size_sampled(cuda_ok):
    """The 560B layer at the prefill batch: sampled pairs and tokens."""
    r = Run(W["prefill_560b_fp8"])
    try:
        r.forward()
        r.check_routing_bitexact()
        rng = np.random.default_rng(2)
        pairs = np.unique(np.concatenate([[0, r.P - 1], rng.integers(0, r.P, 24)]))
        rows = np.unique(np.concatenate([[0, r.T - 1], rng.integers(0, r.T, 6)]))
        _check(r, pairs, rows)
    finally:
        r.close()


def test_fp8_layer_decode_full_size(cuda_ok):
    r = Run(W["decode_560b_fp8"])
    try:
        r.forward()
        r.check_routing_bitexact()
        rng = np.random.default_rng(3)
        _check(r, np.unique(rng.integers(0, r.P, 30)), np.arange(0, r.T, 16))
    finally:
        r.close()


def test_fp8_against_bf16_layer(cuda_ok):
    """The quantization error of the method: the FP8 layer stays within a few percent
    of the bf16 layer on the same weights and tokens (same routing)."""
    wb, wf = W["small_bf16"], W["small_fp8"]
    rb = Run(wb)
    try:
        rf = Run(wf, weights=rb.weights, x=rb.x)
        try:
            rb.forward()
            rf.forward()
            assert np.array_equal(rb.dbg["idx"], rf.dbg["idx"])
            yb = (rb.y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            yf = (rf.y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            rel = np.abs(yf - yb).max(axis=1) / np.abs(yb).max(axis=1)
            assert rel.max() < 0.1 and np.median(rel) < 0.05, (rel.max(), np.median(rel))
            assert rel.max() > 1e-3  # the FP8 path really quantizes
        finally:
            rf.close()
    finally:
        rb.close()
