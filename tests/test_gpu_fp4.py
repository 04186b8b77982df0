"""GPU parity of the W4A4 experts (ZCMOE_FP4 layers: MXFP4, E2M1 codes with one E8M0
scale per 32 elements; zcmoe_quantize_mx4) through the C ABI.

A LongCat-Flash news page (gate.com post) reports W4A4 serving, expert weights
and activations in 4 bits, without naming the format; MXFP4 is the reading.

Tolerances (from the arithmetic):
  * quantizer: bit-exact codes and scales (decisions on exact values);
  * routing: bit-exact (the router is unchanged);
  * expert and layer outputs vs the MXFP4 oracle: max over rows of
    ||err||_inf / ||ref||_inf <= 2e-2 and median row <= 4e-3 -- the products of
    E2M1 codes and power-of-two scales are exact in fp32, so what remains is the
    two bf16 roundings of Y and y (2 * 2^-9), fp32 accumulation, and the rare
    silu(g)*u element on the other side of an E2M1 rounding boundary.
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


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rows,cols", [(1, 256), (77, 512), (300, 768)])
def test_quantizer_mx4_bitexact(cuda_ok, dtype, rows, cols):
    g = torch.Generator(device="cuda").manual_seed(rows * 5 + cols)
    x = torch.randn((rows, cols), generator=g, device="cuda", dtype=torch.float32)
    x *= torch.exp2(torch.randint(-20, 20, (rows, 1), generator=g, device="cuda").float())
    x[0, :32] = 0.0                      # an all-zero block
    x[0, 32:64] = 1e-39                  # a subnormal-only block
    x[0, 64] = 6.0                       # a block whose maximum is exactly representable
    x = x.to(dtype)
    codes, scales = zcmoe.quantize_mx4(x)
    torch.cuda.synchronize()
    ref_c, ref_s = oracle.quantize_mx4(to_host_bits(x))
    assert np.array_equal(scales.cpu().numpy(), ref_s)
    got_c = codes.cpu().numpy()
    bad = np.argwhere(got_c != ref_c)
    assert bad.size == 0, [(int(r), int(c), int(got_c[r, c]), int(ref_c[r, c])) for r, c in bad[:5]]


def _check(r, pairs, rows):
    if r.P:
        assert r.check_expert_outputs(pairs) <= TOL["fp4"]
    r.check_layer_outputs(rows)


def _median_layer_err(r, rows):
    idx = r.dbg["idx"][rows]
    gate = r.dbg["gate"][rows].astype(np.float64)
    ref = oracle.layer_outputs(r.x_host(rows), idx, gate, r.w.n_ffn, r.expert_weights, fp4=True)
    err = row_rel_err(r.y[rows], ref)
    return float(np.median(err)), float(err.max())


def test_fp4_layer_small(cuda_ok):
    r = Run(W["small_fp4"])
    try:
        r.forward()
        r.check_routing_bitexact()
        rng = np.random.default_rng(1)
        pairs = np.unique(np.concatenate([[0, r.P - 1], rng.integers(0, r.P, 150)]))
        rows = np.unique(np.concatenate([[0, r.T - 1], rng.integers(0, r.T, 40)]))
        _check(r, pairs, rows)
        med, worst = _median_layer_err(r, rows)
        assert med <= MEDIAN_TOL and worst <= TOL["fp4"], (med, worst)
    finally:
        r.close()


@pytest.mark.parametrize("T,d,N,inter,Z,k", [
    (1, 512, 8, 256, 4, 3),        # one token
    (333, 512, 5, 256, 3, 4),      # ragged T
    (2000, 512, 3, 256, 1, 2),     # several row blocks per expert, partial last block
    (300, 1024, 9, 768, 0, 5),     # no zero experts; inter not a multiple of 512
])
def test_fp4_layer_ragged(cuda_ok, T, d, N, inter, Z, k):
    w = configs.Workload("ragged_fp4", T=T, d=d, n_ffn=N, inter=inter, n_zero=Z, top_k=k, dtype="fp4", w_std=0.05,
                         bias=("uniform", -0.05, 0.05), seed=3)
    r = Run(w, max_tokens=T + 5)
    try:
        r.forward()
        r.check_routing_bitexact()
        _check(r, range(r.P), np.arange(T))
        med, _ = _median_layer_err(r, np.arange(T))
        assert med <= MEDIAN_TOL, med
    finally:
        r.close()


def test_fp4_layer_prefill_full_size_sampled(cuda_ok):
    r = Run(W["prefill_560b_fp4"])
    try:
        r.forward()
        r.check_routing_bitexact()
        rng = np.random.default_rng(2)
        pairs = np.unique(np.concatenate([[0, r.P - 1], rng.integers(0, r.P, 24)]))
        rows = np.unique(np.concatenate([[0, r.T - 1], rng.integers(0, r.T, 6)]))
        _check(r, pairs, rows)
    finally:
        r.close()


def test_fp4_layer_decode_full_size(cuda_ok):
    r = Run(W["decode_560b_fp4"])
    try:
        r.forward()
        r.check_routing_bitexact()
        rng = np.random.default_rng(3)
        _check(r, np.unique(rng.integers(0, r.P, 30)), np.arange(0, r.T, 16))
    finally:
        r.close()


def test_fp4_against_bf16_layer(cuda_ok):
    """The quantization error of W4A4 on the same weights and tokens: bounded (the oracle
    measures 14-32% of a row's largest value on random experts), and larger than FP8's."""
    rb = Run(W["small_bf16"])
    try:
        r4 = Run(W["small_fp4"], weights=rb.weights, x=rb.x)
        try:
            rb.forward()
            r4.forward()
            assert np.array_equal(rb.dbg["idx"], r4.dbg["idx"])
            yb = (rb.y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            y4 = (r4.y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            rel = np.abs(y4 - yb).max(axis=1) / np.abs(yb).max(axis=1)
            assert rel.max() < 0.5 and np.median(rel) < 0.25, (rel.max(), np.median(rel))
            assert np.median(rel) > 1e-2  # it really quantizes to 4 bits
        finally:
            r4.close()
    finally:
        rb.close()
