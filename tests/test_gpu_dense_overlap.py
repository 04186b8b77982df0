"""GPU parity of the dense FFN path and of the shortcut-connected overlap
(zcmoe_dense_*, zcmoe_forward_overlap) through the C ABI.

LongCat-Flash technical summary (zhangjingwei.cn), 二 架構 part 2 "快捷連接 MoE"
and 模型配置 (dense path 12288 wide): the dense FFN of the preceding block and
the MoE layer do not depend on each other, so they may run at the same time.

Tolerances (from the arithmetic):
  * dense FFN vs the fp64 oracle's SwiGLU FFN: max over rows of
    ||err||_inf / ||ref||_inf <= 2e-2 (bf16 operands, fp32 accumulation, the
    SwiGLU product and the output each rounded once to bf16);
  * overlap vs the two calls one after the other: bit-identical outputs (the same
    deterministic kernels on the same inputs) and identical controller
    accumulators.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_shifted_b200 import configs, zcmoe
from mixture_experts_layer_shifted_b200.zcmoe import LayerShape, ZcDense, ZcMoE, forward_overlap
from tests.gpu_harness import TOL, row_rel_err, to_host_bits

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS


def _dense_workload(T, d, inter, seed=7):
    # only the dense fields matter; the MoE fields are a valid placeholder
    return configs.Workload("dense", T=T, d=d, n_ffn=1, inter=64, n_zero=0, top_k=1, dtype="bf16", w_std=0.05,
                            dense_inter=inter, seed=seed)


def _dense(w, max_tokens=None):
    wts = configs.device_dense_weights(w)
    return ZcDense(*wts, max_tokens=max_tokens or w.T), wts


def _bits(t):
    return t.contiguous().view(torch.int16)


def _check_dense(x, y, wts, rows):
    idx = torch.as_tensor(rows, device="cuda", dtype=torch.long)
    ref = oracle.ffn(to_host_bits(x[idx]), *[to_host_bits(t) for t in wts])
    err = row_rel_err(to_host_bits(y[idx]), ref)
    assert float(err.max()) <= TOL["bf16"], float(err.max())
    return float(err.max())


# ---------------------------------------------------------------- dense FFN

@pytest.mark.parametrize("T,d,inter", [
    (1, 128, 192),       # one token, one partial row block
    (129, 64, 64),       # one row past a full row block; the smallest widths
    (300, 256, 384),     # inter not a multiple of the 128-wide gate/up column tile
    (1000, 320, 448),    # d not a multiple of the 256-wide down column tile
])
def test_dense_ffn_small(cuda_ok, T, d, inter):
    w = _dense_workload(T, d, inter)
    dn, wts = _dense(w)
    try:
        x = configs.device_tokens(w)
        y = dn.forward(x)
        torch.cuda.synchronize()
        dn.check()
        _check_dense(x, y, wts, np.arange(T))
    finally:
        dn.close()


def test_dense_ffn_full_size_sampled_rows(cuda_ok):
    """The 12288-wide dense path on the prefill batch (16384 x 6144), rows
    sampled across the first, middle and last row blocks."""
    w = W["prefill_560b"]
    dn, wts = _dense(w)
    try:
        x = configs.device_tokens(w)
        y = dn.forward(x)
        torch.cuda.synchronize()
        dn.check()
        _check_dense(x, y, wts, [0, 1, 127, 128, 8191, 12345, w.T - 1])
    finally:
        dn.close()


def test_dense_ffn_rows_are_independent_of_the_batch(cuda_ok):
    """A token's output does not depend on the other tokens of the batch or on T:
    the first 77 rows of a 1000-token batch equal a 77-token batch bit for bit."""
    w = _dense_workload(1000, 256, 384)
    dn, _ = _dense(w)
    try:
        x = configs.device_tokens(w)
        y_all = dn.forward(x)
        y_head = dn.forward(x[:77].clone())
        torch.cuda.synchronize()
        assert torch.equal(_bits(y_all[:77]), _bits(y_head))
    finally:
        dn.close()


# ---------------------------------------------------------------- overlap

def _moe(w, T, weights):
    shape = LayerShape(w.d, w.n_ffn, w.n_zero, w.inter, w.top_k, w.dtype)
    return ZcMoE(shape, *weights, max_tokens=T, init_bias=configs.bias_vector(w),
                 logit_offset=configs.logit_offsets(w))


def _overlap_case(w, same_x, T=None):
    """Two MoE handles on the same weights: one runs zcmoe_forward then the dense
    FFN, the other zcmoe_forward_overlap; everything must agree bit for bit."""
    T = w.T if T is None else T
    weights = configs.device_weights(w)
    seq, ovl = _moe(w, T, weights), _moe(w, T, weights)
    dn, _ = _dense(w, T)
    try:
        x = configs.device_tokens(w, T)
        xd = x if same_x else configs.device_tokens(w, T, step=1)
        y_seq = seq.forward(x)
        yd_seq = dn.forward(xd)
        y_ovl, yd_ovl = forward_overlap(ovl, dn, x, xd)
        torch.cuda.synchronize()
        seq.check()
        ovl.check()
        dn.check()
        assert torch.equal(_bits(y_seq), _bits(y_ovl))
        assert torch.equal(_bits(yd_seq), _bits(yd_ovl))
        a, b = seq.state(), ovl.state()
        assert np.array_equal(a["counts"], b["counts"]) and a["tokens"] == b["tokens"] == T
        return y_ovl, yd_ovl
    finally:
        seq.close()
        ovl.close()
        dn.close()


@pytest.mark.parametrize("same_x", [True, False])
def test_overlap_bitexact_small(cuda_ok, same_x):
    _overlap_case(W["small_bf16"], same_x)


@pytest.mark.parametrize("T", [1, 333])
def test_overlap_bitexact_ragged(cuda_ok, T):
    _overlap_case(W["small_bf16"], False, T=T)


def test_overlap_bitexact_prefill_full_size(cuda_ok):
    """The 560B layer at the prefill batch beside its 12288-wide dense path."""
    _overlap_case(W["prefill_560b"], True)


def test_overlap_in_a_cuda_graph(cuda_ok):
    """The overlap captured on one stream (the dense FFN forked onto the dense
    handle's stream and joined back) replays to the same bits as the plain calls."""
    w = W["small_bf16"]
    weights = configs.device_weights(w)
    seq, ovl = _moe(w, w.T, weights), _moe(w, w.T, weights)
    dn, _ = _dense(w)
    try:
        x = configs.device_tokens(w)
        y_seq = seq.forward(x)
        yd_seq = dn.forward(x)
        y_ovl, yd_ovl = torch.empty_like(x), torch.empty_like(x)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            forward_overlap(ovl, dn, x, y_moe=y_ovl, y_dense=yd_ovl)  # first call outside the capture
        torch.cuda.synchronize()
        y_ovl.zero_()
        yd_ovl.zero_()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            forward_overlap(ovl, dn, x, y_moe=y_ovl, y_dense=yd_ovl)
        g.replay()
        torch.cuda.synchronize()
        ovl.check()
        dn.check()
        assert torch.equal(_bits(y_seq), _bits(y_ovl))
        assert torch.equal(_bits(yd_seq), _bits(yd_ovl))
        del g
    finally:
        seq.close()
        ovl.close()
        dn.close()


def test_overlap_argument_checks(cuda_ok):
    w = W["small_bf16"]
    weights = configs.device_weights(w)
    moe = _moe(w, w.T, weights)
    dn, _ = _dense(w)
    small_dn, _ = _dense(w, max_tokens=w.T - 1)
    other_d, _ = _dense(_dense_workload(w.T, 512, 256))
    f32 = W["tiny_f32"]
    f32_moe = ZcMoE(LayerShape(f32.d, f32.n_ffn, f32.n_zero, f32.inter, f32.top_k, f32.dtype),
                    *configs.device_weights(f32), max_tokens=w.T)
    f32_dn, _ = _dense(_dense_workload(w.T, f32.d, 128))
    x = configs.device_tokens(w)
    y = torch.empty_like(x)
    yd = torch.empty_like(x)
    try:
        def code(fn):
            with pytest.raises(zcmoe.ZcmoeError) as ei:
                fn()
            return ei.value.code

        assert code(lambda: forward_overlap(moe, other_d, x, y_moe=y, y_dense=yd)) == zcmoe.ZCMOE_EINVAL
        assert code(lambda: forward_overlap(moe, small_dn, x, y_moe=y, y_dense=yd)) == zcmoe.ZCMOE_ERANGE
        assert code(lambda: forward_overlap(moe, dn, x, y_moe=y, y_dense=y)) == zcmoe.ZCMOE_EINVAL
        assert code(lambda: forward_overlap(moe, dn, x, y_moe=x, y_dense=yd)) == zcmoe.ZCMOE_EINVAL
        assert code(lambda: forward_overlap(moe, dn, x, y_moe=y, y_dense=x)) == zcmoe.ZCMOE_EINVAL
        xf = configs.device_tokens(f32, w.T)
        assert code(lambda: forward_overlap(f32_moe, f32_dn, xf, y_moe=torch.empty_like(xf),
                                            y_dense=torch.empty_like(xf))) == zcmoe.ZCMOE_EUNSUPPORTED
        # nothing was enqueued by the refused calls; a valid call still works
        forward_overlap(moe, dn, x, y_moe=y, y_dense=yd)
        torch.cuda.synchronize()
        moe.check()
        dn.check()
        closed = ZcDense(*configs.device_dense_weights(w), max_tokens=8)
        closed.close()
        assert code(lambda: forward_overlap(moe, closed, x, y_moe=y, y_dense=yd)) == zcmoe.ZCMOE_EINVAL
    finally:
        for o in (moe, dn, small_dn, other_d, f32_moe, f32_dn):
            o.close()
