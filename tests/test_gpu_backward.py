"""GPU parity of the backward pass (zcmoe_backward) against the fp64 oracle backward.

LongCat-Flash technical summary (zhangjingwei.cn), 五 訓練基礎設施: fused GemmAdd for
the weight gradients, deterministic ScatterAdd for the input gradient.

The oracle is given the routing decisions the GPU took (which experts each token
picked; the routing tests check them bit for bit against the oracle's own) and
computes everything else itself in fp64: its own logits and softmax scores, the
expert activations, every gradient.

Tolerances (from the arithmetic): the GPU path rounds dY = g dy, H, dG, dU and the
router's dl to bf16 (relative 2^-9 each) and accumulates in fp32; every gradient
is a few such factors deep, so the error of a value is a few 2^-9 of the scale of
the terms it sums.  dx: max over tokens of ||err||_inf / ||ref||_inf <= 3e-2
(median 1e-2).  Weight gradients: the same bound per matrix (each expert's dW, and
dW_r), relative to the matrix's largest entry -- not per row, because a row of an
expert that saw one token is one outer product (e.g. da_i x) whose da_i can cancel
to 1e-5 of the matrix's scale while its rounding error stays at that scale.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_shifted_b200 import configs, zcmoe
from tests.gpu_harness import Run, row_rel_err, to_host_bits

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS
TOL, MEDIAN_TOL = 3e-2, 1e-2


def _bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _grads(w, init=0.0, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    shapes = {"router": (w.E, w.d), "gate": (w.n_ffn, w.inter, w.d), "up": (w.n_ffn, w.inter, w.d),
              "down": (w.n_ffn, w.d, w.inter)}
    return {k_: (torch.randn(s_, generator=g, device="cuda") * init) for k_, s_ in shapes.items()}


def _run_backward(r, dy, grads, accumulate=True):
    dx = r.layer.backward(r.x, dy, grads=grads, accumulate=accumulate)
    torch.cuda.synchronize()
    r.layer.check()
    return dx


def _oracle_backward(r, dy_host, rows=None, weights=True):
    T = r.T
    rows = np.arange(T) if rows is None else np.asarray(rows)
    x = r.x_host(rows)
    wr = r.router_host()
    l = oracle.router_logits(x, wr, r.offset)
    s = oracle.softmax(l)
    wg, wu, wd = (to_host_bits(t) for t in r.weights[1:])
    return oracle.layer_backward(x, r.dbg["idx"][rows], s, r.shape.routed_scale, dy_host[rows], r.w.n_ffn, wr, wg, wu,
                                 wd, weights=weights)


def _oracle_dx_sampled(r, dy_host, rows):
    """dx of a few tokens with only the experts they use copied to the host: the experts
    are renumbered (those used first; score columns and router rows permuted alike), which
    leaves dx unchanged."""
    rows = np.asarray(rows)
    x = r.x_host(rows)
    wr = r.router_host()
    s = oracle.softmax(oracle.router_logits(x, wr, r.offset))
    idx = r.dbg["idx"][rows]
    N, E = r.w.n_ffn, r.w.E
    used = sorted({int(e) for e in idx.ravel() if e < N})
    order = used + [e for e in range(E) if e not in set(used)]
    inv = np.empty(E, np.int64)
    inv[order] = np.arange(E)
    ws = [r.expert_weights(e) for e in used]
    wg, wu, wd = (np.stack([w_[i] for w_ in ws]) for i in range(3))
    dx, *_ = oracle.layer_backward(x, inv[idx].astype(np.int32), s[:, order], r.shape.routed_scale, dy_host[rows],
                                   len(used), wr[order], wg, wu, wd, weights=False)
    return dx


def _cmp(got, ref, name):
    """dx: one comparison per token row.  Weight gradients: one per matrix (each expert's
    matrix of a [N, rows, cols] gradient; the router's [E, d] as one matrix)."""
    if name == "dx":
        got2, ref2 = got, ref
    elif got.ndim == 3:
        got2, ref2 = got.reshape(got.shape[0], -1), ref.reshape(ref.shape[0], -1)
    else:
        got2, ref2 = got.reshape(1, -1), ref.reshape(1, -1)
    keep = np.abs(ref2).max(axis=1) > 0
    if (~keep).any():  # no contribution (an expert no token picked): nothing added
        assert np.abs(got2[~keep]).max() == 0.0, name
    err = row_rel_err(got2[keep], ref2[keep])
    assert float(err.max()) <= TOL and float(np.median(err)) <= MEDIAN_TOL, (name, float(err.max()),
                                                                             float(np.median(err)))
    return float(err.max())


def _case(w, T=None, init=0.5, saved=False, accumulate=True):
    r = Run(w, T=T, max_tokens=(T or w.T) + 3)
    try:
        if saved:
            r.layer.save_for_backward(True)
        r.forward()
        g = torch.Generator(device="cuda").manual_seed(5)
        dy = (torch.randn((r.T, w.d), generator=g, device="cuda") * 0.1).to(torch.bfloat16)
        grads = _grads(w, init)
        before = {k_: v.clone() for k_, v in grads.items()}
        dx = _run_backward(r, dy, grads, accumulate)
        ref = _oracle_backward(r, _bf16_to_f64(to_host_bits(dy)))
        _cmp(_bf16_to_f64(to_host_bits(dx)), ref[0], "dx")
        for name, i in (("router", 1), ("gate", 2), ("up", 3), ("down", 4)):
            # accumulate: what was added; overwrite: what is there (experts no token
            # picked must then hold exact zeros, whatever the accumulator held before)
            got = (grads[name] - before[name]) if accumulate else grads[name]
            _cmp(got.double().cpu().numpy(), ref[i], name)
        return r, dy
    except BaseException:
        r.close()
        raise


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
def test_backward_small(cuda_ok, saved):
    r, _ = _case(W["small_bf16"], saved=saved)
    r.close()


@pytest.mark.parametrize("T,N", [(600, 64), (1, 8)], ids=["600-tokens", "one-token"])
def test_backward_overwrite_mode(cuda_ok, T, N):
    """ZCMOE_GRAD_OVERWRITE: the gradients replace the accumulators' contents (non-zero
    before); with one token most experts get exact zeros."""
    w = W["small_bf16"] if T > 1 else configs.Workload("one_tok", T=1, d=256, n_ffn=N, inter=128, n_zero=4, top_k=3,
                                                       dtype="bf16", w_std=0.05, bias=("uniform", -0.05, 0.05),
                                                       seed=3)
    r, _ = _case(w, T=T, saved=True, accumulate=False)
    r.close()


@pytest.mark.parametrize("T,d,N,inter,Z,k", [
    (1, 256, 8, 128, 4, 3),        # one token
    (333, 320, 5, 192, 3, 4),      # ragged T; d and inter not multiples of the 256-wide tiles
    (2000, 256, 3, 128, 1, 2),     # several row blocks per expert, partial last block
    (300, 512, 9, 384, 0, 5),      # no zero experts
])
@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
def test_backward_ragged(cuda_ok, T, d, N, inter, Z, k, saved):
    w = configs.Workload("ragged_bwd", T=T, d=d, n_ffn=N, inter=inter, n_zero=Z, top_k=k, dtype="bf16", w_std=0.05,
                         bias=("uniform", -0.05, 0.05), seed=3)
    r, _ = _case(w, saved=saved)
    r.close()


@pytest.mark.parametrize("names", [("router",), ("gate", "down"), ("up",), ("gate", "up"), ()],
                         ids=["router-only", "gate+down", "up-only", "gate+up", "dx-only"])
def test_backward_gradient_subsets(cuda_ok, names):
    """Any subset of the weight gradients (NULL skips one): the requested ones are added,
    dx is unchanged.  dW_g and dW_u together come from one launch over [dG | dU] (two
    accumulators); either alone from a launch of its own."""
    w = W["small_bf16"]
    r = Run(w)
    try:
        r.layer.save_for_backward(True)
        r.forward()
        g = torch.Generator(device="cuda").manual_seed(5)
        dy = (torch.randn((r.T, w.d), generator=g, device="cuda") * 0.1).to(torch.bfloat16)
        grads = {k_: v for k_, v in _grads(w, 0.0).items() if k_ in names}
        dx = _run_backward(r, dy, grads)
        ref = _oracle_backward(r, _bf16_to_f64(to_host_bits(dy)))
        _cmp(_bf16_to_f64(to_host_bits(dx)), ref[0], "dx")
        for name, i in (("router", 1), ("gate", 2), ("up", 3), ("down", 4)):
            if name in grads:
                _cmp(grads[name].double().cpu().numpy(), ref[i], name)
    finally:
        r.close()


def test_saved_activations_leave_the_forward_unchanged(cuda_ok):
    """Training mode only adds stores: y is bit-identical with and without it, and
    switching it off again returns to the recomputing backward with the same results
    within rounding (the saved G and U are bf16, the recomputed ones fp32)."""
    w = W["small_bf16"]
    r = Run(w)
    try:
        y0 = r.layer.forward(r.x).clone()
        r.layer.save_for_backward(True)
        y1 = r.layer.forward(r.x).clone()
        torch.cuda.synchronize()
        assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
        dy = (torch.randn((r.T, w.d), device="cuda") * 0.1).to(torch.bfloat16)
        outs = []
        for on in (True, False):
            r.layer.save_for_backward(on)
            r.layer.forward(r.x)
            grads = _grads(w, 0.0)
            dx = _run_backward(r, dy, grads)
            outs.append((dx.float(), grads))
        (dx_s, g_s), (dx_r, g_r) = outs
        assert float((dx_s - dx_r).abs().max()) <= 2e-2 * float(dx_r.abs().max())
        for k_ in g_s:
            assert float((g_s[k_] - g_r[k_]).abs().max()) <= 2e-2 * float(g_r[k_].abs().max()), k_
    finally:
        r.close()


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
def test_backward_is_deterministic(cuda_ok, saved):
    """Two backward passes of the same forward give the same bits (no atomics anywhere)."""
    w = W["small_bf16"]
    r = Run(w)
    try:
        if saved:
            r.layer.save_for_backward(True)
        r.forward(debug=False)
        dy = (torch.randn((r.T, w.d), device="cuda") * 0.1).to(torch.bfloat16)
        outs = []
        for _ in range(2):
            grads = _grads(w, 0.0)
            dx = _run_backward(r, dy, grads)
            outs.append([dx.view(torch.int16)] + [grads[k_].view(torch.int32) for k_ in ("router", "gate", "up", "down")])
        assert all(torch.equal(a_, b_) for a_, b_ in zip(*outs))
    finally:
        r.close()


def test_backward_prefill_full_size_sampled_rows(cuda_ok):
    """The 560B layer at the prefill batch: dx of sampled tokens against the oracle (a
    token's dx depends only on its own routing); the weight gradients are exercised and
    must be finite (their exact values are checked at the smaller sizes above)."""
    w = W["prefill_560b"]
    r = Run(w)
    try:
        r.layer.save_for_backward(True)  # the configuration the bench times
        r.forward()
        dy = (torch.randn((r.T, w.d), device="cuda") * 0.05).to(torch.bfloat16)
        grads = {"router": torch.zeros((w.E, w.d), device="cuda"),
                 "down": torch.zeros((w.n_ffn, w.d, w.inter), device="cuda")}
        dx = _run_backward(r, dy, grads)
        rows = [0, 1, 4097, 9999, r.T - 1]
        ref = _oracle_dx_sampled(r, _bf16_to_f64(to_host_bits(dy)), rows)
        _cmp(_bf16_to_f64(to_host_bits(dx[torch.as_tensor(rows, device="cuda")])), ref, "dx")
        assert all(torch.isfinite(g_).all() for g_ in grads.values())
        assert grads["down"].abs().sum() > 0 and grads["router"].abs().sum() > 0
    finally:
        r.close()


def test_backward_argument_checks(cuda_ok):
    w = W["small_bf16"]
    r = Run(w)
    try:
        r.forward(debug=False)
        dy = torch.zeros_like(r.x)
        with pytest.raises(zcmoe.ZcmoeError) as ei:
            r.layer.backward(r.x[:-1], dy[:-1])   # T differs from the forward's
        assert ei.value.code == zcmoe.ZCMOE_EINVAL
        with pytest.raises(zcmoe.ZcmoeError) as ei:
            r.layer.backward(r.x, dy, dx=r.x)     # dx overlaps x
        assert ei.value.code == zcmoe.ZCMOE_EINVAL
    finally:
        r.close()
    f = Run(W["small_fp8"])
    try:
        f.forward(debug=False)
        with pytest.raises(zcmoe.ZcmoeError) as ei:
            f.layer.backward(f.x, torch.zeros_like(f.x))
        assert ei.value.code == zcmoe.ZCMOE_EUNSUPPORTED
        with pytest.raises(zcmoe.ZcmoeError) as ei:
            f.layer.save_for_backward(True)
        assert ei.value.code == zcmoe.ZCMOE_EUNSUPPORTED
    finally:
        f.close()
