"""Expert parallelism on one GPU: the CUDA stages (zcmoe_ep_dispatch / experts /
combine) driven by ep.ep_forward, with the ranks of an EP group emulated by host
threads that exchange rows through host-side copies (each rank's kernels finish
before its rows are handed over, so no kernel waits on another rank's).

Every output row of the expert GEMMs depends only on its own input row, and the
combine sums each token's slots in slot order, so the expert-parallel layer must
give the same bits as one handle holding all experts, for every rank's tokens."""
import threading

import numpy as np
import pytest
import torch

from mixture_experts_layer_shifted_b200 import configs, zcmoe
from mixture_experts_layer_shifted_b200.ep import CudaStages, EpMoE
from mixture_experts_layer_shifted_b200.zcmoe import LayerShape, ZcMoE

pytestmark = pytest.mark.gpu


class _Group:
    def __init__(self, size):
        self.size = size
        self.slots = [None] * size
        self.barrier = threading.Barrier(size, timeout=300)


class ThreadComm:
    """all_to_all among threads: each rank publishes its input once its stream is done,
    then copies its blocks out of every rank's input."""

    def __init__(self, group, rank):
        self.group, self.rank, self.size = group, rank, group.size

    def all_to_all(self, out, inp, out_splits, in_splits, async_op=False):
        g = self.group
        torch.cuda.current_stream().synchronize()
        g.slots[self.rank] = (inp, [int(v) for v in in_splits])
        g.barrier.wait()
        o = 0
        for s in range(self.size):
            src, splits = g.slots[s]
            start, n = sum(splits[:self.rank]), splits[self.rank]
            assert n == int(out_splits[s])
            if n:
                out[o:o + n].copy_(src[start:start + n])
            o += n
        torch.cuda.current_stream().synchronize()
        g.barrier.wait()
        return None


def _run_ranks(size, fn):
    """fn(rank, comm) on `size` threads, each with its own stream; returns the results."""
    group = _Group(size)
    res, errs = [None] * size, []

    def body(r):
        try:
            torch.cuda.set_device(0)
            with torch.cuda.stream(torch.cuda.Stream()):
                res[r] = fn(r, ThreadComm(group, r))
                torch.cuda.current_stream().synchronize()
        except BaseException as e:  # noqa: BLE001
            errs.append(e)
            group.barrier.abort()

    ts = [threading.Thread(target=body, args=(r,)) for r in range(size)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    if errs:
        raise errs[0]
    return res


def _layer_inputs(w, sizes):
    weights = configs.device_weights(w)
    xs = [configs.device_tokens(w, max(T, 1), step=r)[:T] for r, T in enumerate(sizes)]
    return weights, xs


def _reference(w, weights, xs):
    shape = LayerShape(w.d, w.n_ffn, w.n_zero, w.inter, w.top_k, "bf16")
    ref = ZcMoE(shape, *weights, max_tokens=max(max(x.shape[0] for x in xs), 1), init_bias=configs.bias_vector(w),
                logit_offset=configs.logit_offsets(w))
    try:
        out = [ref.forward(x).clone() if x.shape[0] else x.clone() for x in xs]
        torch.cuda.synchronize()
        return out
    finally:
        ref.close()


def _ep(w, weights, xs, size, chunks, max_recv_rows=None):
    shape = LayerShape(w.d, w.n_ffn, w.n_zero, w.inter, w.top_k, "bf16")
    wr, wg, wu, wd = weights
    NL = w.n_ffn // size

    def rank_fn(r, comm):
        sl = slice(r * NL, (r + 1) * NL)
        layer = EpMoE(shape, wr, wg[sl], wu[sl], wd[sl], max_tokens=max(max(x.shape[0] for x in xs), 1), comm=comm,
                      chunks=chunks, max_recv_rows=max_recv_rows, init_bias=configs.bias_vector(w),
                      logit_offset=configs.logit_offsets(w))
        try:
            y = layer.forward(xs[r])
            torch.cuda.current_stream().synchronize()
            for lay in layer.layers:
                lay.check()
            return y.clone()
        finally:
            layer.close()

    return _run_ranks(size, rank_fn)


W = configs.WORKLOADS


@pytest.mark.parametrize("size,chunks", [(1, 1), (1, 2), (2, 1), (2, 2), (4, 2)])
def test_ep_equals_one_handle_small(cuda_ok, size, chunks):
    w = W["small_bf16"]
    sizes = [1000 + 77 * r for r in range(size)]
    weights, xs = _layer_inputs(w, sizes)
    ref = _reference(w, weights, xs)
    got = _ep(w, weights, xs, size, chunks)
    for r in range(size):
        assert torch.equal(got[r].view(torch.int16), ref[r].view(torch.int16)), r


def test_ep_ragged_and_empty_ranks(cuda_ok):
    """Four ranks: one token, none, a ragged batch, and a batch whose routing leaves some
    experts empty on some sources."""
    w = configs.Workload("ep_ragged", T=300, d=512, n_ffn=8, inter=256, n_zero=4, top_k=3, dtype="bf16", w_std=0.05,
                         bias=("uniform", -0.05, 0.05), seed=4)
    sizes = [1, 0, 300, 57]
    weights, xs = _layer_inputs(w, sizes)
    ref = _reference(w, weights, xs)
    got = _ep(w, weights, xs, 4, 2)
    for r in range(4):
        assert got[r].shape == ref[r].shape
        assert torch.equal(got[r].view(torch.int16), ref[r].view(torch.int16)), r


def test_ep_prefill_560b_eight_ranks(cuda_ok):
    """The 560B layer shape with its 512 FFN experts spread over eight emulated ranks
    (64 each), 2048 tokens per rank, two chunks."""
    w = W["prefill_560b"]
    sizes = [2048] * 8
    weights, xs = _layer_inputs(w, sizes)
    ref = _reference(w, weights, xs)
    got = _ep(w, weights, xs, 8, 2, max_recv_rows=40000)
    for r in range(8):
        assert torch.equal(got[r].view(torch.int16), ref[r].view(torch.int16)), r


def test_ep_argument_checks(cuda_ok):
    w = W["small_bf16"]
    shape = LayerShape(w.d, w.n_ffn, w.n_zero, w.inter, w.top_k, "bf16")
    wr, wg, wu, wd = configs.device_weights(w)
    NL = w.n_ffn // 2
    lay = ZcMoE(shape, wr, wg[:NL], wu[:NL], wd[:NL], max_tokens=64, ep_rank=0, ep_size=2, max_recv_rows=256)
    try:
        x = configs.device_tokens(w, 64)
        with pytest.raises(zcmoe.ZcmoeError) as ei:   # the whole forward needs every expert
            lay.forward(x)
        assert ei.value.code == zcmoe.ZCMOE_EUNSUPPORTED
        st = CudaStages(lay)
        cap = max(64 * w.top_k, 256)                  # rows one experts call may take
        xr = torch.zeros((cap + 8, w.d), dtype=torch.bfloat16, device="cuda")
        counts = np.zeros((2, NL), np.int32)
        counts[1, 3] = cap + 8
        with pytest.raises(zcmoe.ZcmoeError) as ei:   # more rows than the workspace holds
            st.experts(xr, counts)
        assert ei.value.code == zcmoe.ZCMOE_ERANGE
        with pytest.raises(zcmoe.ZcmoeError) as ei:   # counts that do not add up to the rows
            st.experts(xr[:10], np.ones((2, NL), np.int32))
        assert ei.value.code == zcmoe.ZCMOE_EINVAL
        with pytest.raises(zcmoe.ZcmoeError) as ei:   # combine of another T than the dispatch's
            xs, _ = st.dispatch(x)
            st.combine(x[:10], xs[:10])
        assert ei.value.code == zcmoe.ZCMOE_EINVAL
    finally:
        lay.close()
    n3 = w.n_ffn // 3
    with pytest.raises(zcmoe.ZcmoeError) as ei:       # n_ffn not a multiple of ep_size
        ZcMoE(shape, wr, wg[:n3], wu[:n3], wd[:n3], max_tokens=64, ep_rank=0, ep_size=3, max_recv_rows=256)
    assert ei.value.code == zcmoe.ZCMOE_EINVAL


def test_ep_controller_step_keeps_one_bias(cuda_ok):
    """Two chunk handles per rank and two ranks: after a shared controller step every handle
    holds the same bias as one handle that saw all the tokens."""
    w = W["small_bf16"]
    sizes = [512, 700]
    weights, xs = _layer_inputs(w, sizes)
    shape = LayerShape(w.d, w.n_ffn, w.n_zero, w.inter, w.top_k, "bf16")
    wr, wg, wu, wd = weights
    gains = dict(kp=0.0, ki=0.05, kd=0.0, decay=1.0, target_ffn_per_token=5.0)
    group_counts = [None, None]
    lock = threading.Lock()

    def rank_fn(r, comm):
        NL = w.n_ffn // 2
        sl = slice(r * NL, (r + 1) * NL)
        layer = EpMoE(shape, wr, wg[sl], wu[sl], wd[sl], max_tokens=1024, comm=comm, chunks=2,
                      init_bias=configs.bias_vector(w))
        try:
            layer.forward(xs[r])

            def all_reduce(t):  # the group sum, through the threads
                torch.cuda.current_stream().synchronize()
                with lock:
                    group_counts[r] = t.clone()
                comm.group.barrier.wait()
                t.copy_(group_counts[0] + group_counts[1])
                comm.group.barrier.wait()

            layer.controller_step(all_reduce=all_reduce, **gains)
            return [lay.state()["bias"] for lay in layer.layers]
        finally:
            layer.close()

    got = _run_ranks(2, rank_fn)
    ref = ZcMoE(shape, *weights, max_tokens=2048, init_bias=configs.bias_vector(w))
    try:
        ref.forward(torch.cat(xs, 0))
        ref.update_bias(**gains)
        want = ref.state()["bias"]
    finally:
        ref.close()
    for biases in got:
        for b in biases:
            np.testing.assert_array_equal(b.view(np.uint32), want.view(np.uint32))
