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

import oracle
from mixture_experts_layer_shifted_b200 import configs, zcmoe
from mixture_experts_layer_shifted_b200.ep import CudaStages, EpMoE
from mixture_experts_layer_shifted_b200.zcmoe import LayerShape, ZcDense, ZcMoE
from tests.gpu_harness import TOL, row_rel_err, to_host_bits

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


def _chunk_debug(w, T):
    E, k = w.E, w.top_k
    f = lambda n, dt: torch.empty((max(n, 1),), dtype=dt, device="cuda")  # noqa: E731
    return {"logits": f(T * E, torch.float32), "scores": f(T * E, torch.float32), "idx": f(T * k, torch.int32),
            "gate": f(T * k, torch.float32), "counts": f(E, torch.int32), "offsets": f(w.n_ffn + 1, torch.int32),
            "perm": f(T * k, torch.int32), "pos": f(T * k, torch.int32)}


def _ep(w, weights, xs, size, chunks, max_recv_rows=None, debug=False):
    """Each rank's y; with debug, also each rank's per-chunk routing on the host:
    a list of (token range, {field: array}) per chunk."""
    shape = LayerShape(w.d, w.n_ffn, w.n_zero, w.inter, w.top_k, "bf16")
    wr, wg, wu, wd = weights
    NL = w.n_ffn // size

    def rank_fn(r, comm):
        sl = slice(r * NL, (r + 1) * NL)
        layer = EpMoE(shape, wr, wg[sl], wu[sl], wd[sl], max_tokens=max(max(x.shape[0] for x in xs), 1), comm=comm,
                      chunks=chunks, max_recv_rows=max_recv_rows, init_bias=configs.bias_vector(w),
                      logit_offset=configs.logit_offsets(w))
        try:
            T = xs[r].shape[0]
            bounds = layer.chunk_bounds(T)
            dbg = [_chunk_debug(w, b - a) for a, b in bounds] if debug else None
            y = layer.forward(xs[r], debug=dbg)
            torch.cuda.current_stream().synchronize()
            for lay in layer.layers:
                lay.check()
            if not debug:
                return y.clone()
            E, k = w.E, w.top_k
            routing = []
            for (a, b), dd in zip(bounds, dbg):
                n = b - a
                h = {"logits": dd["logits"][:n * E].view(n, E), "scores": dd["scores"][:n * E].view(n, E),
                     "idx": dd["idx"][:n * k].view(n, k), "gate": dd["gate"][:n * k].view(n, k),
                     "counts": dd["counts"], "offsets": dd["offsets"], "perm": dd["perm"][:n * k],
                     "pos": dd["pos"][:n * k].view(n, k)}
                routing.append(((a, b), {key: v.cpu().numpy() for key, v in h.items()}))
            return y.clone(), routing
        finally:
            layer.close()

    return _run_ranks(size, rank_fn)


def _check_ep_against_oracle(w, weights, xs, got, rows_per_rank=None, seed=0):
    """Each chunk's routing bit-exact against the oracle's fp32 replica fed the chunk's
    logits (and the integer stage on its picks); each rank's y on sampled tokens against
    the fp64 oracle driven by those picks, max row error <= 2e-2 of the row's max."""
    bias = configs.bias_vector(w)
    wr, wg, wu, wd = weights
    expert_weights = lambda e: (to_host_bits(wg[e]), to_host_bits(wu[e]), to_host_bits(wd[e]))  # noqa: E731
    rng = np.random.default_rng(seed)
    for r, (y, routing) in enumerate(got):
        idx_all = np.zeros((xs[r].shape[0], w.top_k), np.int32)
        gate_all = np.zeros((xs[r].shape[0], w.top_k), np.float32)
        for (a, b), d in routing:
            if b == a:
                continue
            idx, gate, scores = oracle.route_replica_f32(d["logits"], bias, w.top_k, 1.0, want_scores=True)
            np.testing.assert_array_equal(d["scores"].view(np.uint32), scores.view(np.uint32))
            np.testing.assert_array_equal(d["idx"], idx)
            np.testing.assert_array_equal(d["gate"].view(np.uint32), gate.view(np.uint32))
            counts, offsets, perm, pos = oracle.integer_stage(idx, w.n_ffn, w.E)
            np.testing.assert_array_equal(d["counts"], counts)
            np.testing.assert_array_equal(d["offsets"], offsets)
            np.testing.assert_array_equal(d["perm"][:int(offsets[-1])], perm)
            np.testing.assert_array_equal(d["pos"], pos)
            idx_all[a:b], gate_all[a:b] = idx, gate
        T = xs[r].shape[0]
        if T == 0:
            continue
        rows = np.arange(T) if rows_per_rank is None or rows_per_rank >= T else \
            np.sort(rng.choice(T, size=rows_per_rank, replace=False))
        x_rows = to_host_bits(xs[r][torch.as_tensor(rows, device="cuda", dtype=torch.long)])
        ref = oracle.layer_outputs(x_rows, idx_all[rows], gate_all[rows].astype(np.float64), w.n_ffn,
                                   expert_weights)
        err = row_rel_err(to_host_bits(y)[rows], ref)
        assert float(err.max()) <= TOL["bf16"], (r, float(err.max()))


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


@pytest.mark.parametrize("size,chunks", [(2, 2), (4, 2)])
def test_ep_against_the_oracle_small(cuda_ok, size, chunks):
    """Two and four emulated ranks: every chunk's routing bit-exact against the oracle's
    replica, every rank's every token against the fp64 oracle layer."""
    w = W["small_bf16"]
    sizes = [600 + 77 * r for r in range(size)]
    weights, xs = _layer_inputs(w, sizes)
    got = _ep(w, weights, xs, size, chunks, debug=True)
    _check_ep_against_oracle(w, weights, xs, got)


def test_ep_ragged_and_empty_ranks(cuda_ok):
    """Four ranks: one token, none, a ragged batch, and a batch whose routing leaves some
    experts empty on some sources."""
    w = configs.Workload("ep_ragged", T=300, d=512, n_ffn=8, inter=256, n_zero=4, top_k=3, dtype="bf16", w_std=0.05,
                         bias=("uniform", -0.05, 0.05), seed=4)
    sizes = [1, 0, 300, 57]
    weights, xs = _layer_inputs(w, sizes)
    ref = _reference(w, weights, xs)
    got = _ep(w, weights, xs, 4, 2, debug=True)
    for r in range(4):
        assert got[r][0].shape == ref[r].shape
        assert torch.equal(got[r][0].view(torch.int16), ref[r].view(torch.int16)), r
    _check_ep_against_oracle(w, weights, xs, got)


def test_ep_prefill_560b_eight_ranks(cuda_ok):
    """The 560B layer shape with its 512 FFN experts spread over eight emulated ranks
    (64 each), 2048 tokens per rank, two chunks."""
    w = W["prefill_560b"]
    sizes = [2048] * 8
    weights, xs = _layer_inputs(w, sizes)
    ref = _reference(w, weights, xs)
    got = _ep(w, weights, xs, 8, 2, max_recv_rows=40000, debug=True)
    for r in range(8):
        assert torch.equal(got[r][0].view(torch.int16), ref[r].view(torch.int16)), r
    # against the oracle: all 16 chunks' routing on every token, 24 sampled tokens per rank
    _check_ep_against_oracle(w, weights, xs, got, rows_per_rank=24, seed=8)


def test_ep_with_the_dense_ffn_alongside(cuda_ok):
    """The shortcut-connected dense FFN handed to the expert-parallel forward runs on its own
    stream while the exchanges and expert GEMMs are in flight: both outputs equal the
    sequential calls bit for bit, and the dense output matches the oracle's SwiGLU FFN."""
    w = W["small_bf16"]
    sizes = [700, 530]
    weights, xs = _layer_inputs(w, sizes)
    ref = _reference(w, weights, xs)
    shape = LayerShape(w.d, w.n_ffn, w.n_zero, w.inter, w.top_k, "bf16")
    wr, wg, wu, wd = weights
    NL = w.n_ffn // 2
    dw = list(configs.device_dense_weights(w))
    dense_ref = ZcDense(*dw, max_tokens=1024)
    try:
        want_dense = [dense_ref.forward(x).clone() for x in xs]
        torch.cuda.synchronize()
    finally:
        dense_ref.close()

    def rank_fn(r, comm):
        sl = slice(r * NL, (r + 1) * NL)
        layer = EpMoE(shape, wr, wg[sl], wu[sl], wd[sl], max_tokens=1024, comm=comm, chunks=2,
                      init_bias=configs.bias_vector(w))
        dense = ZcDense(*dw, max_tokens=1024)
        try:
            y, yd = layer.forward(xs[r], dense=dense)
            torch.cuda.current_stream().synchronize()
            dense.check()
            return y.clone(), yd.clone()
        finally:
            layer.close()
            dense.close()

    got = _run_ranks(2, rank_fn)
    for r in range(2):
        assert torch.equal(got[r][0].view(torch.int16), ref[r].view(torch.int16)), r
        assert torch.equal(got[r][1].view(torch.int16), want_dense[r].view(torch.int16)), r
        rows = np.arange(0, sizes[r], 37)
        x_rows = to_host_bits(xs[r][torch.as_tensor(rows, device="cuda")])
        want = oracle.ffn(x_rows, *(to_host_bits(t) for t in dw))
        err = row_rel_err(to_host_bits(got[r][1])[rows], want)
        assert float(err.max()) <= TOL["bf16"], float(err.max())


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
            xs = st.dispatch(x, torch.empty((w.n_ffn + 1,), dtype=torch.int32, device="cuda"))
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
