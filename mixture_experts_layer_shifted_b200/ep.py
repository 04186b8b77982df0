"""Expert-parallel forward of the layer: one process per GPU, the exchanges through
torch.distributed (NCCL all-to-all on GPUs).

LongCat-Flash technical summary (zhangjingwei.cn), 五 訓練基礎設施: the FFN layers
are partitioned by expert over an EP group, without tensor parallelism; the MoE
layer is split into two chunks along the token dimension so one chunk's
dispatch/combine traffic overlaps the other's computation.

Rank r holds FFN experts [r * n_local, (r + 1) * n_local).  A forward:
  1. dispatch of every chunk: routing on the token's rank; the FFN pairs' rows in
     expert order, so the rows for rank r are one contiguous block (zero-expert
     picks stay local);
  2. ONE exchange of all chunks' per-expert row counts, read on the host with one
     synchronisation (the all-to-all split sizes);
  3. per chunk: the row exchange (asynchronous), the local experts on the received
     rows (source-major rows, regrouped by expert inside the library), and the
     return exchange (asynchronous), so chunk 1's rows move while chunk 0's experts
     compute and chunk 0's outputs return while chunk 1's experts compute;
  4. combine of every chunk on the token's rank.
The shortcut-connected dense FFN (same page, 二 part 2 "快捷連接 MoE": the dense
block's FFN runs while the MoE layer's dispatch and combine traffic is in flight)
can be handed to forward(): it is enqueued on its own stream right after the
dispatches, so it overlaps the exchanges and the expert GEMMs.

The stages are an object with dispatch / experts / combine (CudaStages: the C
ABI on device tensors) and the exchanges a communicator with all_to_all
(TorchComm: a torch.distributed process group), so the protocol is the same code
whatever carries it.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import zcmoe


class TorchComm:
    """all_to_all over a torch.distributed process group (async when asked)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.rank = dist.get_rank(group)
        self.size = dist.get_world_size(group)

    def all_to_all(self, out, inp, out_splits, in_splits, async_op=False):
        return self.dist.all_to_all_single(out, inp, list(out_splits), list(in_splits), group=self.group,
                                           async_op=async_op)


class LocalComm:
    """The one-rank group (every expert local): the exchanges are copies."""

    rank, size = 0, 1

    def all_to_all(self, out, inp, out_splits, in_splits, async_op=False):
        if out.numel():
            out.copy_(inp)
        return None


class CudaStages:
    """The three stages of one chunk through the C ABI; `layer` is a ZcMoE created with
    this rank's ep_rank / ep_size (its routing state belongs to this chunk)."""

    def __init__(self, layer: zcmoe.ZcMoE):
        self.layer = layer
        self.shape = layer.shape

    def dispatch(self, x, offsets, debug: dict | None = None):
        """-> xsend [T*k, d]; fills offsets ([n_ffn + 1] int32 on the device); no host sync.
        debug: zcmoe_debug field names -> device tensors that receive this chunk's routing."""
        T, s = x.shape[0], self.shape
        xsend = torch.empty((max(T * s.top_k, 1), s.d), dtype=x.dtype, device=x.device)
        dbg = zcmoe.zcmoe_debug(**{k_: v.data_ptr() for k_, v in debug.items()}) if debug else None
        zcmoe.zcmoe_ep_dispatch(self.layer.h, ctypes.c_void_p(x.data_ptr()), T, ctypes.c_void_p(xsend.data_ptr()),
                                ctypes.c_void_p(offsets.data_ptr()), dbg=dbg)
        return xsend

    def experts(self, xrecv, counts):
        """counts [ep_size, n_local] host ints -> yrecv (rows in xrecv's order)."""
        c = np.ascontiguousarray(counts, dtype=np.int32).reshape(-1)
        yrecv = torch.empty_like(xrecv)
        zcmoe.zcmoe_ep_experts(self.layer.h, ctypes.c_void_p(xrecv.data_ptr()), c.ctypes.data_as(ctypes.c_void_p),
                               xrecv.shape[0], ctypes.c_void_p(yrecv.data_ptr()))
        return yrecv

    def combine(self, x, yback):
        y = torch.empty_like(x)
        zcmoe.zcmoe_ep_combine(self.layer.h, ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(yback.data_ptr()),
                               x.shape[0], ctypes.c_void_p(y.data_ptr()))
        return y


class _Chunk:
    """Host state of one chunk between the stages."""

    def __init__(self, x, stages):
        self.x, self.stages = x, stages


def _exchange_counts(comm, offsets, R, NL):
    """offsets: [nck, n_ffn + 1] int32 on the device (each chunk's dispatch offsets).
    One all-to-all of every chunk's per-expert counts, then one host read of both sides:
    -> (send_counts [nck, R, NL], recv_counts [nck, R, NL], P [nck]) as host int64."""
    nck = offsets.shape[0]
    send = (offsets[:, 1:] - offsets[:, :-1]).reshape(nck, R, NL).transpose(0, 1).contiguous()  # [dst, chunk, e]
    recv = torch.empty_like(send)                                                                # [src, chunk, e]
    comm.all_to_all(recv.view(-1), send.view(-1), [nck * NL] * R, [nck * NL] * R)
    both = torch.cat([send.view(-1), recv.view(-1)]).cpu().numpy().astype(np.int64)
    half = R * nck * NL
    send_h = both[:half].reshape(R, nck, NL).transpose(1, 0, 2)
    recv_h = both[half:].reshape(R, nck, NL).transpose(1, 0, 2)
    return send_h, recv_h, send_h.sum(axis=(1, 2))


def ep_forward(stages_per_chunk, comm, x, n_ffn: int, dense=None, x_dense=None, y_dense=None, dense_stream=None,
               debug=None):
    """y = layer(x) with the FFN experts spread over comm's ranks.  stages_per_chunk: one
    stage object per chunk (each keeps its chunk's routing until its combine); x is cut into
    that many contiguous token chunks.  dense (optional, a ZcDense, CUDA only): y_dense =
    dense(x_dense) is enqueued on dense_stream after the dispatches and joined before
    returning, so it runs while the exchanges and the expert GEMMs are in flight.  debug
    (optional list, one dict per chunk): routing outputs of each chunk."""
    R = comm.size
    if n_ffn % R:
        raise ValueError("n_ffn must be a multiple of the group size")
    NL = n_ffn // R
    nck = len(stages_per_chunk)
    T = x.shape[0]
    bounds = [T * i // nck for i in range(nck + 1)]
    chunks = [_Chunk(x[bounds[i]:bounds[i + 1]], st) for i, st in enumerate(stages_per_chunk)]
    # 1: every chunk's routing and the copy of its FFN pairs' rows into expert order
    offs = torch.empty((nck, n_ffn + 1), dtype=torch.int32, device=x.device)
    for i, c in enumerate(chunks):
        c.xsend = c.stages.dispatch(c.x, offs[i], debug[i] if debug else None)
    # the dense FFN on its own stream, concurrent with everything below
    if dense is not None:
        main = torch.cuda.current_stream(x.device)
        dense_stream.wait_stream(main)
        y_dense = dense.forward(x_dense, y_dense, stream=dense_stream)
    # 2: one count exchange, one host sync
    send_counts, recv_counts, P = _exchange_counts(comm, offs, R, NL)
    for i, c in enumerate(chunks):
        c.send_rows = send_counts[i].sum(1)
        c.recv_counts = recv_counts[i]
        c.recv_rows = c.recv_counts.sum(1)
        c.P = int(P[i])
        c.xrecv = c.x.new_empty((int(c.recv_rows.sum()), c.x.shape[1]))
        c.work = comm.all_to_all(c.xrecv, c.xsend[:c.P], c.recv_rows.tolist(), c.send_rows.tolist(), async_op=True)
    # 3: the local experts, each chunk's return exchange asynchronous
    for c in chunks:
        if c.work is not None:
            c.work.wait()
        c.yrecv = c.stages.experts(c.xrecv, c.recv_counts)
        c.yback = c.x.new_empty((c.P, c.x.shape[1]))
        c.work = comm.all_to_all(c.yback, c.yrecv, c.send_rows.tolist(), c.recv_rows.tolist(), async_op=True)
    # 4: combine
    ys = []
    for c in chunks:
        if c.work is not None:
            c.work.wait()
        ys.append(c.stages.combine(c.x, c.yback))
    if dense is not None:
        main.wait_stream(dense_stream)
    y = ys[0] if nck == 1 else torch.cat(ys, 0)
    return (y, y_dense) if dense is not None else y


class EpMoE:
    """The layer on one rank of an expert-parallel group: `chunks` handles over the same
    (borrowed) weights, one per token chunk.  max_recv_rows bounds the rows one chunk may
    receive (default: the worst case, every token of every rank picking min(top_k, n_local)
    of this rank's experts; a tighter bound saves workspace, a chunk that exceeds it fails
    with ZCMOE_ERANGE)."""

    def __init__(self, shape: zcmoe.LayerShape, w_router, w_gate_local, w_up_local, w_down_local, max_tokens: int,
                 comm=None, chunks: int = 2, max_recv_rows: int | None = None, init_bias=None, logit_offset=None):
        self.comm = comm if comm is not None else TorchComm()
        self.shape = shape
        R = self.comm.size
        per_chunk = (max_tokens + chunks - 1) // chunks
        cap = max_recv_rows if max_recv_rows is not None else R * per_chunk * min(shape.top_k, shape.n_ffn // R)
        self.layers = [zcmoe.ZcMoE(shape, w_router, w_gate_local, w_up_local, w_down_local, max_tokens=per_chunk,
                                   init_bias=init_bias, logit_offset=logit_offset, ep_rank=self.comm.rank, ep_size=R,
                                   max_recv_rows=cap) for _ in range(chunks)]
        self.stages = [CudaStages(layer) for layer in self.layers]
        self.dense_stream = None

    def forward(self, x, dense=None, x_dense=None, y_dense=None, debug=None):
        """y, or (y, y_dense) when a dense FFN (ZcDense) is given: it runs on its own stream
        while this layer's exchanges and expert GEMMs are in flight (x_dense defaults to x).
        debug: a list of one dict per chunk (zcmoe_debug field names -> device tensors)."""
        if dense is not None:
            if x_dense is None:
                x_dense = x
            if self.dense_stream is None:
                self.dense_stream = torch.cuda.Stream(device=x.device)
        return ep_forward(self.stages, self.comm, x, self.shape.n_ffn, dense=dense, x_dense=x_dense,
                          y_dense=y_dense, dense_stream=self.dense_stream, debug=debug)

    def chunk_bounds(self, T):
        """The token ranges of the chunks a forward of T tokens is cut into."""
        n = len(self.stages)
        return [(T * i // n, T * (i + 1) // n) for i in range(n)]

    def controller_step(self, all_reduce=None, **gains):
        """One bias-controller step shared by the chunk handles and the group: the
        handles' accumulated counts are summed (and over the group by `all_reduce`, a
        function of one int64 device tensor, e.g. dist.all_reduce), written back into every
        handle, and each takes the same bit-exact step, so all biases stay identical."""
        E = self.shape.E
        dev = self.layers[0].weights[0].device
        bufs = [torch.empty(E + 1, dtype=torch.int64, device=dev) for _ in self.layers]
        for layer, b in zip(self.layers, bufs):
            layer.read_counts(b)
        total = torch.stack(bufs).sum(0)
        if all_reduce is not None:
            all_reduce(total)
        for layer in self.layers:
            layer.write_counts(total)
            layer.update_bias(**gains)

    def close(self):
        for layer in self.layers:
            layer.close()
