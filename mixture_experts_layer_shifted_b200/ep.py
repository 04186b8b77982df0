"""Expert-parallel forward of the layer: one process per GPU, the exchanges through
torch.distributed (NCCL all-to-all on GPUs).

LongCat-Flash technical summary (zhangjingwei.cn), 五 訓練基礎設施: the FFN layers
are partitioned by expert over an EP group, without tensor parallelism; the MoE
layer is split into two chunks along the token dimension so one chunk's
dispatch/combine traffic overlaps the other's computation.

Rank r holds FFN experts [r * n_local, (r + 1) * n_local).  Per chunk of tokens:
  1. dispatch: routing on the token's rank; the FFN pairs' rows in expert order, so
     the rows for rank r are one contiguous block (zero-expert picks stay local);
  2. exchange of the per-expert row counts, then of the rows (all-to-all);
  3. the local experts on the received rows (source-major rows, regrouped by
     expert inside the library);
  4. exchange of the outputs back (the reverse all-to-all);
  5. combine on the token's rank.
The counts must reach the host (the all-to-all split sizes), so each chunk syncs
twice; with two chunks, chunk 1's row exchange runs while chunk 0's experts
compute, and chunk 0's return exchange while chunk 1's experts compute.

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

    def dispatch(self, x):
        """-> (xsend [T*k, d], offsets as a host int64 array [n_ffn + 1]); syncs on the offsets."""
        T, s = x.shape[0], self.shape
        xsend = torch.empty((max(T * s.top_k, 1), s.d), dtype=x.dtype, device=x.device)
        off = torch.empty((s.n_ffn + 1,), dtype=torch.int32, device=x.device)
        zcmoe.zcmoe_ep_dispatch(self.layer.h, ctypes.c_void_p(x.data_ptr()), T, ctypes.c_void_p(xsend.data_ptr()),
                                ctypes.c_void_p(off.data_ptr()))
        return xsend, off.cpu().numpy().astype(np.int64)

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


def _exchange_counts(comm, send_counts, device):
    R, NL = send_counts.shape
    sc = torch.as_tensor(send_counts.reshape(-1), dtype=torch.int32).to(device)
    rc = torch.empty_like(sc)
    comm.all_to_all(rc, sc, [NL] * R, [NL] * R)
    return rc.cpu().numpy().astype(np.int64).reshape(R, NL)


def ep_forward(stages_per_chunk, comm, x, n_ffn: int):
    """y = layer(x) with the FFN experts spread over comm's ranks.  stages_per_chunk: one
    stage object per chunk (each keeps its chunk's routing until its combine); x is cut into
    that many contiguous token chunks."""
    R = comm.size
    if n_ffn % R:
        raise ValueError("n_ffn must be a multiple of the group size")
    NL = n_ffn // R
    nck = len(stages_per_chunk)
    T = x.shape[0]
    bounds = [T * i // nck for i in range(nck + 1)]
    chunks = [_Chunk(x[bounds[i]:bounds[i + 1]], st) for i, st in enumerate(stages_per_chunk)]
    # 1-2: dispatch and the row exchange, chunk after chunk (each row exchange asynchronous)
    for c in chunks:
        c.xsend, off = c.stages.dispatch(c.x)
        c.send_counts = np.diff(off).reshape(R, NL)
        c.send_rows = c.send_counts.sum(1)
        c.P = int(off[-1])
        c.recv_counts = _exchange_counts(comm, c.send_counts, c.x.device)
        c.recv_rows = c.recv_counts.sum(1)
        c.xrecv = c.x.new_empty((int(c.recv_rows.sum()), c.x.shape[1]))
        c.work = comm.all_to_all(c.xrecv, c.xsend[:c.P], c.recv_rows.tolist(), c.send_rows.tolist(), async_op=True)
    # 3-4: the local experts, each chunk's return exchange asynchronous
    for c in chunks:
        if c.work is not None:
            c.work.wait()
        c.yrecv = c.stages.experts(c.xrecv, c.recv_counts)
        c.yback = c.x.new_empty((c.P, c.x.shape[1]))
        c.work = comm.all_to_all(c.yback, c.yrecv, c.send_rows.tolist(), c.recv_rows.tolist(), async_op=True)
    # 5: combine
    ys = []
    for c in chunks:
        if c.work is not None:
            c.work.wait()
        ys.append(c.stages.combine(c.x, c.yback))
    return ys[0] if nck == 1 else torch.cat(ys, 0)


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

    def forward(self, x):
        return ep_forward(self.stages, self.comm, x, self.shape.n_ffn)

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
