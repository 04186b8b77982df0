"""The expert-parallel protocol (ep.ep_forward, EpMoE.controller_step) with gloo
ranks on CPU.

The stages run on the oracle here (the CUDA stages are exercised by the GPU tests):
each rank routes its own tokens in fp64, sends the FFN pairs' rows to the ranks that
hold their experts, runs the SwiGLU experts it holds on the rows it received, and
combines the rows that come back.  Every rank's output must equal the oracle's whole
layer on that rank's tokens with all experts in one place, whatever the group size,
the number of token chunks, or a rank with no tokens at all."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from mixture_experts_layer_shifted_b200.ep import TorchComm, ep_forward

D, N, Z, INTER, K = 64, 8, 4, 32, 3
E = N + Z


def _weights():
    rng = np.random.default_rng(7)
    f = lambda *s: (rng.standard_normal(s) * 0.1).astype(np.float32)  # noqa: E731
    return f(E, D), f(N, INTER, D), f(N, INTER, D), f(N, D, INTER), (rng.uniform(-0.05, 0.05, E)).astype(np.float32)


def _tokens(rank, T):
    return np.random.default_rng(100 + rank).standard_normal((T, D)).astype(np.float32)


def _route(x, wr, bias):
    s = oracle.softmax(oracle.router_logits(x, wr))
    idx, gate, _ = oracle.topk(s, bias.astype(np.float64), K)
    return idx, gate


class OracleStages:
    """dispatch / experts / combine on the CPU for rank `rank` of `size`."""

    def __init__(self, rank, size, weights):
        self.rank, self.size = rank, size
        self.wr, self.wg, self.wu, self.wd, self.bias = weights
        self.nl = N // size

    def dispatch(self, x, offsets_out, debug=None):
        xn = x.numpy()
        T = xn.shape[0]
        self.idx, self.gate = _route(xn, self.wr, self.bias) if T else (np.zeros((0, K), np.int32),
                                                                         np.zeros((0, K)))
        _, offsets, perm, pos = oracle.integer_stage(self.idx, N, E)
        self.pos = pos
        xsend = torch.from_numpy(np.ascontiguousarray(xn[perm // K])) if T else torch.zeros((0, D))
        offsets_out.copy_(torch.from_numpy(offsets.astype(np.int32)))
        return xsend

    def experts(self, xrecv, counts):
        # rows from the sources in rank order, each source's rows grouped by local expert
        xr = xrecv.numpy()
        y = np.zeros_like(xr)
        q = 0
        for s in range(self.size):
            for e in range(self.nl):
                n = int(counts[s, e])
                if n:
                    g = self.rank * self.nl + e
                    y[q:q + n] = oracle.ffn(xr[q:q + n], self.wg[g], self.wu[g], self.wd[g])
                q += n
        assert q == xr.shape[0]
        return torch.from_numpy(y)

    def combine(self, x, yback):
        xn, yb = x.numpy().astype(np.float64), yback.numpy().astype(np.float64)
        y = np.zeros_like(xn)
        for t in range(xn.shape[0]):
            for j in range(K):
                e = self.idx[t, j]
                y[t] += self.gate[t, j] * (yb[self.pos[t, j]] if e < N else xn[t])
        return torch.from_numpy(y.astype(np.float32))


def _worker(rank, world, port, sizes, chunks, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _weights()
        x = torch.from_numpy(_tokens(rank, sizes[rank]))
        stages = [OracleStages(rank, world, w) for _ in range(chunks)]
        y = ep_forward(stages, TorchComm(), x, N)
        out[rank] = y.numpy().copy()
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("world,sizes,chunks", [
    (2, (37, 50), 1),
    (2, (37, 50), 2),
    (4, (20, 0, 33, 9), 2),   # a rank with no tokens
    (2, (1, 6), 2),           # one token in two chunks: one chunk of that rank is empty
])
def test_ep_forward_matches_the_whole_layer(world, sizes, chunks):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), sizes, chunks, out), nprocs=world, join=True)
    wr, wg, wu, wd, bias = _weights()
    for r in range(world):
        got = out[r]
        assert got.shape == (sizes[r], D)
        if sizes[r] == 0:
            continue
        x = _tokens(r, sizes[r])
        idx, gate = _route(x, wr, bias)
        want = oracle.layer(x, idx, gate, N, wg, wu, wd)
        err = np.abs(got - want).max() / np.abs(want).max()
        assert err < 1e-6, (r, err)


class OracleControllerLayer:
    """Stands in for one chunk handle in EpMoE.controller_step: its accumulated counts
    and the oracle's controller state, on the CPU."""

    def __init__(self, counts, tokens, b0):
        self.acc = torch.tensor(list(counts) + [tokens], dtype=torch.int64)
        self.b0 = b0
        self.state = oracle.new_controller_state(b0)
        self.weights = (torch.zeros(1),)

    def read_counts(self, buf):
        buf.copy_(self.acc)

    def write_counts(self, buf):
        self.acc.copy_(buf)

    def update_bias(self, kp, ki, kd, decay, target_ffn_per_token):
        counts, tokens = self.acc[:-1].numpy().copy(), self.acc[-1:].numpy().copy()
        oracle.update_bias(counts, tokens, N, Z, K, (kp, ki, kd, decay, target_ffn_per_token), self.b0, self.state)
        self.acc.zero_()


GAINS = dict(kp=0.1, ki=0.05, kd=0.02, decay=0.95, target_ffn_per_token=2.0)


def _chunk_counts(rank, chunk):
    rng = np.random.default_rng(1000 + 10 * rank + chunk)
    T = 13 + 7 * rank + chunk
    return rng.multinomial(T * K, [1 / E] * E).astype(np.int64), T


def _ctl_worker(rank, world, port, out):
    from mixture_experts_layer_shifted_b200.ep import EpMoE
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b0 = np.linspace(-0.01, 0.01, E).astype(np.float32)
        layer = object.__new__(EpMoE)
        layer.shape = type("S", (), {"E": E})()
        layer.layers = [OracleControllerLayer(*_chunk_counts(rank, c), b0) for c in range(2)]
        layer.controller_step(all_reduce=lambda t: dist.all_reduce(t, op=dist.ReduceOp.SUM), **GAINS)
        out[rank] = [lay.state["bias"].copy() for lay in layer.layers]
    finally:
        dist.destroy_process_group()


def test_ep_controller_step_gives_every_handle_the_group_step():
    """Two gloo ranks with two chunk handles each: after EpMoE.controller_step every
    handle holds the bias of one controller that saw all four chunks' counts."""
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_ctl_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    total = np.zeros(E, np.int64)
    tokens = 0
    for r in range(world):
        for c in range(2):
            cnt, T = _chunk_counts(r, c)
            total += cnt
            tokens += T
    b0 = np.linspace(-0.01, 0.01, E).astype(np.float32)
    st = oracle.new_controller_state(b0)
    oracle.update_bias(total, np.array([tokens], np.int64), N, Z, K,
                       tuple(GAINS[k] for k in ("kp", "ki", "kd", "decay", "target_ffn_per_token")), b0, st)
    for r in range(world):
        for bias in out[r]:
            np.testing.assert_array_equal(bias.view(np.uint32), st["bias"].view(np.uint32))
