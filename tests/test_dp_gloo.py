"""The data-parallel controller protocol with two gloo ranks on CPU.

Each rank routes its own batch (oracle routing stands in for the device
forward); the shared step sums the accumulators over the ranks, and every rank
must then hold the same bias, equal to one controller step on the union of
the batches."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from mixture_experts_layer_shifted_b200.dp import controller_step

N, Z, K = 16, 8, 4
E = N + Z
GAINS = dict(kp=0.1, ki=0.05, kd=0.2, decay=0.9, target_ffn_per_token=3.0)


class OracleReplica:
    """CPU replica with the ZcMoE accumulator interface, backed by the oracle."""

    def __init__(self, b0):
        self.b0 = np.asarray(b0, np.float32)
        self.state = oracle.new_controller_state(self.b0)
        self.counts = np.zeros(E, np.int64)
        self.tokens = np.zeros(1, np.int64)

    def forward(self, logits):
        idx, _, _ = oracle.route_replica_f32(logits.astype(np.float32), self.state["bias"], K)
        self.counts += np.bincount(idx.ravel(), minlength=E)
        self.tokens += logits.shape[0]

    def read_counts(self, buf):
        buf[:E] = torch.from_numpy(self.counts)
        buf[E] = int(self.tokens[0])

    def write_counts(self, buf):
        self.counts[:] = buf[:E].numpy()
        self.tokens[0] = int(buf[E])

    def update_bias(self, kp, ki, kd, decay, target_ffn_per_token):
        oracle.update_bias(self.counts, self.tokens, N, Z, K, (kp, ki, kd, decay, target_ffn_per_token), self.b0,
                           self.state)


def _batches(rank, step):
    rng = np.random.default_rng(1000 * step + rank)
    return rng.normal(size=(64 + 16 * rank, E)) * 1.5


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rep = OracleReplica(np.linspace(-0.01, 0.01, E))
        buf = torch.zeros(E + 1, dtype=torch.int64)
        for step in range(5):
            rep.forward(_batches(rank, step))
            controller_step(rep, buf, **GAINS)
        out[rank] = rep.state["bias"].copy()
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_two_rank_controller_matches_single_process():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    b0, b1 = out[0], out[1]
    np.testing.assert_array_equal(b0.view(np.uint32), b1.view(np.uint32))
    # single process over the union of the two ranks' batches
    rep = OracleReplica(np.linspace(-0.01, 0.01, E))
    for step in range(5):
        for r in range(world):
            rep.forward(_batches(r, step))
        rep.update_bias(**GAINS)
    np.testing.assert_array_equal(rep.state["bias"].view(np.uint32), b0.view(np.uint32))
