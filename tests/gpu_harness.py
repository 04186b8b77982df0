"""Shared helpers for the GPU parity tests: run the CUDA layer through the C ABI
(via the ctypes binding) with every debug output, and compare each stage with
the CPU oracle.

Tolerances (from the arithmetic; written in each check):
  * routing, counts, offsets, permutation, positions: bit-exact when the oracle's
    fp32 replica is fed the GPU's own fp32 logits;
  * fp64-routing comparison: indices equal on tokens whose k-th and (k+1)-th
    biased scores differ by at least 1e-5;
  * layer outputs and expert outputs: max over rows of ||err||_inf / ||ref||_inf
    <= 2e-2 (bf16 layers; FP8 / MXFP4 layers against their oracle) or 1e-4 (fp32 layer).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from mixture_experts_layer_shifted_b200 import configs, synth
from mixture_experts_layer_shifted_b200.zcmoe import LayerShape, ZcMoE

TOL = {"bf16": 2e-2, "f32": 1e-4, "fp8": 2e-2, "fp4": 2e-2, "nvfp4": 2e-2}
TIE_MARGIN = 1e-5


def to_host_bits(t):
    """Device tensor -> numpy (bf16 as uint16 bit patterns, fp32 as float32)."""
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return t.contiguous().cpu().numpy()


def as_f64(a):
    if a.dtype == np.uint16:
        return synth.bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def row_rel_err(got, ref):
    got = as_f64(got) if got.dtype != np.float64 else got
    num = np.abs(got - ref).max(axis=1)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return num / den


class Run:
    """One layer + one forward with all debug outputs, kept on the host."""

    def __init__(self, w: configs.Workload, T=None, bias=None, weights=None, x=None, max_tokens=None,
                 routed_scale=1.0):
        self.w = w
        self.T = w.T if T is None else T
        self.shape = LayerShape(w.d, w.n_ffn, w.n_zero, w.inter, w.top_k, w.dtype, routed_scale)
        self.weights = configs.device_weights(w) if weights is None else weights
        self.bias = configs.bias_vector(w) if bias is None else np.asarray(bias, np.float32)
        self.offset = configs.logit_offsets(w)
        self.layer = ZcMoE(self.shape, *self.weights, max_tokens=max_tokens or max(self.T, 1), init_bias=self.bias,
                           logit_offset=self.offset)
        self.x = configs.device_tokens(w, self.T) if x is None else x
        self.cur_bias = self.bias  # the bias the layer routes with now (changes with update_bias)

    def forward(self, debug=True):
        T, E, k, d = self.T, self.w.E, self.w.top_k, self.w.d
        dev = "cuda"
        dbg = None
        if debug:
            dbg = {
                "logits": torch.empty((T, E), dtype=torch.float32, device=dev),
                "scores": torch.empty((T, E), dtype=torch.float32, device=dev),
                "idx": torch.empty((T, k), dtype=torch.int32, device=dev),
                "gate": torch.empty((T, k), dtype=torch.float32, device=dev),
                "counts": torch.empty((E,), dtype=torch.int32, device=dev),
                "offsets": torch.empty((self.w.n_ffn + 1,), dtype=torch.int32, device=dev),
                "perm": torch.empty((T * k,), dtype=torch.int32, device=dev),
                "pos": torch.empty((T, k), dtype=torch.int32, device=dev),
                "expert_out": torch.empty((T * k, d), dtype=self.x.dtype, device=dev),
            }
        y = self.layer.forward(self.x, debug=dbg)
        torch.cuda.synchronize()
        self.layer.check()
        self.y_dev = y
        self.y = to_host_bits(y)
        if debug:
            self.dbg = {k_: to_host_bits(v) for k_, v in dbg.items() if k_ != "expert_out"}
            self.P = int(self.dbg["offsets"][-1])
            self.expert_out = to_host_bits(dbg["expert_out"][: self.P])
        return y

    # ---------------------------------------------------------------- inputs on the host
    def x_host(self, rows=None):
        x = self.x if rows is None else self.x[torch.as_tensor(rows, device="cuda", dtype=torch.long)]
        return to_host_bits(x)

    def expert_weights(self, e):
        _, wg, wu, wd = self.weights
        return to_host_bits(wg[e]), to_host_bits(wu[e]), to_host_bits(wd[e])

    def router_host(self):
        return to_host_bits(self.weights[0])

    # ---------------------------------------------------------------- checks
    def check_routing_bitexact(self):
        """Replica routing on the GPU's fp32 logits and the integer stage on the
        GPU's indices must reproduce every integer and every fp32 value."""
        d = self.dbg
        k = self.w.top_k
        idx, gate, scores = oracle.route_replica_f32(d["logits"], self.cur_bias, k, self.shape.routed_scale,
                                                     want_scores=True)
        np.testing.assert_array_equal(d["scores"].view(np.uint32), scores.view(np.uint32))
        np.testing.assert_array_equal(d["idx"], idx)
        np.testing.assert_array_equal(d["gate"].view(np.uint32), gate.view(np.uint32))
        counts, offsets, perm, pos = oracle.integer_stage(idx, self.w.n_ffn, self.w.E)
        np.testing.assert_array_equal(d["counts"], counts)
        np.testing.assert_array_equal(d["offsets"], offsets)
        np.testing.assert_array_equal(d["perm"][: self.P], perm)
        np.testing.assert_array_equal(d["pos"], pos)
        # invariants the pages fix: per-token FFN picks in [0, k]; every pick counted once
        ffn = (idx < self.w.n_ffn).sum(1)
        assert ffn.min() >= 0 and ffn.max() <= k
        assert counts.sum() == self.T * k

    def check_logits_and_fp64_routing(self, rows):
        """GPU logits vs fp64 logits on `rows`; fp64 routing vs GPU indices away from near-ties."""
        rows = np.asarray(rows)
        ref = oracle.router_logits(self.x_host(rows), self.router_host(), self.offset)
        got = self.dbg["logits"][rows].astype(np.float64)
        # fp32 accumulation of d exact products: |err| <= d * 2^-23 * sum|x||w| (loose bound)
        xs = np.abs(as_f64(self.x_host(rows)))
        ws = np.abs(as_f64(self.router_host()))
        bound = self.w.d * 2.0 ** -23 * (xs @ ws.T) + 1e-6
        assert np.all(np.abs(got - ref) <= bound)
        s = oracle.softmax(ref)
        idx, gate, margin = oracle.topk(s, self.cur_bias.astype(np.float64), self.w.top_k, self.shape.routed_scale)
        ok = margin >= TIE_MARGIN
        np.testing.assert_array_equal(self.dbg["idx"][rows][ok], idx[ok])
        np.testing.assert_allclose(self.dbg["gate"][rows][ok], gate[ok], rtol=1e-4, atol=1e-9)
        return ok.mean()

    def check_expert_outputs(self, pairs):
        """F_e(x_t) for sampled FFN pairs (rows of the permuted order) vs the fp64 oracle."""
        tol = TOL[self.w.dtype]
        perm = self.dbg["perm"]
        k = self.w.top_k
        byexp = {}
        for p in pairs:
            pair = int(perm[p])
            t, j = divmod(pair, k)
            byexp.setdefault(int(self.dbg["idx"][t, j]), []).append((p, t))
        worst = 0.0
        for e, lst in sorted(byexp.items()):
            wg, wu, wd = self.expert_weights(e)
            rows = [t for _, t in lst]
            if self.w.dtype == "nvfp4":
                q = [oracle.quantize_weight_nv4(w_) for w_ in (wg, wu, wd)]
                ref = oracle.ffn_nv4(self.x_host(rows), [c for c, _, _ in q], [s_ for _, s_, _ in q],
                                     [g_ for _, _, g_ in q])
            elif self.w.dtype == "fp4":
                q = [oracle.quantize_mx4(w_) for w_ in (wg, wu, wd)]
                ref = oracle.ffn_fp4(self.x_host(rows), [c for c, _ in q], [s_ for _, s_ in q])
            elif self.w.dtype == "fp8":
                q = [oracle.quantize_blocks(w_, 128) for w_ in (wg, wu, wd)]
                ref = oracle.ffn_fp8(self.x_host(rows), [c for c, _ in q], [s_ for _, s_ in q])
            else:
                ref = oracle.ffn(self.x_host(rows), wg, wu, wd)
            got = self.expert_out[[p for p, _ in lst]]
            err = row_rel_err(got, ref)
            worst = max(worst, float(err.max()))
        assert worst <= tol, worst
        return worst

    def check_layer_outputs(self, rows):
        """y on `rows` vs the fp64 oracle driven by the GPU's routing (all tokens compared)."""
        tol = TOL[self.w.dtype]
        rows = np.asarray(rows)
        idx = self.dbg["idx"][rows]
        gate = self.dbg["gate"][rows].astype(np.float64)
        ref = oracle.layer_outputs(self.x_host(rows), idx, gate, self.w.n_ffn, self.expert_weights,
                                   fp8=self.w.dtype == "fp8", fp4=self.w.dtype == "fp4",
                                   nv4=self.w.dtype == "nvfp4")
        err = row_rel_err(self.y[rows], ref)
        assert float(err.max()) <= tol, float(err.max())
        return float(err.max())

    def close(self):
        self.layer.close()
