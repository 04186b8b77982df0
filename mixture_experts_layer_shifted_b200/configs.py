"""Named layer workloads and their seeded synthetic inputs.

Shapes follow the LongCat-Flash layer (technical summary, zhangjingwei.cn,
二 架構 / 模型配置: hidden 6144, expert width 2048, 512 FFN + 256 zero experts,
top-12) and smaller variants of it.  Inputs are generated on the device by the
seeded generator in ``synth`` (Philox4x32-10, Irwin-Hall normals), so any
element can be regenerated on the host.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import synth


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    n_ffn: int
    inter: int
    n_zero: int
    top_k: int
    dtype: str            # "f32", "bf16", "fp8", "fp4" or "nvfp4" (bf16 interface; FP8 / MXFP4 / NVFP4 experts)
    x_std: float = 1.0
    w_std: float = 0.02
    bias: tuple = ("zero",)   # ("zero",) | ("uniform", lo, hi) | ("zero_experts", value)
    zipf_s: float = 0.0       # > 0: router logits plus Zipf(s) expert offsets
    seed: int = 0
    steps: int = 1            # forward (+ bias update) steps of the workload
    target_ffn: float | None = None
    dense_inter: int = 0      # width of the dense FFN path run beside the layer (ScMoE); 0: none
    notes: str = ""

    @property
    def E(self):
        return self.n_ffn + self.n_zero

    def weight_bytes(self):
        esz = 4 if self.dtype == "f32" else 2  # the caller's weights (bf16 also for fp8 / fp4 / nvfp4 layers)
        return (3 * self.n_ffn * self.inter * self.d + self.E * self.d) * esz

    def with_(self, **kw):
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", T=64, d=256, n_ffn=16, inter=128, n_zero=8, top_k=4, dtype="f32",
                         w_std=0.02, bias=("uniform", -0.1, 0.1)),
    "small_bf16": Workload("small_bf16", T=4096, d=1024, n_ffn=64, inter=512, n_zero=32, top_k=8, dtype="bf16",
                           w_std=0.02, bias=("uniform", -0.2, 0.2), dense_inter=3072),
    "prefill_560b": Workload("prefill_560b", T=16384, d=6144, n_ffn=512, inter=2048, n_zero=256, top_k=12,
                             dtype="bf16", w_std=0.006, bias=("zero",), dense_inter=12288),
    "decode_560b": Workload("decode_560b", T=128, d=6144, n_ffn=512, inter=2048, n_zero=256, top_k=12, dtype="bf16",
                            w_std=0.006, bias=("zero",), dense_inter=12288,
                            notes="bias 0: uniform routing already sends 256/768 = 1/3 of picks to zero experts"),
    "decode_560b_zero_bias": Workload("decode_560b_zero_bias", T=128, d=6144, n_ffn=512, inter=2048, n_zero=256,
                                      top_k=12, dtype="bf16", w_std=0.006, bias=("zero_experts", 0.5),
                                      notes="literal +0.5 on zero experts: every pick is a zero expert"),
    "skewed_4096": Workload("skewed_4096", T=32768, d=4096, n_ffn=256, inter=1024, n_zero=128, top_k=8, dtype="bf16",
                            w_std=0.02, bias=("zero",), zipf_s=1.1, steps=100, target_ffn=6.0),
    # small case of the prefill kernels for profiler captures: a few GB on the device,
    # inputs still larger than L2
    "prefill_probe": Workload("prefill_probe", T=2048, d=6144, n_ffn=32, inter=2048, n_zero=16, top_k=12,
                              dtype="bf16", w_std=0.006, bias=("zero",), dense_inter=12288),
    # the prefill layer's per-expert shape at one eighth of its size (64 FFN + 32 zero experts,
    # 2048 tokens, top-12: ~256 rows per expert as at prefill; 4.8 GB of weights): profiler
    # captures of the expert GEMMs, whose traffic scales to prefill_560b by 8
    "prefill_probe256": Workload("prefill_probe256", T=2048, d=6144, n_ffn=64, inter=2048, n_zero=32, top_k=12,
                                 dtype="bf16", w_std=0.006, bias=("zero",)),
    # the 560B layer's expert shape with 16 experts (1.2 GB of weights): small captures of the
    # backward kernels, ~512 rows per expert as at prefill
    "bwd_probe": Workload("bwd_probe", T=1024, d=6144, n_ffn=16, inter=2048, n_zero=8, top_k=12, dtype="bf16",
                          w_std=0.006, bias=("zero",)),
}
# the same layers with block-scaled FP8 and W4A4 (MXFP4, NVFP4) experts
for _name in ("small_bf16", "prefill_560b", "decode_560b", "skewed_4096", "prefill_probe"):
    for _dt in ("fp8", "fp4", "nvfp4"):
        _n = _name.replace("_bf16", "") + "_" + _dt
        WORKLOADS[_n] = WORKLOADS[_name].with_(name=_n, dtype=_dt)


def bias_vector(w: Workload) -> np.ndarray:
    kind = w.bias[0]
    if kind == "zero":
        return np.zeros(w.E, np.float32)
    if kind == "uniform":
        return synth.uniform((w.E,), synth.TID_BIAS, w.seed, w.bias[1], w.bias[2])
    if kind == "zero_experts":
        b = np.zeros(w.E, np.float32)
        b[w.n_ffn:] = np.float32(w.bias[1])
        return b
    raise ValueError(kind)


def logit_offsets(w: Workload):
    return synth.zipf_logit_offsets(w.E, w.zipf_s, w.seed) if w.zipf_s > 0 else None


def device_weights(w: Workload, device="cuda"):
    """(w_router [E,d], w_gate [N,inter,d], w_up [N,inter,d], w_down [N,d,inter]) on the device."""
    import torch
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    shapes = [(w.E, w.d), (w.n_ffn, w.inter, w.d), (w.n_ffn, w.inter, w.d), (w.n_ffn, w.d, w.inter)]
    tids = [synth.TID_WR, synth.TID_WG, synth.TID_WU, synth.TID_WD]
    out = []
    for shp, tid in zip(shapes, tids):
        t = torch.empty(shp, dtype=dt, device=device)
        synth.fill_normal_(t, tid, w.seed, w.w_std)
        out.append(t)
    return tuple(out)


def device_dense_weights(w: Workload, device="cuda"):
    """(w_gate [I, d], w_up [I, d], w_down [d, I]) of the dense FFN path, I = w.dense_inter, bf16."""
    import torch
    if w.dense_inter <= 0:
        raise ValueError(f"workload {w.name} has no dense FFN path")
    shapes = [(w.dense_inter, w.d), (w.dense_inter, w.d), (w.d, w.dense_inter)]
    tids = [synth.TID_DENSE_G, synth.TID_DENSE_U, synth.TID_DENSE_D]
    out = []
    for shp, tid in zip(shapes, tids):
        t = torch.empty(shp, dtype=torch.bfloat16, device=device)
        synth.fill_normal_(t, tid, w.seed, w.w_std)
        out.append(t)
    return tuple(out)


def device_tokens(w: Workload, T: int | None = None, device="cuda", step: int = 0):
    """x [T, d] on the device; step > 0 gives a fresh batch of the same distribution."""
    import torch
    T = w.T if T is None else T
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    x = torch.empty((T, w.d), dtype=dt, device=device)
    synth.fill_normal_(x, synth.TID_X + 16 * step, w.seed, w.x_std)
    return x
