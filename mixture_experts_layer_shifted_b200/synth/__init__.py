"""Seeded synthetic inputs for the zero-computation-expert MoE layer.

This module is the one place that makes test and benchmark inputs.  It holds
none of the layer's arithmetic: only a counter-based random generator and the
recipes that turn its words into input tensors.  The same generator is written
twice, once here in numpy (any subset of indices, on the host) and once in
``synth.cu`` (whole tensors, on the device), and the two give bit-identical
values, so a host-side checker can regenerate or verify any element.

Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
as easy as 1, 2, 3", SC'11).  Element ``i`` of the tensor with id ``tid`` under
``seed`` uses counter blocks ``(lo32(i), hi32(i), tid, 0)`` and
``(lo32(i), hi32(i), tid, 1)`` with key ``(lo32(seed), hi32(seed))``.

Recipes (all exact or single-rounding in fp32, so host and device agree bit for bit):

* normal(std): Irwin-Hall sum of twelve 16-bit uniforms.  The twelve halves are
  words 0..3 of block 0 and words 0..1 of block 1, low half first.  With
  ``h`` the twelve 16-bit integers, ``z = (sum(h) - 393210) / 65536`` is exact
  in fp32 (mean 0, variance 1 - 2**-32 * ..., support [-6, 6]) and the value is
  ``fl32(z * std)``.
* uniform(a, b): ``u = (2 * (w0 >> 9) + 1) * 2**-24`` (exact, in (0, 1)), value
  ``fl32(a + fl32(fl32(b - a) * u))``.
* bf16 tensors round the fp32 value to nearest-even.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

# Philox4x32 round and key-schedule constants, from the SC'11 paper.
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
MASK32 = 0xFFFFFFFF

# Tensor ids used by the layer recipes.
TID_X = 1
TID_WR = 2
TID_WG = 3
TID_WU = 4
TID_WD = 5
TID_BIAS = 6
TID_ZIPF = 7
TID_DENSE_G = 8   # dense FFN path (ScMoE): W_gate, W_up, W_down
TID_DENSE_U = 9
TID_DENSE_D = 10


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10 on uint32 numpy arrays (or scalars)."""
    c0 = np.asarray(c0, dtype=np.uint64)
    c1 = np.asarray(c1, dtype=np.uint64)
    c2 = np.asarray(c2, dtype=np.uint64)
    c3 = np.asarray(c3, dtype=np.uint64)
    k0 = np.asarray(k0, dtype=np.uint64)
    k1 = np.asarray(k1, dtype=np.uint64)
    m0 = np.uint64(PHILOX_M0)
    m1 = np.uint64(PHILOX_M1)
    w0 = np.uint64(PHILOX_W0)
    w1 = np.uint64(PHILOX_W1)
    mask = np.uint64(MASK32)
    s32 = np.uint64(32)
    for r in range(10):
        if r:
            k0 = (k0 + w0) & mask
            k1 = (k1 + w1) & mask
        p0 = m0 * c0
        p1 = m1 * c2
        hi0, lo0 = p0 >> s32, p0 & mask
        hi1, lo1 = p1 >> s32, p1 & mask
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return (c0.astype(np.uint32), c1.astype(np.uint32),
            c2.astype(np.uint32), c3.astype(np.uint32))


def _blocks(idx, tid, seed, which):
    idx = np.asarray(idx, dtype=np.uint64)
    lo = idx & np.uint64(MASK32)
    hi = idx >> np.uint64(32)
    return philox4x32_10(lo, hi, np.full_like(lo, tid), np.full_like(lo, which),
                         seed & MASK32, (seed >> 32) & MASK32)


def normal_f32(idx, tid, seed, std):
    """fp32 values of the normal recipe at flat indices ``idx``."""
    a = _blocks(idx, tid, seed, 0)
    b = _blocks(idx, tid, seed, 1)
    s = np.zeros(np.shape(idx), dtype=np.int64)
    for w in (a[0], a[1], a[2], a[3], b[0], b[1]):
        w = w.astype(np.int64)
        s += (w & 0xFFFF) + (w >> 16)
    z = (s - 393210).astype(np.float32) / np.float32(65536.0)
    return (z * np.float32(std)).astype(np.float32)


def uniform_f32(idx, tid, seed, lo, hi):
    a = _blocks(idx, tid, seed, 0)
    u = ((a[0] >> np.uint32(9)).astype(np.int64) * 2 + 1).astype(np.float32) * np.float32(2.0 ** -24)
    span = np.float32(np.float32(hi) - np.float32(lo))
    return (np.float32(lo) + (span * u).astype(np.float32)).astype(np.float32)


def f32_to_bf16_bits(v):
    """Round fp32 to bf16 (nearest-even); returns uint16 bit patterns."""
    b = np.asarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = (b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal(shape, tid, seed, std, dtype="f32"):
    """Whole tensor on the host.  ``dtype`` 'f32' -> float32, 'bf16' -> uint16 bits."""
    n = int(np.prod(shape))
    v = normal_f32(np.arange(n, dtype=np.uint64), tid, seed, std).reshape(shape)
    return f32_to_bf16_bits(v) if dtype == "bf16" else v


def uniform(shape, tid, seed, lo, hi):
    n = int(np.prod(shape))
    return uniform_f32(np.arange(n, dtype=np.uint64), tid, seed, lo, hi).reshape(shape)


def zipf_logit_offsets(E, s=1.1, seed=0):
    """Skewed-routing prior: o_e = -s * ln(r_e), r_e in 1..E the rank of expert e
    under a seeded permutation (experts sorted by their Philox word, ties by id).
    Softmax of the offsets alone is proportional to rank**-s (Zipf)."""
    w = _blocks(np.arange(E, dtype=np.uint64), TID_ZIPF, seed, 0)[0].astype(np.int64)
    order = np.lexsort((np.arange(E), w))
    rank = np.empty(E, dtype=np.int64)
    rank[order] = np.arange(1, E + 1)
    return np.array([-s * math.log(r) for r in rank], dtype=np.float64).astype(np.float32)


# ---------------------------------------------------------------------------
# Device fill (libzcsynth.so).  Used by benchmarks and GPU tests to build large
# tensors in HBM without a host round trip.
# ---------------------------------------------------------------------------
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None


def device_lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(_HERE, "libzcsynth.so")
        if not os.path.exists(path):
            raise RuntimeError(f"device generator library missing: {path} (run __graft_entry__.build())")
        lib = ctypes.CDLL(path)
        lib.zcsynth_normal.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint32,
                                       ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p]
        lib.zcsynth_normal.restype = ctypes.c_int
        lib.zcsynth_uniform.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint32,
                                        ctypes.c_uint64, ctypes.c_float, ctypes.c_float, ctypes.c_void_p]
        lib.zcsynth_uniform.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def fill_normal_(tensor, tid, seed, std):
    """Fill a contiguous CUDA tensor (float32 or bfloat16) with the normal recipe."""
    import torch
    assert tensor.is_cuda and tensor.is_contiguous()
    bf16 = {torch.float32: 0, torch.bfloat16: 1}[tensor.dtype]
    stream = torch.cuda.current_stream(tensor.device).cuda_stream
    rc = device_lib().zcsynth_normal(tensor.data_ptr(), tensor.numel(), bf16, tid, seed, std, stream)
    if rc != 0:
        raise RuntimeError(f"zcsynth_normal failed ({rc})")
    return tensor


def fill_uniform_(tensor, tid, seed, lo, hi):
    import torch
    assert tensor.is_cuda and tensor.is_contiguous() and tensor.dtype == torch.float32
    stream = torch.cuda.current_stream(tensor.device).cuda_stream
    rc = device_lib().zcsynth_uniform(tensor.data_ptr(), tensor.numel(), tid, seed, lo, hi, stream)
    if rc != 0:
        raise RuntimeError(f"zcsynth_uniform failed ({rc})")
    return tensor
