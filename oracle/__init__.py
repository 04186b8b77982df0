"""CPU oracle for the zero-computation-expert MoE layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only callers.  Nothing in the product
package imports this module, and this module imports nothing from the product.

The arithmetic lives in ``zcmoe_oracle.c`` (plain C, fp64, plus an fp32 replica
of the routing rule); this file builds it with gcc and wraps it with ctypes.
Python here only marshals arrays, except ``layer_outputs`` which sums the
per-expert fp64 results in numpy and ``brute_force_topk`` which enumerates
subsets with itertools (tiny inputs only).

Parity status: every function is pinned by tests under ``tests/`` (see
test_oracle_pins.py) except the bias controller's convergence rate, which is
"parity unpinned": the pages give no gains and no trajectory.
"""
from __future__ import annotations

import ctypes
import itertools
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zcmoe_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
_PREBUILT = False
_lib = None

F32P = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
F64P = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
I32P = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
I64P = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")


def compile_command(src: str, out: str) -> list:
    """gcc -O2 -ffp-contract=off, no fast-math, OpenMP: the one way the oracle is built."""
    return ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
            "-fvisibility=hidden", "-o", out, src, "-lm"]


def use_library(path: str) -> None:
    """Load the oracle from `path`, a library built elsewhere with compile_command.
    The pins' mutation test uses it to run the pins against deliberately broken
    copies of the source; nothing else calls it."""
    global _SO, _PREBUILT, _lib
    _SO, _PREBUILT, _lib = path, True, None


def build(force: bool = False) -> str:
    """Compile the oracle (nothing to do after use_library)."""
    if _PREBUILT:
        return _SO
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.run(compile_command(_SRC, _SO), check=True)
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        vp, i64, i32, f32, f64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
        L.zo_router_logits.argtypes = [vp, i32, vp, i32, vp, i64, i32, i32, F64P]
        L.zo_router_logits.restype = None
        L.zo_softmax_f64.argtypes = [F64P, i64, i32, F64P]
        L.zo_softmax_f64.restype = None
        L.zo_topk_f64.argtypes = [F64P, vp, i64, i32, i32, f64, I32P, F64P, vp]
        L.zo_topk_f64.restype = None
        L.zo_zexp.argtypes = [f32]
        L.zo_zexp.restype = f32
        L.zo_route_replica_f32.argtypes = [F32P, vp, i64, i32, i32, f32, vp, I32P, F32P]
        L.zo_route_replica_f32.restype = None
        L.zo_integer_stage.argtypes = [I32P, i64, i32, i32, i32, I32P, I32P, I32P, I32P]
        L.zo_integer_stage.restype = i64
        U8P = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
        L.zo_e4m3_encode.argtypes = [f32]
        L.zo_e4m3_encode.restype = ctypes.c_uint8
        L.zo_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.zo_e4m3_decode.restype = f64
        L.zo_e8m0_scale.argtypes = [f32]
        L.zo_e8m0_scale.restype = ctypes.c_uint8
        L.zo_quantize_blocks.argtypes = [vp, i32, i64, i64, i32, U8P, U8P]
        L.zo_quantize_blocks.restype = None
        L.zo_ffn_fp8_f64.argtypes = [vp, i32, i64, U8P, U8P, U8P, U8P, U8P, U8P, i32, i32, F64P]
        L.zo_ffn_fp8_f64.restype = None
        L.zo_e2m1_encode.argtypes = [f32]
        L.zo_e2m1_encode.restype = ctypes.c_uint8
        L.zo_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.zo_e2m1_decode.restype = f64
        L.zo_mx4_scale.argtypes = [f32]
        L.zo_mx4_scale.restype = ctypes.c_uint8
        L.zo_quantize_mx4.argtypes = [vp, i32, i64, i64, U8P, U8P]
        L.zo_quantize_mx4.restype = None
        L.zo_ffn_fp4_f64.argtypes = [vp, i32, i64, U8P, U8P, U8P, U8P, U8P, U8P, i32, i32, F64P]
        L.zo_ffn_fp4_f64.restype = None
        L.zo_nv4_global.argtypes = [f32]
        L.zo_nv4_global.restype = f32
        L.zo_nv4_scale.argtypes = [f32, f32]
        L.zo_nv4_scale.restype = ctypes.c_uint8
        L.zo_quantize_nv4.argtypes = [vp, i32, i64, i64, f32, U8P, U8P]
        L.zo_quantize_nv4.restype = None
        L.zo_ffn_nv4_f64.argtypes = [vp, i32, i64, U8P, U8P, f32, U8P, U8P, f32, U8P, U8P, f32, i32, i32, F64P]
        L.zo_ffn_nv4_f64.restype = None
        L.zo_layer_bwd_f64.argtypes = [vp, i32, i64, i32, i32, i32, i32, i32, vp, vp, vp, vp, i32, I32P, F64P, f64,
                                       F64P, F64P, vp, vp, vp, vp]
        L.zo_layer_bwd_f64.restype = None
        L.zo_ffn_f64.argtypes = [vp, i32, i64, vp, vp, vp, i32, i32, i32, F64P]
        L.zo_ffn_f64.restype = None
        L.zo_layer_f64.argtypes = [vp, i32, i64, I32P, F64P, i32, i32, vp, vp, vp, i32, i32, i32, F64P]
        L.zo_layer_f64.restype = None
        L.zo_update_bias.argtypes = [I64P, I64P, i32, i32, i32, f32, f32, f32, f32, f32, F32P, F32P, F32P,
                                     F32P, F32P]
        L.zo_update_bias.restype = None
        _lib = L
    return _lib


def _arr(a):
    """(pointer, dtype code) for a float32 array or a uint16 bf16-bits array."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return a, 1
    if a.dtype != np.float32:
        raise TypeError(f"oracle inputs are float32 or bf16 bits (uint16), got {a.dtype}")
    return a, 0


def router_logits(x, wr, offset=None):
    """fp64 logits l = x W_r^T + o.  x [T,d], wr [E,d] (float32 or bf16 bits)."""
    x, xd = _arr(x)
    wr, wd = _arr(wr)
    T, d = x.shape
    E = wr.shape[0]
    out = np.empty((T, E), dtype=np.float64)
    off = None if offset is None else np.ascontiguousarray(offset, dtype=np.float32)
    lib().zo_router_logits(x.ctypes.data, xd, wr.ctypes.data, wd, None if off is None else off.ctypes.data,
                           T, d, E, out)
    return out


def softmax(logits):
    l = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = l.shape
    out = np.empty_like(l)
    lib().zo_softmax_f64(l, T, E, out)
    return out


def topk(scores, bias, k, scale=1.0):
    """fp64 bias-shifted top-k.  Returns idx [T,k] int32, gate [T,k] f64, margin [T] f64."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    T, E = s.shape
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    idx = np.empty((T, k), dtype=np.int32)
    gate = np.empty((T, k), dtype=np.float64)
    margin = np.empty(T, dtype=np.float64)
    lib().zo_topk_f64(s, None if b is None else b.ctypes.data, T, E, k, float(scale), idx, gate, margin.ctypes.data)
    return idx, gate, margin


def zexp(x: float) -> float:
    return float(lib().zo_zexp(float(x)))


def route_replica_f32(logits_f32, bias_f32, k, scale=1.0, want_scores=False):
    """fp32 replica of the routing rule, fed fp32 logits.  Returns (idx, gate, scores|None)."""
    l = np.ascontiguousarray(logits_f32, dtype=np.float32)
    T, E = l.shape
    b = None if bias_f32 is None else np.ascontiguousarray(bias_f32, dtype=np.float32)
    idx = np.empty((T, k), dtype=np.int32)
    gate = np.empty((T, k), dtype=np.float32)
    scores = np.empty((T, E), dtype=np.float32) if want_scores else None
    lib().zo_route_replica_f32(l, None if b is None else b.ctypes.data, T, E, k, float(scale),
                               None if scores is None else scores.ctypes.data, idx, gate)
    return idx, gate, scores


def integer_stage(idx, N, E):
    """counts [E], offsets [N+1], perm [P] (entries t*k+j), pos [T,k] (-1 for zero slots)."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(N + 1, dtype=np.int32)
    perm = np.empty(max(T * k, 1), dtype=np.int32)
    pos = np.empty((T, k), dtype=np.int32)
    P = lib().zo_integer_stage(idx, T, k, N, E, counts, offsets, perm, pos)
    return counts, offsets, perm[:P].copy(), pos


def ffn(xs, wg, wu, wd):
    """fp64 SwiGLU expert on rows xs [n,d]; wg,wu [inter,d], wd [d,inter]."""
    xs, xd = _arr(xs)
    wg, gd = _arr(wg)
    wu, _ = _arr(wu)
    wd_, _ = _arr(wd)
    n, d = xs.shape
    inter = wg.shape[0]
    out = np.empty((n, d), dtype=np.float64)
    lib().zo_ffn_f64(xs.ctypes.data, xd, n, wg.ctypes.data, wu.ctypes.data, wd_.ctypes.data, gd, d, inter, out)
    return out


def layer(x, idx, gate, N, wg, wu, wd):
    """fp64 layer output for all tokens, all weights in memory."""
    x, xd = _arr(x)
    wg, gd = _arr(wg)
    wu, _ = _arr(wu)
    wd_, _ = _arr(wd)
    T, d = x.shape
    k = idx.shape[1]
    inter = wg.shape[1]
    y = np.empty((T, d), dtype=np.float64)
    lib().zo_layer_f64(x.ctypes.data, xd, T, np.ascontiguousarray(idx, dtype=np.int32),
                       np.ascontiguousarray(gate, dtype=np.float64), k, N, wg.ctypes.data, wu.ctypes.data,
                       wd_.ctypes.data, gd, d, inter, y)
    return y


def layer_outputs(x_rows, idx, gate, N, expert_weights, fp8=False, expert_fn=None, fp4=False, nv4=False):
    """fp64 layer output for a few tokens when the expert weights are fetched one
    expert at a time.  ``expert_weights(e) -> (wg, wu, wd)``.  Sums
    g * F_e(x) over the token's FFN slots plus (sum of zero-slot gates) * x.
    fp8: F_e is the block-scaled FP8 expert (ffn_fp8) on weights quantized here
    per [128,128].  fp4: the MXFP4 expert (ffn_fp4) on weights quantized here per
    [1,32].  nv4: the NVFP4 expert (ffn_nv4) on weights quantized here per [1,16]
    with one fp32 scale per matrix.  expert_fn(e, rows) -> F_e(rows), if given,
    replaces these."""
    x_rows = np.ascontiguousarray(x_rows)
    n, d = x_rows.shape
    xf = x_rows.astype(np.float64) if x_rows.dtype == np.float32 else \
        (x_rows.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    y = np.zeros((n, d), dtype=np.float64)
    zsum = np.zeros(n, dtype=np.float64)
    users = {}
    for r in range(n):
        for j in range(idx.shape[1]):
            e = int(idx[r, j])
            if e >= N:
                zsum[r] += float(gate[r, j])
            else:
                users.setdefault(e, []).append((r, j))
    for e in sorted(users):
        rows = [r for r, _ in users[e]]
        if expert_fn is not None:
            f = expert_fn(e, x_rows[rows])
            for i, (r, j) in enumerate(users[e]):
                y[r] += float(gate[r, j]) * f[i]
            continue
        wg, wu, wd = expert_weights(e)
        if nv4:
            q = [quantize_weight_nv4(w) for w in (wg, wu, wd)]
            f = ffn_nv4(x_rows[rows], [c for c, _, _ in q], [s_ for _, s_, _ in q], [g_ for _, _, g_ in q])
        elif fp4:
            q = [quantize_mx4(w) for w in (wg, wu, wd)]
            f = ffn_fp4(x_rows[rows], [c for c, _ in q], [s_ for _, s_ in q])
        elif fp8:
            q = [quantize_blocks(w, 128) for w in (wg, wu, wd)]
            f = ffn_fp8(x_rows[rows], [c for c, _ in q], [s_ for _, s_ in q])
        else:
            f = ffn(x_rows[rows], wg, wu, wd)
        for i, (r, j) in enumerate(users[e]):
            y[r] += float(gate[r, j]) * f[i]
    y += zsum[:, None] * xf
    return y


def update_bias(counts, tokens, N, Z, k, gains, b0, state):
    """One controller step in place.  counts int64 [E], tokens int64 [1];
    gains = (kp, ki, kd, decay, target_ffn); state = dict(eta [1], integ [E], eprev [E], bias [E])."""
    kp, ki, kd, decay, target = gains
    lib().zo_update_bias(counts, tokens, N, Z, k, kp, ki, kd, decay, target, np.ascontiguousarray(b0, np.float32),
                         state["eta"], state["integ"], state["eprev"], state["bias"])


def new_controller_state(b0):
    E = len(b0)
    return {"eta": np.ones(1, np.float32), "integ": np.zeros(E, np.float32), "eprev": np.zeros(E, np.float32),
            "bias": np.array(b0, dtype=np.float32)}


def brute_force_topk(v, k):
    """Enumerate all k-subsets of v (tiny E only); the chosen set maximises sum(v)
    with ties broken towards the lexicographically smaller sorted index tuple.
    Returns the indices ordered by v descending, then index ascending."""
    E = len(v)
    best, best_sum = None, None
    for comb in itertools.combinations(range(E), k):
        s = sum(float(v[i]) for i in comb)
        if best is None or s > best_sum:
            best, best_sum = comb, s
    return sorted(best, key=lambda i: (-float(v[i]), i))


# ----------------------------------------------------------------- block-scaled FP8
def e4m3_encode(v: float) -> int:
    """E4M3 code of v (round to nearest even, saturating at 448)."""
    return int(lib().zo_e4m3_encode(float(v)))


def e4m3_decode(code: int) -> float:
    return float(lib().zo_e4m3_decode(int(code)))


def e8m0_scale(amax: float) -> int:
    """E8M0 code of the smallest power of two s with amax <= 448 s (127 for amax 0)."""
    return int(lib().zo_e8m0_scale(float(amax)))


def quantize_blocks(src, block_rows):
    """(codes [rows, cols] uint8, scales [ceil(rows/block_rows), cols/128] uint8) of a
    2-D fp32 array or bf16 bit array; block_rows 1 or 128."""
    src, dt = _arr(src)
    rows, cols = src.shape
    if cols % 128:
        raise ValueError("cols must be a multiple of 128")
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty(((rows + block_rows - 1) // block_rows, cols // 128), np.uint8)
    lib().zo_quantize_blocks(src.ctypes.data, dt, rows, cols, block_rows, codes, scales)
    return codes, scales


def dequantize_blocks(codes, scales, block_rows):
    """fp64 values codes * 2^(scale - 127) (NaN codes give NaN)."""
    table = np.array([e4m3_decode(c) for c in range(256)], np.float64)
    rows, cols = codes.shape
    sc = np.repeat(np.repeat(scales.astype(np.int64) - 127, block_rows, 0)[:rows], 128, 1)
    return np.ldexp(table[codes], sc)


def ffn_fp8(xs, wq, sq):
    """fp64 SwiGLU expert on FP8 operands: xs [n, d] (fp32 or bf16 bits) quantized per
    [1,128] inside; wq = (wg, wu, wd) codes, sq = their [128,128] scales."""
    xs, xd = _arr(xs)
    n, d = xs.shape
    wg, wu, wd = (np.ascontiguousarray(w, np.uint8) for w in wq)
    sg, su, sd = (np.ascontiguousarray(s_, np.uint8) for s_ in sq)
    inter = wg.shape[0]
    out = np.empty((n, d), np.float64)
    lib().zo_ffn_fp8_f64(xs.ctypes.data, xd, n, wg, sg, wu, su, wd, sd, d, inter, out)
    return out


# ----------------------------------------------------------------- W4A4 (MXFP4)
def e2m1_encode(v: float) -> int:
    return int(lib().zo_e2m1_encode(float(v)))


def e2m1_decode(code: int) -> float:
    return float(lib().zo_e2m1_decode(int(code)))


def mx4_scale(amax: float) -> int:
    """E8M0 code of the smallest power of two s with amax <= 6 s (127 for amax 0)."""
    return int(lib().zo_mx4_scale(float(amax)))


def quantize_mx4(src):
    """(codes [rows, cols/2] uint8, two per byte with the even element low; scales
    [rows, cols/32] uint8) of a 2-D fp32 array or bf16 bit array."""
    src, dt = _arr(src)
    rows, cols = src.shape
    if cols % 32:
        raise ValueError("cols must be a multiple of 32")
    codes = np.empty((rows, cols // 2), np.uint8)
    scales = np.empty((rows, cols // 32), np.uint8)
    lib().zo_quantize_mx4(src.ctypes.data, dt, rows, cols, codes, scales)
    return codes, scales


def dequantize_mx4(codes, scales):
    table = np.array([e2m1_decode(c) for c in range(16)], np.float64)
    rows = codes.shape[0]
    nib = np.empty((rows, codes.shape[1] * 2), np.uint8)
    nib[:, 0::2] = codes & 0xF
    nib[:, 1::2] = codes >> 4
    return np.ldexp(table[nib], np.repeat(scales.astype(np.int64) - 127, 32, 1))


def ffn_fp4(xs, wq, sq):
    """fp64 SwiGLU expert on MXFP4 operands: xs [n, d] quantized per [1,32] inside;
    wq = (wg, wu, wd) packed codes, sq = their [1,32] scales."""
    xs, xd = _arr(xs)
    n, d = xs.shape
    wg, wu, wd = (np.ascontiguousarray(w, np.uint8) for w in wq)
    sg, su, sd = (np.ascontiguousarray(s_, np.uint8) for s_ in sq)
    inter = wg.shape[0]
    out = np.empty((n, d), np.float64)
    lib().zo_ffn_fp4_f64(xs.ctypes.data, xd, n, wg, sg, wu, su, wd, sd, d, inter, out)
    return out


# ----------------------------------------------------------------- W4A4 as NVFP4
def nv4_global(amax: float) -> float:
    """fp32 tensor scale of a weight matrix: fl32(amax / (6 * 448)), 1 for amax 0."""
    return float(lib().zo_nv4_global(float(amax)))


def nv4_scale(amax: float, g: float = 1.0) -> int:
    """UE4M3 code of the smallest block scale s with amax <= 6 s g (decided in fp32)."""
    return int(lib().zo_nv4_scale(float(amax), float(g)))


def quantize_nv4(src, g=1.0):
    """(codes [rows, cols/2] uint8, two per byte with the even element low; scales
    [rows, cols/16] uint8 UE4M3) of a 2-D fp32 array or bf16 bit array, tensor scale g."""
    src, dt = _arr(src)
    rows, cols = src.shape
    if cols % 16:
        raise ValueError("cols must be a multiple of 16")
    codes = np.empty((rows, cols // 2), np.uint8)
    scales = np.empty((rows, cols // 16), np.uint8)
    lib().zo_quantize_nv4(src.ctypes.data, dt, rows, cols, float(g), codes, scales)
    return codes, scales


def dequantize_nv4(codes, scales, g=1.0):
    table = np.array([e2m1_decode(c) for c in range(16)], np.float64)
    lo, hi = table[codes & 0xF], table[codes >> 4]
    vals = np.empty((codes.shape[0], codes.shape[1] * 2), np.float64)
    vals[:, 0::2], vals[:, 1::2] = lo, hi
    s = np.array([e4m3_decode(int(c)) for c in range(256)], np.float64)[scales]
    return vals * np.repeat(s, 16, axis=1) * float(g)


def quantize_weight_nv4(w):
    """A weight matrix's NVFP4 form: (codes, scales, g) with g from its largest magnitude."""
    w_arr, _ = _arr(w)
    vals = (w_arr.astype(np.uint32) << 16).view(np.float32) if w_arr.dtype == np.uint16 else w_arr
    g = nv4_global(float(np.abs(vals).max()) if vals.size else 0.0)
    codes, scales = quantize_nv4(w, g)
    return codes, scales, g


def ffn_nv4(xs, wq, sq, gq):
    """fp64 SwiGLU expert on NVFP4 operands: xs [n, d] quantized per [1,16] inside (g = 1);
    wq = (wg, wu, wd) packed codes, sq = their [1,16] UE4M3 scales, gq = their fp32 scales."""
    xs, xd = _arr(xs)
    n, d = xs.shape
    wg, wu, wd = (np.ascontiguousarray(w, np.uint8) for w in wq)
    sg, su, sd = (np.ascontiguousarray(s_, np.uint8) for s_ in sq)
    inter = wg.shape[0]
    out = np.empty((n, d), np.float64)
    lib().zo_ffn_nv4_f64(xs.ctypes.data, xd, n, wg, sg, float(gq[0]), wu, su, float(gq[1]), wd, sd, float(gq[2]),
                         d, inter, out)
    return out


# ----------------------------------------------------------------- backward (training)
def layer_backward(x, idx, scores, scale, dy, N, wr, wg, wu, wd, weights=True):
    """fp64 gradients of the layer for fixed routing: returns (dx [T,d], dW_r [E,d],
    dW_g [N,inter,d], dW_u [N,inter,d], dW_d [N,d,inter]); weights=False computes dx
    only (the others are None).  scores [T,E] are the forward's softmax scores; the
    bias and the logit offset get no gradient."""
    x, xd = _arr(x)
    wr, gd = _arr(wr)
    wg, _ = _arr(wg)
    wu, _ = _arr(wu)
    wd_, _ = _arr(wd)
    T, d = x.shape
    E = wr.shape[0]
    inter = wg.shape[1]
    k = idx.shape[1]
    dx = np.zeros((T, d))
    ws = [np.zeros((E, d)), np.zeros((N, inter, d)), np.zeros((N, inter, d)), np.zeros((N, d, inter))] if weights \
        else [None] * 4
    lib().zo_layer_bwd_f64(x.ctypes.data, xd, T, d, E, N, k, inter, wr.ctypes.data, wg.ctypes.data, wu.ctypes.data,
                           wd_.ctypes.data, gd, np.ascontiguousarray(idx, np.int32),
                           np.ascontiguousarray(scores, np.float64), float(scale),
                           np.ascontiguousarray(dy, np.float64), dx,
                           *[None if w_ is None else w_.ctypes.data for w_ in ws])
    return (dx, *ws)
