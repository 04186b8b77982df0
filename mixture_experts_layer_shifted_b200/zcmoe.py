"""ctypes binding of libzcmoe.so (C ABI in include/zcmoe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and streams.  There is no fallback:
if the library is missing or the device is not an sm_100 part, calls fail.

The functions carry the C names; ``ZcMoE`` is a small owner object that keeps
the weight tensors alive for the handle's lifetime.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch  # noqa: F401  (loads the CUDA runtime the library links against)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzcmoe.so")

ZCMOE_OK = 0
ZCMOE_EINVAL = -1
ZCMOE_ERANGE = -2
ZCMOE_ENOMEM = -3
ZCMOE_ECUDA = -4
ZCMOE_EUNSUPPORTED = -5
ZCMOE_ETIMEOUT = -6
ZCMOE_F32 = 0
ZCMOE_BF16 = 1
ZCMOE_FP8 = 2
ZCMOE_FP4 = 3
ZCMOE_NVFP4 = 4
_DTYPES = {"f32": ZCMOE_F32, "bf16": ZCMOE_BF16, "fp8": ZCMOE_FP8, "fp4": ZCMOE_FP4, "nvfp4": ZCMOE_NVFP4}

EXPORTED = ("zcmoe_create", "zcmoe_forward", "zcmoe_forward_host", "zcmoe_update_bias", "zcmoe_read_counts",
            "zcmoe_write_counts", "zcmoe_get_state", "zcmoe_set_bias", "zcmoe_check", "zcmoe_profile_begin",
            "zcmoe_profile_end", "zcmoe_selftest_wait", "zcmoe_route_noalloc", "zcmoe_destroy",
            "zcmoe_dense_create", "zcmoe_dense_forward", "zcmoe_forward_overlap", "zcmoe_dense_check",
            "zcmoe_dense_destroy", "zcmoe_quantize_e4m3", "zcmoe_quantize_mx4", "zcmoe_quantize_nv4", "zcmoe_backward",
            "zcmoe_save_for_backward", "zcmoe_backward_ex", "zcmoe_forward_host_async",
            "zcmoe_forward_host_flush", "zcmoe_create_ep", "zcmoe_ep_dispatch", "zcmoe_ep_experts",
            "zcmoe_ep_combine", "zcmoe_get_controller", "zcmoe_set_controller", "zcmoe_last_error")
STAGES = ("router", "softmax_topk", "integer", "gather", "gate_up", "down", "combine")


class ZcmoeError(RuntimeError):
    def __init__(self, code, where, msg):
        super().__init__(f"{where} failed with code {code}: {msg}")
        self.code = code


class zcmoe_config(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("n_ffn", ctypes.c_int32), ("n_zero", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("top_k", ctypes.c_int32), ("max_tokens", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("routed_scale", ctypes.c_float),
                ("init_bias", ctypes.POINTER(ctypes.c_float)), ("logit_offset", ctypes.POINTER(ctypes.c_float))]


class zcmoe_weights(ctypes.Structure):
    _fields_ = [("w_router", ctypes.c_void_p), ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p),
                ("w_down", ctypes.c_void_p)]


class zcmoe_gains(ctypes.Structure):
    _fields_ = [("kp", ctypes.c_float), ("ki", ctypes.c_float), ("kd", ctypes.c_float), ("decay", ctypes.c_float),
                ("target_ffn_per_token", ctypes.c_float)]


class zcmoe_debug(ctypes.Structure):
    _fields_ = [("logits", ctypes.c_void_p), ("scores", ctypes.c_void_p), ("idx", ctypes.c_void_p),
                ("gate", ctypes.c_void_p), ("counts", ctypes.c_void_p), ("offsets", ctypes.c_void_p),
                ("perm", ctypes.c_void_p), ("pos", ctypes.c_void_p), ("expert_out", ctypes.c_void_p)]


class zcmoe_dense_config(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("inter", ctypes.c_int32), ("max_tokens", ctypes.c_int32)]


class zcmoe_dense_weights(ctypes.Structure):
    _fields_ = [("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p)]


_lib = None


def lib():
    """Loads libzcmoe.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.zcmoe_create.argtypes = [ctypes.POINTER(zcmoe_config), ctypes.POINTER(zcmoe_weights), ctypes.POINTER(vp)]
        L.zcmoe_forward.argtypes = [vp, vp, i64, vp, vp, ctypes.POINTER(zcmoe_debug)]
        L.zcmoe_forward_host.argtypes = [vp, vp, i64, vp, vp]
        L.zcmoe_forward_host_async.argtypes = [vp, vp, i64, vp, vp]
        L.zcmoe_forward_host_flush.argtypes = [vp, vp]
        L.zcmoe_update_bias.argtypes = [vp, ctypes.POINTER(zcmoe_gains), vp]
        L.zcmoe_read_counts.argtypes = [vp, vp, vp]
        L.zcmoe_write_counts.argtypes = [vp, vp, vp]
        L.zcmoe_get_state.argtypes = [vp, vp, vp, vp, vp]
        L.zcmoe_set_bias.argtypes = [vp, vp]
        L.zcmoe_get_controller.argtypes = [vp, vp, vp, vp, vp, vp, vp]
        L.zcmoe_set_controller.argtypes = [vp, vp, vp, vp, vp, vp, vp]
        L.zcmoe_check.argtypes = [vp]
        L.zcmoe_destroy.argtypes = [vp]
        L.zcmoe_profile_begin.argtypes = [vp]
        L.zcmoe_profile_end.argtypes = [vp, vp, vp]
        L.zcmoe_selftest_wait.argtypes = [vp, i64, vp]
        L.zcmoe_route_noalloc.argtypes = [vp, vp, i64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                                          vp, vp, vp, vp, vp, vp, vp]
        L.zcmoe_dense_create.argtypes = [ctypes.POINTER(zcmoe_dense_config), ctypes.POINTER(zcmoe_dense_weights),
                                         ctypes.POINTER(vp)]
        L.zcmoe_dense_forward.argtypes = [vp, vp, i64, vp, vp]
        L.zcmoe_forward_overlap.argtypes = [vp, vp, vp, vp, i64, vp, vp, vp]
        L.zcmoe_dense_check.argtypes = [vp]
        L.zcmoe_quantize_e4m3.argtypes = [vp, ctypes.c_int32, i64, i64, ctypes.c_int32, vp, vp, vp]
        L.zcmoe_quantize_mx4.argtypes = [vp, ctypes.c_int32, i64, i64, vp, vp, vp]
        L.zcmoe_quantize_nv4.argtypes = [vp, ctypes.c_int32, i64, i64, ctypes.c_float, vp, vp, vp, vp]
        L.zcmoe_backward.argtypes = [vp, vp, vp, i64, vp, vp, vp, vp, vp, vp]
        L.zcmoe_backward_ex.argtypes = [vp, vp, vp, i64, vp, vp, vp, vp, vp, ctypes.c_uint32, vp]
        L.zcmoe_save_for_backward.argtypes = [vp, ctypes.c_int32]
        L.zcmoe_create_ep.argtypes = [ctypes.POINTER(zcmoe_config), ctypes.POINTER(zcmoe_weights), ctypes.c_int32,
                                      ctypes.c_int32, i64, ctypes.POINTER(vp)]
        L.zcmoe_ep_dispatch.argtypes = [vp, vp, i64, vp, vp, vp, ctypes.POINTER(zcmoe_debug)]
        L.zcmoe_ep_experts.argtypes = [vp, vp, vp, i64, vp, vp]
        L.zcmoe_ep_combine.argtypes = [vp, vp, vp, i64, vp, vp]
        L.zcmoe_dense_destroy.argtypes = [vp]
        for f in EXPORTED[:-1]:
            getattr(L, f).restype = i32
        L.zcmoe_last_error.argtypes = []
        L.zcmoe_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(rc, where):
    if rc != ZCMOE_OK:
        raise ZcmoeError(rc, where, lib().zcmoe_last_error().decode(errors="replace"))


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _expect(t, name, shape, dtype, cuda=True):
    """The library sees only a pointer, so the binding checks what the pointer must
    hold: a contiguous tensor of exactly `shape` (None matches any extent) and
    `dtype`, on the GPU (cuda=True) or in host memory.  Raises ValueError."""
    ok = (t.dim() == len(shape) and all(w is None or int(n) == w for n, w in zip(t.shape, shape))
          and t.dtype == dtype and t.is_contiguous() and bool(t.is_cuda) == cuda)
    if not ok:
        want = "[" + ", ".join("*" if w is None else str(w) for w in shape) + "]"
        where = "device" if cuda else "host"
        raise ValueError(f"{name}: expected a contiguous {where} tensor {want} {dtype}, got {list(t.shape)} "
                         f"{t.dtype} on {t.device}{'' if t.is_contiguous() else ' (not contiguous)'}")


def _expect_at_least(t, name, numel, dtype):
    """A device output buffer the library fills from its start: contiguous, of `dtype`,
    holding at least `numel` elements."""
    if t.dtype != dtype or not t.is_contiguous() or not t.is_cuda or t.numel() < numel:
        raise ValueError(f"{name}: expected a contiguous device {dtype} buffer of at least {numel} elements, got "
                         f"{list(t.shape)} {t.dtype} on {t.device}")


# ----------------------------------------------------------------- C names
def zcmoe_create(cfg: zcmoe_config, w: zcmoe_weights) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(lib().zcmoe_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)), "zcmoe_create")
    return h


def zcmoe_create_ep(cfg: zcmoe_config, w: zcmoe_weights, ep_rank: int, ep_size: int,
                    max_recv_rows: int) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(lib().zcmoe_create_ep(ctypes.byref(cfg), ctypes.byref(w), ep_rank, ep_size, max_recv_rows, ctypes.byref(h)),
           "zcmoe_create_ep")
    return h


def zcmoe_ep_dispatch(h, x_ptr, T, xsend_ptr, offsets_ptr, stream=None, dbg=None):
    _check(lib().zcmoe_ep_dispatch(h, x_ptr, T, xsend_ptr, offsets_ptr, _stream(stream),
                                   ctypes.byref(dbg) if dbg is not None else None), "zcmoe_ep_dispatch")


def zcmoe_ep_experts(h, xrecv_ptr, counts_host_ptr, P_recv, yrecv_ptr, stream=None):
    _check(lib().zcmoe_ep_experts(h, xrecv_ptr, counts_host_ptr, P_recv, yrecv_ptr, _stream(stream)),
           "zcmoe_ep_experts")


def zcmoe_ep_combine(h, x_ptr, yback_ptr, T, y_ptr, stream=None):
    _check(lib().zcmoe_ep_combine(h, x_ptr, yback_ptr, T, y_ptr, _stream(stream)), "zcmoe_ep_combine")


def zcmoe_forward(h, x_ptr, T, y_ptr, stream=None, dbg: zcmoe_debug | None = None):
    _check(lib().zcmoe_forward(h, x_ptr, T, y_ptr, _stream(stream), ctypes.byref(dbg) if dbg is not None else None),
           "zcmoe_forward")


def zcmoe_forward_host(h, x_host_ptr, T, y_host_ptr, stream=None):
    _check(lib().zcmoe_forward_host(h, x_host_ptr, T, y_host_ptr, _stream(stream)), "zcmoe_forward_host")


def zcmoe_forward_host_async(h, x_host_ptr, T, y_host_ptr, stream=None):
    _check(lib().zcmoe_forward_host_async(h, x_host_ptr, T, y_host_ptr, _stream(stream)), "zcmoe_forward_host_async")


def zcmoe_forward_host_flush(h, stream=None):
    _check(lib().zcmoe_forward_host_flush(h, _stream(stream)), "zcmoe_forward_host_flush")


def zcmoe_update_bias(h, gains: zcmoe_gains, stream=None):
    _check(lib().zcmoe_update_bias(h, ctypes.byref(gains), _stream(stream)), "zcmoe_update_bias")


def zcmoe_read_counts(h, dst_ptr, stream=None):
    _check(lib().zcmoe_read_counts(h, dst_ptr, _stream(stream)), "zcmoe_read_counts")


def zcmoe_write_counts(h, src_ptr, stream=None):
    _check(lib().zcmoe_write_counts(h, src_ptr, _stream(stream)), "zcmoe_write_counts")


def zcmoe_get_state(h, bias_ptr=None, counts_ptr=None, tokens_ptr=None, eta_ptr=None):
    _check(lib().zcmoe_get_state(h, bias_ptr, counts_ptr, tokens_ptr, eta_ptr), "zcmoe_get_state")


def zcmoe_set_bias(h, bias_ptr):
    _check(lib().zcmoe_set_bias(h, bias_ptr), "zcmoe_set_bias")


def zcmoe_get_controller(h, bias_ptr=None, integ_ptr=None, eprev_ptr=None, eta_ptr=None, counts_ptr=None,
                         tokens_ptr=None):
    _check(lib().zcmoe_get_controller(h, bias_ptr, integ_ptr, eprev_ptr, eta_ptr, counts_ptr, tokens_ptr),
           "zcmoe_get_controller")


def zcmoe_set_controller(h, bias_ptr, integ_ptr, eprev_ptr, eta_ptr, counts_ptr, tokens_ptr):
    _check(lib().zcmoe_set_controller(h, bias_ptr, integ_ptr, eprev_ptr, eta_ptr, counts_ptr, tokens_ptr),
           "zcmoe_set_controller")


def zcmoe_check(h):
    _check(lib().zcmoe_check(h), "zcmoe_check")


def zcmoe_profile_begin(h):
    _check(lib().zcmoe_profile_begin(h), "zcmoe_profile_begin")


def zcmoe_profile_end(h):
    """Returns ({stage: total ms}, number of forwards recorded)."""
    ms = (ctypes.c_float * len(STAGES))()
    n = ctypes.c_int32()
    _check(lib().zcmoe_profile_end(h, ms, ctypes.byref(n)), "zcmoe_profile_end")
    return dict(zip(STAGES, [float(v) for v in ms])), int(n.value)


def zcmoe_selftest_wait(h, limit_ns, stream=None):
    _check(lib().zcmoe_selftest_wait(h, int(limit_ns), _stream(stream)), "zcmoe_selftest_wait")


def zcmoe_route_noalloc(logits, bias, T, n_ffn, n_zero, top_k, routed_scale, idx, gate, counts, offsets, perm, pos,
                        stream=None):
    """Routing stage with no device allocation; every argument is a device pointer
    (or tensor data_ptr) except the sizes and the scale."""
    _check(lib().zcmoe_route_noalloc(logits, bias, T, n_ffn, n_zero, top_k, routed_scale, idx, gate, counts, offsets,
                                     perm, pos, _stream(stream)), "zcmoe_route_noalloc")


def zcmoe_destroy(h):
    _check(lib().zcmoe_destroy(h), "zcmoe_destroy")


def zcmoe_dense_create(cfg: zcmoe_dense_config, w: zcmoe_dense_weights) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(lib().zcmoe_dense_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)), "zcmoe_dense_create")
    return h


def zcmoe_dense_forward(h, x_ptr, T, y_ptr, stream=None):
    _check(lib().zcmoe_dense_forward(h, x_ptr, T, y_ptr, _stream(stream)), "zcmoe_dense_forward")


def zcmoe_forward_overlap(moe, dense, x_moe_ptr, x_dense_ptr, T, y_moe_ptr, y_dense_ptr, stream=None):
    _check(lib().zcmoe_forward_overlap(moe, dense, x_moe_ptr, x_dense_ptr, T, y_moe_ptr, y_dense_ptr, _stream(stream)),
           "zcmoe_forward_overlap")


def zcmoe_dense_check(h):
    _check(lib().zcmoe_dense_check(h), "zcmoe_dense_check")


def zcmoe_dense_destroy(h):
    _check(lib().zcmoe_dense_destroy(h), "zcmoe_dense_destroy")


def zcmoe_quantize_e4m3(src_ptr, src_dtype, rows, cols, block_rows, codes_ptr, scales_ptr, stream=None):
    _check(lib().zcmoe_quantize_e4m3(src_ptr, src_dtype, rows, cols, block_rows, codes_ptr, scales_ptr,
                                     _stream(stream)), "zcmoe_quantize_e4m3")


def quantize_e4m3(src, block_rows, stream=None):
    """(codes uint8 [rows, cols], scales uint8 [ceil(rows/block_rows), cols/128]) of a
    2-D bf16 or fp32 device tensor (block-scaled FP8, the rule of ZCMOE_FP8 layers)."""
    rows, cols = src.shape
    codes = torch.empty((rows, cols), dtype=torch.uint8, device=src.device)
    scales = torch.empty(((rows + block_rows - 1) // block_rows, cols // 128), dtype=torch.uint8, device=src.device)
    dt = ZCMOE_BF16 if src.dtype == torch.bfloat16 else ZCMOE_F32
    zcmoe_quantize_e4m3(ctypes.c_void_p(src.data_ptr()), dt, rows, cols, block_rows, ctypes.c_void_p(codes.data_ptr()),
                        ctypes.c_void_p(scales.data_ptr()), stream)
    return codes, scales


ZCMOE_GRAD_OVERWRITE = 1


def zcmoe_backward(h, x_ptr, dy_ptr, T, dx_ptr, g_router=None, g_gate=None, g_up=None, g_down=None, stream=None,
                   flags=0):
    if flags:
        _check(lib().zcmoe_backward_ex(h, x_ptr, dy_ptr, T, dx_ptr, g_router, g_gate, g_up, g_down, flags,
                                       _stream(stream)), "zcmoe_backward_ex")
    else:
        _check(lib().zcmoe_backward(h, x_ptr, dy_ptr, T, dx_ptr, g_router, g_gate, g_up, g_down, _stream(stream)),
               "zcmoe_backward")


def zcmoe_save_for_backward(h, on):
    _check(lib().zcmoe_save_for_backward(h, 1 if on else 0), "zcmoe_save_for_backward")


def zcmoe_quantize_mx4(src_ptr, src_dtype, rows, cols, codes_ptr, scales_ptr, stream=None):
    _check(lib().zcmoe_quantize_mx4(src_ptr, src_dtype, rows, cols, codes_ptr, scales_ptr, _stream(stream)),
           "zcmoe_quantize_mx4")


def quantize_mx4(src, stream=None):
    """(codes uint8 [rows, cols/2], scales uint8 [rows, cols/32]) of a 2-D bf16 or fp32
    device tensor (MXFP4, the rule of ZCMOE_FP4 layers)."""
    rows, cols = src.shape
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=src.device)
    scales = torch.empty((rows, cols // 32), dtype=torch.uint8, device=src.device)
    dt = ZCMOE_BF16 if src.dtype == torch.bfloat16 else ZCMOE_F32
    zcmoe_quantize_mx4(ctypes.c_void_p(src.data_ptr()), dt, rows, cols, ctypes.c_void_p(codes.data_ptr()),
                       ctypes.c_void_p(scales.data_ptr()), stream)
    return codes, scales


def zcmoe_quantize_nv4(src_ptr, src_dtype, rows, cols, global_scale, codes_ptr, scales_ptr, global_out_ptr,
                       stream=None):
    _check(lib().zcmoe_quantize_nv4(src_ptr, src_dtype, rows, cols, global_scale, codes_ptr, scales_ptr,
                                    global_out_ptr, _stream(stream)), "zcmoe_quantize_nv4")


def quantize_nv4(src, global_scale=1.0, stream=None):
    """(codes uint8 [rows, cols/2], scales uint8 [rows, cols/16], g float32 [1]) of a 2-D
    bf16 or fp32 device tensor (NVFP4, the rule of ZCMOE_NVFP4 layers).  global_scale
    g > 0 quantizes under g; 0 derives g from the tensor as the layer does for a weight
    matrix (amax / 2688)."""
    rows, cols = src.shape
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=src.device)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=src.device)
    g = torch.full((1,), float(global_scale), dtype=torch.float32, device=src.device)
    dt = ZCMOE_BF16 if src.dtype == torch.bfloat16 else ZCMOE_F32
    zcmoe_quantize_nv4(ctypes.c_void_p(src.data_ptr()), dt, rows, cols, float(global_scale),
                       ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
                       ctypes.c_void_p(g.data_ptr()), stream)
    return codes, scales, g


def zcmoe_last_error() -> str:
    return lib().zcmoe_last_error().decode(errors="replace")


# ----------------------------------------------------------------- owner object
@dataclass
class LayerShape:
    d: int
    n_ffn: int
    n_zero: int
    inter: int
    top_k: int
    dtype: str = "bf16"  # "bf16", "f32", "fp8", "fp4" or "nvfp4" (bf16 interface; FP8 / MXFP4 / NVFP4 experts)
    routed_scale: float = 1.0

    @property
    def E(self):
        return self.n_ffn + self.n_zero

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


class ZcMoE:
    """Owns a handle plus references to its (borrowed) device weights."""

    def __init__(self, shape: LayerShape, w_router, w_gate, w_up, w_down, max_tokens: int, init_bias=None,
                 logit_offset=None, ep_rank: int = 0, ep_size: int = 1, max_recv_rows: int = 0):
        """ep_size > 1: rank ep_rank of an expert-parallel group; w_gate, w_up, w_down then hold
        only this rank's n_ffn / ep_size experts (see ep.py for the forward)."""
        import numpy as np
        self.shape = shape
        self.weights = (w_router, w_gate, w_up, w_down)
        self.ep_rank, self.ep_size = ep_rank, ep_size
        E, NL = shape.E, shape.n_ffn // max(ep_size, 1)
        for t, want in zip(self.weights, [(E, shape.d), (NL, shape.inter, shape.d),
                                          (NL, shape.inter, shape.d), (NL, shape.d, shape.inter)]):
            if tuple(t.shape) != want or t.dtype != shape.torch_dtype or not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"weight of shape {tuple(t.shape)} {t.dtype}; expected {want} {shape.torch_dtype}")
        self._bias0 = None if init_bias is None else np.ascontiguousarray(init_bias, dtype=np.float32)
        self._offset = None if logit_offset is None else np.ascontiguousarray(logit_offset, dtype=np.float32)
        fp = ctypes.POINTER(ctypes.c_float)
        cfg = zcmoe_config(shape.d, shape.n_ffn, shape.n_zero, shape.inter, shape.top_k, max_tokens,
                           _DTYPES[shape.dtype], shape.routed_scale,
                           None if self._bias0 is None else self._bias0.ctypes.data_as(fp),
                           None if self._offset is None else self._offset.ctypes.data_as(fp))
        w = zcmoe_weights(w_router.data_ptr(), w_gate.data_ptr(), w_up.data_ptr(), w_down.data_ptr())
        self.max_tokens = max_tokens
        self.h = (zcmoe_create(cfg, w) if ep_size == 1 and max_recv_rows == 0
                  else zcmoe_create_ep(cfg, w, ep_rank, ep_size, max_recv_rows))

    def forward(self, x, y=None, stream=None, debug: dict | None = None):
        """y = layer(x); ``debug`` maps zcmoe_debug field names to device tensors to fill."""
        s = self.shape
        _expect(x, "x", (None, s.d), s.torch_dtype)
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        _expect(y, "y", (T, s.d), s.torch_dtype)
        dbg = None
        if debug:
            k, E = s.top_k, s.E
            need = {"logits": (T * E, torch.float32), "scores": (T * E, torch.float32), "idx": (T * k, torch.int32),
                    "gate": (T * k, torch.float32), "counts": (E, torch.int32), "offsets": (s.n_ffn + 1, torch.int32),
                    "perm": (T * k, torch.int32), "pos": (T * k, torch.int32),
                    "expert_out": (T * k * s.d, s.torch_dtype)}
            for name, t in debug.items():
                if name not in need:
                    raise ValueError(f"debug: unknown field {name!r}; fields: {sorted(need)}")
                _expect_at_least(t, f"debug[{name!r}]", *need[name])
            dbg = zcmoe_debug(**{k_: v.data_ptr() for k_, v in debug.items()})
        zcmoe_forward(self.h, ctypes.c_void_p(x.data_ptr()), T, ctypes.c_void_p(y.data_ptr()), stream, dbg)
        return y

    def forward_host(self, x_host, y_host, stream=None, pipelined=False):
        """y_host = layer(x_host), both page-locked host tensors.  pipelined: y_host is complete
        once the stream has passed the next forward_host call or flush_host()."""
        s = self.shape
        _expect(x_host, "x_host", (None, s.d), s.torch_dtype, cuda=False)
        _expect(y_host, "y_host", (x_host.shape[0], s.d), s.torch_dtype, cuda=False)
        fn = zcmoe_forward_host_async if pipelined else zcmoe_forward_host
        fn(self.h, ctypes.c_void_p(x_host.data_ptr()), x_host.shape[0], ctypes.c_void_p(y_host.data_ptr()), stream)
        return y_host

    def flush_host(self, stream=None):
        zcmoe_forward_host_flush(self.h, stream)

    def backward(self, x, dy, dx=None, grads: dict | None = None, stream=None, accumulate=True):
        """dx of the last forward (x must be the tensor it read); adds the weight gradients
        into the fp32 tensors of ``grads`` (keys router, gate, up, down; missing: skipped), or
        writes them there with accumulate=False."""
        s = self.shape
        _expect(x, "x", (None, s.d), s.torch_dtype)
        T = x.shape[0]
        _expect(dy, "dy", (T, s.d), s.torch_dtype)
        dx = torch.empty_like(x) if dx is None else dx
        _expect(dx, "dx", (T, s.d), s.torch_dtype)
        g = grads or {}
        NL = s.n_ffn // max(self.ep_size, 1)
        gshape = {"router": (s.E, s.d), "gate": (NL, s.inter, s.d), "up": (NL, s.inter, s.d),
                  "down": (NL, s.d, s.inter)}
        for name, t in g.items():
            if name not in gshape:
                raise ValueError(f"grads: unknown key {name!r}; keys: {sorted(gshape)}")
            _expect(t, f"grads[{name!r}]", gshape[name], torch.float32)
        ptr = lambda name: ctypes.c_void_p(g[name].data_ptr()) if name in g else None  # noqa: E731
        zcmoe_backward(self.h, ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(dy.data_ptr()), x.shape[0],
                       ctypes.c_void_p(dx.data_ptr()), ptr("router"), ptr("gate"), ptr("up"), ptr("down"), stream,
                       flags=0 if accumulate else ZCMOE_GRAD_OVERWRITE)
        return dx

    def save_for_backward(self, on=True):
        """Training mode: later forwards store G and U for the backward (no recompute)."""
        zcmoe_save_for_backward(self.h, on)

    def update_bias(self, kp=0.0, ki=0.0, kd=0.0, decay=1.0, target_ffn_per_token=None, stream=None):
        K = float(self.shape.top_k if target_ffn_per_token is None else target_ffn_per_token)
        zcmoe_update_bias(self.h, zcmoe_gains(kp, ki, kd, decay, K), stream)

    def read_counts(self, dst, stream=None):
        _expect(dst, "dst", (self.shape.E + 1,), torch.int64)
        zcmoe_read_counts(self.h, ctypes.c_void_p(dst.data_ptr()), stream)

    def write_counts(self, src, stream=None):
        _expect(src, "src", (self.shape.E + 1,), torch.int64)
        zcmoe_write_counts(self.h, ctypes.c_void_p(src.data_ptr()), stream)

    def state(self):
        import numpy as np
        E = self.shape.E
        bias = np.empty(E, np.float32)
        counts = np.empty(E, np.int64)
        tokens = np.empty(1, np.int64)
        eta = np.empty(1, np.float32)
        zcmoe_get_state(self.h, bias.ctypes.data, counts.ctypes.data, tokens.ctypes.data, eta.ctypes.data)
        return {"bias": bias, "counts": counts, "tokens": int(tokens[0]), "eta": float(eta[0])}

    def set_bias(self, bias):
        import numpy as np
        b = np.ascontiguousarray(bias, dtype=np.float32)
        if b.shape != (self.shape.E,):
            raise ValueError(f"bias: expected {self.shape.E} values, got shape {b.shape}")
        zcmoe_set_bias(self.h, b.ctypes.data)

    CONTROLLER_FIELDS = ("bias", "integ", "eprev", "eta", "counts", "tokens")

    def controller_state(self):
        """The whole controller state as host arrays (a checkpoint): bias, integ, eprev
        [E] float32, eta [1] float32, counts [E] int64, tokens [1] int64."""
        import numpy as np
        E = self.shape.E
        st = {"bias": np.empty(E, np.float32), "integ": np.empty(E, np.float32), "eprev": np.empty(E, np.float32),
              "eta": np.empty(1, np.float32), "counts": np.empty(E, np.int64), "tokens": np.empty(1, np.int64)}
        zcmoe_get_controller(self.h, *(st[k].ctypes.data for k in self.CONTROLLER_FIELDS))
        return st

    def load_controller_state(self, st):
        """Restores a controller_state() checkpoint (the handle must have been created
        with the same init_bias for the steps to continue identically)."""
        import numpy as np
        E = self.shape.E
        want = {"bias": (E, np.float32), "integ": (E, np.float32), "eprev": (E, np.float32), "eta": (1, np.float32),
                "counts": (E, np.int64), "tokens": (1, np.int64)}
        arrs = {}
        for k, (n, dt) in want.items():
            a = np.ascontiguousarray(st[k], dtype=dt).reshape(-1)
            if a.shape != (n,):
                raise ValueError(f"{k}: expected {n} values, got {a.size}")
            arrs[k] = a
        zcmoe_set_controller(self.h, *(arrs[k].ctypes.data for k in self.CONTROLLER_FIELDS))

    def check(self):
        zcmoe_check(self.h)

    def profile_begin(self):
        zcmoe_profile_begin(self.h)

    def profile_end(self):
        return zcmoe_profile_end(self.h)

    def close(self):
        if self.h is not None:
            zcmoe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class ZcDense:
    """Owns a dense-FFN handle plus references to its (borrowed) bf16 weights:
    w_gate [inter, d], w_up [inter, d], w_down [d, inter]."""

    def __init__(self, w_gate, w_up, w_down, max_tokens: int):
        inter, d = w_gate.shape
        self.d, self.inter, self.max_tokens = d, inter, max_tokens
        self.weights = (w_gate, w_up, w_down)
        for t, want in zip(self.weights, [(inter, d), (inter, d), (d, inter)]):
            if tuple(t.shape) != want or t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"weight of shape {tuple(t.shape)} {t.dtype}; expected {want} bfloat16")
        cfg = zcmoe_dense_config(d, inter, max_tokens)
        w = zcmoe_dense_weights(w_gate.data_ptr(), w_up.data_ptr(), w_down.data_ptr())
        self.h = zcmoe_dense_create(cfg, w)

    def forward(self, x, y=None, stream=None):
        _expect(x, "x", (None, self.d), torch.bfloat16)
        if y is None:
            y = torch.empty_like(x)
        _expect(y, "y", (x.shape[0], self.d), torch.bfloat16)
        zcmoe_dense_forward(self.h, ctypes.c_void_p(x.data_ptr()), x.shape[0], ctypes.c_void_p(y.data_ptr()), stream)
        return y

    def check(self):
        zcmoe_dense_check(self.h)

    def close(self):
        if self.h is not None:
            zcmoe_dense_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def forward_overlap(moe: ZcMoE, dense: ZcDense, x_moe, x_dense=None, y_moe=None, y_dense=None, stream=None):
    """(y_moe, y_dense): the MoE layer and the dense FFN over the same tokens, run
    concurrently (zcmoe_forward_overlap).  x_dense defaults to x_moe."""
    x_dense = x_moe if x_dense is None else x_dense
    if x_dense.shape[0] != x_moe.shape[0]:
        raise ValueError("x_moe and x_dense must hold the same number of tokens")
    y_moe = torch.empty_like(x_moe) if y_moe is None else y_moe
    y_dense = torch.empty_like(x_dense) if y_dense is None else y_dense
    # the tensors are checked against the MoE layer's row width and dtype; a dense handle
    # that does not match the layer is refused by the library
    s = moe.shape
    for name, t in (("x_moe", x_moe), ("x_dense", x_dense), ("y_moe", y_moe), ("y_dense", y_dense)):
        _expect(t, name, (x_moe.shape[0], s.d), s.torch_dtype)
    zcmoe_forward_overlap(moe.h, dense.h, ctypes.c_void_p(x_moe.data_ptr()), ctypes.c_void_p(x_dense.data_ptr()),
                          x_moe.shape[0], ctypes.c_void_p(y_moe.data_ptr()), ctypes.c_void_p(y_dense.data_ptr()),
                          stream)
    return y_moe, y_dense
