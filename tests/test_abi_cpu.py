"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point the header declares, and rejects bad arguments before it
touches the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zcmoe.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"ZCMOE_API\s+[\w\s\*]+?\b(zcmoe_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def zc():
    from mixture_experts_layer_shifted_b200 import build
    build.build()
    from mixture_experts_layer_shifted_b200 import zcmoe
    return zcmoe


def test_header_declares_the_four_calls():
    names = _declared()
    for n in ("zcmoe_create", "zcmoe_forward", "zcmoe_update_bias", "zcmoe_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(zc):
    lib = zc.lib()
    for name in _declared():
        assert hasattr(lib, name), name
    assert sorted(zc.EXPORTED) == _declared()


def test_synth_library_exports():
    from mixture_experts_layer_shifted_b200 import build, synth
    build.build()
    lib = synth.device_lib()
    assert hasattr(lib, "zcsynth_normal") and hasattr(lib, "zcsynth_uniform")


def test_bad_arguments_are_rejected_on_the_host(zc):
    lib = zc.lib()
    h = ctypes.c_void_p()
    cfg = zc.zcmoe_config(256, 16, 8, 128, 4, 64, zc.ZCMOE_F32, 1.0, None, None)
    w = zc.zcmoe_weights(16, 16, 16, 16)
    assert lib.zcmoe_create(None, ctypes.byref(w), ctypes.byref(h)) == zc.ZCMOE_EINVAL
    assert lib.zcmoe_create(ctypes.byref(cfg), ctypes.byref(w), None) == zc.ZCMOE_EINVAL
    for bad in [dict(d=100), dict(inter=0), dict(top_k=0), dict(top_k=33), dict(n_ffn=0), dict(n_zero=2000),
                dict(max_tokens=0), dict(dtype=7)]:
        c = zc.zcmoe_config(256, 16, 8, 128, 4, 64, zc.ZCMOE_F32, 1.0, None, None)
        for k_, v in bad.items():
            setattr(c, k_, v)
        assert lib.zcmoe_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == zc.ZCMOE_EINVAL, bad
        assert h.value is None
        assert zc.zcmoe_last_error() != ""
    w_bad = zc.zcmoe_weights(16, 17, 16, 16)  # misaligned
    assert lib.zcmoe_create(ctypes.byref(cfg), ctypes.byref(w_bad), ctypes.byref(h)) == zc.ZCMOE_EINVAL
    w_null = zc.zcmoe_weights(16, None, 16, 16)
    assert lib.zcmoe_create(ctypes.byref(cfg), ctypes.byref(w_null), ctypes.byref(h)) == zc.ZCMOE_EINVAL
    # handles that were never created are refused, not dereferenced
    fake = ctypes.c_void_p(0x1000)
    assert lib.zcmoe_forward(fake, None, 1, None, None, None) == zc.ZCMOE_EINVAL
    assert lib.zcmoe_update_bias(fake, None, None) == zc.ZCMOE_EINVAL
    assert lib.zcmoe_check(fake) == zc.ZCMOE_EINVAL
    assert lib.zcmoe_destroy(fake) == zc.ZCMOE_EINVAL
    assert lib.zcmoe_destroy(None) == zc.ZCMOE_OK


def test_create_without_a_device_fails_cleanly(zc):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    lib = zc.lib()
    h = ctypes.c_void_p()
    cfg = zc.zcmoe_config(256, 16, 8, 128, 4, 64, zc.ZCMOE_F32, 1.0, None, None)
    w = zc.zcmoe_weights(16, 16, 16, 16)
    rc = lib.zcmoe_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h))
    assert rc in (zc.ZCMOE_ECUDA, zc.ZCMOE_EUNSUPPORTED)
    assert h.value is None


def test_dense_and_overlap_arguments_are_rejected_on_the_host(zc):
    lib = zc.lib()
    h = ctypes.c_void_p()
    w = zc.zcmoe_dense_weights(16, 16, 16)
    cfg = zc.zcmoe_dense_config(256, 384, 64)
    assert lib.zcmoe_dense_create(None, ctypes.byref(w), ctypes.byref(h)) == zc.ZCMOE_EINVAL
    assert lib.zcmoe_dense_create(ctypes.byref(cfg), ctypes.byref(w), None) == zc.ZCMOE_EINVAL
    for bad in [dict(d=100), dict(d=0), dict(inter=32), dict(inter=100), dict(max_tokens=0),
                dict(max_tokens=(1 << 20) + 1)]:
        c = zc.zcmoe_dense_config(256, 384, 64)
        for k_, v in bad.items():
            setattr(c, k_, v)
        assert lib.zcmoe_dense_create(ctypes.byref(c), ctypes.byref(w), ctypes.byref(h)) == zc.ZCMOE_EINVAL, bad
        assert h.value is None
        assert zc.zcmoe_last_error() != ""
    assert lib.zcmoe_dense_create(ctypes.byref(cfg), ctypes.byref(zc.zcmoe_dense_weights(16, 24, 16)),
                                  ctypes.byref(h)) == zc.ZCMOE_EINVAL  # misaligned
    assert lib.zcmoe_dense_create(ctypes.byref(cfg), ctypes.byref(zc.zcmoe_dense_weights(16, 16, None)),
                                  ctypes.byref(h)) == zc.ZCMOE_EINVAL
    # handles that were never created are refused, not dereferenced; a MoE handle
    # is not a dense handle
    fake = ctypes.c_void_p(0x1000)
    assert lib.zcmoe_dense_forward(fake, None, 1, None, None) == zc.ZCMOE_EINVAL
    assert lib.zcmoe_dense_check(fake) == zc.ZCMOE_EINVAL
    assert lib.zcmoe_dense_destroy(fake) == zc.ZCMOE_EINVAL
    assert lib.zcmoe_dense_destroy(None) == zc.ZCMOE_OK
    assert lib.zcmoe_forward_overlap(fake, fake, None, None, 1, None, None, None) == zc.ZCMOE_EINVAL


def test_training_ep_and_host_entry_points_refuse_unknown_handles(zc):
    """The backward, training-mode, expert-parallel and pipelined host entry points check the
    handle (and their own arguments) on the host before any device work."""
    lib = zc.lib()
    fake = ctypes.c_void_p(0x1000)
    E = zc.ZCMOE_EINVAL
    assert lib.zcmoe_backward(fake, None, None, 1, None, None, None, None, None, None) == E
    assert lib.zcmoe_backward_ex(fake, None, None, 1, None, None, None, None, None, 0, None) == E
    assert lib.zcmoe_save_for_backward(fake, 1) == E
    assert lib.zcmoe_ep_dispatch(fake, None, 1, None, None, None, None) == E
    assert lib.zcmoe_ep_experts(fake, None, None, 0, None, None) == E
    assert lib.zcmoe_ep_combine(fake, None, None, 1, None, None) == E
    assert lib.zcmoe_forward_host_async(fake, None, 1, None, None) == E
    assert lib.zcmoe_forward_host_flush(fake, None) == E
    # create_ep: the group arguments are checked before the device is touched
    h = ctypes.c_void_p()
    cfg = zc.zcmoe_config(256, 16, 8, 128, 4, 64, zc.ZCMOE_BF16, 1.0, None, None)
    w = zc.zcmoe_weights(16, 16, 16, 16)
    for rank, size, cap in [(0, 3, 0), (2, 2, 0), (-1, 2, 0), (0, 0, 0), (0, 2, -1)]:
        assert lib.zcmoe_create_ep(ctypes.byref(cfg), ctypes.byref(w), rank, size, cap, ctypes.byref(h)) == E
        assert h.value is None
    cfg32 = zc.zcmoe_config(256, 16, 8, 128, 4, 64, zc.ZCMOE_F32, 1.0, None, None)
    assert lib.zcmoe_create_ep(ctypes.byref(cfg32), ctypes.byref(w), 0, 2, 0,
                               ctypes.byref(h)) == zc.ZCMOE_EUNSUPPORTED


def test_binding_tensor_checks(zc):
    """The binding passes bare pointers, so it checks each tensor's dims, dtype,
    contiguity and memory kind before the call; a mismatch is a ValueError."""
    import torch
    ok = torch.zeros((5, 64), dtype=torch.bfloat16)
    zc._expect(ok, "x", (None, 64), torch.bfloat16, cuda=False)
    zc._expect(ok, "x", (5, 64), torch.bfloat16, cuda=False)
    bad = [
        (ok, (None, 32), torch.bfloat16, False),            # width
        (ok, (4, 64), torch.bfloat16, False),               # rows
        (ok, (None, 64), torch.float32, False),             # dtype
        (ok, (None, 64), torch.bfloat16, True),             # host memory where device memory is needed
        (ok.reshape(-1), (None, 64), torch.bfloat16, False),  # dims
        (torch.zeros((64, 5), dtype=torch.bfloat16).t(), (None, 64), torch.bfloat16, False),  # not contiguous
    ]
    for t, shape, dtype, cuda in bad:
        with pytest.raises(ValueError):
            zc._expect(t, "x", shape, dtype, cuda=cuda)
    with pytest.raises(ValueError):
        zc._expect_at_least(torch.zeros(8, dtype=torch.int32), "perm", 8, torch.int32)   # host buffer


def test_layer_methods_check_tensors_before_the_library(zc):
    """A layer object whose handle is not live: a call that passed the binding's checks
    would reach the library and fail there with EINVAL, so each ValueError below shows
    the check ran first, and the ZcmoeError shows well-formed tensors get through."""
    import numpy as np
    import torch
    lay = object.__new__(zc.ZcMoE)
    lay.shape = zc.LayerShape(64, 4, 2, 32, 2, "bf16")
    lay.ep_size = 1
    lay.h = ctypes.c_void_p(0x1000)
    try:
        x = torch.zeros((5, 64), dtype=torch.bfloat16)
        y = torch.zeros((5, 64), dtype=torch.bfloat16)
        with pytest.raises(ValueError):
            lay.forward(x, y, stream=0)                     # host tensors for a device call
        with pytest.raises(ValueError):
            lay.backward(x, y, y.clone(), stream=0)
        with pytest.raises(ValueError):
            lay.read_counts(torch.zeros(7, dtype=torch.int64), stream=0)
        with pytest.raises(ValueError):
            lay.set_bias(np.zeros(5, np.float32))           # E = 6 values needed
        with pytest.raises(ValueError):
            lay.forward_host(x, torch.zeros((4, 64), dtype=torch.bfloat16), stream=0)   # y rows
        with pytest.raises(ValueError):
            lay.forward_host(torch.zeros((5, 32), dtype=torch.bfloat16), y, stream=0)   # width
        with pytest.raises(ValueError):
            lay.forward_host(x.float(), y.float(), stream=0)                            # dtype
        with pytest.raises(zc.ZcmoeError) as ei:
            lay.forward_host(x, y, stream=0)
        assert ei.value.code == zc.ZCMOE_EINVAL
        with pytest.raises(zc.ZcmoeError) as ei:
            lay.set_bias(np.zeros(6, np.float32))
        assert ei.value.code == zc.ZCMOE_EINVAL
    finally:
        lay.h = None


def test_controller_checkpoint_entry_points_refuse_unknown_handles(zc):
    lib = zc.lib()
    fake = ctypes.c_void_p(0x1000)
    assert lib.zcmoe_get_controller(fake, None, None, None, None, None, None) == zc.ZCMOE_EINVAL
    assert lib.zcmoe_set_controller(fake, None, None, None, None, None, None) == zc.ZCMOE_EINVAL
    assert "handle" in zc.zcmoe_last_error()


def test_load_controller_state_checks_sizes_before_the_library(zc):
    import numpy as np
    lay = object.__new__(zc.ZcMoE)
    lay.shape = zc.LayerShape(64, 4, 2, 32, 2, "bf16")
    lay.h = ctypes.c_void_p(0x1000)
    try:
        E = lay.shape.E
        good = {"bias": np.zeros(E), "integ": np.zeros(E), "eprev": np.zeros(E), "eta": [1.0],
                "counts": np.zeros(E, np.int64), "tokens": [0]}
        with pytest.raises(ValueError):
            lay.load_controller_state(dict(good, integ=np.zeros(E - 1)))
        with pytest.raises(zc.ZcmoeError) as ei:      # well-formed: reaches the library, which refuses the handle
            lay.load_controller_state(good)
        assert ei.value.code == zc.ZCMOE_EINVAL
    finally:
        lay.h = None


def test_create_checks_quantized_shapes_scale_and_group_on_the_host(zc):
    """Refusals that come before any device call: FP8 / MXFP4 shape rules, a routed
    scale that is not finite, and expert-parallel group arguments."""
    import math
    lib = zc.lib()
    h = ctypes.c_void_p()
    w = zc.zcmoe_weights(16, 16, 16, 16)

    def cfg(**kw):
        c = zc.zcmoe_config(512, 16, 8, 256, 4, 64, zc.ZCMOE_BF16, 1.0, None, None)
        for k_, v in kw.items():
            setattr(c, k_, v)
        return c

    for bad in [dict(dtype=zc.ZCMOE_FP8, d=256), dict(dtype=zc.ZCMOE_FP8, inter=192),
                dict(dtype=zc.ZCMOE_FP4, d=768), dict(dtype=zc.ZCMOE_FP4, inter=128),
                dict(dtype=zc.ZCMOE_NVFP4, d=768), dict(dtype=zc.ZCMOE_NVFP4, inter=128),
                dict(routed_scale=math.nan), dict(routed_scale=math.inf)]:
        assert lib.zcmoe_create(ctypes.byref(cfg(**bad)), ctypes.byref(w), ctypes.byref(h)) == zc.ZCMOE_EINVAL, bad
        assert h.value is None
    c = cfg()
    for rank, size, cap in [(-1, 2, 0), (2, 2, 0), (0, 0, 0), (0, 3, 0), (0, 2, -1), (0, 2, 1 << 31)]:
        assert lib.zcmoe_create_ep(ctypes.byref(c), ctypes.byref(w), rank, size, cap, ctypes.byref(h)) == \
            zc.ZCMOE_EINVAL, (rank, size, cap)
        assert h.value is None
    for dt in (zc.ZCMOE_FP8, zc.ZCMOE_FP4, zc.ZCMOE_NVFP4):
        assert lib.zcmoe_create_ep(ctypes.byref(cfg(dtype=dt)), ctypes.byref(w), 0, 2, 0,
                                   ctypes.byref(h)) == zc.ZCMOE_EUNSUPPORTED


def test_quantizers_refuse_bad_arguments_on_the_host(zc):
    """zcmoe_quantize_e4m3 / _mx4 / _nv4 check dtype, shape, pointers, alignment and (NVFP4) the
    tensor scale before they touch the device; zero rows is a no-op."""
    import math
    lib = zc.lib()
    p16 = ctypes.c_void_p(0x10000)   # never dereferenced: every call below is refused first
    p_odd = ctypes.c_void_p(0x10008)
    BF16, F32 = zc.ZCMOE_BF16, zc.ZCMOE_F32
    E = zc.ZCMOE_EINVAL
    # E4M3: cols a multiple of 128, block_rows 1 or 128
    assert lib.zcmoe_quantize_e4m3(p16, 7, 4, 128, 1, p16, p16, None) == E
    assert lib.zcmoe_quantize_e4m3(p16, BF16, 4, 100, 1, p16, p16, None) == E
    assert lib.zcmoe_quantize_e4m3(p16, BF16, 4, 128, 64, p16, p16, None) == E
    assert lib.zcmoe_quantize_e4m3(None, BF16, 4, 128, 1, p16, p16, None) == E
    assert lib.zcmoe_quantize_e4m3(p_odd, BF16, 4, 128, 1, p16, p16, None) == E
    assert lib.zcmoe_quantize_e4m3(None, BF16, 0, 128, 1, None, None, None) == zc.ZCMOE_OK
    # MXFP4: cols a multiple of 256
    assert lib.zcmoe_quantize_mx4(p16, F32, 4, 128, p16, p16, None) == E
    assert lib.zcmoe_quantize_mx4(p16, 3, 4, 256, p16, p16, None) == E
    assert lib.zcmoe_quantize_mx4(p16, BF16, 4, 256, None, p16, None) == E
    assert lib.zcmoe_quantize_mx4(p16, BF16, 4, 256, p_odd, p16, None) == E
    assert lib.zcmoe_quantize_mx4(None, BF16, 0, 256, None, None, None) == zc.ZCMOE_OK
    # NVFP4: cols a multiple of 256; the tensor scale finite and >= 0; 0 derives it and needs global_out
    assert lib.zcmoe_quantize_nv4(p16, BF16, 4, 128, 1.0, p16, p16, None, None) == E
    for g in (-1.0, math.nan, math.inf):
        assert lib.zcmoe_quantize_nv4(p16, BF16, 4, 256, g, p16, p16, p16, None) == E, g
    assert lib.zcmoe_quantize_nv4(p16, BF16, 4, 256, 0.0, p16, p16, None, None) == E
    assert lib.zcmoe_quantize_nv4(p16, BF16, 4, 256, 0.0, p16, p16, ctypes.c_void_p(0x10002), None) == E
    assert lib.zcmoe_quantize_nv4(p16, 5, 4, 256, 1.0, p16, p16, None, None) == E
    assert lib.zcmoe_quantize_nv4(p_odd, BF16, 4, 256, 1.0, p16, p16, None, None) == E
    assert lib.zcmoe_quantize_nv4(None, BF16, 0, 256, 1.0, None, None, None, None) == zc.ZCMOE_OK


def test_noalloc_refuses_on_the_host_at_its_exact_limits(zc):
    """zcmoe_route_noalloc checks its arguments before it touches the device, so the
    refusals run without a GPU.  Its scratch layout is align8(ceil(T/256) E 4) +
    (E+1) 8 + (N+1) 4 + 16 bytes of a 1 MiB array: T = 86,528 fits at E = 768,
    N = 512 and the next 256-token block does not; a routed scale that is not a
    finite number is refused like zcmoe_create refuses it."""
    lib = zc.lib()
    p = ctypes.c_void_p(16)
    def call(T, N=512, Z=256, k=12, scale=1.0):
        return lib.zcmoe_route_noalloc(p, p, T, N, Z, k, scale, p, p, p, p, p, p, None)
    def need(T, N, E):
        nb = -(-T // 256)
        return ((nb * E * 4 + 7) & ~7) + (E + 1) * 8 + (N + 1) * 4 + 16
    assert need(86_528, 512, 768) <= 1 << 20 < need(86_529, 512, 768)
    assert call(86_529) == zc.ZCMOE_ERANGE
    msg = zc.lib().zcmoe_last_error().decode()
    assert "86528" in msg and "scratch" in msg, msg
    assert need(698_112, 64, 96) <= 1 << 20 < need(698_113, 64, 96)
    assert call(698_113, N=64, Z=32, k=8) == zc.ZCMOE_ERANGE
    assert "698112" in zc.lib().zcmoe_last_error().decode()
    for bad in (float("nan"), float("inf"), -float("inf")):
        assert call(1024, scale=bad) == zc.ZCMOE_EINVAL
    assert call(-1) == zc.ZCMOE_ERANGE
    assert call(1024, k=0) == zc.ZCMOE_EINVAL
