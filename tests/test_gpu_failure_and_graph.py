"""Failure detection without a GPU fault, and CUDA-graph replay.

* A kernel wait that nothing releases gives up after its limit, records a
  timeout that zcmoe_check reports, and leaves the context usable.
* A device allocation failure at create is reported as ZCMOE_ENOMEM and
  leaves nothing behind.
* A forward captured in a CUDA graph replays to the same bits as eager.
* A destroyed handle is refused by every entry point (double destroy, use after
  destroy) instead of being dereferenced."""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_layer_shifted_b200 import configs
from mixture_experts_layer_shifted_b200 import zcmoe as Z
from tests.gpu_harness import Run

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_context_survives(cuda_ok):
    r = Run(configs.WORKLOADS["small_bf16"], T=512)
    try:
        y0 = r.forward(debug=False).clone()
        Z.zcmoe_selftest_wait(r.layer.h, 50_000_000)  # 50 ms
        with pytest.raises(Z.ZcmoeError) as ei:
            r.layer.check()
        assert ei.value.code == Z.ZCMOE_ETIMEOUT
        assert "99" in str(ei.value)
        r.layer.check()  # the flag was cleared by the report
        y1 = r.forward(debug=False)
        assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
        with pytest.raises(Z.ZcmoeError) as ei:
            Z.zcmoe_selftest_wait(r.layer.h, 5_000_000_000)
        assert ei.value.code == Z.ZCMOE_EINVAL
    finally:
        r.close()


def test_device_allocation_failure_is_reported(cuda_ok):
    w = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    p = w.data_ptr()
    # the 560B layer shape with room for 2^20 tokens needs ~200 GB of workspace
    cfg = Z.zcmoe_config(6144, 512, 256, 2048, 12, 1 << 20, Z.ZCMOE_BF16, 1.0, None, None)
    wts = Z.zcmoe_weights(p, p, p, p)
    h = ctypes.c_void_p()
    free0, _ = torch.cuda.mem_get_info()
    rc = Z.lib().zcmoe_create(ctypes.byref(cfg), ctypes.byref(wts), ctypes.byref(h))
    assert rc == Z.ZCMOE_ENOMEM and h.value is None
    assert "cudaMalloc" in Z.zcmoe_last_error()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 >= free0 - (64 << 20)  # nothing of the partial allocation is kept
    # the device is still usable: a normal layer works
    r = Run(configs.WORKLOADS["tiny_f32"])
    try:
        r.forward()
        r.check_routing_bitexact()
    finally:
        r.close()


def test_forward_in_cuda_graph_matches_eager(cuda_ok):
    r = Run(configs.WORKLOADS["small_bf16"])
    try:
        y_eager = r.forward(debug=False).clone()
        tok0 = r.layer.state()["tokens"]
        y = torch.empty_like(r.x)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            r.layer.forward(r.x, y)  # warm-up on the capture stream
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            r.layer.forward(r.x, y)
        y.zero_()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        r.layer.check()
        assert torch.equal(y.view(torch.int16), y_eager.view(torch.int16))
        # every replay ran the whole forward, counts included
        assert r.layer.state()["tokens"] == tok0 + 4 * r.T
    finally:
        r.close()


def test_destroyed_handle_is_refused(cuda_ok):
    r = Run(configs.WORKLOADS["tiny_f32"])
    raw = r.layer.h
    lib = Z.lib()
    y = torch.empty_like(r.x)
    bias = np.zeros(r.w.E, np.float32)
    assert lib.zcmoe_destroy(raw) == Z.ZCMOE_OK
    r.layer.h = None                                    # the owner no longer holds it
    assert lib.zcmoe_destroy(raw) == Z.ZCMOE_EINVAL      # double destroy
    xp, yp = ctypes.c_void_p(r.x.data_ptr()), ctypes.c_void_p(y.data_ptr())
    assert lib.zcmoe_forward(raw, xp, r.x.shape[0], yp, None, None) == Z.ZCMOE_EINVAL
    gains = Z.zcmoe_gains(0.0, 0.02, 0.0, 1.0, 2.0)
    assert lib.zcmoe_update_bias(raw, ctypes.byref(gains), None) == Z.ZCMOE_EINVAL
    assert lib.zcmoe_get_state(raw, bias.ctypes.data, None, None, None) == Z.ZCMOE_EINVAL
    assert lib.zcmoe_check(raw) == Z.ZCMOE_EINVAL
    assert "handle" in Z.zcmoe_last_error()
