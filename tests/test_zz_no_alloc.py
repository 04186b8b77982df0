"""The allocation-free routing entry point, zcmoe_route_noalloc.

It exists for callers that cannot call cudaMalloc (code inside a framework's
memory pool or a fixed memory budget, and latency-critical loops where an
allocation could synchronise the device).  Its scratch is a fixed device array
inside the library.  This file is collected last so that a run stopping at the
first failure has already run every other test; it also passes on its own in
a fresh process.

The check: the routing outputs of two back-to-back calls (the second one
reusing the scratch the first one left behind) equal, bit for bit, what the
regular zcmoe_forward computes for the same logits and bias (routing is
compared bit-exactly everywhere in these tests)."""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_layer_shifted_b200 import configs
from mixture_experts_layer_shifted_b200 import zcmoe as Z
from tests.gpu_harness import Run

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("name,T", [("small_bf16", None), ("prefill_probe", 3000)])
def test_noalloc_routing_matches_forward_twice(cuda_ok, name, T):
    w = configs.WORKLOADS[name]
    r = Run(w, T=T)
    try:
        r.forward()
        Tn, E, k, N = r.T, w.E, w.top_k, w.n_ffn
        logits = torch.from_numpy(r.dbg["logits"]).cuda()
        bias = torch.from_numpy(r.cur_bias).cuda()
        for call in range(2):
            out = {
                "idx": torch.full((Tn, k), -7, dtype=torch.int32, device="cuda"),
                "gate": torch.full((Tn, k), -7.0, dtype=torch.float32, device="cuda"),
                "counts": torch.full((E,), -7, dtype=torch.int32, device="cuda"),
                "offsets": torch.full((N + 1,), -7, dtype=torch.int32, device="cuda"),
                "perm": torch.full((Tn * k,), -7, dtype=torch.int32, device="cuda"),
                "pos": torch.full((Tn, k), -7, dtype=torch.int32, device="cuda"),
            }
            Z.zcmoe_route_noalloc(_p(logits), _p(bias), Tn, N, w.n_zero, k, 1.0, _p(out["idx"]), _p(out["gate"]),
                                  _p(out["counts"]), _p(out["offsets"]), _p(out["perm"]), _p(out["pos"]))
            torch.cuda.synchronize()
            got = {key: v.cpu().numpy() for key, v in out.items()}
            np.testing.assert_array_equal(got["idx"], r.dbg["idx"])
            np.testing.assert_array_equal(got["gate"].view(np.uint32), r.dbg["gate"].view(np.uint32))
            np.testing.assert_array_equal(got["counts"], r.dbg["counts"])
            np.testing.assert_array_equal(got["offsets"], r.dbg["offsets"])
            P = int(r.dbg["offsets"][-1])
            np.testing.assert_array_equal(got["perm"][:P], r.dbg["perm"][:P])
            np.testing.assert_array_equal(got["pos"], r.dbg["pos"])
    finally:
        r.close()


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_ok):
    E, k, N = 768, 12, 512
    T = 100_000  # needs ~1.2 MB of routing scratch; the fixed array holds 1 MiB
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(Z.ZcmoeError) as ei:
        Z.zcmoe_route_noalloc(_p(dummy), _p(dummy), T, N, E - N, k, 1.0, *([_p(dummy)] * 6))
    assert ei.value.code == Z.ZCMOE_ERANGE
    assert "scratch" in Z.zcmoe_last_error()
