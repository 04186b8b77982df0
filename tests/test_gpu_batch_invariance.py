"""A token's routing does not depend on the batch it arrives in.

The router GEMM picks its tile width by batch size: 256-column tiles when the batch
has enough row blocks to fill the SMs, 32-column tiles for a batch of a few row
blocks (decode), so that more SMs share the work.  Every logit is still the same
sequence of K = 16 tensor-core steps accumulated in fp32 in the same order, so the
logits, and with them every routing decision, must be bit-identical whichever
width ran; the expert outputs of a token (same rows, same weights) then agree as
well.  Expert parallelism relies on this: a token routed in a chunk of another
size must pick the same experts.
"""
import numpy as np
import pytest

from mixture_experts_layer_shifted_b200 import configs
from tests.gpu_harness import Run

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,T_big,T_small", [
    ("small_bf16", 8192, 128),     # E = 96: 3 narrow tiles per row block; 64 row blocks take 256-wide tiles
    ("decode_560b", 1024, 128),    # E = 768: 24 narrow tiles; 8 row blocks (192 > 148 SMs) take 256-wide
    ("small_bf16", 8192, 77),      # a ragged small batch (one partly valid row block, M = 64 MMAs)
])
def test_logits_and_routing_do_not_depend_on_the_batch(cuda_ok, name, T_big, T_small):
    w = configs.WORKLOADS[name]
    big = Run(w, T=T_big)
    try:
        big.forward()
        big.check_routing_bitexact()
        for start in (0, T_big - T_small, 300):
            small = Run(w, T=T_small, weights=big.weights, x=big.x[start:start + T_small].contiguous())
            try:
                small.forward()
                rows = slice(start, start + T_small)
                np.testing.assert_array_equal(small.dbg["logits"].view(np.uint32), big.dbg["logits"][rows].view(np.uint32))
                np.testing.assert_array_equal(small.dbg["idx"], big.dbg["idx"][rows])
                np.testing.assert_array_equal(small.dbg["gate"].view(np.uint32), big.dbg["gate"][rows].view(np.uint32))
                np.testing.assert_array_equal(small.y, big.y[rows])
            finally:
                small.close()
    finally:
        big.close()
