"""GPU parity at the full layer sizes, in the launch configuration the benchmark
times: routing, counts and permutation are compared bit for bit over every
token; expert and layer outputs on sampled pairs/tokens that the fp64 oracle
can compute one by one."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_shifted_b200 import configs, synth
from tests.gpu_harness import TOL, Run

pytestmark = pytest.mark.gpu

W = configs.WORKLOADS


def _sample_pairs(r, n, seed=0):
    rng = np.random.default_rng(seed)
    offs = r.dbg["offsets"]
    hit = [e for e in range(r.w.n_ffn) if offs[e + 1] > offs[e]]
    edges = []
    for e in rng.choice(hit, size=min(6, len(hit)), replace=False):
        edges += [int(offs[e]), int(offs[e + 1]) - 1]
        if offs[e + 1] - offs[e] > 128:
            edges += [int(offs[e]) + 127, int(offs[e]) + 128]  # row-block boundary
    rand = rng.choice(r.P, size=min(n, r.P), replace=False).tolist()
    return sorted(set(rand) | set(edges))


@pytest.fixture(scope="module")
def big_weights(cuda_ok):
    w = configs.device_weights(W["prefill_560b"])
    yield w
    del w
    torch.cuda.empty_cache()


def test_generator_device_matches_host(cuda_ok):
    t = torch.empty((1 << 20,), dtype=torch.bfloat16, device="cuda")
    synth.fill_normal_(t, synth.TID_WG, 0, 0.006)
    idx = np.random.default_rng(1).choice(t.numel(), 4096, replace=False).astype(np.uint64)
    host = synth.f32_to_bf16_bits(synth.normal_f32(idx, synth.TID_WG, 0, 0.006))
    dev = t.view(torch.int16).cpu().numpy().view(np.uint16)[idx.astype(np.int64)]
    np.testing.assert_array_equal(dev, host)
    u = torch.empty((100003,), dtype=torch.float32, device="cuda")
    synth.fill_uniform_(u, synth.TID_BIAS, 7, -0.2, 0.2)
    np.testing.assert_array_equal(u.cpu().numpy(), synth.uniform((100003,), synth.TID_BIAS, 7, -0.2, 0.2))


def test_prefill_560b(big_weights):
    r = Run(W["prefill_560b"], weights=big_weights)
    try:
        r.forward()
        r.check_routing_bitexact()
        assert r.check_logits_and_fp64_routing(np.arange(0, r.T, 64)) > 0.2
        r.check_expert_outputs(_sample_pairs(r, 40))
        r.check_layer_outputs([0, 1, 4097, r.T - 1])
        y0 = r.y.copy()
        r.forward(debug=False)
        np.testing.assert_array_equal(r.y, y0)  # bitwise run-to-run determinism
        # uniform routing: ~ k * N / E = 8 FFN experts per token
        assert 7.0 < r.P / r.T < 9.0
    finally:
        r.close()


def test_decode_560b(big_weights):
    r = Run(W["decode_560b"], weights=big_weights)
    try:
        r.forward()
        r.check_routing_bitexact()
        r.check_expert_outputs(_sample_pairs(r, 40, seed=1))
        r.check_layer_outputs([0, 5, 77, r.T - 1])
        zero_frac = 1.0 - r.P / (r.T * r.w.top_k)
        assert 0.2 < zero_frac < 0.45
    finally:
        r.close()


def test_decode_560b_literal_zero_bias(big_weights):
    r = Run(W["decode_560b_zero_bias"], weights=big_weights)
    try:
        r.forward()
        r.check_routing_bitexact()
        assert r.P == 0 and np.all(r.dbg["idx"] >= r.w.n_ffn)
        z = np.zeros(r.T, np.float32)
        for j in range(r.w.top_k):
            z = (z + r.dbg["gate"][:, j]).astype(np.float32)
        x = synth.bf16_bits_to_f32(r.x_host())
        np.testing.assert_array_equal(r.y, synth.f32_to_bf16_bits((z[:, None] * x).astype(np.float32)))
    finally:
        r.close()


def test_skewed_routing_with_bias_control(cuda_ok):
    """Zipf(1.1) logit offsets; 100 x (forward + update_bias) toward 6 FFN experts
    per token.  Every controller step is bit-exact against the oracle given the
    GPU's counts; routing is bit-exact on the first and last step."""
    w = W["skewed_4096"]
    r = Run(w)
    gains = (0.0, 0.02, 0.0, 1.0, w.target_ffn)
    st = oracle.new_controller_state(r.bias)
    traj = []
    try:
        for step in range(w.steps):
            r.x = configs.device_tokens(w, step=step)
            r.cur_bias = st["bias"].copy()
            first_or_last = step in (0, w.steps - 1)
            r.forward(debug=first_or_last)
            if first_or_last:
                r.check_routing_bitexact()
                # the oracle uses the same offsets: its logits include them
                assert r.check_logits_and_fp64_routing(np.arange(0, r.T, 512)) > 0.3
            s = r.layer.state()
            traj.append(float(s["counts"][: w.n_ffn].sum()) / s["tokens"])
            counts = s["counts"].copy()
            tokens = np.array([s["tokens"]], np.int64)
            oracle.update_bias(counts, tokens, w.n_ffn, w.n_zero, w.top_k, gains, r.bias, st)
            r.layer.update_bias(*gains[:4], target_ffn_per_token=gains[4])
            s2 = r.layer.state()
            np.testing.assert_array_equal(s2["bias"].view(np.uint32), st["bias"].view(np.uint32))
        r.check_expert_outputs(_sample_pairs(r, 30, seed=2))
        r.check_layer_outputs([0, 1, r.T // 2, r.T - 1])
        # skew: the busiest expert takes far more than the mean share in the first step
        print("ffn experts per token, first/last step:", traj[0], traj[-1])
        late = float(np.mean(traj[-10:]))
        assert abs(late - w.target_ffn) < abs(traj[0] - w.target_ffn)
    finally:
        r.close()
