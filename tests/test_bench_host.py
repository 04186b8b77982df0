"""Host-side arithmetic of bench.py, on CPU.

The roofline figures the bench reports rest on two functions: the algorithmic
work of one forward (FLOPs and HBM bytes from the realised routing) and the
roofline time max(tensor time, HBM time).  They are checked here against
figures computed by hand, stage by stage, for the three large layer shapes:
- the 560B prefill batch (16384 tokens, d 6144, 512 + 256 experts, inter 2048,
  top-12), at P = 131072 pairs, with all 512 FFN experts hit;
- the decode batch of 128 tokens, with the 442.8 experts that uniform routing
  hits on average;
- the skewed batch (32768 tokens, d 4096, 256 + 128 experts, inter 1024, top-8),
  at 6 FFN picks per token.

The clock record's parser and the check of the recorded DRAM traffic against
the GEMM source hash are covered as well."""
import hashlib
import json
import os
import shutil
import time

import pytest

import bench
from mixture_experts_layer_shifted_b200 import configs

W = configs.WORKLOADS
PEAKS = {"bf16_tflops_sustained": 1668.1, "hbm_gbs": 6547.2}


def _by_stage(T, d, N, Z, inter, P, distinct, wbytes=2):
    """FLOPs: the router GEMM, then per FFN pair the gate, up and down GEMMs.
    Bytes: each expert hit streams its three matrices once; the router weight;
    x read and y written once."""
    E = N + Z
    router = T * E * (2 * d)
    per_pair = 3 * (2 * d * inter)
    flops = router + P * per_pair
    weights = distinct * (inter * d + inter * d + d * inter) * wbytes
    return flops, weights + E * d * 2 + T * d * 2 + T * d * 2


@pytest.mark.parametrize("name,P,distinct,F_quoted,B_quoted,ms_quoted", [
    ("prefill_560b", 131072, 512, 10.05e12, 39.07e9, 6.03),
    ("decode_560b", 1024, 442.8, 78.5e9, 33.45e9, 5.11),
    ("skewed_4096", 196608, 256, 5.05e12, 6.98e9, 3.03),
])
def test_algorithmic_work_and_roofline(name, P, distinct, F_quoted, B_quoted, ms_quoted):
    wl = W[name]
    F, B = bench.algorithmic_work(wl, P, distinct)
    f2, b2 = _by_stage(wl.T, wl.d, wl.n_ffn, wl.n_zero, wl.inter, P, distinct)
    assert F == pytest.approx(f2, rel=1e-12)
    assert B == pytest.approx(b2, rel=1e-12)
    assert F == pytest.approx(F_quoted, rel=3e-3)
    assert B == pytest.approx(B_quoted, rel=3e-3)
    assert bench.roofline_ms(wl, F, B, PEAKS) == pytest.approx(ms_quoted, rel=3e-3)


def test_roofline_picks_the_slower_side():
    wl = W["prefill_560b"]
    F, B = bench.algorithmic_work(wl, 131072, 512)
    t_tensor = 1e3 * F / (PEAKS["bf16_tflops_sustained"] * 1e12)
    t_hbm = 1e3 * B / (PEAKS["hbm_gbs"] * 1e9)
    assert t_tensor > t_hbm   # the prefill shape sits just on the tensor side of the ridge
    assert bench.roofline_ms(wl, F, B, PEAKS) == pytest.approx(t_tensor, rel=1e-12)
    wl = W["decode_560b"]
    F, B = bench.algorithmic_work(wl, 1024, 442.8)
    assert bench.roofline_ms(wl, F, B, PEAKS) == pytest.approx(1e3 * B / (PEAKS["hbm_gbs"] * 1e9), rel=1e-12)


@pytest.mark.parametrize("fmt,wbytes,mult", [("fp8", 1, 2), ("fp4", 0.5 + 1 / 32, 4), ("nvfp4", 0.5 + 1 / 16, 4)])
def test_low_precision_experts(fmt, wbytes, mult):
    """FP8 / MXFP4 / NVFP4 experts: weights stream at 1 / 0.5 bytes per element (codes)
    plus one scale byte per 32 (MXFP4) or 16 (NVFP4) elements, the router and x, y stay
    bf16, and the expert GEMMs run at 2x / 4x / 4x the bf16 rate."""
    wl = W[f"prefill_560b_{fmt}"]
    P, distinct = 131072, 512
    F, B = bench.algorithmic_work(wl, P, distinct)
    f2, b2 = _by_stage(wl.T, wl.d, wl.n_ffn, wl.n_zero, wl.inter, P, distinct, wbytes=wbytes)
    assert (F, B) == (pytest.approx(f2, rel=1e-12), pytest.approx(b2, rel=1e-12))
    p = PEAKS["bf16_tflops_sustained"] * 1e12
    router = 2.0 * wl.T * wl.d * wl.E
    want = 1e3 * max(router / p + (F - router) / (mult * p), B / (PEAKS["hbm_gbs"] * 1e9))
    assert bench.roofline_ms(wl, F, B, PEAKS) == pytest.approx(want, rel=1e-12)


def _line(sm, smax=1965, power_cap=False, reason=None):
    flags = {r: "Not Active" for r in bench.THROTTLE_REASONS + ("sw_power_cap",)}
    if power_cap:
        flags["sw_power_cap"] = "Active"
    if reason:
        flags[reason] = "Active"
    f = ["0", str(sm), str(smax), "812.40", "0x0000000000000004"] + [flags[r] for r in
                                                                     bench.THROTTLE_REASONS + ("sw_power_cap",)]
    return ", ".join(f)


def test_clock_record_unthrottled_and_power_capped():
    c = bench.parse_clock_lines([_line(1965), _line(1950), _line(1957)])
    assert c["sm_mhz"] == 1957 and c["sm_max_mhz"] == 1965 and c["reasons"] == [] and c["samples"] == 3
    assert "rejected" not in c
    c = bench.parse_clock_lines([_line(1100, power_cap=True), _line(1150, power_cap=True), _line(1965)])
    assert c["reasons"] == ["sw_power_cap"] and c["sm_mhz"] == 1150
    assert "rejected" not in c   # the power cap is kept and noted


@pytest.mark.parametrize("reason", bench.THROTTLE_REASONS)
def test_clock_record_rejects_slowdowns(reason):
    c = bench.parse_clock_lines([_line(1965), _line(1400, reason=reason), _line(1965)])
    assert reason in c["reasons"]
    assert reason in c["rejected"]


def test_clock_record_rejects_a_clock_lock():
    c = bench.parse_clock_lines([_line(900), _line(900), _line(910)])
    assert c["reasons"] == [] and "no reason active" in c["rejected"]


def test_clock_record_skips_malformed_lines():
    c = bench.parse_clock_lines(["", "garbage", "0, [N/A], [N/A], 1, 0x0, a, b, c, d", _line(1965)])
    assert c["samples"] == 1 and c["sm_mhz"] == 1965
    c = bench.parse_clock_lines([])
    assert c["sm_mhz"] is None and c["samples"] == 0 and "rejected" not in c


def test_recorded_traffic_follows_the_gemm_source(tmp_path, monkeypatch):
    """The committed DRAM counts apply only while the GEMM source they were taken
    on is unchanged: a one-byte edit of the kernel must drop them."""
    rec = os.path.join(bench.ROOT, "profiles", "gemm_dram_traffic_prefill_560b.json")
    if not os.path.exists(rec):
        pytest.skip("no recorded traffic")
    src = os.path.join(bench.ROOT, "mixture_experts_layer_shifted_b200", "csrc")
    (tmp_path / "profiles").mkdir()
    shutil.copy(rec, tmp_path / "profiles")
    dst = tmp_path / "mixture_experts_layer_shifted_b200" / "csrc"
    dst.mkdir(parents=True)
    for f in ("gemm_tc.cu", "zc_ptx.cuh"):
        shutil.copy(os.path.join(src, f), dst / f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    data = json.load(open(rec))
    h = hashlib.sha256()
    for f in ("gemm_tc.cu", "zc_ptx.cuh"):
        h.update((dst / f).read_bytes())
    t = bench.recorded_traffic("prefill_560b", "gate_up")
    if data["kernel_source_sha256"] == h.hexdigest():
        assert t == data["gate_up"]["dram_read_bytes"] + data["gate_up"]["dram_write_bytes"]
    else:
        assert t is None
    assert bench.recorded_traffic("prefill_560b", "no_such_kernel") is None
    assert bench.recorded_traffic("decode_560b", "gate_up") is None
    with open(dst / "gemm_tc.cu", "ab") as fh:
        fh.write(b"\n")
    assert bench.recorded_traffic("prefill_560b", "gate_up") is None


def test_clock_sampler_with_a_fake_nvidia_smi(tmp_path, monkeypatch):
    """The sampler end to end: a stand-in nvidia-smi on PATH prints two samples
    under the power cap and then waits to be terminated, as the real one does."""
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\n"
                    f"echo '{_line(1200, power_cap=True)}'\n"
                    f"echo '{_line(1300, power_cap=True)}'\n"
                    "exec sleep 30\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    s = bench.ClockSampler(0)
    s.start()
    for _ in range(100):
        if len(s.lines) >= 2:
            break
        time.sleep(0.05)
    c = s.stop()
    assert c["samples"] == 2 and c["sm_mhz"] == 1250 and c["reasons"] == ["sw_power_cap"]
    assert "rejected" not in c


def test_reference_arm_other_ranks_exit_without_work():
    """Under torchrun the reference arm runs on rank 0 alone: any other rank exits 0 at
    once, prints nothing and forms no process group (no rendezvous is reachable here,
    so joining one would fail or hang)."""
    import subprocess
    import sys
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1", MASTER_PORT="9")
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
