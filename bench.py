"""Benchmark of the zero-computation-expert MoE layer forward on B200.

One step = one pass of the whole hot path over one batch: router GEMM +
softmax/top-k + integer stage + row scatter + grouped gate/up GEMM + grouped down
GEMM + combine (zcmoe_forward), then the bias controller step
(zcmoe_update_bias; with N > 1 ranks the selection counts are summed over the
ranks with one NCCL all-reduce first, so every replica takes the same step).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl zcmoe|reference]

Prints one JSON line (rank 0).  Inputs are seeded synthetic tensors made on the
device; the weights (tens of GB) and the token batch are far larger than the
126 MB L2, so no flush is needed between steps.  ``--impl reference`` times the
CPU oracle on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ZC-MoE layer tokens/s on 1 B200; % of BF16 tensor / HBM roofline"
DEFAULT_WORKLOAD = "prefill_560b"
GAINS = dict(kp=0.0, ki=0.02, kd=0.0, decay=1.0)


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks/throttle sampling while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        return parse_clock_lines(self.lines)


THROTTLE_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def parse_clock_lines(lines):
    """Summary of nvidia-smi samples in ClockSampler.FIELDS order (csv, no header,
    no units): median SM clock, the max SM clock, every throttle reason seen
    active, and `rejected` when the record disqualifies the timed region — a
    hardware or thermal slowdown, or an SM clock far below its max with no
    reason active (a clock lock left by someone else).  sw_power_cap is normal
    for a 1 kW part under dense GEMMs and is only listed."""
    sm, smax, reasons = [], None, set()
    names = THROTTLE_REASONS + ("sw_power_cap",)
    for line in lines:
        f = [v.strip() for v in line.split(",")]
        if len(f) < 9:
            continue
        try:
            sm.append(float(f[1]))
            smax = float(f[2])
        except ValueError:
            continue
        for n, v in zip(names, f[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
           "samples": len(sm)}
    bad = [r for r in THROTTLE_REASONS if r in reasons]
    if bad:
        out["rejected"] = "throttled: " + ", ".join(bad)
    elif sm and smax and not reasons and out["sm_mhz"] < 0.6 * smax:
        out["rejected"] = f"SM clock {out['sm_mhz']:.0f} of {smax:.0f} MHz with no reason active"
    return out


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
        return dist, dist.get_rank(), ws, local
    return None, 0, 1, 0


def recorded_traffic(workload, kernel):
    """DRAM bytes per launch from the committed ncu capture, or None when the
    GEMM source changed since the capture (the counters no longer apply)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"gemm_dram_traffic_{workload}.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path))
    h = hashlib.sha256()
    for f in ("gemm_tc.cu", "zc_ptx.cuh"):
        h.update(open(os.path.join(ROOT, "mixture_experts_layer_shifted_b200", "csrc", f), "rb").read())
    if rec.get("kernel_source_sha256") != h.hexdigest() or kernel not in rec:
        return None
    return rec[kernel]["dram_read_bytes"] + rec[kernel]["dram_write_bytes"]


def algorithmic_work(wl, P, distinct):
    """FLOPs and bytes per forward from the realised routing: P FFN pairs and
    `distinct` FFN experts hit.  F = 2 T d E + 6 d inter P;
    B = distinct * 3 d inter * w + E d * 2 + 2 T d * 2 (bf16; expert weights w = 2
    bytes per element, 1 for FP8 experts, 0.5 + 1/32 for MXFP4 (codes + one scale byte
    per 32) and 0.5 + 1/16 for NVFP4 (one per 16); fp32 layers 4 throughout)."""
    esz = 4 if wl.dtype == "f32" else 2
    wsz = {"fp8": 1, "fp4": 0.5 + 1 / 32, "nvfp4": 0.5 + 1 / 16}.get(wl.dtype, esz)
    F = 2.0 * wl.T * wl.d * wl.E + 6.0 * wl.d * wl.inter * P
    B = distinct * 3.0 * wl.d * wl.inter * wsz + wl.E * wl.d * esz + 2.0 * wl.T * wl.d * esz
    return F, B


def roofline_ms(wl, F, B, peaks):
    """max(tensor time, HBM time); FP8 experts at twice the measured bf16 rate (the
    nominal 4.5 / 2.25 PFLOP/s ratio), the router in bf16."""
    p = peaks["bf16_tflops_sustained"] * 1e12
    f_router = 2.0 * wl.T * wl.d * wl.E
    mult = {"fp8": 2, "fp4": 4, "nvfp4": 4}.get(wl.dtype, 1)
    t_tensor = f_router / p + (F - f_router) / (mult * p)
    return 1e3 * max(t_tensor, B / (peaks["hbm_gbs"] * 1e9))


def to_host_bits(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return t.contiguous().cpu().numpy()


def cpu_oracle_sample(wl, weights, x, bias, offset, n_tokens, min_s=10.0):
    """Times the oracle on the first tokens of the batch (router, routing, experts,
    combine) with the weights it needs already on the host, repeating the sample
    until at least min_s seconds of CPU work.  Returns (tokens, seconds, cores)."""
    import oracle
    import torch
    cores = len(os.sched_getaffinity(0))
    xs = to_host_bits(x[:n_tokens])
    wr = to_host_bits(weights[0])
    # routing first (cheap) to learn which experts the sample needs; fetch them before timing
    l = oracle.router_logits(xs, wr, offset)
    idx, gate, _ = oracle.topk(oracle.softmax(l), bias.astype(np.float64), wl.top_k)
    need = sorted({int(e) for e in idx.ravel() if e < wl.n_ffn})
    cache = {e: tuple(to_host_bits(w[e]) for w in weights[1:]) for e in need}
    efn = None
    if wl.dtype == "fp8":  # weights quantized once, as the layer does at create
        q8 = {e: [oracle.quantize_blocks(w, 128) for w in cache[e]] for e in need}
        efn = lambda e, rows: oracle.ffn_fp8(rows, [c for c, _ in q8[e]], [s_ for _, s_ in q8[e]])
    elif wl.dtype == "fp4":
        q4 = {e: [oracle.quantize_mx4(w) for w in cache[e]] for e in need}
        efn = lambda e, rows: oracle.ffn_fp4(rows, [c for c, _ in q4[e]], [s_ for _, s_ in q4[e]])
    elif wl.dtype == "nvfp4":
        qn = {e: [oracle.quantize_weight_nv4(w) for w in cache[e]] for e in need}
        efn = lambda e, rows: oracle.ffn_nv4(rows, [c for c, _, _ in qn[e]], [s_ for _, s_, _ in qn[e]],
                                             [g_ for _, _, g_ in qn[e]])
    done = 0
    t0 = time.perf_counter()
    while True:  # the sample is processed again until the time budget is spent
        for t in range(n_tokens):
            l = oracle.router_logits(xs[t:t + 1], wr, offset)
            i1, g1, _ = oracle.topk(oracle.softmax(l), bias.astype(np.float64), wl.top_k)
            oracle.layer_outputs(xs[t:t + 1], i1, g1, wl.n_ffn, lambda e: cache[e], expert_fn=efn)
            done += 1
        if time.perf_counter() - t0 > min_s:
            break
    dt = time.perf_counter() - t0
    del cache
    torch.cuda.empty_cache()
    return done, dt, cores


def run_reference(args, wl, rank, ws):
    """Reference arm: the CPU oracle, timed on the host cores on a bounded sample per step."""
    if rank != 0:
        return
    import torch
    from mixture_experts_layer_shifted_b200 import configs
    weights = configs.device_weights(wl)
    x = configs.device_tokens(wl)
    bias = configs.bias_vector(wl)
    offset = configs.logit_offsets(wl)
    per_step = 4 if wl.d >= 4096 else 16
    for _ in range(args.warmup):
        cpu_oracle_sample(wl, weights, x, bias, offset, 1, min_s=0.0)
    tot_tok, tot_s, cores = 0, 0.0, 1
    for _ in range(args.steps):
        n, s, cores = cpu_oracle_sample(wl, weights, x, bias, offset, per_step, min_s=0.0)
        tot_tok += n
        tot_s += s
    v = tot_tok / tot_s
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "T": wl.T, "d": wl.d, "n_ffn": wl.n_ffn, "n_zero": wl.n_zero,
                       "inter": wl.inter, "top_k": wl.top_k, "parallelism": "dp1"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{per_step} tokens per step of the {wl.name} batch, full layer in fp64"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def measure_overlap(wl, layer, x, stream, peaks, reps=10):
    """The dense FFN path beside the layer on the same batch (shortcut-connected
    MoE): device time of the layer alone, the dense FFN alone, the two one after
    the other, and the two through zcmoe_forward_overlap; each a replayed graph."""
    import torch
    from mixture_experts_layer_shifted_b200 import configs
    from mixture_experts_layer_shifted_b200.zcmoe import ZcDense, forward_overlap

    dense = ZcDense(*configs.device_dense_weights(wl), max_tokens=wl.T)
    y, yd = torch.empty_like(x), torch.empty_like(x)
    variants = {
        "moe": lambda: layer.forward(x, y),
        "dense": lambda: dense.forward(x, yd),
        "sequential": lambda: (layer.forward(x, y), dense.forward(x, yd)),
        "overlap": lambda: forward_overlap(layer, dense, x, y_moe=y, y_dense=yd),
    }
    ms = {}
    for name, fn in variants.items():
        fn()  # first calls outside the capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        ms[name] = a.elapsed_time(b) / reps
        del g
    dense.check()
    layer.check()
    dense.close()
    f_dense = 6.0 * wl.T * wl.d * wl.dense_inter
    hidden = ms["sequential"] - ms["overlap"]
    tflops = f_dense / (ms["dense"] * 1e-3) / 1e12
    return {"dense_inter": wl.dense_inter, "ms_moe": ms["moe"], "ms_dense": ms["dense"],
            "ms_sequential": ms["sequential"], "ms_overlap": ms["overlap"], "hidden_ms": hidden,
            "hidden_frac_of_dense": hidden / ms["dense"], "speedup": ms["sequential"] / ms["overlap"],
            "dense_tflops": tflops, "dense_frac": tflops / peaks["bf16_tflops_sustained"],
            "note": "each variant one replayed CUDA graph, %d replays after 3; same batch for both paths" % reps}


def graph_ms(fn, stream, reps=10):
    """Device time of fn() as one replayed CUDA graph (first call outside the capture)."""
    import torch
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / reps


def measure_lowp(layer, weights, x, stream, peaks, fmt="fp8"):
    """The same layer with block-scaled FP8 or W4A4 (MXFP4) experts, on the same weights
    and batch: forward time against the bf16 layer, the expert GEMMs against the
    format's peak (2x or 4x the measured sustained bf16 peak, the nominal 4.5 and
    9 PFLOP/s against 2.25), and the decode batch against HBM."""
    import torch
    from mixture_experts_layer_shifted_b200 import configs
    from mixture_experts_layer_shifted_b200.zcmoe import LayerShape, ZcMoE

    out = {}
    mult = 2 if fmt == "fp8" else 4
    for name, layer_b in ((f"prefill_560b_{fmt}", layer), (f"decode_560b_{fmt}", None)):
        wf = configs.WORKLOADS[name]
        xf = x if layer_b is not None else configs.device_tokens(wf)
        shp = LayerShape(wf.d, wf.n_ffn, wf.n_zero, wf.inter, wf.top_k, fmt)
        l8 = ZcMoE(shp, *weights, max_tokens=wf.T, init_bias=configs.bias_vector(wf),
                   logit_offset=configs.logit_offsets(wf))
        lb = layer_b
        if lb is None:
            lb = ZcMoE(LayerShape(wf.d, wf.n_ffn, wf.n_zero, wf.inter, wf.top_k, "bf16"), *weights,
                       max_tokens=wf.T, init_bias=configs.bias_vector(wf), logit_offset=configs.logit_offsets(wf))
        y8, yb = torch.empty_like(xf), torch.empty_like(xf)
        ms8 = graph_ms(lambda: l8.forward(xf, y8), stream)
        msb = graph_ms(lambda: lb.forward(xf, yb), stream)
        offs = torch.empty((wf.n_ffn + 1,), dtype=torch.int32, device=xf.device)
        l8.forward(xf, y8, debug={"offsets": offs})
        torch.cuda.synchronize()
        cnt = np.diff(offs.cpu().numpy())
        P, distinct = int(cnt.sum()), int((cnt > 0).sum())
        F, B = algorithmic_work(wf, P, distinct)
        l8.profile_begin()
        for _ in range(5):
            l8.forward(xf, y8)
        st, nf = l8.profile_end()
        st = {k_: v / nf for k_, v in st.items()}
        p8 = mult * peaks["bf16_tflops_sustained"]
        gu = 4.0 * wf.d * wf.inter * P / (st["gate_up"] * 1e-3) / 1e12
        dn = 2.0 * wf.d * wf.inter * P / (st["down"] * 1e-3) / 1e12
        rec = {"tokens_per_s": wf.T / (ms8 * 1e-3), "ms_per_forward": ms8, "bf16_ms_per_forward": msb,
               "speedup_vs_bf16": msb / ms8, "stage_ms": st,
               "gate_up": {"tflops": gu, "frac_peak": gu / p8},
               "down": {"tflops": dn, "frac_peak": dn / p8},
               "layer_roofline_ms": roofline_ms(wf, F, B, peaks), "P": P}
        if layer_b is None:
            rec["hbm_gbs"] = B / (ms8 * 1e-3) / 1e9
            rec["hbm_frac"] = rec["hbm_gbs"] / peaks["hbm_gbs"]
            lb.close()
        l8.check()
        l8.close()
        out[name] = rec
    out["peak_note"] = (f"{fmt} dense peak = {mult} x measured sustained bf16 "
                        f"(nominal {'4.5' if mult == 2 else '9'}/2.25 PFLOP/s ratio)")
    return out


def measure_backward(wl, layer, x, stream, peaks, P):
    """zcmoe_backward after a forward of the same batch, in training mode (the forward
    stores G and U; the backward reads them): dx only, and dx plus the four weight
    gradients added into fp32 accumulators (fused GemmAdd); each a replayed graph.
    Also the recomputing backward (training mode off) and the forward's cost of storing."""
    import torch
    g = torch.Generator(device=x.device).manual_seed(11)
    dy = (torch.randn(x.shape, generator=g, device=x.device) * 0.05).to(torch.bfloat16)
    dx = torch.empty_like(x)
    y = torch.empty_like(x)
    layer.forward(x, y)
    ms_dx_recompute = graph_ms(lambda: layer.backward(x, dy, dx), stream)
    ms_fwd = graph_ms(lambda: layer.forward(x, y), stream)
    layer.save_for_backward(True)
    ms_fwd_saving = graph_ms(lambda: layer.forward(x, y), stream)
    layer.forward(x, y)
    ms_dx = graph_ms(lambda: layer.backward(x, dy, dx), stream)
    grads = {"router": torch.zeros((wl.E, wl.d), device=x.device),
             "gate": torch.zeros((wl.n_ffn, wl.inter, wl.d), device=x.device),
             "up": torch.zeros((wl.n_ffn, wl.inter, wl.d), device=x.device),
             "down": torch.zeros((wl.n_ffn, wl.d, wl.inter), device=x.device)}
    ms_full = graph_ms(lambda: layer.backward(x, dy, dx, grads=grads), stream, reps=3)
    ms_full_ow = graph_ms(lambda: layer.backward(x, dy, dx, grads=grads, accumulate=False), stream, reps=3)
    layer.check()
    ok = all(bool(torch.isfinite(t).all()) for t in grads.values())
    del grads
    layer.save_for_backward(False)
    torch.cuda.empty_cache()
    dpi = float(wl.d) * wl.inter * P
    f_dx = 6.0 * dpi + 2.0 * wl.T * wl.E * wl.d       # dH, dX, router dx
    f_w = 6.0 * dpi + 2.0 * wl.T * wl.E * wl.d        # dW_d, dW_g, dW_u, dW_r
    acc_bytes = 8.0 * (3 * wl.n_ffn * wl.inter * wl.d + wl.E * wl.d)  # fp32 read + write of the accumulators
    return {"ms_dx_only": ms_dx, "ms_with_weight_grads": ms_full, "tflops_dx_only": f_dx / (ms_dx * 1e-3) / 1e12,
            "tflops_total": (f_dx + f_w) / (ms_full * 1e-3) / 1e12, "gemmadd_accumulator_bytes": acc_bytes,
            "gemmadd_hbm_ms": 1e3 * acc_bytes / (peaks["hbm_gbs"] * 1e9), "finite": ok,
            "ms_with_weight_grads_overwrite": ms_full_ow, "ms_dx_only_recompute": ms_dx_recompute, "ms_forward": ms_fwd, "ms_forward_saving_gu": ms_fwd_saving,
            "note": "training mode (forward stores G, U); weight gradients added into fp32 accumulators "
                    "(3 x 25.8 GB + router); each a replayed graph"}


def run_ep(args, wl, dist, rank, ws, local, peaks):
    """--ep: the expert-parallel layer (ep.py): rank r holds FFN experts [r N/ws, (r+1) N/ws)
    and routes its own batch of wl.T tokens; dispatch and combine are NCCL all-to-alls (one
    GPU: copies), two token chunks.  A step = forward + the shared controller step.  Eager
    launches (the all-to-all split sizes go through the host)."""
    import torch
    from mixture_experts_layer_shifted_b200 import configs
    from mixture_experts_layer_shifted_b200.ep import CudaStages, EpMoE, LocalComm, TorchComm
    from mixture_experts_layer_shifted_b200.zcmoe import LayerShape

    dev = torch.device("cuda", local)
    shape = LayerShape(wl.d, wl.n_ffn, wl.n_zero, wl.inter, wl.top_k, "bf16")
    if wl.n_ffn % ws:
        raise SystemExit(f"--ep needs n_ffn ({wl.n_ffn}) to be a multiple of the GPU count")
    NL = wl.n_ffn // ws
    full = configs.device_weights(wl)
    sl = slice(rank * NL, (rank + 1) * NL)
    wr = full[0]
    wg, wu, wd = (t[sl].clone() for t in full[1:])
    keep_full = ws == 1 and not args.no_cpu_baseline  # the oracle sample reads them
    if not keep_full:
        del full
        torch.cuda.empty_cache()
    comm = TorchComm() if dist else LocalComm()
    # rows one chunk's experts call may receive: twice a chunk's own FFN pairs (about 3x the balanced share)
    # chunks per step: the pages cut the layer in two so that one chunk's exchange overlaps the
    # other's experts; a one-rank group has no exchange to hide, so it runs one chunk unless asked
    nck = max(1, args.ep_chunks if args.ep_chunks > 0 else (2 if ws > 1 else 1))
    cap = 2 * wl.T * wl.top_k // nck
    layer = EpMoE(shape, wr, wg, wu, wd, max_tokens=wl.T, comm=comm, chunks=nck, max_recv_rows=cap,
                  init_bias=configs.bias_vector(wl), logit_offset=configs.logit_offsets(wl))
    # the expert stage timed with events on the launch stream
    ev_pairs, recv_rows = [], []

    class TimedStages(CudaStages):
        def experts(self, xrecv, counts):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            y = super().experts(xrecv, counts)
            b.record()
            ev_pairs.append((a, b))
            recv_rows.append(int(xrecv.shape[0]))
            return y

    layer.stages = [TimedStages(lay) for lay in layer.layers]
    xs = [configs.device_tokens(wl, step=rank * 4 + i) for i in range(2)]
    target = wl.target_ffn if wl.target_ffn is not None else wl.top_k * wl.n_ffn / wl.E
    red = (lambda t: dist.all_reduce(t, op=dist.ReduceOp.SUM)) if dist else None

    def step(i):
        y = layer.forward(xs[i % 2])
        layer.controller_step(all_reduce=red, target_ffn_per_token=target, **GAINS)
        return y

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    ev_pairs.clear()
    recv_rows.clear()
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1)
    exp_ms = sum(a.elapsed_time(b) for a, b in ev_pairs) / args.steps
    exp_rows = sum(recv_rows) / args.steps
    if dist:
        t = torch.tensor([ms, exp_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, exp_ms = float(t[0]), float(t[1])
    value = wl.T * ws * args.steps / (ms / 1e3)
    # end to end: x from pinned host memory, y back to it, every step
    xh = xs[0].cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, min(args.steps, 10))
    a.record(stream)
    for _ in range(n_e2e):
        xd = xh.to(dev, non_blocking=True)
        yh.copy_(layer.forward(xd), non_blocking=True)
        layer.controller_step(all_reduce=red, target_ffn_per_token=target, **GAINS)
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / n_e2e
    if dist:
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    io = xh.numel() * xh.element_size()
    flops = 6.0 * wl.d * wl.inter * exp_rows
    peak = peaks["bf16_tflops_sustained"]
    achieved = flops / (exp_ms * 1e-3) / 1e12 if exp_ms > 0 else 0.0
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        n_tok = 8 if wl.d >= 4096 else 64
        n, sec, cores = cpu_oracle_sample(wl, full, xs[0], configs.bias_vector(wl), configs.logit_offsets(wl), n_tok,
                                          min_s=12.0)
        cpu = {"value": n / sec, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"first {n_tok} tokens of the {wl.name} batch, {n} tokens in {sec:.1f} s"}
    for lay in layer.layers:
        lay.check()
    layer.close()
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Philox, random-init weights)",
            "config": {"workload": wl.name, "T_per_rank": wl.T, "d": wl.d, "n_ffn": wl.n_ffn, "n_zero": wl.n_zero,
                       "inter": wl.inter, "top_k": wl.top_k, "parallelism": f"ep{ws}", "chunks": nck,
                       "l2": "inputs larger than L2; no flush"},
            "roofline": {"bound": "tensor", "kernel": "zcmoe_ep_experts (regroup + grouped gate/up + down)",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "traffic": None, "peak_kind": f"bf16 dense, sustained, {peaks['source']}",
                         "per_launch": {"flops": flops, "ms": exp_ms, "units": f"{exp_rows:.0f} received rows x 6 d inter per step"}},
            "cpu_baseline": cpu,
            "e2e": {"value": wl.T * ws / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": io,
                    "d2h_bytes_per_step": io, "ms_per_step": e2e_ms},
            # per chunk: router GEMM, softmax/top-k, the integer stage (one kernel up to 1024 tokens,
            # else three), the row scatter, the two expert GEMMs (+ 2 regroups with ws > 1), combine;
            # per step one bias update per chunk handle
            "gpu_launches": args.steps * (nck * (6 + (1 if wl.T // nck <= 1024 else 3) + (2 if ws > 1 else 0)) + nck),
            "clocks": clocks, "peaks": peaks,
            "launch": "eager (host-side split sizes)"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="zcmoe", choices=["zcmoe", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--secondary", default="decode,fp8,fp4,nvfp4,backward,overlap",
                    help="comma list of the secondary measurements to run after the headline")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism over the GPUs (ep.py) instead of data-parallel replicas")
    ap.add_argument("--ep-chunks", type=int, default=0,
                    help="--ep: token chunks per step (default: 2 with more than one rank, 1 with one)")
    ap.add_argument("--eager", action="store_true",
                    help="launch every step eagerly instead of replaying one captured CUDA graph (N=1)")
    args = ap.parse_args()
    sec = set() if args.no_secondary else {s_.strip() for s_ in args.secondary.split(",") if s_.strip()}
    unknown = sec - {"decode", "fp8", "fp4", "nvfp4", "backward", "overlap"}
    if unknown:
        ap.error(f"unknown secondary measurement(s): {sorted(unknown)}")
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        # the CPU oracle runs on rank 0 alone; the other ranks exit 0 without work, and no
        # process group is formed (nothing would be exchanged)
        rank, ws = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))
        if rank != 0:
            return
        import torch
        from mixture_experts_layer_shifted_b200 import configs
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        run_reference(args, configs.WORKLOADS[args.workload], rank, ws)
        return

    import torch
    from mixture_experts_layer_shifted_b200 import configs
    from mixture_experts_layer_shifted_b200.dp import controller_step
    from mixture_experts_layer_shifted_b200.zcmoe import LayerShape, ZcMoE

    dist, rank, ws, local = _dist()
    wl = configs.WORKLOADS[args.workload]

    peaks = _peaks()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.ep:
        run_ep(args, wl, dist, rank, ws, local, peaks)
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return
    weights = configs.device_weights(wl)
    xs = [configs.device_tokens(wl, step=rank * 4 + i) for i in range(2)]
    bias = configs.bias_vector(wl)
    offset = configs.logit_offsets(wl)
    shape = LayerShape(wl.d, wl.n_ffn, wl.n_zero, wl.inter, wl.top_k, wl.dtype)
    layer = ZcMoE(shape, *weights, max_tokens=wl.T, init_bias=bias, logit_offset=offset)
    y = torch.empty_like(xs[0])
    counts_buf = torch.empty(wl.E + 1, dtype=torch.int64, device=dev)
    target = wl.target_ffn if wl.target_ffn is not None else wl.top_k * wl.n_ffn / wl.E
    stream = torch.cuda.current_stream()

    def step(i):
        layer.forward(xs[i % 2], y)
        if dist:
            controller_step(layer, counts_buf, target_ffn_per_token=target, **GAINS)
        else:
            layer.update_bias(target_ffn_per_token=target, **GAINS)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    layer.check()
    use_graph = not dist and not args.eager
    if use_graph:
        # one step (forward on each of the two batches + bias update) captured once;
        # replays launch the same kernels with no host work in between
        graphs = []
        for i in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(i)
            graphs.append(g)
        torch.cuda.synchronize()

        def step(i):  # noqa: F811
            graphs[i % 2].replay()

    # ---------------------------------------------------------------- timed region (device time)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    ms = ev0.elapsed_time(ev1)
    if dist:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    layer.check()
    tokens = wl.T * ws * args.steps
    value = tokens / (ms / 1e3)

    # ---------------------------------------------------------------- realised routing of one batch
    E, k = wl.E, wl.top_k
    idx = torch.empty((wl.T, k), dtype=torch.int32, device=dev)
    offs = torch.empty((wl.n_ffn + 1,), dtype=torch.int32, device=dev)
    layer.forward(xs[0], y, debug={"idx": idx, "offsets": offs})
    torch.cuda.synchronize()
    cnt = np.diff(offs.cpu().numpy())
    P = int(cnt.sum())
    distinct = int((cnt > 0).sum())
    F, B = algorithmic_work(wl, P, distinct)

    # ---------------------------------------------------------------- per-stage device time (events on the launch stream)
    layer.profile_begin()
    nprof = max(3, min(args.steps, 10))
    for i in range(nprof):
        layer.forward(xs[i % 2], y)
    stage_ms, nf = layer.profile_end()
    stage_avg = {s: v / nf for s, v in stage_ms.items()}
    gu_ms = stage_avg["gate_up"]
    gu_flops = 4.0 * wl.d * wl.inter * P
    fp8 = wl.dtype in ("fp8", "fp4", "nvfp4")
    mult = {"fp8": 2, "fp4": 4, "nvfp4": 4}.get(wl.dtype, 1)
    tensor_peak = peaks["bf16_tflops_sustained"] * mult
    achieved = gu_flops / (gu_ms * 1e-3) / 1e12
    kname = (f"grouped {wl.dtype.upper()} gate/up GEMM + SwiGLU + quantize (k_fp8_gemm<1>)" if fp8
             else "grouped gate/up GEMM + SwiGLU (k_tc_gemm<1>)")
    roofline = {"bound": "tensor", "kernel": kname, "achieved": achieved,
                "peak": tensor_peak, "unit": "TFLOP/s", "frac": achieved / tensor_peak,
                "traffic": None if fp8 else recorded_traffic(wl.name, "gate_up"),
                "peak_kind": (f"{wl.dtype} dense = {mult} x bf16 dense sustained ({peaks['source']}; nominal ratio)" if fp8
                              else f"bf16 dense, sustained, {peaks['source']}"),
                "per_launch": {"flops": gu_flops, "ms": gu_ms, "units": f"{P} FFN (token, expert) pairs x 4 d inter"}}
    fwd_ms = sum(stage_avg.values())
    t_roof_ms = roofline_ms(wl, F, B, peaks)
    layer_roof = {"forward_ms": fwd_ms, "roofline_ms": t_roof_ms, "frac": t_roof_ms / fwd_ms,
                  "flops": F, "bytes": B, "stage_ms": stage_avg,
                  "down": {"ms": stage_avg["down"],
                           "tflops": 2.0 * wl.d * wl.inter * P / (stage_avg["down"] * 1e-3) / 1e12}}

    # ---------------------------------------------------------------- e2e through host buffers (C ABI, pinned)
    # pipelined: step i's y download and step i+1's x upload run beside the forwards; the
    # flush before the closing event waits for the last download
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty_like(xh[0]).pin_memory() for _ in range(2)]
    for i in range(2):
        layer.forward_host(xh[i], yh[i], pipelined=True)
    layer.flush_host()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, min(args.steps, 10))
    e0.record(stream)
    for i in range(n_e2e):
        layer.forward_host(xh[i % 2], yh[i % 2], pipelined=True)
        layer.update_bias(target_ffn_per_token=target, **GAINS)
    layer.flush_host()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / n_e2e
    if dist:
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    io_bytes = xh[0].numel() * xh[0].element_size()
    e2e = {"value": wl.T * ws / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": io_bytes,
           "d2h_bytes_per_step": io_bytes, "ms_per_step": e2e_ms}

    # ---------------------------------------------------------------- CPU oracle baseline (rank 0, N = 1)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        n_tok = 8 if wl.d >= 4096 else 64
        n, s, cores = cpu_oracle_sample(wl, weights, xs[0], bias, offset, n_tok, min_s=12.0)
        cpu = {"value": n / s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"first {n_tok} tokens of the {wl.name} batch, processed {n // n_tok} times ({n} tokens, "
                         f"{s:.1f} s): fp64 router, routing, experts and combine; the needed expert weights "
                         f"copied to the host beforehand, not timed"}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic (seeded Philox, random-init weights)",
            "config": {"workload": wl.name, "T": wl.T, "d": wl.d, "n_ffn": wl.n_ffn, "n_zero": wl.n_zero,
                       "inter": wl.inter, "top_k": wl.top_k, "parallelism": f"dp{ws}",
                       "l2": "inputs larger than L2 (weights %.1f GB, x %.0f MB); no flush" %
                             (wl.weight_bytes() / 1e9, xs[0].numel() * xs[0].element_size() / 1e6),
                       "realised": {"P": P, "ffn_per_token": P / wl.T, "distinct_experts": distinct,
                                    "zero_fraction": 1.0 - P / (wl.T * k)}},
            "roofline": roofline, "layer_roofline": layer_roof, "cpu_baseline": cpu, "e2e": e2e,
            # router GEMM, softmax/top-k, the integer stage (one kernel up to 1024 tokens, else
            # three), the row scatter (or quantizing gather), gate/up, down, combine, bias update
            "gpu_launches": (7 + (1 if wl.T <= 1024 else 3)) * args.steps, "clocks": clocks, "peaks": peaks,
            "launch": "cuda graph per step" if use_graph else "eager"}

    # the controller over the workload's steps (Zipf-skewed routing): FFN experts per token per
    # step, from a fresh layer, a batch per step; outside the timed region (reads counts each step)
    if rank == 0 and ws == 1 and wl.steps > 1:
        ctl = ZcMoE(shape, *weights, max_tokens=wl.T, init_bias=bias, logit_offset=offset)
        traj = []
        yc = torch.empty_like(xs[0])
        for i in range(wl.steps):
            ctl.forward(configs.device_tokens(wl, step=i), yc)
            st = ctl.state()
            traj.append(float(st["counts"][: wl.n_ffn].sum()) / st["tokens"])
            ctl.update_bias(target_ffn_per_token=target, **GAINS)
        ctl.check()
        ctl.close()
        line["controller"] = {"target_ffn_per_token": target, "steps": wl.steps, "gains": GAINS,
                              "ffn_per_token_first": traj[0], "ffn_per_token_last": traj[-1],
                              "ffn_per_token_mean_last10": float(np.mean(traj[-10:])),
                              "trajectory_every_10": traj[::10]}

    # secondary workload (decode): reported beside the headline, not as the headline
    if rank == 0 and ws == 1 and "decode" in sec and wl.name == "prefill_560b":
        wd = configs.WORKLOADS["decode_560b"]
        xd = configs.device_tokens(wd)
        layer2 = ZcMoE(LayerShape(wd.d, wd.n_ffn, wd.n_zero, wd.inter, wd.top_k, wd.dtype), *weights,
                       max_tokens=wd.T, init_bias=configs.bias_vector(wd))
        yd = torch.empty_like(xd)
        for _ in range(5):
            layer2.forward(xd, yd)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        nd = 20
        a.record(stream)
        for _ in range(nd):
            layer2.forward(xd, yd)
        b.record(stream)
        torch.cuda.synchronize()
        dms = a.elapsed_time(b) / nd
        offs2 = torch.empty((wd.n_ffn + 1,), dtype=torch.int32, device=dev)
        layer2.forward(xd, yd, debug={"offsets": offs2})
        cnt2 = np.diff(offs2.cpu().numpy())
        F2, B2 = algorithmic_work(wd, int(cnt2.sum()), int((cnt2 > 0).sum()))
        hbm = B2 / (dms * 1e-3) / 1e9
        line["decode"] = {"workload": wd.name, "tokens_per_s": wd.T / (dms * 1e-3), "ms_per_forward": dms,
                          "hbm_gbs": hbm, "hbm_frac": hbm / peaks["hbm_gbs"], "bytes": B2,
                          "P": int(cnt2.sum()), "distinct_experts": int((cnt2 > 0).sum())}
        layer2.close()

    # secondary: the same layer with block-scaled FP8 experts (bf16 headline unchanged)
    if rank == 0 and ws == 1 and wl.name == "prefill_560b":
        for fmt in ("fp8", "fp4", "nvfp4"):
            if fmt in sec:
                line[fmt] = measure_lowp(layer, weights, xs[0], stream, peaks, fmt)

    # secondary: the backward pass (training) of the same batch
    if rank == 0 and ws == 1 and "backward" in sec and wl.dtype == "bf16":
        line["backward"] = measure_backward(wl, layer, xs[0], stream, peaks, P)

    # secondary: the dense FFN path run beside the layer (shortcut-connected MoE)
    if rank == 0 and ws == 1 and "overlap" in sec and wl.dense_inter > 0:
        line["scmoe_overlap"] = measure_overlap(wl, layer, xs[0], stream, peaks)

    layer.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
