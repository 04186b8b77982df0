"""The oracle's pins, tested by planted mistakes.

A pin is worth something only if a plausible mistake in the oracle makes it
fail.  Each case below copies oracle/zcmoe_oracle.c and plants one such mistake
in the copy: a dropped term, a wrong sign, an index off by one, a transposed
operand, a changed rounding or tie rule.  The copy is built the way the oracle
is built, and tests/test_oracle_pins.py runs against it (oracle.use_library, in
worker processes that each take a share of the copies).

The second test does the same for the oracle's Python glue (oracle/__init__.py):
each mistake goes into a copy of the package, which a worker imports in place of
the repository's.

Every mutant must fail at least one pin.  An unchanged copy built the same way
must pass them all, so a broken harness cannot pass for a caught mutant.  The
mistakes live only in the temporary copies, on the CPU."""
import concurrent.futures
import json
import os
import shutil
import subprocess
import sys

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "zcmoe_oracle.c")
PY_SRC = os.path.join(ROOT, "oracle", "__init__.py")

# (name, text in the source, replacement, which occurrence)
MUTANTS = [
    # router logits and softmax
    ("logit offset dropped", "if (offset) acc += (double)offset[e];", "if (offset) acc += 0.0;", 0),
    ("router operand transposed", "elem(wr, w_dtype, (int64_t)e * d + c)", "elem(wr, w_dtype, (int64_t)c * E + e)", 0),
    ("softmax sum skips expert 0", "for (int e = 0; e < E; ++e) sum += exp(lt[e] - m);",
     "for (int e = 1; e < E; ++e) sum += exp(lt[e] - m);", 0),
    # top-k and gates
    ("ties to the higher index", "if (best < 0 || v > bv) { best = e; bv = v; } /* strict",
     "if (best < 0 || v >= bv) { best = e; bv = v; } /* strict", 0),
    ("bias in the gate", "gate[t * k + j] = scale * st[best];", "gate[t * k + j] = scale * bv;", 0),
    ("bias ignored in selection", "double v = key64(st[e] + (bias ? bias[e] : 0.0));\n        if (best < 0",
     "double v = key64(st[e]);\n        if (best < 0", 0),
    ("routed scale dropped", "gate[t * k + j] = scale * st[best];", "gate[t * k + j] = st[best];", 0),
    # fp32 replica
    ("replica ties to the higher index", "float v = key32(u[e] + (bias ? bias[e] : 0.0f));\n        if (best < 0 || v > bv)",
     "float v = key32(u[e] + (bias ? bias[e] : 0.0f));\n        if (best < 0 || v >= bv)", 0),
    ("NaN biased score not ranked last (fp64)", "static double key64(double v) { return v != v ? -INFINITY : v; }",
     "static double key64(double v) { return v; }", 0),
    ("NaN biased score not ranked last (replica)", "static float key32(float v) { return v != v ? -INFINITY : v; }",
     "static float key32(float v) { return v; }", 0),
    ("replica max starts at the first logit", "float m = -INFINITY;\n    for (int e = 0; e < E; ++e)\n      if (lt[e] > m) m = lt[e];",
     "float m = lt[0];\n    for (int e = 1; e < E; ++e)\n      if (lt[e] > m) m = lt[e];", 0),
    ("NVFP4 block scale rounds past an exact fit", "if ((float)zo_e4m3_decode((uint8_t)c) >= t) return (uint8_t)c;",
     "if ((float)zo_e4m3_decode((uint8_t)c) > t) return (uint8_t)c;", 0),
    ("NVFP4 tensor scale for 448 instead of 6 * 448", "const float r = amax / 2688.0f;", "const float r = amax / 448.0f;", 0),
    ("NVFP4 W_d tensor scale dropped", "out[r * d + c] = acc * (double)gd;", "out[r * d + c] = acc;", 0),
    ("NVFP4 gate and up tensor scales swapped", "g *= (double)gg;\n      u *= (double)gu;",
     "g *= (double)gu;\n      u *= (double)gg;", 0),
    ("NVFP4 scale read for blocks of 32", "return tab[code] * zo_e4m3_decode(scales[r * (cols / 16) + c / 16]);",
     "return tab[code] * zo_e4m3_decode(scales[r * (cols / 16) + c / 32]);", 0),
    ("NVFP4 codes scaled without the tensor scale", "const float sg = (float)zo_e4m3_decode(sc) * g;",
     "const float sg = (float)zo_e4m3_decode(sc);", 0),
    ("replica sum tree reads its own partial", "nxt[p] = part[p] + part[p ^ w];", "nxt[p] = part[p] + part[p];", 0),
    ("replica max not subtracted", "u[e] = zo_zexp(lt[e] - m);", "u[e] = zo_zexp(lt[e]);", 0),
    ("zexp coefficient 1/3! wrong", "0x1.555556p-3f);  /* 1/3! */", "0x1.555556p-2f);  /* 1/3! */", 0),
    ("zexp C2 term dropped", "r = fmaf(-n, C2, r);", "r = r;", 0),
    # integer stage
    ("permutation in descending token order", "for (int64_t t = 0; t < T; ++t) {\n    for (int j = 0; j < k; ++j) {\n      int e = idx[t * k + j];",
     "for (int64_t t = T - 1; t >= 0; --t) {\n    for (int j = 0; j < k; ++j) {\n      int e = idx[t * k + j];", 0),
    ("zero experts enter the permutation offsets", "for (int e = 0; e < N; ++e) offsets[e + 1] = offsets[e] + counts[e];",
     "for (int e = 0; e < N; ++e) offsets[e + 1] = offsets[e] + counts[e] + (e == N - 1 ? counts[E - 1] : 0);", 0),
    # SwiGLU expert and layer
    ("silu sign", "h[i] = g / (1.0 + exp(-g)) * u;", "h[i] = g / (1.0 + exp(g)) * u;", 0),
    ("gate and up swapped", "h[i] = g / (1.0 + exp(-g)) * u;", "h[i] = u / (1.0 + exp(-u)) * g;", 0),
    ("W_d transposed", "acc += elem(wd, w_dtype, (int64_t)c * inter + i) * h[i];",
     "acc += elem(wd, w_dtype, (int64_t)i * d + c) * h[i];", 0),
    ("zero experts return nothing", "yt[c] += zsum * elem(x, x_dtype, t * d + c);",
     "yt[c] += 0.0 * elem(x, x_dtype, t * d + c);", 0),
    ("expert output not gated", "for (int c = 0; c < d; ++c) yt[c] += g * f[c];",
     "for (int c = 0; c < d; ++c) yt[c] += f[c];", 0),
    # bias controller
    ("controller error sign", "const float err = tau - load;", "const float err = load - tau;", 0),
    ("decay applied after the step", "const float et = *eta * decay;\n  *eta = et;",
     "const float et = *eta;\n  *eta = et * decay;", 0),
    ("initial bias dropped", "bias[i] = s2 + b0[i];", "bias[i] = s2;", 0),
    ("derivative term sign", "const float dd = kde * (err - eprev[i]);",
     "const float dd = kde * (err + eprev[i]);", 0),
    ("zero-expert target from N", "((float)k - target_ffn) / (float)Z", "((float)k - target_ffn) / (float)N", 0),
    ("accumulators not reset", "    counts[i] = 0;\n  }\n  *tokens = 0;", "  }\n  *tokens = 0;", 0),
    # FP8
    ("E4M3 ties rounded up", "if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) == 1.0)) r += 1.0;\n  const double val = r * q; /* <= 448",
     "if (frac >= 0.5) r += 1.0;\n  const double val = r * q; /* <= 448", 0),
    ("E8M0 scale one step small", "? k - 8 : k - 7;", "? k - 8 : k - 8;", 0),
    ("E4M3 subnormal spacing", "q = ldexp(1.0, -9);\n  } else {", "q = ldexp(1.0, -8);\n  } else {", 0),
    ("FP8 expert gate and up swapped", "h32[i] = (float)(g / (1.0 + exp(-g)) * u);",
     "h32[i] = (float)(u / (1.0 + exp(-u)) * g);", 0),
    ("FP8 H not quantized", "for (int i = 0; i < inter; ++i) hv[i] = ldexp(zo_e4m3_decode(hq[i]), (int)hs_sc[i / 128] - 127);",
     "for (int i = 0; i < inter; ++i) hv[i] = h32[i];", 0),
    # MXFP4
    ("E2M1 ties rounded up", "if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) == 1.0)) r += 1.0;\n  const double val = r * q;\n  if (val < 1.0)",
     "if (frac >= 0.5) r += 1.0;\n  const double val = r * q;\n  if (val < 1.0)", 0),
    ("MX scale one step small", "? k - 2 : k - 1;", "? k - 2 : k - 2;", 0),
    ("nibble order", "codes[r * (cols / 2) + c / 2] = (uint8_t)(lo | (hi << 4));",
     "codes[r * (cols / 2) + c / 2] = (uint8_t)(hi | (lo << 4));", 0),
    ("FP4 expert gate and up swapped", "h32[i] = (float)(g / (1.0 + exp(-g)) * u);",
     "h32[i] = (float)(u / (1.0 + exp(-u)) * g);", 1),
    # backward
    ("silu derivative term dropped", "const double da = dh[i] * b[i] * sg * (1.0 + a[i] * (1.0 - sg));",
     "const double da = dh[i] * b[i] * sg;", 0),
    ("softmax Jacobian mean dropped", "dl[e] = s[t * E + e] * (ds[e] - sds);", "dl[e] = s[t * E + e] * ds[e];", 0),
    ("zero-expert dx dropped", "dxt[c] += g * dyt[c];", "dxt[c] += 0.0 * dyt[c];", 0),
    ("dW_d uses the gated input", "dwd[eo + (int64_t)c * inter + i] += dF[c] * hh[i];",
     "dwd[eo + (int64_t)c * inter + i] += dyt[c] * hh[i];", 0),
    ("up gradient without silu", "const double db = dh[i] * a[i] * sg;", "const double db = dh[i] * a[i];", 0),
    ("dW_u from the gate's gradient", "if (dwu) dwu[eo + (int64_t)i * d + c] += db * xv[c];",
     "if (dwu) dwu[eo + (int64_t)i * d + c] += da * xv[c];", 0),
    ("router part of dx dropped", "dxt[c] += elem(wr, w_dtype, (int64_t)e * d + c) * dl[e];",
     "dxt[c] += 0.0 * elem(wr, w_dtype, (int64_t)e * d + c) * dl[e];", 0),
    # more routing and integer-stage slips
    ("replica gate from the biased score", "gate[t * k + j] = scale * u[best];", "gate[t * k + j] = scale * bv;", 0),
    ("replica bias ignored", "float v = key32(u[e] + (bias ? bias[e] : 0.0f));", "float v = key32(u[e]);", 0),
    ("margin sign", "margin[t] = found ? last - next : INFINITY;", "margin[t] = found ? next - last : INFINITY;", 0),
    ("zero experts left out of the counts", "for (int64_t i = 0; i < T * k; ++i) counts[idx[i]]++;",
     "for (int64_t i = 0; i < T * k; ++i) if (idx[i] < N) counts[idx[i]]++;", 0),
    ("zero slot position not -1", "pos[t * k + j] = -1;", "pos[t * k + j] = 0;", 0),
    # more quantized-expert slips
    ("FP4 H not quantized", "for (int i = 0; i < inter; ++i) hv[i] = mx4_value(hq, hsc, inter, 0, i, tab);",
     "for (int i = 0; i < inter; ++i) hv[i] = h32[i];", 0),
    ("FP8 x not quantized", "for (int c = 0; c < d; ++c) xv[c] = ldexp(zo_e4m3_decode(xq[c]), (int)xs_sc[c / 128] - 127);",
     "for (int c = 0; c < d; ++c) xv[c] = elem(xs, x_dtype, r * d + c);", 0),
    ("FP8 weight scale of the first column block only", "const double sgv = ldexp(1.0, (int)sg[(i / 128) * dkb + c / 128] - 127);",
     "const double sgv = ldexp(1.0, (int)sg[(i / 128) * dkb] - 127);", 0),
    ("FP4 x not quantized", "for (int c = 0; c < d; ++c) xv[c] = mx4_value(xq, xsc, d, 0, c, tab);",
     "for (int c = 0; c < d; ++c) xv[c] = elem(xs, x_dtype, r * d + c);", 0),
    ("softmax numerator without the max", "s[t * E + e] = exp(lt[e] - m) / sum;", "s[t * E + e] = exp(lt[e]) / sum;", 0),
    ("top-k never marks a pick taken", "taken[best] = 1;\n      idx[t * k + j] = best;\n      gate[t * k + j] = scale * st[best];",
     "taken[best] = 0;\n      idx[t * k + j] = best;\n      gate[t * k + j] = scale * st[best];", 0),
    ("zero expert returns token 0", "yt[c] += zsum * elem(x, x_dtype, t * d + c);", "yt[c] += zsum * elem(x, x_dtype, c);", 0),
    ("load per pick instead of per token", "const float tf = (float)*tokens;", "const float tf = (float)(*tokens * k);", 0),
    ("block amax from the first row only", "for (int64_t r = r0; r < r1; ++r)\n        for (int64_t c = cb * 128; c < cb * 128 + 128; ++c) {\n          const double a",
     "for (int64_t r = r0; r < r0 + 1; ++r)\n        for (int64_t c = cb * 128; c < cb * 128 + 128; ++c) {\n          const double a", 0),
    ("FP8 down scale index transposed", "ldexp(1.0, (int)sd[(c / 128) * ikb + i / 128] - 127)",
     "ldexp(1.0, (int)sd[(i / 128) * dkb + c / 128] - 127)", 0),
    ("router scale dropped in the backward", "ds[e] += scale * dg;\n      for (int i = 0; i < inter; ++i) {",
     "ds[e] += dg;\n      for (int i = 0; i < inter; ++i) {", 0),
    ("softmax Jacobian mean without s", "for (int e = 0; e < E; ++e) sds += s[t * E + e] * ds[e];",
     "for (int e = 0; e < E; ++e) sds += ds[e];", 0),
    ("up uses the gate weights", "u += elem(wu, w_dtype, (int64_t)i * d + c) * xv;", "u += elem(wg, w_dtype, (int64_t)i * d + c) * xv;", 0),
    ("FP4 weight scale of the first block only", "const double sgv = ldexp(1.0, (int)sg[(int64_t)i * (d / 32) + c / 32] - 127);",
     "const double sgv = ldexp(1.0, (int)sg[(int64_t)i * (d / 32)] - 127);", 0),
]


# Mistakes in the Python glue (oracle/__init__.py): each runs against its own copy
# of the package, with the unchanged C library.
PY_MUTANTS = [
    ("layer outputs: zero-expert term dropped", "y += zsum[:, None] * xf", "y += 0.0 * zsum[:, None] * xf", 0),
    ("layer outputs: expert output not gated", "y[r] += float(gate[r, j]) * f[i]", "y[r] += f[i]", 1),
    ("layer outputs: bf16 rows decoded with the wrong shift", "(x_rows.astype(np.uint32) << 16)",
     "(x_rows.astype(np.uint32) << 8)", 0),
    ("layer outputs: FP8 weights quantized per [1,128]",
     "q = [quantize_blocks(w, 128) for w in (wg, wu, wd)]\n            f = ffn_fp8",
     "q = [quantize_blocks(w, 1) for w in (wg, wu, wd)]\n            f = ffn_fp8", 0),
    ("dequantize: scale ignored", "return np.ldexp(table[codes], sc)", "return table[codes]", 0),
    ("dequantize MXFP4: nibbles swapped", "nib[:, 0::2] = codes & 0xF\n    nib[:, 1::2] = codes >> 4",
     "nib[:, 0::2] = codes >> 4\n    nib[:, 1::2] = codes & 0xF", 0),
    ("router logits: offset not passed", "off = None if offset is None else np.ascontiguousarray(offset, dtype=np.float32)",
     "off = None", 0),
    ("top-k: scale not passed", "float(scale), idx, gate, margin.ctypes.data", "1.0, idx, gate, margin.ctypes.data", 0),
    ("integer stage: the whole perm buffer returned", "perm[:P].copy()", "perm.copy()", 0),
    ("brute force: ties to the later subset", "if best is None or s > best_sum:", "if best is None or s >= best_sum:", 0),
    ("controller state: eta starts at 0", '"eta": np.ones(1, np.float32)', '"eta": np.zeros(1, np.float32)', 0),
]


def _mutate(src, old, new, nth):
    start = -1
    for _ in range(nth + 1):
        start = src.find(old, start + 1)
        assert start >= 0, f"text not found (occurrence {nth}): {old!r}"
    return src[:start] + new + src[start + len(old):]


def _build(job):
    """Writes one copy of the source and builds it as the oracle is built."""
    out_dir, text = job
    os.makedirs(out_dir, exist_ok=True)
    c_path, so_path = os.path.join(out_dir, "oracle.c"), os.path.join(out_dir, "liboracle.so")
    with open(c_path, "w") as f:
        f.write(text)
    subprocess.run(oracle.compile_command(c_path, so_path), check=True, capture_output=True)
    return so_path


def _run_worker(paths, oracle_dir=None):
    """The pins against each library in `paths`, in one worker process (importing the
    oracle package from `oracle_dir` when given)."""
    env = dict(os.environ, OMP_NUM_THREADS="2")
    pre = ["--oracle-dir", oracle_dir] if oracle_dir else []
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "oracle_mutant_worker.py"), *pre, *paths],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    rcs = {}
    for line in r.stdout.splitlines():
        if line.startswith("ZCMOE-MUTANT "):
            rec = json.loads(line[len("ZCMOE-MUTANT "):])
            rcs[rec["lib"]] = rec["rc"]
    return rcs, r.stdout[-3000:] + r.stderr[-3000:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    src = open(SRC).read()
    jobs = [("control", src)] + [(name, _mutate(src, old, new, nth)) for name, old, new, nth in MUTANTS]
    for name, text in jobs[1:]:
        assert text != src, name
    assert len({name for name, _ in jobs}) == len(jobs)
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        libs = list(ex.map(_build, [(str(tmp_path / f"m{i}"), text) for i, (_, text) in enumerate(jobs)]))
    shares = [libs[w::workers] for w in range(workers)]
    rcs, logs = {}, []
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        for got, log in ex.map(_run_worker, shares):
            rcs.update(got)
            logs.append(log)
    assert len(rcs) == len(libs), "a worker stopped early:\n" + "\n".join(logs)
    names = {lib: name for lib, (name, _) in zip(libs, jobs)}
    assert rcs[libs[0]] == 0, "the unchanged copy must pass every pin:\n" + "\n".join(logs)
    survivors = [names[lib] for lib in libs[1:] if rcs[lib] != 1]
    assert not survivors, f"mistakes that no pin caught (pytest exit code other than 1): {survivors}"


def _py_copy(job):
    """A copy of the oracle package with `text` as its Python glue and the repository's
    C source and library; returns (package parent dir, library path)."""
    out_dir, text = job
    pkg = os.path.join(out_dir, "oracle")
    os.makedirs(pkg, exist_ok=True)
    with open(os.path.join(pkg, "__init__.py"), "w") as f:
        f.write(text)
    shutil.copy2(SRC, os.path.join(pkg, "zcmoe_oracle.c"))
    so = os.path.join(pkg, "liboracle.so")
    shutil.copy2(oracle.build(), so)
    return out_dir, so


def test_every_planted_mistake_in_the_python_glue_fails_a_pin(tmp_path):
    src = open(PY_SRC).read()
    jobs = [("control", src)] + [(name, _mutate(src, old, new, nth)) for name, old, new, nth in PY_MUTANTS]
    for name, text in jobs[1:]:
        assert text != src, name
    copies = [_py_copy((str(tmp_path / f"p{i}"), text)) for i, (_, text) in enumerate(jobs)]
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        results = list(ex.map(lambda c: _run_worker([c[1]], oracle_dir=c[0]), copies))
    rcs = [got.get(so) for (got, _), (_, so) in zip(results, copies)]
    logs = [log for _, log in results]
    assert rcs[0] == 0, "the unchanged copy must pass every pin:\n" + logs[0]
    survivors = [name for (name, _), rc in zip(jobs[1:], rcs[1:]) if rc != 1]
    assert not survivors, f"mistakes that no pin caught (pytest exit code other than 1): {survivors}"
