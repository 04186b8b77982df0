"""Worker for tests/test_gpu_threads.py, run in a fresh process so that the
library's first-use set-up (tensor-map encoder lookup, per-device shared-memory
attributes of every GEMM kernel) happens inside the racing threads.

Four host threads each create their own layer handle on the same weights and run
forwards on their own CUDA stream at the same time (ctypes releases the GIL
during library calls); every output must equal, bit for bit, the output of the
same forward run afterwards on one thread."""
import sys
import threading

import numpy as np
import torch


def main() -> int:
    from mixture_experts_layer_shifted_b200 import configs
    from mixture_experts_layer_shifted_b200.zcmoe import LayerShape, ZcMoE

    torch.cuda.set_device(0)
    outs = {}
    errors = []
    cases = []
    for i, (name, dt) in enumerate([("small_bf16", "bf16"), ("small_bf16", "fp8"), ("small_bf16", "fp4"),
                                    ("small_bf16", "bf16")]):
        w = configs.WORKLOADS[name].with_(dtype=dt, seed=i)
        weights = configs.device_weights(w.with_(dtype="bf16"))
        x = configs.device_tokens(w.with_(dtype="bf16"), 2048 + 128 * i)
        cases.append((w, weights, x))
    torch.cuda.synchronize()
    start = threading.Barrier(len(cases))

    def run(i):
        try:
            w, weights, x = cases[i]
            shape = LayerShape(w.d, w.n_ffn, w.n_zero, w.inter, w.top_k, w.dtype, 1.0)
            s = torch.cuda.Stream()
            start.wait()
            layer = ZcMoE(shape, *weights, max_tokens=x.shape[0], init_bias=configs.bias_vector(w))
            with torch.cuda.stream(s):
                ys = [layer.forward(x, stream=s) for _ in range(3)]
            s.synchronize()
            layer.check()
            outs[i] = [y.view(torch.int16).cpu().numpy() for y in ys]
            layer.close()
        except Exception as e:  # reported by the main thread
            errors.append((i, repr(e)))

    threads = [threading.Thread(target=run, args=(i,)) for i in range(len(cases))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    if errors or len(outs) != len(cases):
        print("FAILED", errors, sorted(outs))
        return 1
    for i, (w, weights, x) in enumerate(cases):
        shape = LayerShape(w.d, w.n_ffn, w.n_zero, w.inter, w.top_k, w.dtype, 1.0)
        layer = ZcMoE(shape, *weights, max_tokens=x.shape[0], init_bias=configs.bias_vector(w))
        y = layer.forward(x).view(torch.int16).cpu().numpy()
        layer.close()
        for j, got in enumerate(outs[i]):
            if not np.array_equal(got, y):
                print(f"FAILED case {i} ({w.dtype}) forward {j}: differs from the serial result")
                return 1
    print("OK", len(cases), "threads")
    return 0


if __name__ == "__main__":
    sys.exit(main())
