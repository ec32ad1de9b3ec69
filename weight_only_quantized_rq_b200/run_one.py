"""Run one product y = x * w_hat^T a few times on cuda:0 (for profiling a
single launch, or a quick timing of one shape).

    python -m weight_only_quantized_rq_b200.run_one --fmt w4g64 --K 4096 --N 16384 --M 16 [--reps 3] [--time]

The weights are N(0, 0.02) and RTN-packed (one candidate); x is N(0, 1) in
bf16. With --time the command also prints the mean time of 40 back-to-back
calls measured with CUDA events.
"""
from __future__ import annotations

import argparse
import json


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--fmt", default="w4g64", choices=["w4g64", "w8g16", "w4sb32"])
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--N", type=int, default=4096)
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--time", action="store_true")
    a = ap.parse_args()

    import torch
    import weight_only_quantized_rq_b200 as rq

    torch.cuda.set_device(0)
    g = torch.Generator(device="cuda").manual_seed(0)
    W = torch.randn(a.N, a.K, device="cuda", generator=g) * 0.02
    p = rq.rq_quantize_pack(W, a.fmt, None, 1, 1.0, 1.0)
    del W
    x = torch.randn(a.M, a.K, device="cuda", generator=g).to(torch.bfloat16)
    y = torch.empty(a.M, a.N, device="cuda")
    for _ in range(a.reps):
        rq.rq_wgemm(x, p, y)
    torch.cuda.synchronize()
    out = {"fmt": a.fmt, "K": a.K, "N": a.N, "M": a.M, "packed_bytes": p.nbytes}
    if a.time:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(40):
            rq.rq_wgemm(x, p, y)
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / 40
        out.update(us=round(us, 2), GB_s=round(p.nbytes / us / 1e3, 1),
                   TFLOP_s=round(2 * a.M * a.K * a.N / us / 1e6, 1))
    out["device_status"] = rq.rq_device_status()
    print(json.dumps(out))
    return 0 if out["device_status"] == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
