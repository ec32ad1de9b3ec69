"""Benchmark of the decode hot path: the int4 group-64 (E[x^2]-searched)
weight-only product over the RWKV-7 1.5B layer set, 24 layers x (r, k, v, o
2048x2048, channel-mix key 2048->8192, value 8192->2048), M = 1 activation
row, on one B200 per process.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload IDX] [--M ROWS] [--no-graph]

A step is one pass of rq_wgemm over all 144 matrices (the packing is done
once, before timing; it is offline work in the method). The metric is the
effective weight-stream bandwidth: packed bytes of all matrices / step time.
Inputs are synthetic (seeded), weights drawn on the GPU; the packed set
(642 MB) is larger than the 126 MB L2, so no flush is needed between steps.

Under torchrun (N > 1) every rank runs the same workload on its own GPU
(independent replicas, no collective in the data path: weak scaling); rank 0
prints the aggregate. ``--impl reference`` times the CPU oracle instead, on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4g64 GEMV effective weight GB/s and % of HBM peak at M=1 (1×B200)"
HBM_FALLBACK = 6650.0
NOMINAL_HBM = 8000.0


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return HBM_FALLBACK, "fallback"


def tensor_peak():
    """Dense bf16 tensor throughput (TFLOP/s) for a kernel timed in a short
    burst: the measured one when available."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(ms: float, ws: int, device) -> float:
    """The largest of the ranks' times (every rank takes part, in the same
    order, whatever its value)."""
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if ws > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(ws: int, bytes_per_rank: float, ms_max: float) -> float:
    """Weak scaling: every rank streams bytes_per_rank per step; the job's
    rate is all ranks' bytes over the slowest rank's step time."""
    return ws * bytes_per_rank / (ms_max * 1e-3) / 1e9


# ----------------------------------------------------------- clocks -------
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"rq_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ oracle ------
def oracle_sample(w, seconds: float, seed: int = 0):
    """Time the CPU oracle's product (exact dequant + fp64 sums) over a
    bounded sample of the workload's rows: for each matrix shape of one
    layer, a few rows (packed by the oracle from CPU-drawn weights). Returns
    (packed bytes processed per second, description, threads)."""
    import numpy as np

    import oracle
    from weight_only_quantized_rq_b200 import workloads as wl
    oracle.build()
    rng = np.random.default_rng(seed)
    shapes = []
    for j, layer, m in w.matrices():
        if layer > 0:
            break
        rows = 128
        g = wl.random_matrix(10_000 + j, rows, m.K).numpy()
        a = wl.act_sq(w, m.K)
        codes, scales = oracle.pack(m.fmt, g, a if m.n_cand > 1 else None, n_cand=m.n_cand,
                                    t_lo=0.7 if m.n_cand > 1 else 1.0)
        x = wl.bf16_bits(wl.activations(w, j, m.K, 1))
        cshape, _, sshape = oracle.packed_shapes(m.fmt, m.K, m.N)
        per_row = cshape[1] + (2 * sshape[1] if sshape else 0)          # packed bytes of one row
        shapes.append((m, codes, scales, x, rows, per_row))
    done_bytes, t0 = 0.0, time.perf_counter()
    reps = 0
    while True:
        for m, codes, scales, x, rows, per_row in shapes:
            oracle.wgemm(m.fmt, x, m.K, rows, codes, scales)
            done_bytes += rows * per_row
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    desc = (f"oracle product (exact dequant + fp64 ascending-k sums) over 128 rows of each of the "
            f"{len(shapes)} matrix shapes of one layer, M=1, repeated {reps}x ({el:.1f} s)")
    return done_bytes / el / 1e9, desc, oracle.threads(), el


def host_cpu():
    """CPU model and the cores this process may run on."""
    model = "unknown"
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    return model, cores


def oracle_pack_rate(w, seconds: float):
    """The oracle's quantize-pack (the E[x^2]-weighted search of the method,
    rwkv-quant article "Two presets and six sizes") over a few rows of each
    matrix shape of one layer of the workload, repeated for about `seconds`:
    weights per second."""
    import numpy as np

    import oracle
    from weight_only_quantized_rq_b200 import workloads as wl
    oracle.build()
    sample = []
    for j, layer, m in w.matrices():
        if layer > 0:
            break
        rows = 8
        sample.append((m, wl.random_matrix(20_000 + j, rows, m.K).numpy(), wl.act_sq(w, m.K)))
    done, t0, reps = 0, time.perf_counter(), 0
    while True:
        for m, W, a in sample:
            oracle.pack(m.fmt, W, a if m.n_cand > 1 else None, n_cand=m.n_cand,
                        t_lo=0.7 if m.n_cand > 1 else 1.0)
            done += W.size
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return done / el, f"8 rows of each of the {len(sample)} matrix shapes of one layer, {reps}x ({el:.1f} s)"


def run_reference(args, w, M):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    per_step = 2.0
    for _ in range(args.warmup):
        oracle_sample(w, per_step / 4)
    vals, secs = [], []
    for _ in range(args.steps):
        v, desc, thr, el = oracle_sample(w, per_step)
        vals.append(v)
        secs.append(el)
    value = statistics.median(vals)
    hbm, src = peaks()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * statistics.median(secs), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, M),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": thr, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, M):
    return {"workload": w.name, "M": M, "matrices": len(w.matrices()),
            "formats": sorted({m.fmt for m in w.per_layer}),
            "l2": "packed set larger than the 126 MB L2; no flush between steps",
            "inputs": "weights N(0,0.02) drawn on the GPU from seeded generators, act_sq closed form"}


def kernel_hash() -> str:
    h = hashlib.sha1()
    for f in ("rq_gemv.cu", "rq_device.cuh"):
        with open(os.path.join(ROOT, "weight_only_quantized_rq_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(p))
        e = d[kernel]
        return e["bytes_per_launch"] if e.get("source_hash") == kernel_hash() else None
    except Exception:
        return None


# -------------------------------------------------------------- ours ------
def pack_workload(w, dev):
    """Quantize-pack every matrix of a workload on the GPU (not timed)."""
    import torch
    import weight_only_quantized_rq_b200 as rq
    from weight_only_quantized_rq_b200 import workloads as wl
    mats = []
    for j, layer, m in w.matrices():
        W = wl.weights(w, j, m, device=str(dev))
        a = torch.from_numpy(wl.act_sq(w, m.K)).to(dev) if m.n_cand > 1 else None
        p = rq.rq_quantize_pack(W, m.fmt, a, m.n_cand, 0.7 if m.n_cand > 1 else 1.0, 1.0)
        mats.append((j, m, p))
        del W
    torch.cuda.synchronize()
    return mats


class Problem:
    """One M over a packed workload: every product's x in one device block,
    every y in another, and the step as batched launches (one per format and
    chunk of at most 160 products; the products are independent)."""

    def __init__(self, w, mats, M, dev, ydtype=None):
        import torch
        import weight_only_quantized_rq_b200 as rq
        from weight_only_quantized_rq_b200 import workloads as wl
        self.M = M
        ydtype = torch.float32 if ydtype is None else ydtype
        ysz = 4 if ydtype == torch.float32 else 2
        xs_elems = sum(M * m.K + 8 for _, m, _ in mats)
        ys_elems = sum(M * m.N + 8 for _, m, _ in mats)
        self.xdev = torch.empty(xs_elems, dtype=torch.bfloat16, device=dev)
        self.ydev = torch.empty(ys_elems, dtype=ydtype, device=dev)
        self.calls, xo, yo = [], 0, 0
        for j, m, p in mats:
            x = self.xdev[xo:xo + M * m.K].view(M, m.K)
            x.copy_(wl.activations(w, j, m.K, M, device=str(dev)))
            y = self.ydev[yo:yo + M * m.N].view(M, m.N)
            self.calls.append((x, p, y, m))
            xo += (M * m.K + 7) // 8 * 8
            yo += (M * m.N + 7) // 8 * 8
        self.packed_bytes = sum(p.nbytes for _, _, p in mats)
        self.alg_bytes = sum(p.nbytes + 2 * M * p.K + ysz * M * p.N for _, _, p in mats)
        self.flops = sum(2 * M * p.K * p.N for _, _, p in mats)
        self.h2d = sum(M * m.K * 2 for _, m, _ in mats)
        self.d2h = sum(M * m.N * ysz for _, m, _ in mats)
        self.batches = []
        self.kernel_launches = 0     # launches the library issues per step
        for fmt in sorted({m.fmt for *_, m in self.calls}):
            cs = [c for c in self.calls if c[3].fmt == fmt]
            for i in range(0, len(cs), rq.MAX_BATCH):
                ch = cs[i:i + rq.MAX_BATCH]
                self.batches.append(rq.WgemmBatch([c[0] for c in ch], [c[1] for c in ch], [c[2] for c in ch]))
                tc = rq.tc_path(fmt, M)
                self.kernel_launches += -(-len(ch) // rq.TC_MAX_ITEMS) if tc else 1
        torch.cuda.synchronize()

    def step(self, stream):
        for b in self.batches:
            b(stream=stream)

    def roofline_s(self, hbm_gbs, tflops):
        """Lower bound on the step time: per product, the slower of its
        weight/x/y traffic at the HBM rate and its flops at the tensor rate."""
        t = 0.0
        for x, p, y, m in self.calls:
            b = p.nbytes + 2 * self.M * p.K + 4 * self.M * p.N
            f = 2 * self.M * p.K * p.N
            t += max(b / (hbm_gbs * 1e9), f / (tflops * 1e12))
        return t


def run_ours(args, w, M):
    import torch
    import weight_only_quantized_rq_b200 as rq

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    # CPU baseline first, before heavy GPU work (rank 0, single GPU only)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        import oracle
        v, desc, thr, _ = oracle_sample(w, args.cpu_seconds)
        nthr = oracle.threads()
        oracle.set_threads(1)
        v1, desc1, _, _ = oracle_sample(w, args.cpu_seconds / 3)
        oracle.set_threads(nthr)
        model, aff = host_cpu()
        cpu = {"value": round(v, 4), "unit": "GB/s", "cores": thr, "kind": "oracle", "sample": desc,
               "one_core": {"value": round(v1, 4), "unit": "GB/s", "sample": desc1},
               "cpu_model": model, "cores_available": aff}

    mats = pack_workload(w, dev)
    prob = Problem(w, mats, M, dev)
    calls, packed_bytes, alg_bytes = prob.calls, prob.packed_bytes, prob.alg_bytes
    stream = torch.cuda.Stream(device=dev)

    def step():
        prob.step(stream)

    # the decode chain of a real token: per layer, the independent r/k/v
    # projections in one launch, then o, ffn key, ffn value, each depending on
    # the previous one (programmatic dependent launch overlaps their weight
    # streams)
    per = len(w.per_layer)
    names = [m.name for m in w.per_layer]
    rkv = [i for i, n in enumerate(names) if n in ("r", "k", "v")]
    chain_parts = []
    for L0 in range(0, len(calls), per):
        lay = calls[L0:L0 + per]
        if rkv:
            chain_parts.append(rq.WgemmBatch([lay[i][0] for i in rkv], [lay[i][1] for i in rkv], [lay[i][2] for i in rkv]))
        chain_parts.extend([lay[i] for i in range(per) if i not in rkv])

    def chain_step():
        for part in chain_parts:
            if isinstance(part, rq.WgemmBatch):
                part(stream=stream)
            else:
                rq.rq_wgemm(part[0], part[1], part[2], stream=stream)

    graphs = []

    def capture(fn):
        with torch.cuda.stream(stream):
            fn()
            stream.synchronize()
            if args.no_graph:
                return fn
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn()
        torch.cuda.synchronize()
        graphs.append(g)
        return g.replay

    run = capture(step)
    run_chain = capture(chain_step)

    def barrier():
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    def timed(fn, steps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                fn()
            barrier()
            e0.record(stream)
            for _ in range(steps):
                fn()
            e1.record(stream)
        barrier()
        return max_over_ranks(e0.elapsed_time(e1) / steps, ws, dev)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ms_max = timed(run, args.steps)
    clk = clocks.stop()
    value = whole_job_gbs(ws, packed_bytes, ms_max)
    ms_chain = timed(run_chain, args.steps)
    chain_val = whole_job_gbs(ws, packed_bytes, ms_chain)

    # end to end through the public API: pinned host x in, host y out
    xh = torch.empty(prob.xdev.shape, dtype=prob.xdev.dtype, pin_memory=True)
    yh = torch.empty(prob.ydev.shape, dtype=prob.ydev.dtype, pin_memory=True)
    xh.copy_(prob.xdev)

    def e2e_step():
        prob.xdev.copy_(xh, non_blocking=True)
        run()
        yh.copy_(prob.ydev, non_blocking=True)

    ms_serial = timed(e2e_step, args.steps)
    e2e_serial = whole_job_gbs(ws, packed_bytes, ms_serial)

    # The same, double-buffered as a serving loop runs it: two sets of x/y
    # buffers (the weights are shared), the copies on their own stream, so
    # step i's host copies overlap the neighbouring steps' kernels. Every
    # step still moves its own x in and its own y out inside the timed region.
    prob2 = Problem(w, mats, M, dev)
    run2 = capture(lambda: prob2.step(stream))
    xh2 = torch.empty(xh.shape, dtype=xh.dtype, pin_memory=True)
    yh2 = torch.empty(yh.shape, dtype=yh.dtype, pin_memory=True)
    xh2.copy_(prob2.xdev)
    sets = [(prob, run, xh, yh), (prob2, run2, xh2, yh2)]
    hstream = torch.cuda.Stream(device=dev)             # host -> device copies
    dstream = torch.cuda.Stream(device=dev)             # device -> host copies
    ev = {(k, b): torch.cuda.Event() for k in ("h2d", "comp", "d2h") for b in (0, 1)}
    for e in ev.values():
        e.record(stream)

    def pipelined(n):
        for i in range(n):
            b = i & 1
            P, R, xhb, yhb = sets[b]
            hstream.wait_event(ev["comp", b])            # step i - 2 has read x_b
            with torch.cuda.stream(hstream):
                P.xdev.copy_(xhb, non_blocking=True)
            ev["h2d", b].record(hstream)
            stream.wait_event(ev["h2d", b])
            stream.wait_event(ev["d2h", b])              # y_b of step i - 2 is on the host
            with torch.cuda.stream(stream):
                R()
            ev["comp", b].record(stream)
            dstream.wait_event(ev["comp", b])
            with torch.cuda.stream(dstream):
                yhb.copy_(P.ydev, non_blocking=True)
            ev["d2h", b].record(dstream)
        stream.wait_event(ev["d2h", 0])
        stream.wait_event(ev["d2h", 1])

    pipelined(max(args.warmup, 2))
    barrier()
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    hstream.wait_event(p0)
    dstream.wait_event(p0)
    pipelined(args.steps)
    p1.record(stream)
    barrier()
    ms_e2e = max_over_ranks(p0.elapsed_time(p1) / args.steps, ws, dev)
    e2e_val = whole_job_gbs(ws, packed_bytes, ms_e2e)
    launches = prob.kernel_launches
    hbm, src = peaks()
    tc_peak, tc_src = tensor_peak()
    per_launch_bytes = alg_bytes / launches
    per_launch_s = ms_max * 1e-3 / launches
    achieved = per_launch_bytes / per_launch_s / 1e9
    traffic = recorded_traffic("gemv_batch_w4g64_m1")

    # every configuration at each of its activation-row counts (the headline
    # workload at its other M, and the other four configurations), one
    # batched step per (configuration, M)
    from weight_only_quantized_rq_b200 import workloads as wl
    def measure(w2, mats2, Ms):
        entry = {"workload": w2.name, "packed_bytes_per_step": sum(p.nbytes for _, _, p in mats2)}
        for m2 in Ms:
            pr = Problem(w2, mats2, m2, dev)
            f = capture(lambda pr=pr: pr.step(stream))
            ms2 = timed(f, min(args.steps, 10))
            t_roof = pr.roofline_s(hbm, tc_peak)
            entry[str(m2)] = {
                "ms_per_step": round(ms2, 5),
                "GB_s": round(ws * pr.packed_bytes / (ms2 * 1e-3) / 1e9, 2),
                "pct_hbm_measured": round(100 * pr.packed_bytes / (ms2 * 1e-3) / 1e9 / hbm, 2),
                "TFLOP_s": round(ws * pr.flops / (ms2 * 1e-3) / 1e12, 2),
                "pct_bf16_peak_measured": round(100 * pr.flops / (ms2 * 1e-3) / 1e12 / tc_peak, 2),
                "roofline_frac": round(t_roof / (ms2 * 1e-3), 4),
                "launches_per_step": pr.kernel_launches,
                "kernel": "tc_kernel" if all(rq.tc_path(c[3].fmt, m2) for c in pr.calls) else "gemv_kernel"}
            del pr
        return entry

    configs, variants = {}, {}
    if not args.quick:
        for w2 in wl.WORKLOADS:
            Ms = [m for m in w2.Ms if not (w2 is w and m == M)]
            if not Ms:
                continue
            mats2 = mats if w2 is w else pack_workload(w2, dev)
            configs[w2.name.split(" ")[0]] = measure(w2, mats2, Ms)
            if w2 is not w:
                del mats2
                torch.cuda.empty_cache()
        # the preset's wider-code matrices (5- and 6-bit superblocks)
        for w2 in wl.VARIANTS:
            mats2 = pack_workload(w2, dev)
            variants[w2.name.split(" ")[0] + "/" + w2.per_layer[0].name] = measure(w2, mats2, list(w2.Ms))
            del mats2
            torch.cuda.empty_cache()
    # quantize-pack (offline: the E[x^2]-weighted search, code emission and
    # packing) of one layer of every configuration on the GPU, and the
    # oracle's pack of a few rows of the same shapes on 1 core and on all
    # cores (rank 0 only): weights per second
    pack = None
    if not args.quick:
        pack = {}
        for w2 in list(wl.WORKLOADS) + list(wl.VARIANTS):
            shapes = [m for j2, layer2, m in w2.matrices() if layer2 == 0]
            Ws = [wl.weights(w2, j2, m, device=str(dev)) for j2, layer2, m in w2.matrices() if layer2 == 0]
            acts = [torch.from_numpy(wl.act_sq(w2, m.K)).to(dev) if m.n_cand > 1 else None for m in shapes]
            outs = [rq.alloc_packed(m.fmt, m.K, m.N, dev) for m in shapes]

            def pack_all(shapes=shapes, Ws=Ws, acts=acts, outs=outs):
                for m, Wd, a, o in zip(shapes, Ws, acts, outs):
                    rq.rq_quantize_pack(Wd, m.fmt, a, m.n_cand, 0.7 if m.n_cand > 1 else 1.0, 1.0, out=o,
                                        stream=stream)
            with torch.cuda.stream(stream):
                pack_all()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                pack_all()
                e1.record(stream)
            e1.synchronize()
            ms_p = e0.elapsed_time(e1)
            nw = sum(m.K * m.N for m in shapes)
            ent = {"matrices": [f"{m.fmt} {m.K}->{m.N} n_cand={m.n_cand}" for m in shapes],
                   "gpu_ms": round(ms_p, 3), "gpu_Mweights_per_s": round(nw / (ms_p * 1e-3) / 1e6, 1)}
            if rank == 0 and ws == 1 and not args.no_cpu_baseline:      # the CPU-baseline leg
                import oracle
                nthr = oracle.threads()
                r_all, d_all = oracle_pack_rate(w2, 1.0)
                oracle.set_threads(1)
                r_one, d_one = oracle_pack_rate(w2, 1.0)
                oracle.set_threads(nthr)
                ent["oracle_Mweights_per_s"] = {"all_cores": round(r_all / 1e6, 3), "cores": nthr,
                                                "one_core": round(r_one / 1e6, 3), "sample": d_all}
                ent["gpu_over_oracle_all_cores"] = round(nw / (ms_p * 1e-3) / r_all, 1)
            pack[w2.name.split(" ")[0]] = ent
            del Ws, acts, outs
        torch.cuda.empty_cache()
    # config 1 as a single 768^2 product in one launch (launch-bound by
    # construction; the configuration's line streams 2048 distinct copies)
    single768 = None
    if not args.quick:
        w0 = wl.WORKLOADS[0]
        m0 = w0.per_layer[0]
        W0 = wl.weights(w0, 0, m0, device=str(dev))
        p0 = rq.rq_quantize_pack(W0, m0.fmt, None, 1, 1.0, 1.0)
        x0 = wl.activations(w0, 0, m0.K, 1, device=str(dev))
        y0 = torch.empty(1, m0.N, device=dev)
        f0 = capture(lambda: rq.rq_wgemm(x0, p0, y0, stream=stream))
        ms0 = timed(f0, args.steps)
        single768 = {"ms_per_call": round(ms0, 5), "calls_per_s": round(1e3 / ms0, 1),
                     "GB_s": round(p0.nbytes / (ms0 * 1e-3) / 1e9, 2),
                     "note": "one 313 KB matrix per launch: resident in L2 and bound by the launch, not by HBM"}
        del W0, p0, x0, y0
    # the E[x^2] statistic of the scale search over a calibration batch of
    # 7.2B width (32768 rows x 4096 channels of bf16, 256 MB > L2)
    act_stats = None
    if not args.quick:
        R_c, K_c = 32768, 4096
        g_c = torch.Generator(device=dev).manual_seed(77)
        xa = torch.randn(R_c, K_c, device=dev, generator=g_c).to(torch.bfloat16)
        ss = torch.zeros(K_c, dtype=torch.float64, device=dev)
        f = capture(lambda: rq.rq_act_sumsq(xa, ss, stream=stream))
        ms_a = timed(f, min(args.steps, 10))
        gbs = R_c * K_c * 2 / (ms_a * 1e-3) / 1e9
        act_stats = {"rows": R_c, "K": K_c, "ms_per_call": round(ms_a, 5), "GB_s": round(gbs, 2),
                     "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": hbm, "unit": "GB/s",
                                  "frac": round(gbs / hbm, 4),
                                  "note": "algorithmic bytes = R * K * 2 (x read once) per call"},
                     "kernel": "act_sumsq_kernel"}
        del xa, ss
    # the headline step with the bf16-output epilogue (y rounded once to bf16
    # in the same launches)
    bf16_out = None
    if not args.quick:
        pr16 = Problem(w, mats, M, dev, ydtype=torch.bfloat16)
        f16 = capture(lambda: pr16.step(stream))
        ms16 = timed(f16, args.steps)
        bf16_out = {"ms_per_step": round(ms16, 5), "GB_s": round(ws * pr16.packed_bytes / (ms16 * 1e-3) / 1e9, 2),
                    "pct_hbm_measured": round(100 * pr16.packed_bytes / (ms16 * 1e-3) / 1e9 / hbm, 2),
                    "launches_per_step": pr16.kernel_launches}
        del pr16
    # GPTQ on the preset grid for one 1.5B projection (2048 -> 2048, int4 g64)
    # from 4096 calibration rows: the three device steps, each timed alone
    gptq = None
    if not args.quick:
        K_g, N_g, R_g = 2048, 2048, 4096
        g_g = torch.Generator(device=dev).manual_seed(91)
        basis = torch.randn(256, K_g, device=dev, generator=g_g)
        xg = (torch.randn(R_g, 256, device=dev, generator=g_g) @ basis
              + 0.1 * torch.randn(R_g, K_g, device=dev, generator=g_g)).to(torch.bfloat16)
        Wg = torch.randn(N_g, K_g, device=dev, generator=g_g) * 0.02
        Hg = torch.zeros(K_g, K_g, dtype=torch.float64, device=dev)
        Ug = torch.empty(K_g, K_g, dtype=torch.float64, device=dev)
        dg = torch.empty(K_g, dtype=torch.uint8, device=dev)
        outg = rq.alloc_packed("w4g64", K_g, N_g, dev)

        def ev_time(fn, reps):
            with torch.cuda.stream(stream):
                fn()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(reps):
                    fn()
                e1.record(stream)
            e1.synchronize()
            return e0.elapsed_time(e1) / reps

        ms_h = ev_time(lambda: rq.rq_hessian_accum(xg, Hg, stream=stream), 3)
        Hg.zero_()
        rq.rq_hessian_accum(xg, Hg, stream=stream)
        ms_p = ev_time(lambda: rq.rq_gptq_prepare(Hg, 0.01, Ug, dg, stream=stream), 2)
        ms_q = ev_time(lambda: rq.rq_gptq_quantize_pack(Wg, "w4g64", Ug, dg, None, 64, 0.7, 1.0, outg,
                                                        stream=stream), 2)
        gptq = {"K": K_g, "N": N_g, "rows": R_g, "fmt": "w4g64",
                "hessian_ms": round(ms_h, 3), "hessian_fp64_TFLOP_s": round(2.0 * K_g * K_g * R_g / (ms_h * 1e-3) / 1e12, 2),
                "prepare_ms": round(ms_p, 3), "pack_ms": round(ms_q, 3),
                "pack_fp64_GFLOP_s": round(N_g * K_g * K_g / (ms_q * 1e-3) / 1e9, 1),
                "kernels": "hessian_kernel; gptq_reverse/chol_block_diag + chol_block_panel (per 32 columns)/"
                           "chol_pivots/trinv/gptq_finish; gptq_sym_kernel",
                "note": "offline calibration steps, measured for reference; not part of the decode step"}
        del xg, Wg, Hg, Ug, dg, outg, basis
    status = rq.rq_device_status(stream)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {**config_of(w, M), "packed_bytes_per_step": packed_bytes, "step": "batched rq_wgemm_batch "
                   "launches over the layer set's independent products", "graph": not args.no_graph, "pdl": True,
                   "parallelism": f"replicas{ws}" if ws > 1 else "single",
                   "pct_hbm_measured": round(100 * value / ws / hbm, 2),
                   "pct_hbm_nominal_8TBs": round(100 * value / ws / NOMINAL_HBM, 2)},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": hbm, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "traffic": traffic,
                     "kernel": "gemv_kernel<w4g64, M=1> (batched launch)" if M <= 2 else "tc_kernel",
                     "peak_source": src,
                     "note": "algorithmic bytes (packed weights + x + y) per launch / CUDA-event time per launch"},
        "decode_chain": {"value": round(chain_val, 2), "unit": "GB/s", "ms_per_step": round(ms_chain, 5),
                         "launches_per_step": len(chain_parts),
                         "structure": "per layer: r/k/v in one batched launch, then o, ffn key, ffn value, "
                                      "each dependent on the previous launch"},
        "configs": configs,
        "configs_note": "per (configuration, M): one graph-captured step of batched launches over the "
                        "configuration's products; roofline_frac = sum over products of max(bytes / HBM peak, "
                        "flops / bf16 peak) divided by the step time",
        "preset_variants": variants,
        "bf16_out": bf16_out,
        "act_stats": act_stats,
        "pack": pack,
        "single_768": single768,
        "gptq": gptq,
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "h2d_bytes_per_step": prob.h2d,
                "d2h_bytes_per_step": prob.d2h, "ms_per_step": round(ms_e2e, 5),
                "pipelining": "two x/y buffer sets; host-to-device and device-to-host copies on their own "
                              "streams, overlapping the neighbouring steps' kernels",
                "serial": {"value": round(e2e_serial, 2), "ms_per_step": round(ms_serial, 5),
                           "note": "copy in, step, copy out on one stream, nothing overlapped"}},
        "gpu_launches": launches * args.steps,
        "clocks": clk,
        "device_status": status,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        del run, run_chain
        graphs.clear()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--quick", action="store_true", help="headline line only (no other configurations)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    from weight_only_quantized_rq_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w, args.M)
    return run_ours(args, w, args.M)


if __name__ == "__main__":
    sys.exit(main())
