#!/usr/bin/env python
"""Benchmark of the W4A4 rotated linear layer on B200.

One step = one pass of the whole hot path over one batch: hq_rotate_quant (K1:
grouped Hadamard rotation + per-token int4 quantisation) followed by
w4a4_linear (K2: int4 x int4 GEMM with the fused SERQ term and dequantising
epilogue).  Weights are prepared once, offline, by the library's own kernels.

Default workload: the decode-shaped Llama-7B MLP up-projection, 16 tokens,
K = 4096, N = 11008, group-128 asymmetric int4 weights, Hadamard group 128,
rank-16 SERQ term, fp16 in/out.  Other workloads: --workload attn|down|large|tiny.

Timing: the P steps of one pass over a rotating pool of layers (distinct
weights and activations, more bytes than the 126 MB L2) are captured in a CUDA
graph; the timed region replays it, bracketed by a barrier and a device
synchronise, with CUDA events; the value is the max over ranks.  Per-kernel
launch durations (for the roofline) come from graphs holding one kernel kind,
timed with CUDA events on the launch stream.  SM clocks are sampled with
nvidia-smi during the timed region.  With --gpus N (torchrun) every rank runs
an independent replica (weak scaling; the layer has no exchange step).

Prints ONE JSON line on rank 0.
"""
import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024

DEFAULT_STEPS = {"tiny": 20000, "decode": 100000, "attn": 20000, "down": 4000, "large": 400}
DEFAULT_M = {"tiny": 16, "decode": 16, "attn": 2048, "down": 4096, "large": 8192}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d.get("bf16_tflops_sustained"),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(DEFAULT_M), default="decode")
    ap.add_argument("--m", type=int, default=None, help="tokens per step (default: the workload's)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


# ----------------------------------------------------------------- algorithmic work per launch
def k1_bytes(M, K, xbytes=2):
    return M * K * xbytes + M * K // 2 + 4 * M


def k2_bytes(M, N, K, gw, r, ybytes=2):
    b = N * K // 2                                  # packed weights
    b += (2 * (K // gw) * N * 2) if gw else 2 * N   # scales (+ zero points)
    b += N * r // 2 + 2 * N + 4 * r                 # Rq, sr, sal
    b += M * K // 2 + 4 * M                         # Xq, sx
    b += M * N * ybytes                             # Y
    return b


def k2_ops(M, N, K):
    return 2 * M * N * K


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        rows = [ln.strip().split(",") for ln in open(self.f.name) if ln.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- CPU oracle timing
def oracle_step_sample(wl, M, seed, n_rows, n_cols, sample_seed=0):
    """Builds the oracle's own prepared weights for a column sample and returns a
    callable doing one sampled step (rotate/quant of the sampled rows + the
    layer on those rows and columns), plus the ops it performs."""
    import numpy as np

    import oracle as O
    from w4a4_bit_gemm_hq_b200 import synth

    rng = np.random.default_rng(sample_seed)
    X = synth.activations(wl, seed=seed, M=M)
    W = synth.weights(wl, seed=seed)
    d = synth.hadamard_signs(wl.g, seed=seed)
    rows = np.sort(rng.choice(M, size=min(n_rows, M), replace=False))
    cols = np.sort(rng.choice(wl.N, size=min(n_cols, wl.N), replace=False))
    Wc = W[cols]
    Wrot = O.rotate_normalised(Wc, wl.wdtype, wl.g, d)
    Wq, sw, zw = O.w4_pack(Wrot, "f32", wl.gw)
    _, sal = O.salient_channels(X[rows], wl.xdtype, wl.g, d, wl.r)
    Rq, sr = O.serq_prepare(Wrot, Wq, sw, zw, wl.gw, sal)
    Xs = np.ascontiguousarray(X[rows])

    def step():
        Xq, sx = O.rotate_quant(Xs, wl.xdtype, wl.g, d)
        O.linear_rows_f64(Xq, sx, wl.K, Wq, sw, zw, wl.gw, Rq, sr, sal, np.arange(len(rows)))

    return step, 2 * len(rows) * len(cols) * wl.K, len(rows), len(cols)


def omp_threads():
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v and v.isdigit() else (os.cpu_count() or 1)


def cpu_baseline(wl, M, budget_s=12.0):
    # size the sample: one calibration step with a small column sample, then scale
    step, ops, nr, nc = oracle_step_sample(wl, M, 0, n_rows=1, n_cols=64)
    t = time.perf_counter()
    step()
    per_col = max((time.perf_counter() - t) / nc, 1e-7)
    n_rows = min(M, 16)
    n_cols = int(min(wl.N, max(64, budget_s / 3 / (per_col * n_rows))))
    step, ops, nr, nc = oracle_step_sample(wl, M, 0, n_rows=n_rows, n_cols=n_cols)
    times = []
    t_end = time.perf_counter() + budget_s
    while time.perf_counter() < t_end or not times:
        t = time.perf_counter()
        step()
        times.append(time.perf_counter() - t)
    tmed = statistics.median(times)
    return {"value": ops / tmed / 1e12, "unit": "TOPS", "cores": omp_threads(), "kind": "oracle",
            "sample": "%d rows x %d of %d output channels of the %s layer (K=%d), rotate/quant of those rows "
                      "+ integer GEMM + fp64 epilogue, median of %d runs" % (nr, nc, wl.N, wl.name, wl.K,
                                                                             len(times))}


def run_reference(args, wl, M, rank, world):
    """The comparison arm: the CPU oracle as it stands, on the host cores, each
    step a bounded sample of the same workload."""
    if rank != 0:
        return
    steps = args.steps if args.steps is not None else 20
    warm = max(args.warmup, 3)
    budget = 90.0
    step, ops, nr, nc = oracle_step_sample(wl, M, 0, n_rows=1, n_cols=64)
    t = time.perf_counter()
    step()
    per_col = max((time.perf_counter() - t) / nc, 1e-7)
    n_cols = int(min(wl.N, max(8, budget / (steps + warm) / per_col)))
    step, ops, nr, nc = oracle_step_sample(wl, M, 0, n_rows=1, n_cols=n_cols)
    for _ in range(warm):
        step()
    t = time.perf_counter()
    for _ in range(steps):
        step()
    el = time.perf_counter() - t
    value = ops * steps / el / 1e12
    sample = "1 row x %d of %d output channels of the %s layer per step (K=%d)" % (nc, wl.N, wl.name, wl.K)
    print(json.dumps({
        "impl": "reference", "metric": metric_name(), "value": value, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": steps, "warmup": warm, "ms_per_step": el / steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int64", "data": "synthetic",
        "config": config_dict(wl, M, None, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": omp_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def metric_name():
    return "W4A4 linear TOPS & rotate/quant GB/s at Llama-7B shapes, % of B200 roofline"


def config_dict(wl, M, pool, n):
    c = {"workload": "%s: W4A4 linear M=%d K=%d N=%d (Hadamard group %d, weight group %s, SERQ rank %d, %s in/out)"
                     % (wl.name, M, wl.K, wl.N, wl.g, wl.gw if wl.gw else "per-channel", wl.r, wl.xdtype),
         "M": M, "K": wl.K, "N": wl.N, "hadamard_group": wl.g, "weight_group": wl.gw, "serq_rank": wl.r,
         "parallelism": "replicas x%d" % n}
    if pool is not None:
        c["l2"] = "rotating pool of %d layers and batches (%.0f MB > 126 MB L2)" % pool
    return c


# ----------------------------------------------------------------- ranks
# One process per GPU, each a full replica of the layer on its own token
# batches (the layer has no exchange step); these helpers are the only
# cross-rank logic and work with any torch.distributed backend.
def max_over_ranks(ms, pg, device):
    """The slowest rank's duration: the job is done when every replica is."""
    if pg is None:
        return ms
    import torch

    t = torch.tensor([ms], device=device, dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_tops(ops_per_unit, units_per_rank, world, ms):
    """Whole-job throughput: the work all ranks did over the slowest rank's time."""
    return ops_per_unit * units_per_rank * world / (ms * 1e-3) / 1e12


def replica_seed(rank, i):
    """Seed of token batch i of rank `rank`: replicas process different batches."""
    return 1000 * rank + i


# ----------------------------------------------------------------- main
def main():
    args = parse()
    wl0 = None
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    from w4a4_bit_gemm_hq_b200 import synth

    wl0 = synth.WORKLOADS[args.workload]
    M = args.m if args.m is not None else DEFAULT_M[args.workload]
    wl = wl0.with_m(M)

    if args.impl == "reference":
        run_reference(args, wl, M, rank, world)
        return

    import numpy as np
    import torch

    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist

    from w4a4_bit_gemm_hq_b200 import hq

    dev = torch.device("cuda", local)
    steps = args.steps if args.steps is not None else DEFAULT_STEPS[args.workload]
    warm = max(args.warmup, 3)
    peaks = measured_peaks()
    xdt = torch.float16 if wl.xdtype == "f16" else torch.bfloat16

    def to_dev(a, dt):
        if dt == "bf16":
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(a).to(dev)

    # ---- one prepared layer, then a pool of distinct copies
    X0 = synth.activations(wl, seed=replica_seed(rank, 0), M=M)
    W0 = synth.weights(wl, seed=rank)
    d = torch.from_numpy(synth.hadamard_signs(wl.g, seed=rank)).to(dev)
    Xd0 = to_dev(X0, wl.xdtype)
    base = hq.W4A4Linear.prepare(to_dev(W0, wl.wdtype), wl.g, wl.gw, wl.r, d, X_calib=Xd0, out_dtype=xdt)
    del W0
    per_step = k1_bytes(M, wl.K) + k2_bytes(M, wl.N, wl.K, wl.gw, wl.r) + M * wl.K * 2
    P = int(min(16, max(1, math.ceil(2 * L2_BYTES / per_step))))
    layers, Xs, Xqs, sxs, Ys = [], [], [], [], []
    for i in range(P):
        clone = lambda t: None if t is None else t.clone()
        layers.append(hq.W4A4Linear(base.group, base.gw, base.H_signs, clone(base.Wq), clone(base.sw),
                                    clone(base.zw), clone(base.Rq), clone(base.sr), base.sal_idx, wl.K, wl.N, xdt))
        Xs.append(Xd0 if i == 0 else torch.from_numpy(synth.activations(wl, seed=replica_seed(rank, i), M=M).view(
            np.int16 if wl.xdtype == "bf16" else np.float16)).view(xdt).to(dev))
        Xqs.append(torch.empty((M, wl.K // 2), dtype=torch.uint8, device=dev))
        sxs.append(torch.empty((M,), dtype=torch.float32, device=dev))
        Ys.append(torch.empty((M, wl.N), dtype=xdt, device=dev))
    pool_mb = P * per_step / 1e6

    def k1(i):
        hq.hq_rotate_quant(Xs[i], wl.g, layers[i].H_signs, Xqs[i], sxs[i])

    def k2(i):
        L = layers[i]
        hq.w4a4_linear(Xqs[i], sxs[i], L.Wq, L.sw, L.zw, L.gw, L.Rq, L.sr, L.sal_idx, xdt, Ys[i],
                       L.workspace(M, dev))

    def step(i):
        k1(i)
        k2(i)

    # ---- warm-up (eager), then graphs
    for w in range(warm):
        step(w % P)
    torch.cuda.synchronize()
    assert hq.hq_last_device_status() == 0

    def capture(fn_list):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for fn in fn_list:
                fn()
        torch.cuda.current_stream().wait_stream(s)
        with torch.cuda.graph(g):
            for fn in fn_list:
                fn()
        return g

    g_full = capture([lambda i=i: step(i) for i in range(P)])
    rem = steps % P
    g_rem = capture([lambda i=i: step(i) for i in range(rem)]) if rem else None
    reps = steps // P

    def barrier():
        if pg is not None:
            pg.barrier()

    # ---- timed region
    torch.cuda.synchronize()
    barrier()
    clk = ClockSampler(local)
    clk.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g_full.replay()
    if g_rem is not None:
        g_rem.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    clocks = clk.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), pg, dev)
    assert hq.hq_last_device_status() == 0

    # ---- per-kernel launch durations (graphs of one kernel kind, CUDA events)
    def kernel_ms(fn):
        g = capture([lambda i=i: fn(i) for i in range(P)])
        r = max(1, min(reps, 2000))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(r):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / (r * P)

    t_k1 = kernel_ms(k1)
    t_k2 = kernel_ms(k2)

    # ---- end to end through the public call, host buffers, copies inside
    e2e = None
    if not args.no_e2e:
        Xh = [torch.empty((M, wl.K), dtype=xdt, pin_memory=True) for _ in range(P)]
        Yh = [torch.empty((M, wl.N), dtype=xdt, pin_memory=True) for _ in range(P)]
        for i in range(P):
            Xh[i].copy_(Xs[i].cpu())

        def e2e_step(i):
            Xs[i].copy_(Xh[i], non_blocking=True)
            layers[i](Xs[i], Ys[i], Xqs[i], sxs[i])
            Yh[i].copy_(Ys[i], non_blocking=True)

        g_e2e = capture([lambda i=i: e2e_step(i) for i in range(P)])
        r = max(1, min(reps, 20000))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier()
        a.record()
        for _ in range(r):
            g_e2e.replay()
        b.record()
        torch.cuda.synchronize()
        barrier()
        e_ms = max_over_ranks(a.elapsed_time(b), pg, dev)
        e2e = {"value": job_tops(k2_ops(M, wl.N, wl.K), r * P, world, e_ms), "unit": "TOPS",
               "h2d_bytes_per_step": M * wl.K * 2, "d2h_bytes_per_step": M * wl.N * 2,
               "ms_per_step": e_ms / (r * P)}

    ops = k2_ops(M, wl.N, wl.K)
    value = job_tops(ops, steps, world, ms)
    # ---- roofline of the dominant kernel
    b1 = k1_bytes(M, wl.K)
    b2 = k2_bytes(M, wl.N, wl.K, wl.gw, wl.r)
    k1_gbs = b1 / (t_k1 * 1e-3) / 1e9
    int8_peak = 2.0 * peaks["bf16"]          # dense int8 = 2 x dense bf16 (nominal 4.5 vs 2.25 PF)
    decode_like = M <= 64
    if t_k2 >= t_k1:
        if decode_like:
            roof = {"kernel": "k_gemm_small (w4a4_linear)", "bound": "hbm", "achieved": b2 / (t_k2 * 1e-3) / 1e9,
                    "peak": peaks["hbm"], "unit": "GB/s", "bytes_per_launch": b2}
        else:
            roof = {"kernel": "k_gemm_pf (w4a4_linear)", "bound": "tensor",
                    "achieved": ops / (t_k2 * 1e-3) / 1e12, "peak": int8_peak, "unit": "TOP/s",
                    "ops_per_launch": ops}
    else:
        roof = {"kernel": "k_rotate (hq_rotate_quant)", "bound": "hbm", "achieved": k1_gbs, "peak": peaks["hbm"],
                "unit": "GB/s", "bytes_per_launch": b1}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = peaks["src"] + (" (int8 = 2 x measured bf16 burst)" if roof["bound"] == "tensor" else
                                          " HBM copy, burst")
    roof["traffic"] = committed_traffic(args.workload, M, roof["kernel"])

    out = {
        "metric": metric_name(), "value": value, "unit": "TOPS", "n_gpus": world, "steps": steps, "warmup": warm,
        "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4", "data": "synthetic", "config": config_dict(wl, M, (P, pool_mb), world),
        "roofline": roof,
        "kernels": {"k1_rotate_quant": {"ms": t_k1, "GB/s": k1_gbs, "frac_hbm": k1_gbs / peaks["hbm"],
                                        "bytes_per_launch": b1},
                    "k2_linear": {"ms": t_k2, "TOP/s": ops / (t_k2 * 1e-3) / 1e12,
                                  "GB/s": b2 / (t_k2 * 1e-3) / 1e9, "frac_int8": ops / (t_k2 * 1e-3) / 1e12 / int8_peak,
                                  "frac_hbm": b2 / (t_k2 * 1e-3) / 1e9 / peaks["hbm"], "bytes_per_launch": b2}},
        "gpu_launches": 2 * steps,
        "clocks": clocks,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, M)
    if rank == 0:
        print(json.dumps(out), flush=True)
    del g_full, g_rem
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


def committed_traffic(workload, M, kernel):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary (profiles/ncu_traffic.json), when it matches this workload and the
    current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get("%s:M=%d" % (workload, M))
        if not e or e.get("sources_sha") != sources_sha(e.get("sources")):
            return None
        return e["dram_bytes_per_launch"]
    except (ValueError, KeyError):
        return None


def sources_sha(files=None):
    """Hash of the CUDA sources a captured kernel is built from (all of csrc/
    when the entry names none): a committed traffic figure is used only while
    they are unchanged."""
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "w4a4_bit_gemm_hq_b200", "csrc")
    for f in sorted(files if files else os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:12]


if __name__ == "__main__":
    main()
