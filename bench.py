#!/usr/bin/env python
"""Benchmark of the W4A4 rotated linear layer on B200.

One step = one pass of the whole hot path over one batch: hq_rotate_quant (K1:
grouped Hadamard rotation + per-token int4 quantisation) followed by
w4a4_linear (K2: int4 x int4 GEMM with the fused SERQ term and dequantising
epilogue).  Weights are prepared once, offline, by the library's own kernels.

The JSON line's headline (value, ms_per_step, roofline, e2e, cpu_baseline) is
the Llama-7B MLP down-projection: 4096 tokens, K = 11008 (86 Hadamard groups
of 128), N = 4096, group-128 asymmetric int4 weights, rank-32 SERQ term, bf16
in/out.  The same run also measures every other layer shape of the suite and
reports them under "workloads": decode (M = 1, 4, 16; 4096 -> 11008), the
attention projection (M = 2048; 4096 -> 4096, one Hadamard group of 4096) and
the Llama-70B MLP shape (M = 512, 2048, 8192; 8192 -> 28672), each with K1's
HBM throughput and fraction of the HBM roofline and K2's TOP/s and fraction of
the dense int8 tensor peak (of HBM for decode).  "serq_overhead" compares K2
with and without the SERQ term on the same weights; "activation_variants"
times the W4A8 and OffQ activations on the decode and down layers;
"calibration" times the offline calibration kernels of the down layer.

"e2e" is the same metric through the public call (W4A4Linear) with pinned host
buffers: every step copies its activations in and its output back, on three
streams (copy in, compute, copy out) with events guarding buffer reuse, so a
later step's copy in overlaps the compute and copy out of earlier ones.

Timing: every layer shape runs over a rotating pool of layers and batches
(distinct weights and activations) holding more bytes than 2x the 126 MB L2;
steps are captured in CUDA graphs and timed with CUDA events on the launching
stream; per-kernel launch durations come from graphs holding one kernel kind.
SM clocks are sampled with nvidia-smi during the headline's timed region.
With --gpus N (torchrun) every rank runs an independent replica (weak scaling;
the layer has no exchange step), durations are the max over ranks.

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
HEADLINE = ("down", 4096)
# (workload, M) of the suite; the large Llama-70B shape is measured at three M
SUITE = [("decode", 1), ("decode", 4), ("decode", 16), ("attn", 2048), ("down", 4096), ("large", 512),
         ("large", 2048), ("large", 8192)]
# shapes where K1 and the prefill GEMM have roofline targets (M >= 2048)
TARGET_SHAPES = [("attn", 2048), ("down", 4096), ("large", 8192)]
K1_TARGET, K2_TARGET = 0.70, 0.60
# shapes also measured with W4A8 and OffQ activations
VARIANT_SHAPES = [("decode", 16), ("down", 4096)]
DEFAULT_STEPS = 500
NOMINAL_INT8_PER_BF16 = 2.0   # dense int8 / dense bf16 tensor throughput (4.5 / 2.25 PF nominal)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d.get("bf16_tflops_sustained"),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def parse():
    from w4a4_bit_gemm_hq_b200 import synth

    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(synth.WORKLOADS), default=HEADLINE[0],
                    help="headline workload (default: the down-projection)")
    ap.add_argument("--m", type=int, default=None, help="tokens per step of the headline (default: the workload's)")
    ap.add_argument("--headline-only", action="store_true", help="skip the other shapes (profiling runs)")
    ap.add_argument("--calibration-only", action="store_true",
                    help="time the offline calibration kernels of the down layer only (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


# ----------------------------------------------------------------- algorithmic work per launch
def k1_bytes(M, K, xbytes=2):
    """Read X (16-bit), write packed codes (0.5 B / element) and sx (4 B / row)."""
    return M * K * xbytes + M * K // 2 + 4 * M


def k2_bytes(M, N, K, gw, r, ybytes=2):
    """Every operand of w4a4_linear read once and Y written once."""
    b = N * K // 2                                  # packed weights
    b += (2 * (K // gw) * N * 2) if gw else 2 * N   # scales (+ zero points)
    b += N * r // 2 + 2 * N + 4 * r                 # Rq, sr, sal
    b += M * K // 2 + 4 * M                         # Xq, sx
    b += M * N * ybytes                             # Y
    return b


def k2_ops(M, N, K):
    """Main-term integer ops (the SERQ term's 2 M N r are not counted)."""
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
    rows = np.sort(rng.choice(M, size=min(n_rows, M), replace=False))
    X = synth.activations(wl, seed=seed, M=M)[rows]
    cols = np.sort(rng.choice(wl.N, size=min(n_cols, wl.N), replace=False))
    Wc = synth.weights(wl, seed=seed)[cols]
    d = synth.hadamard_signs(wl.g, seed=seed)
    Wrot = O.rotate_normalised(Wc, wl.wdtype, wl.g, d)
    Wq, sw, zw = O.w4_pack(Wrot, "f32", wl.gw)
    _, sal = O.salient_channels(X, wl.xdtype, wl.g, d, wl.r)
    Rq, sr = O.serq_prepare(Wrot, Wq, sw, zw, wl.gw, sal)
    Xs = np.ascontiguousarray(X)

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


def describe(wl, M):
    return "%s: W4A4 linear M=%d K=%d N=%d (Hadamard group %d, weight group %s, SERQ rank %d, %s in/out)" % (
        wl.name, M, wl.K, wl.N, wl.g, wl.gw if wl.gw else "per-channel", wl.r, wl.xdtype)


def config_dict(wl, M, pool, n):
    c = {"workload": describe(wl, M), "M": M, "K": wl.K, "N": wl.N, "hadamard_group": wl.g,
         "weight_group": wl.gw, "serq_rank": wl.r, "parallelism": "replicas x%d" % n}
    if pool is not None:
        c["l2"] = "rotating pool of %d layers and batches (%.0f MB > 2 x 126 MB L2)" % pool
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


# ----------------------------------------------------------------- GPU measurement
class Runner:
    """Device, peaks and helpers shared by every measured shape."""

    def __init__(self, torch, hq, synth, rank, dev):
        self.torch, self.hq, self.synth, self.rank, self.dev = torch, hq, synth, rank, dev
        self.peaks = measured_peaks()
        self.int8_peak = NOMINAL_INT8_PER_BF16 * self.peaks["bf16"]
        self.int8_peak_sus = NOMINAL_INT8_PER_BF16 * self.peaks["bf16_sus"] if self.peaks["bf16_sus"] else None

    def to_dev(self, a, dt):
        import numpy as np

        if dt == "bf16":
            return self.torch.from_numpy(a.view(np.int16)).to(self.dev).view(self.torch.bfloat16)
        return self.torch.from_numpy(a).to(self.dev)

    def capture(self, fns):
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for fn in fns:
                fn()
        torch.cuda.current_stream().wait_stream(s)
        with torch.cuda.graph(g):
            for fn in fns:
                fn()
        return g

    def time_graph(self, g, reps):
        torch = self.torch
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(reps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    def launch_ms(self, fn, P, budget_ms=25.0):
        """Average duration of one launch of fn(i), from a graph of P launches
        (one per pool entry) replayed until about budget_ms have passed."""
        g = self.capture([lambda i=i: fn(i) for i in range(P)])
        g.replay()
        est = max(self.time_graph(g, 1), 1e-3)
        reps = int(max(2, min(2000, budget_ms / est)))
        ms = self.time_graph(g, reps) / (reps * P)
        del g
        return ms


class Shape:
    """One prepared layer shape: a pool of P layers (distinct weights) and P
    token batches (distinct activations), all resident on the device."""

    def __init__(self, R, wl, M, base=None, r=None):
        torch, hq, synth = R.torch, R.hq, R.synth
        self.R, self.wl, self.M = R, wl, M
        self.r = wl.r if r is None else r
        self.xdt = torch.float16 if wl.xdtype == "f16" else torch.bfloat16
        X0 = R.to_dev(synth.activations(wl, seed=replica_seed(R.rank, 0), M=M), wl.xdtype)
        if base is None:
            W = R.to_dev(synth.weights(wl, seed=R.rank), wl.wdtype)
            d = torch.from_numpy(synth.hadamard_signs(wl.g, seed=R.rank)).to(R.dev)
            base = hq.W4A4Linear.prepare(W, wl.g, wl.gw, self.r, d, X_calib=X0, out_dtype=self.xdt)
            del W
        self.base = base
        per_step = k1_bytes(M, wl.K) + k2_bytes(M, wl.N, wl.K, wl.gw, self.r) + M * wl.K * 2
        self.per_step = per_step
        self.P = int(min(16, max(1, math.ceil(2.2 * L2_BYTES / per_step))))
        clone = lambda t: None if t is None else t.clone()
        b = base
        self.layers = [b] + [hq.W4A4Linear(b.group, b.gw, b.H_signs, clone(b.Wq), clone(b.sw), clone(b.zw),
                                           clone(b.Rq), clone(b.sr), b.sal_idx, wl.K, wl.N, self.xdt)
                             for _ in range(self.P - 1)]
        # distinct batches: the seeded batch and row rotations of it (different
        # bytes at different addresses; the values' statistics are unchanged)
        self.X = [X0] + [X0.roll(i, 0).contiguous() for i in range(1, self.P)]
        self.Xq = [torch.empty((M, wl.K // 2), dtype=torch.uint8, device=R.dev) for _ in range(self.P)]
        self.sx = [torch.empty((M,), dtype=torch.float32, device=R.dev) for _ in range(self.P)]
        self.Y = [torch.empty((M, wl.N), dtype=self.xdt, device=R.dev) for _ in range(self.P)]
        self.ws = [L.workspace(M, R.dev) for L in self.layers]

    def k1(self, i):
        self.R.hq.hq_rotate_quant(self.X[i], self.wl.g, self.layers[i].H_signs, self.Xq[i], self.sx[i])

    def k2(self, i):
        L = self.layers[i]
        self.R.hq.w4a4_linear(self.Xq[i], self.sx[i], L.Wq, L.sw, L.zw, L.gw, L.Rq, L.sr, L.sal_idx, self.xdt,
                              self.Y[i], self.ws[i])

    def step(self, i):
        self.k1(i)
        self.k2(i)

    def record(self, decode_like):
        """K1, K2 and whole-step measurements of this shape."""
        R, wl, M, P = self.R, self.wl, self.M, self.P
        for i in range(P):
            self.step(i)
        R.torch.cuda.synchronize()
        assert R.hq.hq_last_device_status() == 0
        t1 = R.launch_ms(self.k1, P)
        t2 = R.launch_ms(self.k2, P)
        ts = R.launch_ms(self.step, P)
        b1, b2, ops = k1_bytes(M, wl.K), k2_bytes(M, wl.N, wl.K, wl.gw, self.r), k2_ops(M, wl.N, wl.K)
        rec = {"workload": wl.name, "M": M, "K": wl.K, "N": wl.N, "hadamard_group": wl.g, "weight_group": wl.gw,
               "serq_rank": self.r, "pool": P,
               "k1_us": t1 * 1e3, "k1_bytes": b1, "k1_GBs": b1 / (t1 * 1e-3) / 1e9,
               "k1_frac_hbm": b1 / (t1 * 1e-3) / 1e9 / R.peaks["hbm"],
               "k2_us": t2 * 1e3, "k2_ops": ops, "k2_bytes": b2, "k2_TOPs": ops / (t2 * 1e-3) / 1e12,
               "k2_GBs": b2 / (t2 * 1e-3) / 1e9,
               "step_us": ts * 1e3, "step_TOPS": ops / (ts * 1e-3) / 1e12}
        if decode_like:
            rec["k2_bound"] = "hbm"
            rec["k2_frac_hbm"] = rec["k2_GBs"] / R.peaks["hbm"]
        else:
            rec["k2_bound"] = "tensor (int8)"
            rec["k2_frac_int8"] = rec["k2_TOPs"] / R.int8_peak
        return rec

    def variants(self, decode_like):
        """The same layers with W4A8 activations (8-bit per-token codes) and,
        for Hadamard groups of 128, OffQ activations (per-group scale and
        zero point): K1, K2 and step times of each."""
        R, wl, M, P = self.R, self.wl, self.M, self.P
        torch, hq = R.torch, R.hq
        out = []
        Xq8 = [torch.empty((M, wl.K), dtype=torch.int8, device=R.dev) for _ in range(P)]
        k1_8 = lambda i: hq.hq_rotate_quant8(self.X[i], wl.g, self.layers[i].H_signs, Xq8[i], self.sx[i])

        def k2_8(i):
            L = self.layers[i]
            hq.w4a8_linear(Xq8[i], self.sx[i], L.Wq, L.sw, L.zw, L.gw, L.Rq, L.sr, L.sal_idx, self.xdt, self.Y[i],
                           self.ws[i])
        b1 = 2 * M * wl.K + M * wl.K + 4 * M
        b2 = k2_bytes(M, wl.N, wl.K, wl.gw, self.r) + M * wl.K // 2
        out.append(self._variant("w4a8", k1_8, k2_8, b1, b2, decode_like))
        del Xq8
        if wl.g == 128:
            G = wl.K // 128
            sxa = [torch.empty((M, G), dtype=torch.float32, device=R.dev) for _ in range(P)]
            zxa = [torch.empty((M, G), dtype=torch.int32, device=R.dev) for _ in range(P)]
            k1_a = lambda i: hq.hq_rotate_quant_asym(self.X[i], wl.g, self.layers[i].H_signs, self.Xq[i], sxa[i],
                                                     zxa[i])

            def k2_a(i):
                L = self.layers[i]
                hq.w4a4_linear_asym(self.Xq[i], sxa[i], zxa[i], L.Wq, L.sw, L.zw, L.gw, L.Rq, L.sr, L.sal_idx,
                                    self.xdt, self.Y[i])
            b1 = 2 * M * wl.K + M * wl.K // 2 + 8 * M * G
            b2 = k2_bytes(M, wl.N, wl.K, wl.gw, self.r) + 8 * M * G - 4 * M
            out.append(self._variant("offq", k1_a, k2_a, b1, b2, decode_like))
            del sxa, zxa
        if not decode_like:
            # MXFP4: hq_rotate (fp32 rows) + hq_quant_mxfp4, then hq_mxfp4_linear on
            # MXFP4 weights (one weight set, quantised once, shared by the pool)
            G = wl.K // 32
            V = [torch.empty((M, wl.K), dtype=torch.float32, device=R.dev) for _ in range(P)]
            qx = [torch.empty((M, wl.K // 2), dtype=torch.uint8, device=R.dev) for _ in range(P)]
            sbx = [torch.empty((M, G), dtype=torch.uint8, device=R.dev) for _ in range(P)]
            Wf = R.to_dev(R.synth.weights(wl), wl.wdtype)
            qw, sbw = hq.hq_quant_mxfp4(hq.hq_rotate(Wf, wl.g, self.layers[0].H_signs))
            del Wf
            Ymx = [torch.empty((M, wl.N), dtype=torch.float32, device=R.dev) for _ in range(P)]

            def k1_m(i):
                hq.hq_rotate(self.X[i], wl.g, self.layers[i].H_signs, V[i])
                hq.hq_quant_mxfp4(V[i], qx[i], sbx[i])

            k2_m = lambda i: hq.hq_mxfp4_linear(qx[i], sbx[i], qw, sbw, Ymx[i])
            b1 = 2 * M * wl.K + 2 * 4 * M * wl.K + M * wl.K // 2 + M * G
            b2 = wl.N * wl.K // 2 + wl.N * G + M * wl.K // 2 + M * G + 4 * M * wl.N
            rec = self._variant("mxfp4 (rotate to fp32 + block quantiser; int8 mma.sync GEMM)", k1_m, k2_m, b1, b2,
                                decode_like)
            out.append(rec)
            del V, qx, sbx, qw, sbw, Ymx
        return out

    def _variant(self, name, k1, k2, b1, b2, decode_like):
        R, wl, M, P = self.R, self.wl, self.M, self.P
        for i in range(P):
            k1(i)
            k2(i)
        R.torch.cuda.synchronize()
        assert R.hq.hq_last_device_status() == 0
        t1 = R.launch_ms(k1, P)
        t2 = R.launch_ms(k2, P)
        ts = R.launch_ms(lambda i: (k1(i), k2(i)), P)
        ops = k2_ops(M, wl.N, wl.K)
        rec = {"workload": wl.name, "M": M, "activations": name, "k1_us": t1 * 1e3, "k1_bytes": b1,
               "k1_frac_hbm": b1 / (t1 * 1e-3) / 1e9 / R.peaks["hbm"], "k2_us": t2 * 1e3, "k2_bytes": b2,
               "k2_TOPs": ops / (t2 * 1e-3) / 1e12, "step_us": ts * 1e3, "step_TOPS": ops / (ts * 1e-3) / 1e12}
        if decode_like:
            rec["k2_frac_hbm"] = b2 / (t2 * 1e-3) / 1e9 / R.peaks["hbm"]
        else:
            rec["k2_frac_int8"] = rec["k2_TOPs"] / R.int8_peak
        return rec

    def free(self):
        for name in ("layers", "X", "Xq", "sx", "Y", "ws", "base"):
            setattr(self, name, None)


def calibration_record(R, S=32, L=128, iters=100):
    """Offline calibration of the down-projection layer (K = 11008) on a
    synthetic calibration batch of S sequences x L tokens: each kernel timed
    alone with CUDA events (median of 5 after one warm-up), with its
    algorithmic bytes where it streams HBM.  Offline work: reported, not part
    of the step."""
    import numpy as np

    torch, hq, synth = R.torch, R.hq, R.synth
    wl = synth.WORKLOADS["down"]
    Xh, _, _ = synth.calibration_activations(wl, S, L)
    X = R.to_dev(Xh, wl.xdtype)
    W = R.to_dev(synth.weights(wl), wl.wdtype)
    M, K, N = S * L, wl.K, wl.N
    st = {}

    def timed(name, fn, nbytes=None):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            out = fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ms = float(np.median(ts))
        rec = {"us": ms * 1e3}
        if nbytes is not None:
            rec["bytes"] = nbytes
            rec["GB/s"] = nbytes / (ms * 1e-3) / 1e9
            rec["frac_hbm"] = rec["GB/s"] / R.peaks["hbm"]
        st[name] = rec
        return out

    tok, T = timed("extreme_tokens", lambda: hq.hq_calib_extreme_tokens(X, S, L), 2 * M * K + 4 * S * K)
    v, lam = timed("top1_pca (%d iterations, cluster of 8 CTAs, T in shared memory)" % iters, lambda: hq.hq_calib_top1_pca(T, iters))
    Xr = timed("householder (activations)", lambda: hq.hq_calib_householder(X, v), 2 * M * K + 4 * M * K)
    Wr = timed("householder (weights)", lambda: hq.hq_calib_householder(W, v), 2 * N * K + 4 * N * K)
    amax = timed("channel_absmax", lambda: hq.hq_calib_channel_absmax(Xr), 4 * M * K)
    perm = timed("sorted_perm (K^2 comparisons)", lambda: hq.hq_calib_sorted_perm(amax))
    timed("permute_channels (weights)", lambda: hq.hq_permute_channels(Wr, perm), 8 * N * K)
    assert hq.hq_last_device_status() == 0
    total = sum(r["us"] for r in st.values())
    return {"workload": "down: calibration batch %d sequences x %d tokens, K=%d, W %dx%d" % (S, L, K, N, K),
            "kernels": st, "total_us": total, "lambda": float(lam.item())}


def int8_gemm_crosscheck(R):
    """cuBLASLt int8 GEMM (torch._int_mm) at 8192^3, best of 10: a cross-check
    of the int8 denominator, which is 2 x the measured bf16 burst peak."""
    torch = R.torch
    try:
        n = 8192
        A = torch.randint(-8, 8, (n, n), dtype=torch.int8, device=R.dev)
        B = torch.randint(-8, 8, (n, n), dtype=torch.int8, device=R.dev)
        for _ in range(3):
            torch._int_mm(A, B.t())
        ts = []
        for _ in range(10):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            torch._int_mm(A, B.t())
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        del A, B
        return 2 * n ** 3 / min(ts) / 1e9
    except Exception as e:  # noqa: BLE001 (report, never fail the bench on the cross-check)
        return "unavailable: %s" % type(e).__name__


# ----------------------------------------------------------------- main
def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    from w4a4_bit_gemm_hq_b200 import synth

    head_name = args.workload
    head_M = args.m if args.m is not None else (HEADLINE[1] if head_name == HEADLINE[0]
                                                  else synth.WORKLOADS[head_name].M)
    wl_head = synth.WORKLOADS[head_name].with_m(head_M)

    if args.impl == "reference":
        run_reference(args, wl_head, head_M, rank, world)
        return

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
    R = Runner(torch, hq, synth, rank, dev)
    if args.calibration_only:
        # every rank calibrates its own copy (no collective); rank 0 prints
        rec = calibration_record(R)
        if rank == 0:
            print(json.dumps({"calibration": rec}), flush=True)
        if pg is not None:
            pg.barrier()
            pg.destroy_process_group()
        return
    steps = args.steps if args.steps is not None else DEFAULT_STEPS
    warm = max(args.warmup, 3)

    # ---- the headline shape: timed region of exactly `steps` steps
    S = Shape(R, wl_head, head_M)
    P = S.P
    for w in range(warm):
        S.step(w % P)
    torch.cuda.synchronize()
    assert hq.hq_last_device_status() == 0
    g_full = R.capture([lambda i=i: S.step(i) for i in range(P)])
    rem = steps % P
    g_rem = R.capture([lambda i=i: S.step(i) for i in range(rem)]) if rem else None
    reps = steps // P
    torch.cuda.synchronize()
    if pg is not None:
        pg.barrier()
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
    if pg is not None:
        pg.barrier()
    clocks = clk.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), pg, dev)
    assert hq.hq_last_device_status() == 0
    del g_full, g_rem
    decode_like = head_M <= 64
    head = S.record(decode_like)

    # ---- end to end through the public call, host buffers, copies inside
    e2e = None
    if not args.no_e2e:
        M, K, N = head_M, wl_head.K, wl_head.N
        Xh = [torch.empty((M, K), dtype=S.xdt, pin_memory=True) for _ in range(P)]
        Yh = [torch.empty((M, N), dtype=S.xdt, pin_memory=True) for _ in range(P)]
        for i in range(P):
            Xh[i].copy_(S.X[i].cpu())

        # three streams: the copy in of step j waits only for the compute that last
        # read its input buffer, the compute for its input and for the copy out
        # that last read its output buffer, the copy out for its compute; so the
        # host-to-device copies of later steps overlap the compute and the
        # device-to-host copies of earlier ones (buffers reused round-robin)
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_steps(nsteps):
            cur = torch.cuda.current_stream()
            for st_ in (s_in, s_cmp, s_out):
                st_.wait_stream(cur)
            ev_cmp, ev_out = [], []
            for j in range(nsteps):
                i = j % P
                with torch.cuda.stream(s_in):
                    if j >= P:
                        s_in.wait_event(ev_cmp[j - P])
                    S.X[i].copy_(Xh[i], non_blocking=True)
                    e_in = torch.cuda.Event()
                    e_in.record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(e_in)
                    if j >= P:
                        s_cmp.wait_event(ev_out[j - P])
                    S.layers[i](S.X[i], S.Y[i], S.Xq[i], S.sx[i])
                    ev_cmp.append(torch.cuda.Event())
                    ev_cmp[-1].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[j])
                    Yh[i].copy_(S.Y[i], non_blocking=True)
                    ev_out.append(torch.cuda.Event())
                    ev_out[-1].record(s_out)
            for st_ in (s_in, s_cmp, s_out):
                cur.wait_stream(st_)

        def e2e_time(nsteps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record()
            e2e_steps(nsteps)
            b.record()
            torch.cuda.synchronize()
            return a.elapsed_time(b)

        e2e_steps(2 * P)
        est = max(e2e_time(2 * P) / (2 * P), 1e-3)
        r = int(max(4 * P, min(20000, 400.0 / est)))
        if pg is not None:
            pg.barrier()
        e_ms = max_over_ranks(e2e_time(r), pg, dev)
        e2e = {"value": job_tops(k2_ops(M, N, K), r, world, e_ms), "unit": "TOPS",
               "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2, "ms_per_step": e_ms / r,
               "steps": r, "pipelined": "copy in, compute and copy out on three streams; step j's copy in "
                                        "overlaps the compute and copy out of earlier steps"}
        del Xh, Yh
    variants = [] if args.headline_only else S.variants(decode_like)
    S.free()
    del S
    torch.cuda.empty_cache()

    # ---- every other shape of the suite
    workloads = [head]
    serq = []
    calib = None
    if not args.headline_only:
        base, prev = None, None
        for name, M in SUITE:
            if (name, M) == (head_name, head_M):
                continue
            if name != prev:   # the M values of one workload share one prepared layer
                base, prev = None, name
                torch.cuda.empty_cache()
            wl = synth.WORKLOADS[name].with_m(M)
            Sh = Shape(R, wl, M, base=base)
            base = Sh.base
            workloads.append(Sh.record(M <= 64))
            if (name, M) in VARIANT_SHAPES:
                variants += Sh.variants(M <= 64)
            Sh.free()
            del Sh
        base = None
        torch.cuda.empty_cache()
        # SERQ term's cost in K2: the same weights without the term (r = 0)
        for name, M in [("attn", 2048), ("down", 4096), ("large", 8192)]:
            wl = synth.WORKLOADS[name].with_m(M)
            with_r = next(w for w in workloads if w["workload"] == name and w["M"] == M)
            S0 = Shape(R, wl, M, r=0)
            t0 = R.launch_ms(S0.k2, S0.P)
            serq.append({"workload": name, "M": M, "serq_rank": wl.r, "k2_us_with_term": with_r["k2_us"],
                         "k2_us_without_term": t0 * 1e3,
                         "overhead_pct": 100.0 * (with_r["k2_us"] / (t0 * 1e3) - 1.0)})
            S0.free()
            del S0
            torch.cuda.empty_cache()
        workloads.sort(key=lambda w: [n for n, _ in SUITE].index(w["workload"]) * 100000 + w["M"])
        calib = calibration_record(R)
        torch.cuda.empty_cache()

    targets = {}
    for name, M in TARGET_SHAPES:
        w = next((w for w in workloads if w["workload"] == name and w["M"] == M), None)
        if w is not None:
            targets["%s M=%d" % (name, M)] = {
                "k1_frac_hbm": w["k1_frac_hbm"], "k1_target": K1_TARGET, "k1_met": w["k1_frac_hbm"] >= K1_TARGET,
                "k2_frac_int8": w["k2_frac_int8"], "k2_target": K2_TARGET,
                "k2_met": w["k2_frac_int8"] >= K2_TARGET}

    # ---- roofline of the headline's dominant kernel
    if head["k2_us"] >= head["k1_us"]:
        if decode_like:
            roof = {"kernel": "k_gemm_small (w4a4_linear)", "bound": "hbm", "achieved": head["k2_GBs"],
                    "peak": R.peaks["hbm"], "unit": "GB/s", "bytes_per_launch": head["k2_bytes"]}
        else:
            roof = {"kernel": "k_gemm_pf (w4a4_linear)", "bound": "tensor", "achieved": head["k2_TOPs"],
                    "peak": R.int8_peak, "unit": "TOP/s", "ops_per_launch": head["k2_ops"]}
    else:
        roof = {"kernel": "k_rotq (hq_rotate_quant)", "bound": "hbm", "achieved": head["k1_GBs"],
                "peak": R.peaks["hbm"], "unit": "GB/s", "bytes_per_launch": head["k1_bytes"]}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = (R.peaks["src"] + (" bf16 burst x %.0f (nominal dense int8 / bf16 ratio)" %
                                             NOMINAL_INT8_PER_BF16 if roof["bound"] == "tensor" else " HBM copy"))
    if roof["bound"] == "tensor" and R.int8_peak_sus:
        roof["frac_of_sustained"] = roof["achieved"] / R.int8_peak_sus
    roof["traffic"] = committed_traffic(head_name, head_M, roof["kernel"])

    ops = k2_ops(head_M, wl_head.N, wl_head.K)
    out = {
        "metric": metric_name(), "value": job_tops(ops, steps, world, ms), "unit": "TOPS", "n_gpus": world,
        "steps": steps, "warmup": warm, "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int4", "data": "synthetic (seeded; Llama-shaped activation statistics)",
        "config": config_dict(wl_head, head_M, (P, P * head["k1_bytes"] / 1e6 + P * head["k2_bytes"] / 1e6), world),
        "roofline": roof,
        "kernels": {"k1_rotate_quant": {"ms": head["k1_us"] / 1e3, "GB/s": head["k1_GBs"],
                                        "frac_hbm": head["k1_frac_hbm"], "bytes_per_launch": head["k1_bytes"]},
                    "k2_linear": {"ms": head["k2_us"] / 1e3, "TOP/s": head["k2_TOPs"], "GB/s": head["k2_GBs"],
                                  "frac_int8": head["k2_TOPs"] / R.int8_peak,
                                  "frac_hbm": head["k2_GBs"] / R.peaks["hbm"], "bytes_per_launch": head["k2_bytes"]}},
        "targets": targets,
        "workloads": workloads,
        "serq_overhead": serq,
        "activation_variants": variants,
        "calibration": calib,
        "peaks": {"hbm_GBs": R.peaks["hbm"], "bf16_TFs_burst": R.peaks["bf16"], "bf16_TFs_sustained": R.peaks["bf16_sus"],
                  "int8_TOPs_denominator": R.int8_peak, "source": R.peaks["src"],
                  "int8_cublaslt_8192_TOPs_live": int8_gemm_crosscheck(R)},
        "gpu_launches": 2 * steps,
        "clocks": clocks,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl_head, head_M)
    if rank == 0:
        print(json.dumps(out), flush=True)
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
