#!/usr/bin/env python
"""Benchmark of the fused SVDQuant W4A4 linear layer on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload qkv] [--impl ours|reference]
                    [--extra fc1,fc2,large] [--strong]

A step is one forward pass of the layer over one batch: svdq_quantize_act
(smoothing, NVFP4 encode, fused down-projection) then svdq_linear (NVFP4
tcgen05 GEMM with the fused up-projection and bias).  The residual weight is
packed once beforehand (it is static per layer).  Between steps the L2 cache
is kept cold by rotating over 4 independent copies of the layer and of its
input/output buffers (together several times the 126 MB L2).

Headline: TFLOP/s of the layer on the FLUX QKV projection, counting
2MNK + 2Mr(K+N) per step, over exactly K steps replayed from one CUDA graph.
Every other time (the kernels alone, the layer without its low-rank branch,
the in-house unfused pipeline, L2-warm and L2-flushed steps, the other FLUX
shapes) comes from one protocol: a CUDA graph of S launches, replayed R times,
each replay timed with CUDA events; the line reports the median and the 10th
and 90th percentiles of the per-launch time.

Under torchrun each rank runs its own replica of the layer (no collective on
the data path): by default each rank processes its own batch of M rows (weak
scaling); with --strong one batch of M rows is split into row blocks, one per
rank (strong scaling).  Step times are the maximum over ranks.

--impl reference times the CPU oracle (test infrastructure) on the same
workload; rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused SVDQuant W4A4 linear TFLOP/s and % of B200 dense NVFP4 peak (1 GPU)"
FALLBACK_BF16_TFLOPS = 1590.0       # earlier measurement on this machine (burst)
FALLBACK_HBM_GBS = 6650.0
FP4_OVER_BF16 = 4.0                 # nominal dense ratio (9 / 2.25 PFLOP/s)
N_COPIES = 4
GRAPH_LAUNCHES = 20                 # S: launches (or steps) per timed graph
GRAPH_REPLAYS = 50                  # R: timed replays per graph
FLUSH_BYTES = 256 << 20             # written between steps of the L2-flushed leg (L2 is 126 MB)
# DRAM bytes (read + write) of one k_linear launch on the QKV layer from an ncu capture, valid only
# for the kernel sources it was taken on (sha256 prefix of csrc/linear.cuh + csrc/common.cuh);
# any other source -> traffic null.
LINEAR_TRAFFIC = {"qkv": {"bytes": 26676224.0 + 35307776.0, "sources": "e190fe53fa6d20b5"}}


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="qkv")
    p.add_argument("--extra", default="fc1,fc2,large",
                   help="other FLUX-sized workloads measured with the same protocol ('' for none)")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--strong", action="store_true", help="split one batch of M rows across the ranks")
    p.add_argument("--cpu-sample-rows", type=int, default=0, help="oracle rows (0 = every row of the batch)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--profile-case", action="store_true",
                   help="run each kernel of the step once on one copy of the headline layer, then the fused "
                        "fc1 GEMM of the MLP pair once, and exit (the case the ncu captures are taken on)")
    return p.parse_args(argv)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, FALLBACK_HBM_GBS, "fallback"


def linear_sources_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("linear.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "w4a4_rank_absorbed_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def linear_traffic(workload: str):
    t = LINEAR_TRAFFIC.get(workload)
    return t["bytes"] if t and t["sources"] == linear_sources_hash() else None


def layer_flops(M, K, N, r):
    """2MNK + 2Mr(K+N): the 4-bit GEMM, the down-projection and the up-projection."""
    return 2.0 * M * N * K + 2.0 * M * r * (K + N)


def linear_flops(M, K, N, r):
    """Work of kernel 3 alone: the 4-bit GEMM and the up-projection."""
    return 2.0 * M * N * K + 2.0 * M * N * r


def quantize_bytes(M, K, r):
    """Algorithmic bytes of kernel 2: X read once, codes, scales, the low-rank product (bf16)."""
    return 2.0 * M * K + M * K / 2 + M * K / 16 + 2.0 * M * r


def unfused_extra_bytes(M, K, N, r):
    """What the unfused pipeline moves on top of the fused one: X read again by the separate
    down-projection, and Y read and written again by the separate up-projection (bf16)."""
    return 2.0 * M * K + 4.0 * M * N


def row_block(M: int, rank: int, world: int):
    """Rows [lo, hi) of a batch of M rows that rank `rank` of `world` takes (contiguous, sizes differ by
    at most one)."""
    lo = rank * M // world
    hi = (rank + 1) * M // world
    return lo, hi


def stats(samples):
    """Median and 10th / 90th percentiles of a list of times (ms)."""
    a = np.sort(np.asarray(samples, dtype=np.float64))
    return {"median": float(np.median(a)), "p10": float(np.percentile(a, 10)), "p90": float(np.percentile(a, 90)),
            "n": int(a.size)}


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(flops_per_rank_step, world, ms_per_step_max):
    """Whole-job TFLOP/s: the work of all ranks over the slowest rank's step time."""
    return flops_per_rank_step * world / (ms_per_step_max * 1e-3) / 1e12


def cpu_cores():
    """Host cores (nproc) and the BLAS thread count the oracle's float64 products run on."""
    nproc = os.cpu_count() or 1
    blas = None
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        blas = max((i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"), default=None)
    except Exception:
        pass
    return nproc, blas


# --------------------------------------------------------------- clocks ------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
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
        self.file.flush()
        self.file.seek(0)
        rows = [l.strip().split(",") for l in self.file.read().splitlines() if l.strip()]
        self.file.close()
        os.unlink(self.file.name)
        return self.summarize(rows)

    @staticmethod
    def summarize(rows):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ oracle arm -----
def oracle_forward(dec, pw, X, bias):
    from oracle import linear as OL
    qa = OL.quantize_act(X, dec.inv_s, dec.gs_x, dec.L1f)
    return OL.linear(qa, dec.gs_x, pw, dec.L2b, bias)


def oracle_setup(wl):
    from oracle import decompose as OD
    from oracle import linear as OL
    dec = OD.decompose(wl.X, wl.W, wl.r, wl.alpha, wl.lora_A, wl.lora_B)
    return dec, OL.pack_weight(dec.R32)


def cpu_baseline(wl, rows: int):
    dec, pw = oracle_setup(wl)
    t0 = time.perf_counter()
    oracle_forward(dec, pw, wl.X[:rows], wl.bias)
    dt = time.perf_counter() - t0
    fl = layer_flops(rows, wl.K, wl.N, wl.r_eff)
    nproc, blas = cpu_cores()
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": nproc, "blas_threads": blas, "kind": "oracle",
            "sample": f"oracle forward (quantize_act + linear, float64 from dequantized values) of {rows} of "
                      f"{wl.M} rows of the {wl.name} layer, weight packed beforehand; {dt:.2f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from w4a4_rank_absorbed_b200.synth import make_workload
    wl = make_workload(args.workload)
    dec, pw = oracle_setup(wl)
    # Each step is the oracle's forward over `rows` rows of the batch, every row by default (the same
    # sample as the cpu_baseline of our arm); fewer when K + W steps of the whole batch would take more
    # than about 150 s.
    rows = min(args.cpu_sample_rows or wl.M, wl.M)
    t0 = time.perf_counter()
    oracle_forward(dec, pw, wl.X[:rows], wl.bias)
    t_one = time.perf_counter() - t0
    budget = 150.0
    if (args.steps + args.warmup) * t_one > budget:
        rows = max(128, int(rows * budget / ((args.steps + args.warmup) * t_one)))
    times = []
    for i in range(args.warmup + args.steps):
        lo = (i * rows) % max(1, wl.M - rows + 1)
        t0 = time.perf_counter()
        oracle_forward(dec, pw, wl.X[lo:lo + rows], wl.bias)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    dt = float(np.median(times))
    fl = layer_flops(rows, wl.K, wl.N, wl.r_eff)
    val = fl / dt / 1e12
    nproc, blas = cpu_cores()
    sample = f"oracle forward of {rows} of {wl.M} rows of the {wl.name} layer per step (weight packed beforehand)"
    out = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": workload_config(wl, args),
           "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": nproc, "blas_threads": blas,
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def workload_config(wl, args=None):
    strong = bool(args and getattr(args, "strong", False))
    return {"workload": f"{wl.name}: SVDQuant linear M={wl.M} K={wl.K} N={wl.N} r={wl.r_eff} alpha={wl.alpha}, "
                        f"NVFP4 group 16, bf16 in/out",
            "M": wl.M, "K": wl.K, "N": wl.N, "r": wl.r_eff,
            "flops_per_step": layer_flops(wl.M, wl.K, wl.N, wl.r_eff),
            "l2": f"inputs larger than L2: the loop rotates over {N_COPIES} copies of the layer and its buffers",
            "launch": "the timed steps replayed from one CUDA graph (2 kernel launches per step)",
            "ranks": "one batch of M rows split into row blocks across ranks" if strong else
                     "each rank runs its own batch of M rows (replicas, no collective)"}


# --------------------------------------------------------------- our arm -----
class Timer:
    """Capture a function of the launch index into a CUDA graph of S launches and time its replays."""

    def __init__(self, torch, dev):
        self.torch = torch
        self.dev = dev

    def capture(self, fn, n):
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(device=self.dev)
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            # thread_local: under torchrun the process group's watchdog thread queries CUDA events
            # while we capture; the default (global) mode would invalidate the capture.
            with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
                for i in range(n):
                    fn(i)
        torch.cuda.current_stream().wait_stream(cap)
        return g

    def replay_ms(self, g):
        torch = self.torch
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    def per_launch(self, fn, n=GRAPH_LAUNCHES, reps=GRAPH_REPLAYS, name="graph"):
        """Per-launch times of a graph of n launches replayed reps times (an NVTX range per leg)."""
        with self.torch.cuda.nvtx.range(name):
            g = self.capture(fn, n)
            g.replay()
            self.torch.cuda.synchronize()
            samples = [self.replay_ms(g) / n for _ in range(reps)]
            del g
        return samples


def build_layer_set(name, dev, rows=None, fc1_layer=None):
    """Layer copies and buffers of one workload (calibrated on its own batch)."""
    import torch

    from w4a4_rank_absorbed_b200 import svdq as C
    from w4a4_rank_absorbed_b200.calib import calibrate
    from w4a4_rank_absorbed_b200.layer import SVDQLinear
    from w4a4_rank_absorbed_b200.synth import make_workload

    wl = make_workload(name)
    if name == "fc2":
        # fc2's input is GELU-tanh of fc1's output (the MLP pair), computed here on the GPU
        Y1 = fc1_layer.forward(torch.from_numpy(make_workload("fc1").X.astype(np.float32)).to(torch.bfloat16)
                               .to(dev))
        X2 = torch.nn.functional.gelu(Y1.float(), approximate="tanh").to(torch.bfloat16)
        wl.X = X2.double().cpu().numpy()
        del Y1, X2
    data = calibrate(wl.X, wl.W, wl.r, wl.alpha, bias=wl.bias, lora_A=wl.lora_A, lora_B=wl.lora_B)
    lo, hi = rows if rows is not None else (0, wl.M)
    M = hi - lo
    K, N, r = wl.K, wl.N, data.r
    layers = [SVDQLinear(data, device=dev) for _ in range(N_COPIES)]
    X0 = torch.from_numpy(wl.X[lo:hi].astype(np.float32)).to(torch.bfloat16)
    s = {"wl": wl, "data": data, "M": M, "K": K, "N": N, "r": r, "layers": layers, "X0": X0,
         "Xs": [X0.to(dev) for _ in range(N_COPIES)],
         "Ys": [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(N_COPIES)],
         "LA": [torch.empty((M, 2 * r), dtype=torch.bfloat16, device=dev) if r else None for _ in range(N_COPIES)],
         "ws": [C.new_workspace(M, K, r, dev) for _ in range(N_COPIES)]}
    for L in layers:
        L.act_buffers(M)
    torch.cuda.synchronize()
    return s


def layer_fns(s):
    from w4a4_rank_absorbed_b200 import svdq as C
    M, K, N, r = s["M"], s["K"], s["N"], s["r"]
    layers, Xs, Ys, LA, ws = s["layers"], s["Xs"], s["Ys"], s["LA"], s["ws"]

    def quantize(i):
        return layers[i % N_COPIES].quantize(Xs[i % N_COPIES])

    def gemm(i):
        L = layers[i % N_COPIES]
        Xq, SFx, LAs = L.act_buffers(M)
        L.gemm(Xq, SFx, LAs, Ys[i % N_COPIES])

    def step(i):
        quantize(i)
        gemm(i)

    def plain_qa(i):
        L = layers[i % N_COPIES]
        Xq, SFx, _ = L.act_buffers(M)
        C.svdq_quantize_act(Xs[i % N_COPIES], M, K, L.inv_s, L.gs_x, None, 0, 1.0, Xq, SFx, None)

    def plain_ln(i):
        L = layers[i % N_COPIES]
        Xq, SFx, _ = L.act_buffers(M)
        C.svdq_linear(Xq, SFx, L.gs_x, L.Wq, L.SFw, L.gs_w, None, None, 0, L.bias, Ys[i % N_COPIES], 0, M, N, K)

    def plain(i):
        plain_qa(i)
        plain_ln(i)

    def down(i):
        L = layers[i % N_COPIES]
        C.svdq_lowrank_down(Xs[i % N_COPIES], M, K, L.L1fT, r, 1.0, LA[i % N_COPIES], ws[i % N_COPIES])

    def up(i):
        L = layers[i % N_COPIES]
        C.svdq_lowrank_up(LA[i % N_COPIES], L.L2p, r, 1.0, Ys[i % N_COPIES], 0, M, N)

    def unfused(i):
        plain_qa(i)
        down(i)
        plain_ln(i)
        up(i)

    return {"quantize": quantize, "gemm": gemm, "step": step, "plain": plain, "plain_qa": plain_qa,
            "plain_ln": plain_ln, "down": down, "up": up, "unfused": unfused}


def measure_set(s, timer, dev, flush_buf):
    """Every per-launch distribution of one workload, from the same graph protocol."""
    import torch
    fns = layer_fns(s)
    r = s["r"]
    for i in range(N_COPIES):          # eager once: lazily created state outside the graphs
        fns["unfused"](i) if r else fns["plain"](i)
        fns["step"](i)
    torch.cuda.synchronize()
    out = {}
    for key in ("step", "quantize", "gemm", "plain", "plain_qa", "plain_ln"):
        out[key] = timer.per_launch(fns[key], name=key)
    if r:
        for key in ("unfused", "down", "up"):
            out[key] = timer.per_launch(fns[key], name=key)
    # L2-warm: one layer copy over and over (its inputs, codes and weight stay in the L2 between steps).
    out["step_l2_warm"] = timer.per_launch(lambda i: fns["step"](0), name="step_l2_warm")
    # L2-flushed: a 256 MB write before every step on one copy, minus the same writes alone.
    flush = lambda i: flush_buf.fill_(i & 0xFF)                       # noqa: E731
    both = timer.per_launch(lambda i: (flush(i), fns["step"](0)))
    alone = timer.per_launch(flush)
    out["step_l2_flushed"] = [b - a for b, a in zip(both, alone)]
    return out


def mlp_chain_report(s1, s2, timer, dev):
    """The MLP pair fc1 -> GELU -> fc2 over one batch, fused (fc1's GEMM epilogue applies GELU and
    quantizes fc2's input: svdq_linear_gelu_quantize) against the unfused in-house pair (fc1's layer
    writes Y1, svdq_gelu_bf16, fc2's layer reads X2), same graph protocol, rotating layer copies."""
    import torch

    from w4a4_rank_absorbed_b200 import svdq as C
    from w4a4_rank_absorbed_b200.layer import SVDQMLP
    M = s1["M"]
    L1s, L2s, X1s = s1["layers"], s2["layers"], s1["Xs"]
    n = min(len(L1s), len(L2s))
    mlps = [SVDQMLP(L1s[i], L2s[i]) for i in range(n)]
    Y2s = [torch.empty((M, L2s[0].N), dtype=torch.bfloat16, device=dev) for _ in range(n)]

    def fused(i):
        mlps[i % n].forward(X1s[i % n], out=Y2s[i % n], fused=True)

    def unfused(i):
        mlps[i % n].forward(X1s[i % n], out=Y2s[i % n], fused=False)

    def fc1_fused_gemm(i):
        L1, L2 = L1s[i % n], L2s[i % n]
        L1.gemm_gelu_quantize(*L1.act_buffers(M), L2)

    def gelu_only(i):
        Y1, X2 = mlps[i % n]._mid[M]
        C.svdq_gelu_bf16(Y1, Y1.numel(), X2)

    for i in range(n):
        unfused(i)
        fused(i)
    torch.cuda.synchronize()
    d = {k: stats(timer.per_launch(f, name="mlp_" + k)) for k, f in (("fused", fused), ("unfused", unfused),
                                                     ("fc1_fused_gemm", fc1_fused_gemm), ("gelu", gelu_only))}
    K1, N1, r1 = s1["K"], s1["N"], s1["r"]
    N2, r2 = s2["N"], s2["r"]
    fl = layer_flops(M, K1, N1, r1) + layer_flops(M, N1, N2, r2)
    out = {"M": M, "fc1": [K1, N1, r1], "fc2": [N1, N2, r2], "ms": d,
           "tflops_fused": fl / (d["fused"]["median"] * 1e-3) / 1e12,
           "tflops_unfused": fl / (d["unfused"]["median"] * 1e-3) / 1e12,
           "speedup_fused": d["unfused"]["median"] / d["fused"]["median"],
           "intermediate_bytes_avoided": 4.0 * M * N1,
           "fused": "fc1 quantize, fc1 GEMM + GELU + fc2 quantize/down-projection (+ reduction), fc2 GEMM",
           "unfused": "fc1 quantize, fc1 GEMM -> Y1 bf16, svdq_gelu_bf16, fc2 quantize, fc2 GEMM"}
    del mlps, Y2s
    torch.cuda.empty_cache()
    return out


def workload_report(s, dist_ms, hbm_peak, fp4_peak):
    M, K, N, r = s["M"], s["K"], s["N"], s["r"]
    st = {k: stats(v) for k, v in dist_ms.items()}
    med = {k: v["median"] for k, v in st.items()}
    ln_fl = linear_flops(M, K, N, r)
    qa_b = quantize_bytes(M, K, r)
    rep = {
        "M": M, "K": K, "N": N, "r": r,
        "ms": st,
        "tflops_step": layer_flops(M, K, N, r) / (med["step"] * 1e-3) / 1e12,
        "roofline": {"bound": "tensor", "kernel": "svdq_linear (k_linear)",
                     "achieved": ln_fl / (med["gemm"] * 1e-3) / 1e12, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": ln_fl / (med["gemm"] * 1e-3) / 1e12 / fp4_peak,
                     "flops_per_launch": ln_fl, "ms_per_launch": med["gemm"]},
        "svdq_quantize_act": {"ms": med["quantize"], "GB_per_s": qa_b / (med["quantize"] * 1e-3) / 1e9,
                              "frac": qa_b / (med["quantize"] * 1e-3) / 1e9 / hbm_peak,
                              "algorithmic_bytes": qa_b},
        "lowrank_branch": {"fused_overhead": med["step"] / med["plain"] - 1.0, "gate_fused_overhead": 0.15},
    }
    if r:
        extra = unfused_extra_bytes(M, K, N, r)
        rep["lowrank_branch"].update({
            "unfused_overhead": med["unfused"] / med["plain"] - 1.0,
            "unfused": "in-house: kernel 2 at r = 0, svdq_lowrank_down (re-reads X), kernel 3 at r = 0, "
                       "svdq_lowrank_up (reads and rewrites Y)",
            "unfused_extra_bytes": extra,
            "down_GB_per_s": (2.0 * M * K + 2.0 * M * r) / (med["down"] * 1e-3) / 1e9,
            "up_GB_per_s": (4.0 * M * N + 4.0 * M * r) / (med["up"] * 1e-3) / 1e9})
    return rep


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from w4a4_rank_absorbed_b200 import build
    build.build()
    from w4a4_rank_absorbed_b200 import svdq as C
    from w4a4_rank_absorbed_b200.synth import make_workload

    bf16_peak, hbm_peak, peak_kind = peaks()
    fp4_peak = bf16_peak * FP4_OVER_BF16
    timer = Timer(torch, dev)
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    wl0 = make_workload(args.workload)
    rows = row_block(wl0.M, rank, world) if (args.strong and world > 1) else None
    del wl0
    fc1_layer = fc1_set = None
    names = [args.workload] + [w for w in (args.extra.split(",") if args.extra else []) if w and w != args.workload]
    if "fc2" in names and "fc1" not in names:
        names.insert(names.index("fc2"), "fc1")
    reports, clk_all, head = {}, [], None
    for name in names:
        s = build_layer_set(name, dev, rows=rows if name == args.workload else None, fc1_layer=fc1_layer)
        clocks = ClockSampler(local)
        clocks.start()
        time.sleep(0.2)
        d = measure_set(s, timer, dev, flush_buf)
        if name == args.workload:
            head = headline_steps(s, args, timer, dev, world, dist)
        clk_all.append(clocks.stop())
        st, site = C.svdq_get_device_error()
        if st != 0:
            raise SystemExit(f"device error {st} at {site:#x}")
        keys = sorted(d)
        maxed = max_over_ranks([x for k in keys for x in d[k]], device=dev)
        pos = 0
        for k in keys:
            d[k], pos = maxed[pos:pos + len(d[k])], pos + len(d[k])
        reports[name] = workload_report(s, d, hbm_peak, fp4_peak)
        if name == args.workload:
            e2e = None if args.no_e2e else e2e_leg(s, args, dev, world, dist)
            head_set = {"M": s["M"], "K": s["K"], "N": s["N"], "r": s["r"], "wl": s["wl"], "data": s["data"]}
        if name == "fc2" and fc1_set is not None:
            reports["mlp_chain"] = mlp_chain_report(fc1_set, s, timer, dev)
            fc1_set = None
        if name == "fc1":
            fc1_layer = s["layers"][0]
            if "fc2" in names:
                fc1_set = {k: s[k] for k in ("layers", "Xs", "M", "K", "N", "r")}
            else:
                s["layers"] = s["layers"][:1]
        del s
        torch.cuda.empty_cache()
    # Kernel 1 (offline weight packing, HBM-bound) on the headline layer: one packing of its residual R.
    pack = pack_leg(head_set["data"], dev, timer)
    del fc1_layer

    M, K, N, r = head_set["M"], head_set["K"], head_set["N"], head_set["r"]
    ms = max_over_ranks([head], device=dev)[0]
    fl = layer_flops(M, K, N, r)
    value = job_throughput(fl, world, ms)
    hr = reports[args.workload]
    clk = ClockSampler.summarize([]) if not clk_all else {
        "sm_mhz": statistics.median([c["sm_mhz"] for c in clk_all if c["sm_mhz"] is not None] or [0]),
        "sm_max_mhz": max((c["sm_max_mhz"] or 0) for c in clk_all),
        "reasons": sorted({x for c in clk_all for x in c["reasons"]}),
        "samples": sum(c.get("samples", 0) for c in clk_all)}
    roof = dict(hr["roofline"])
    roof.update({"traffic": linear_traffic(args.workload),
                 "peak_source": f"{peak_kind} bf16 {bf16_peak:.1f} TFLOP/s x {FP4_OVER_BF16:.0f} (nominal "
                                f"NVFP4:bf16 dense ratio), burst: kernels timed in graphs of {GRAPH_LAUNCHES}",
                 "timing": f"median over {GRAPH_REPLAYS} replays of a graph of {GRAPH_LAUNCHES} launches"})
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong" if (args.strong and world > 1) else "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic (seeded PCG64, random-init layer)",
        "config": workload_config(head_set["wl"], args),
        "pct_of_nvfp4_peak": 100.0 * (value / world) / fp4_peak,
        "roofline": roof,
        "kernels": {"svdq_quantize_act": dict(hr["svdq_quantize_act"], hbm_peak_GB_per_s=hbm_peak),
                    "svdq_linear": {"ms": hr["roofline"]["ms_per_launch"], "TFLOP_per_s": hr["roofline"]["achieved"]},
                    "svdq_pack_weight": pack},
        "lowrank_branch": hr["lowrank_branch"],
        "l2": {"rotating_ms": hr["ms"]["step"], "warm_ms": hr["ms"]["step_l2_warm"],
               "flushed_ms": hr["ms"]["step_l2_flushed"]},
        "workloads": {k: v for k, v in reports.items()},
        "protocol": f"every 'ms' distribution: a CUDA graph of {GRAPH_LAUNCHES} launches (or steps) replayed "
                    f"{GRAPH_REPLAYS} times, each replay timed with CUDA events, max over ranks; median, p10, p90 "
                    f"per launch; the headline ms_per_step is one replay of a graph of exactly --steps steps",
        "clocks": clk,
        "gpu_launches": 2 * args.steps,
    }
    if e2e is not None:
        out["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        wl = make_workload(args.workload)
        out["cpu_baseline"] = cpu_baseline(wl, min(args.cpu_sample_rows or wl.M, wl.M))
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


def headline_steps(s, args, timer, dev, world, dist):
    """The contract's timed region: W untimed warm-up steps, then exactly K steps in one graph replay,
    bracketed by a barrier and a device synchronisation on both sides."""
    import torch
    fns = layer_fns(s)
    for i in range(args.warmup):
        fns["step"](i)
    torch.cuda.synchronize()
    g = timer.capture(fns["step"], args.steps)
    g.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ms = timer.replay_ms(g) / args.steps
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    del g
    return ms


def e2e_leg(s, args, dev, world, dist):
    """End to end through the public API with host buffers: every step copies its X in from pinned host
    memory and its Y out to pinned host memory inside the timed region (the layer's streamed call overlaps
    step i's kernels with step i+1's copy in and step i-1's copy out)."""
    import torch
    M, K, N, r = s["M"], s["K"], s["N"], s["r"]
    Xh = s["X0"].pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    Yhs = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    L0 = s["layers"][0]
    X_devs, Y_devs = s["Xs"][:2], s["Ys"][:2]
    L0.forward_host_stream([Xh] * 2, Yhs, X_devs, Y_devs)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record()
    L0.forward_host_stream([Xh] * e2e_steps, [Yhs[i % 2] for i in range(e2e_steps)], X_devs, Y_devs)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([e0.elapsed_time(e1) / e2e_steps], device=dev)[0]
    fl = layer_flops(M, K, N, r)
    return {"value": job_throughput(fl, world, e2e_ms), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(M * K * 2), "d2h_bytes_per_step": int(M * N * 2), "ms_per_step": e2e_ms}


def pack_leg(data, dev, timer):
    import torch

    from w4a4_rank_absorbed_b200 import svdq as C
    K, N, r = data.K, data.N, data.r
    R_dev = data.R.to(dev, torch.float32).contiguous()
    L2b_dev = data.L2b.to(dev).contiguous() if r else None
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    SFw = torch.empty(C.svdq_sf_bytes(N, K), dtype=torch.uint8, device=dev)
    gsw = torch.empty(1, dtype=torch.float32, device=dev)
    L2p = torch.empty((N, r), dtype=torch.bfloat16, device=dev) if r else None

    def pack(i):
        C.svdq_pack_weight(R_dev, L2b_dev, K, N, r, Wq, SFw, gsw, L2p, sync=False)

    pack(0)
    torch.cuda.synchronize()
    st = stats(timer.per_launch(pack, n=4, reps=10))
    pack_bytes = 4.0 * K * N + K * N / 2 + K * N / 16 + 2.0 * r * N + 2.0 * N * r
    return {"ms": st["median"], "GB_per_s": pack_bytes / (st["median"] * 1e-3) / 1e9, "algorithmic_bytes": pack_bytes,
            "note": "offline, once per layer; not in the step"}


def run_profile_case(args):
    """One launch of each kernel on one layer copy (calibrated on the GPU), few launches in all: the
    small case the full ncu captures are taken on.  Device memory: a few hundred MB."""
    import torch

    from w4a4_rank_absorbed_b200 import build
    build.build()
    from w4a4_rank_absorbed_b200 import svdq as C
    from w4a4_rank_absorbed_b200.calib import calibrate_gpu
    from w4a4_rank_absorbed_b200.layer import SVDQLinear
    from w4a4_rank_absorbed_b200.synth import make_workload
    dev = torch.device("cuda", 0)
    wl = make_workload(args.workload)
    L = SVDQLinear(calibrate_gpu(wl.X, wl.W, wl.r, wl.alpha, bias=wl.bias, device=dev), device=dev)
    X = torch.from_numpy(wl.X.astype(np.float32)).to(torch.bfloat16).to(dev)
    Y = torch.empty((wl.M, wl.N), dtype=torch.bfloat16, device=dev)
    L.gemm(*L.quantize(X), Y)
    torch.cuda.synchronize()
    del L, X, Y
    w1, w2 = make_workload("fc1"), make_workload("fc2")
    X1 = torch.from_numpy(w1.X.astype(np.float32)).to(torch.bfloat16).to(dev)
    L1 = SVDQLinear(calibrate_gpu(w1.X, w1.W, w1.r, w1.alpha, bias=w1.bias, device=dev), device=dev)
    X2 = torch.empty((w1.M, w1.N), dtype=torch.bfloat16, device=dev)
    Y1 = L1.forward(X1)
    C.svdq_gelu_bf16(Y1, Y1.numel(), X2)
    L2 = SVDQLinear(calibrate_gpu(X2.float().cpu(), w2.W, w2.r, w2.alpha, bias=w2.bias, device=dev), device=dev)
    del Y1
    L1.gemm_gelu_quantize(*L1.quantize(X1), L2)
    torch.cuda.synchronize()
    st, site = C.svdq_get_device_error()
    if st != 0:
        raise SystemExit(f"device error {st} at {site:#x}")
    print("profile case done", flush=True)


def main():
    args = parse()
    if args.profile_case:
        run_profile_case(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
