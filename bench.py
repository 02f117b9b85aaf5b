#!/usr/bin/env python
"""Benchmark of the fused SVDQuant W4A4 linear layer on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload qkv] [--impl ours|reference]

A step is one forward pass of the layer over one batch: svdq_quantize_act
(smoothing, NVFP4 encode, fused down-projection) then svdq_linear (NVFP4
tcgen05 GEMM with the fused up-projection and bias).  The residual weight is
packed once beforehand (it is static per layer).  To keep the L2 cache cold
between steps, the timed loop rotates over 4 independent copies of the layer
and of its input/output buffers (together several times the 126 MB L2).

Metric: TFLOP/s of the layer, counting 2MNK + 2Mr(K+N) per step, and the
fraction of the NVFP4 dense tensor peak.  Under torchrun each rank runs the
same layer on its own batch (weak scaling, no collective on the data path);
the step time is the maximum over ranks.

--impl reference times the CPU oracle (test infrastructure) on a bounded
sample of the same workload; rank 0 only.
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
# DRAM bytes (read + write) of one k_linear launch from an ncu capture of this bench
# (profiles/k_linear_qkv.md), valid only for the kernel sources it was taken on: the
# sha256 prefix of csrc/linear.cuh + csrc/common.cuh.  Any other source -> traffic null.
LINEAR_TRAFFIC = {"qkv": {"bytes": 26.841600e6 + 35.598336e6, "sources": "126cf5ca30aee97e"}}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="qkv")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--cpu-sample-rows", type=int, default=0, help="oracle rows per step (0 = auto)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


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
    """Whole-job TFLOP/s: the work of all ranks over the slowest rank's step time (weak scaling)."""
    return flops_per_rank_step * world / (ms_per_step_max * 1e-3) / 1e12


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
def oracle_forward_sample(wl, rows: int):
    """Time the oracle's forward (quantize_act + linear) on the first `rows` rows; weight packed beforehand."""
    from oracle import decompose as OD
    from oracle import linear as OL
    dec = OD.decompose(wl.X, wl.W, wl.r, wl.alpha, wl.lora_A, wl.lora_B)
    pw = OL.pack_weight(dec.R32)
    X = wl.X[:rows]
    t0 = time.perf_counter()
    qa = OL.quantize_act(X, dec.inv_s, dec.gs_x, dec.L1f)
    OL.linear(qa, dec.gs_x, pw, dec.L2b, wl.bias)
    dt = time.perf_counter() - t0
    return dt, dec, pw


def cpu_cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"), default=None)
        if n:
            return int(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(wl, rows: int):
    dt, _, _ = oracle_forward_sample(wl, rows)
    fl = layer_flops(rows, wl.K, wl.N, wl.r_eff)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"oracle forward (quantize_act + linear, float64 from dequantized values) of the first "
                      f"{rows} of {wl.M} rows of the {wl.name} layer, weight packed beforehand; "
                      f"{dt:.2f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from w4a4_rank_absorbed_b200.synth import make_workload
    wl = make_workload(args.workload)
    rows = args.cpu_sample_rows or 256
    from oracle import decompose as OD
    from oracle import linear as OL
    dec = OD.decompose(wl.X, wl.W, wl.r, wl.alpha, wl.lora_A, wl.lora_B)
    pw = OL.pack_weight(dec.R32)
    times = []
    for i in range(args.warmup + args.steps):
        lo = (i * rows) % max(1, wl.M - rows + 1)
        X = wl.X[lo:lo + rows]
        t0 = time.perf_counter()
        qa = OL.quantize_act(X, dec.inv_s, dec.gs_x, dec.L1f)
        OL.linear(qa, dec.gs_x, pw, dec.L2b, wl.bias)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    dt = float(np.mean(times))
    fl = layer_flops(rows, wl.K, wl.N, wl.r_eff)
    val = fl / dt / 1e12
    sample = f"oracle forward of {rows} of {wl.M} rows of the {wl.name} layer per step (weight packed beforehand)"
    out = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": workload_config(wl),
           "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def workload_config(wl):
    return {"workload": f"{wl.name}: SVDQuant linear M={wl.M} K={wl.K} N={wl.N} r={wl.r_eff} alpha={wl.alpha}, "
                        f"NVFP4 group 16, bf16 in/out",
            "M": wl.M, "K": wl.K, "N": wl.N, "r": wl.r_eff,
            "flops_per_step": layer_flops(wl.M, wl.K, wl.N, wl.r_eff),
            "l2": f"inputs larger than L2: the loop rotates over {N_COPIES} copies of the layer and its buffers",
            "launch": "the timed steps replayed from one CUDA graph (2 kernel launches per step)"}


# --------------------------------------------------------------- our arm -----
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
    from w4a4_rank_absorbed_b200.calib import calibrate
    from w4a4_rank_absorbed_b200.layer import SVDQLinear
    from w4a4_rank_absorbed_b200.synth import make_workload

    wl = make_workload(args.workload, seed_offset=0)
    data = calibrate(wl.X, wl.W, wl.r, wl.alpha, bias=wl.bias, lora_A=wl.lora_A, lora_B=wl.lora_B)
    M, K, N, r = wl.M, wl.K, wl.N, data.r
    layers = [SVDQLinear(data, device=dev) for _ in range(N_COPIES)]
    X0 = torch.from_numpy(wl.X.astype(np.float32)).to(torch.bfloat16)
    Xs = [X0.to(dev) for _ in range(N_COPIES)]
    Ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(N_COPIES)]
    for L in layers:
        L.act_buffers(M)
    torch.cuda.synchronize()

    def quantize(i):
        return layers[i % N_COPIES].quantize(Xs[i % N_COPIES])

    def gemm(i):
        L = layers[i % N_COPIES]
        Xq, SFx, LAs = L.act_buffers(M)
        L.gemm(Xq, SFx, LAs, Ys[i % N_COPIES])

    for i in range(args.warmup):
        quantize(i)
        gemm(i)
    torch.cuda.synchronize()

    from w4a4_rank_absorbed_b200 import svdq as C

    # The K timed steps are captured in one CUDA graph (step i: kernel 2 then kernel 3 on layer
    # copy i % N_COPIES) and the timed region is one replay of it: device time, without the
    # Python/ctypes launch overhead or the gaps between separately launched graphs.  The
    # per-kernel averages come from two more graphs holding only kernel 2 or only kernel 3
    # launches over the same copies, timed the same way right after.
    def capture(fn, n):
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(device=dev)
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            # thread_local: under torchrun the process group's watchdog thread queries CUDA events
            # while we capture; the default (global) mode would invalidate the capture.
            with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
                for i in range(n):
                    fn(i)
        torch.cuda.current_stream().wait_stream(cap)
        return g

    def step(i):
        quantize(i)
        gemm(i)

    n_kernel = 4 * N_COPIES
    g_steps = capture(step, args.steps)
    g_qa = capture(quantize, n_kernel)
    g_ln = capture(gemm, n_kernel)
    for g in (g_steps, g_qa, g_ln):        # warm replays, untimed
        g.replay()
    torch.cuda.synchronize()

    def timed(g):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ms = timed(g_steps) / args.steps
    if world > 1:
        dist.barrier()
    t_qa = timed(g_qa) / n_kernel
    t_ln = timed(g_ln) / n_kernel
    clk = clocks.stop()
    st, site = C.svdq_get_device_error()
    if st != 0:
        raise SystemExit(f"device error {st} at {site:#x}")
    # The same layer without its low-rank branch (kernel 2 with r = 0, kernel 3 with r = 0) and
    # with the branch unfused (down-projection X L1f and up-projection Y += LA L2 as separate
    # cuBLAS calls that re-read X and re-read and re-write Y): the cost of the branch, fused and not.

    def plain(i):
        L = layers[i % N_COPIES]
        Xq, SFx, _ = L.act_buffers(M)
        C.svdq_quantize_act(Xs[i % N_COPIES], M, K, L.inv_s, L.gs_x, None, 0, 1.0, Xq, SFx, None)
        C.svdq_linear(Xq, SFx, L.gs_x, L.Wq, L.SFw, L.gs_w, None, None, 0, L.bias, Ys[i % N_COPIES], 0, M, N, K)

    lr = []
    for L in layers:
        if r:
            lr.append((L.L1fT.t().contiguous(), L.L2p[:, :r].t().contiguous(),
                       torch.empty((M, r), dtype=torch.bfloat16, device=dev)))

    def unfused(i):
        plain(i)
        if r:
            L1f, L2b, LA = lr[i % N_COPIES]
            torch.matmul(Xs[i % N_COPIES], L1f, out=LA)
            Ys[i % N_COPIES].addmm_(LA, L2b)

    for i in range(N_COPIES):              # eager first: creates the cuBLAS handle and workspace
        unfused(i)
    torch.cuda.synchronize()
    g_plain = capture(plain, n_kernel)
    g_unf = capture(unfused, n_kernel)
    g_plain.replay()
    g_unf.replay()
    torch.cuda.synchronize()
    t_plain = timed(g_plain) / n_kernel
    t_unf = timed(g_unf) / n_kernel
    # L2-warm step: the same two kernels on one layer copy over and over (its inputs, codes and
    # weight stay in the 126 MB L2 between steps).
    g_warm = capture(lambda i: step(0), n_kernel)
    g_warm.replay()
    torch.cuda.synchronize()
    t_warm = timed(g_warm) / n_kernel
    # Kernel 1 (offline weight packing, HBM-bound): one packing of the layer's residual R.
    L0 = layers[0]
    R_dev = data.R.to(dev, torch.float32).contiguous()
    L2b_dev = L0.L2p[:, :r].t().contiguous() if r else None
    Wq_t, SFw_t = torch.empty_like(L0.Wq), torch.empty_like(L0.SFw)
    gsw_t = torch.empty(1, dtype=torch.float32, device=dev)
    L2p_t = torch.empty_like(L0.L2p) if r else None

    def pack(i):
        C.svdq_pack_weight(R_dev, L2b_dev, K, N, r, Wq_t, SFw_t, gsw_t, L2p_t)

    pack(0)
    torch.cuda.synchronize()
    g_pack = capture(pack, 4)
    g_pack.replay()
    torch.cuda.synchronize()
    t_pack = timed(g_pack) / 4
    del R_dev
    ms, t_qa, t_ln, t_plain, t_unf, t_warm, t_pack = max_over_ranks(
        [ms, t_qa, t_ln, t_plain, t_unf, t_warm, t_pack], device=dev)
    del g_steps, g_qa, g_ln, g_plain, g_unf, g_warm, g_pack

    # End to end through the public API with host buffers: every step copies its X in from pinned
    # host memory and its Y out to pinned host memory inside the timed region.  The layer's
    # streamed call overlaps step i's kernels with step i+1's copy in and step i-1's copy out.
    Xh = X0.pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    Yhs = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    X_devs, Y_devs = Xs[:2], Ys[:2]
    L0 = layers[0]
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
    value = job_throughput(fl, world, ms)
    bf16_peak, hbm_peak, peak_kind = peaks()
    fp4_peak = bf16_peak * FP4_OVER_BF16
    lin_flops = 2.0 * M * N * K + 2.0 * M * N * r
    lin_tf = lin_flops / (t_ln * 1e-3) / 1e12
    qa_bytes = 2.0 * M * K + M * K / 2 + M * K / 16 + 2.0 * M * r
    pack_bytes = 4.0 * K * N + K * N / 2 + K * N / 16 + 2.0 * r * N + 4.0 * N * r
    qa_gbs = qa_bytes / (t_qa * 1e-3) / 1e9

    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic (seeded PCG64, random-init layer)",
        "config": workload_config(wl),
        "pct_of_nvfp4_peak": 100.0 * (value / world) / fp4_peak,
        "roofline": {"bound": "tensor", "kernel": "svdq_linear (k_linear)", "achieved": lin_tf, "peak": fp4_peak,
                     "unit": "TFLOP/s", "frac": lin_tf / fp4_peak, "traffic": linear_traffic(args.workload),
                     "peak_source": f"{peak_kind} bf16 {bf16_peak:.1f} TFLOP/s x {FP4_OVER_BF16:.0f} (nominal "
                                    f"NVFP4:bf16 dense ratio)",
                     "flops_per_launch": lin_flops, "ms_per_launch": t_ln},
        "kernels": {"svdq_quantize_act": {"ms": t_qa, "GB_per_s": qa_gbs, "hbm_peak_GB_per_s": hbm_peak,
                                          "frac": qa_gbs / hbm_peak, "algorithmic_bytes": qa_bytes},
                    "svdq_linear": {"ms": t_ln, "TFLOP_per_s": lin_tf},
                    "svdq_pack_weight": {"ms": t_pack, "GB_per_s": pack_bytes / (t_pack * 1e-3) / 1e9,
                                         "algorithmic_bytes": pack_bytes,
                                         "note": "offline, once per layer; not in the step"}},
        "l2_warm_ms_per_step": t_warm,
        "lowrank_branch": {"fused_ms_per_step": ms, "without_branch_ms_per_step": t_plain,
                           "unfused_ms_per_step": t_unf, "fused_overhead": ms / t_plain - 1.0,
                           "unfused_overhead": t_unf / t_plain - 1.0, "gate_fused_overhead": 0.15,
                           "unfused": "kernel 2 and 3 at r = 0, then X L1f and Y += LA L2 as cuBLAS bf16 calls"},
        "clocks": clk,
        "e2e": {"value": job_throughput(fl, world, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(M * K * 2), "d2h_bytes_per_step": int(M * N * 2), "ms_per_step": e2e_ms},
        "gpu_launches": 2 * args.steps,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = min(args.cpu_sample_rows or M, M)       # default: every row of the step (a few s of CPU)
        out["cpu_baseline"] = cpu_baseline(wl, rows)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
