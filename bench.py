"""Benchmark of the QLoRA frozen-NF4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload proj7b | smallm --n N --m M | adamw]

One step = the whole hot path on one batch: NF4 + double quantisation of the
bf16 weight, the forward (T = X·A, fused dequant GEMM Y = X·W_hatᵀ + sT·B) and
the backward (U = dY·Bᵀ, fused dequant GEMM dX = dY·W_hat + sU·Aᵀ, dA, dB).
Workload: a single 7B-class projection, W 4096 x 4096, X 4096 tokens
(batch 4 x seq 1024), LoRA r = 64, alpha = 16, synthetic seeded inputs.
value = algorithmic fwd+bwd flops per step / device time (TFLOP/s).

--workload smallm: the decode-sized forward (K = 8192, N = 8192 or 28672 W rows,
M = 1..64 tokens, r = 64; the weight quantised once and resident, rotated over
enough copies to exceed L2); value = packed-weight bytes streamed per forward /
device time (GB/s).

--workload adamw: the fused AdamW step on the 14 adapter tensors (r = 64) of
one LLaMA-7B decoder layer (q, k, v, o: 4096 x 4096; gate, up: 11008 x 4096;
down: 4096 x 11008), 5.0 M parameters, float32 master values and moments plus
the bfloat16 copies, in one launch; value = bytes moved per step / device time
(GB/s), 30 bytes per parameter.

Multi-GPU: data parallel.  Every rank runs the layer on its own 4096-token
shard (same weight, same adapters); the adapter gradients dA and dB, one
float32 bucket, are summed over the ranks by one NCCL all-reduce per step, as
a data-parallel training step needs.  value sums the ranks' work over the
slowest rank's time (weak scaling).  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s; packed-weight GB/s; fraction of roofline"
WORKLOAD = "single 7B-class projection: W 4096x4096 NF4+DQ, X 4096 tokens (4x1024), LoRA r=64 alpha=16"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# DRAM traffic (read + write bytes per launch) of the fused dequant GEMMs from the
# ncu capture summarised in profiles/fused_dequant_gemm_proj7b.md.  Reported only
# while the kernel sources hash to the build that capture was taken of.
KERNEL_SOURCES = ["gemm_pair.cuh", "gemm.cuh", "nf4_decode.cuh", "ptx.cuh", "launch.cuh", "linear.cu"]
TRAFFIC_CAPTURE = {"sources_sha1": "118f0767b267fedf5a145b9c8a726560220b6710",
                   "fwd_y": 46_729_344, "bwd_dx": 45_281_792}


# Same for the small-M kernel (profiles/smallm_dequant_gemm_8192x8192_m16.md), per (N, M).
SMALLM_SOURCES = ["gemm_smallm.cuh", "gemm.cuh", "nf4_decode.cuh", "ptx.cuh", "launch.cuh", "linear.cu"]
SMALLM_TRAFFIC = {"sources_sha1": "be7e178431def2548439e796db2b1528aaaa2b5c", (8192, 16): 35_976_960}


# Same for the AdamW kernel (profiles/adamw_llama7b_layer_adapters.md).
ADAMW_SOURCES = ["adamw.cu", "ptx.cuh", "launch.cuh"]
ADAMW_TRAFFIC = {"sources_sha1": "0064428f763192ff27c64743df1b67afd4a73e71", "bytes": 90_732_000}


def kernel_sources_sha1(files=None) -> str:
    h = hashlib.sha1()
    for f in files or KERNEL_SOURCES:
        with open(os.path.join(ROOT, "bit_nf4_quantised_codebook_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs;
    only samples stamped inside [mark_start, mark_end] are kept."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None
        self.t0 = None
        self.t1 = None

    def mark_start(self):
        self.t0 = datetime.datetime.now()

    def mark_end(self):
        self.t1 = datetime.datetime.now()

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
            if self.gpu_id:
                cmd += ["-i", self.gpu_id]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows, all_rows = [], []
        with open(self.path) as f:
            for ln in f:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) < 9:
                    continue
                all_rows.append(parts)
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                except ValueError:
                    continue
                if self.t0 and self.t1 and self.t0 <= ts <= self.t1:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:  # timed region shorter than the sampling period: keep the nearest samples
            rows = all_rows[-3:]
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows if r[3].replace(".", "").isdigit()), default=None)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, device) -> float:
    """The slowest rank's value (device time), so every rank reports the same job time."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(work_per_replica: float, world: int, seconds: float) -> float:
    """Replicas only: every rank runs the same workload, so the job does `world` times the work."""
    return work_per_replica * world / seconds


def run_ours(args):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from bit_nf4_quantised_codebook_b200 import api, inputs

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    api.lib()
    dev = torch.device("cuda", local)
    case = inputs.proj_7b()
    M, N, K, r, s = case.M, case.N, case.K, case.r, case.s
    flops = case.flops_fwd() + case.flops_bwd()

    # Input sets rotated so that consecutive steps never find their inputs in L2
    # (one set: W 33.5 MB + X 33.5 MB + dY 33.5 MB; outputs 67 MB more).
    NSETS = 3
    sets = []
    for i in range(NSETS):
        c = inputs.LinearCase(case.name, M, N, K, r, case.alpha, case.w_std, case.a_std, case.b_std,
                              seed=case.seed + 10 * i)
        sets.append({k: api.bits_to_tensor(getattr(c, k)(), dev) for k in ("W", "X", "A", "B", "dY")})
    wq = api.alloc_weight(N, K, dev)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    sT = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    # dA and dB share one float32 bucket: with several ranks (data parallel, one token
    # shard per rank) the adapter gradients are summed by one all-reduce per step
    gbucket = torch.empty(K * r + r * N, dtype=torch.float32, device=dev)
    dA = gbucket[:K * r].view(K, r)
    dB = gbucket[K * r:].view(r, N)
    ws_q = torch.empty(api.qlora_workspace_size(api.QLORA_OP_QUANTIZE, 0, N, K, 0), dtype=torch.uint8, device=dev)
    ws_f = torch.empty(api.qlora_workspace_size(api.QLORA_OP_FORWARD, M, N, K, r), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(api.qlora_workspace_size(api.QLORA_OP_BACKWARD, M, N, K, r), dtype=torch.uint8, device=dev)
    err = api.new_error_word(dev)

    def step(i, Win=None, Xin=None, Ain=None, Bin=None, dYin=None):
        st = sets[i % NSETS]
        Wt = st["W"] if Win is None else Win
        Xt = st["X"] if Xin is None else Xin
        At = st["A"] if Ain is None else Ain
        Bt = st["B"] if Bin is None else Bin
        dYt = st["dY"] if dYin is None else dYin
        api.qlora_quantize(Wt, out=wq, ws=ws_q, dev_err=err)
        api.qlora_linear_forward(wq, Xt, At, Bt, s, Y=Y, T_save=sT, ws=ws_f, dev_err=err)
        api.qlora_linear_backward(wq, Xt, dYt, At, Bt, s, T_saved=sT, dX=dX, dA=dA, dB=dB, ws=ws_b, dev_err=err)
        if world > 1:
            dist.all_reduce(gbucket)  # sum of the ranks' adapter gradients (NCCL)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if int(err[0].item()) != 0:
        raise RuntimeError(f"device error word {int(err[0].item())} during warm-up")

    # dominant-kernel events (fused dequant GEMMs), one pair per step
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for quad in ev:          # torch creates events lazily: record once so each has a handle
        for e in quad:
            e.record()
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = api.qlora_kernel_launch_count()
    sampler.mark_start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        api.qlora_set_timing_events(*ev[i])
        step(i)
    t1.record()
    torch.cuda.synchronize()
    sampler.mark_end()
    api.qlora_set_timing_events()
    launches = api.qlora_kernel_launch_count() - launches0
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1)
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    bwd_ms = sum(e[2].elapsed_time(e[3]) for e in ev) / args.steps
    if world > 1:
        ms = max_over_ranks(ms, dev)
    torch.cuda.synchronize()
    if int(err[0].item()) != 0:
        raise RuntimeError(f"device error word {int(err[0].item())} during timing")
    ms_step = ms / args.steps
    value = whole_job_rate(flops, world, ms_step * 1e-3) / 1e12

    # the quantiser alone (block kernel, mean, E4M3 constants), events around each call
    # and a write of a buffer larger than L2 before it, so that W comes from HBM
    qsteps = max(3, min(50, args.steps))
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    qev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(qsteps)]
    for i in range(qsteps):
        flush.zero_()
        qev[i][0].record()
        api.qlora_quantize(sets[i % NSETS]["W"], out=wq, ws=ws_q, dev_err=err)
        qev[i][1].record()
    torch.cuda.synchronize()
    q_ms = sum(a.elapsed_time(b) for a, b in qev) / qsteps
    del flush

    # end to end through the public API with pinned host buffers: H2D of the step's
    # inputs (W, X, A, B, dY), the step, D2H of its results (Y, dX, dA, dB)
    e2e_steps = max(3, min(20, args.steps // 10))
    host_in = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in sets[0].items()}
    for k in host_in:
        host_in[k].copy_(sets[0][k])
    dev_in = {k: torch.empty_like(v) for k, v in sets[0].items()}
    host_out = [torch.empty_like(t, device="cpu").pin_memory() for t in (Y, dX, dA, dB)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(e2e_steps):
        for k in dev_in:
            dev_in[k].copy_(host_in[k], non_blocking=True)
        step(i, dev_in["W"], dev_in["X"], dev_in["A"], dev_in["B"], dev_in["dY"])
        for h, d in zip(host_out, (Y, dX, dA, dB)):
            h.copy_(d, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        e2e_ms = max_over_ranks(e2e_ms, dev)
    e2e_value = whole_job_rate(flops, world, e2e_ms / e2e_steps * 1e-3) / 1e12

    hbm, bf16_burst, bf16_sus, peak_src = _peaks()
    # dominant kernel: the fused dequant GEMM of the backward (dX) or forward (Y), whichever is longer
    dom = "bwd_dx" if bwd_ms >= fwd_ms else "fwd_y"
    dom_ms = max(bwd_ms, fwd_ms)
    dom_flops = 2.0 * M * N * K + 2.0 * M * r * (K if dom == "bwd_dx" else N)
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    packed = wq.nbytes()
    traffic = None
    if TRAFFIC_CAPTURE["sources_sha1"] and TRAFFIC_CAPTURE["sources_sha1"] == kernel_sources_sha1():
        traffic = TRAFFIC_CAPTURE.get(dom)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy N(0,std) rounded to bf16)",
        "config": {"workload": WORKLOAD, "M": M, "N": N, "K": K, "r": r, "alpha": case.alpha,
                   "global_batch": 4 * world, "seq_len": 1024,
                   "parallelism": (f"data parallel x{world}: a 4096-token shard per rank, dA/dB summed by one "
                                   f"NCCL all-reduce per step" if world > 1 else "one GPU"),
                   "step": "quantise(W) + forward + backward",
                   "l2": f"inputs larger than L2: {NSETS} rotating input sets (W, X, dY 33.5 MB each) + 67 MB outputs"},
        "packed_weight_gbs": round(2 * packed / (ms_step * 1e-3) / 1e9, 2),
        "kernels": {"fwd_fused_ms": round(fwd_ms, 4), "bwd_fused_ms": round(bwd_ms, 4),
                    "quantize_ms": round(q_ms, 4)},
        "quantiser": {"params_per_s": round(N * K / (q_ms * 1e-3), 1),
                      "gbs": round((2 * N * K + packed) / (q_ms * 1e-3) / 1e9, 1),
                      "hbm_frac": round((2 * N * K + packed) / (q_ms * 1e-3) / 1e9 / hbm, 4),
                      "bytes": "bf16 W read + stored weight written, per call (3 kernels), L2 flushed before each"},
        "roofline": {"kernel": f"fused dequant GEMM ({dom})", "bound": "tensor",
                     "achieved": round(achieved, 2), "peak": bf16_burst, "unit": "TFLOP/s",
                     "frac": round(achieved / bf16_burst, 4), "peak_source": f"{peak_src} bf16 burst",
                     "traffic": traffic, "traffic_unit": "bytes per launch (ncu dram read+write)"},
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_smallm(args):
    """Forward only at decode batch sizes: T = X·A, then the small-M dequant GEMM."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from bit_nf4_quantised_codebook_b200 import api, inputs

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    api.lib()
    dev = torch.device("cuda", local)
    case = inputs.small_m(args.n, args.m)
    M, N, K, r, s = case.M, case.N, case.K, case.r, case.s
    W = api.bits_to_tensor(case.W(), dev)
    ncopy = max(2, -(-3 * 128 * 2**20 // (N * K // 2)))  # weight copies: > 3x L2 in total
    qs = [api.qlora_quantize(W) for _ in range(ncopy)]
    del W
    packed = qs[0].nbytes()
    X, A, B = (api.bits_to_tensor(getattr(case, k)(), dev) for k in ("X", "A", "B"))
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    sT = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(1, api.qlora_workspace_size(api.QLORA_OP_FORWARD, M, N, K, r)), dtype=torch.uint8,
                     device=dev)
    err = api.new_error_word(dev)

    def step(i, Xin=None):
        api.qlora_linear_forward(qs[i % ncopy], X if Xin is None else Xin, A, B, s, Y=Y, T_save=sT, ws=ws,
                                 dev_err=err)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for pair in ev:
        for e in pair:
            e.record()
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = api.qlora_kernel_launch_count()
    sampler.mark_start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        step(i)
    t1.record()
    torch.cuda.synchronize()
    sampler.mark_end()
    launches = api.qlora_kernel_launch_count() - launches0
    # the dominant kernel alone: events around it (they end the programmatic overlap
    # with the X·A kernel, so this loop is timed separately from the step loop)
    for i in range(args.steps):
        api.qlora_set_timing_events(ev[i][0], ev[i][1])
        step(i)
    torch.cuda.synchronize()
    api.qlora_set_timing_events()
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1)
    kern_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    if world > 1:
        ms = max_over_ranks(ms, dev)
    if int(err[0].item()) != 0:
        raise RuntimeError(f"device error word {int(err[0].item())}")
    ms_step = ms / args.steps
    value = whole_job_rate(packed, world, ms_step * 1e-3) / 1e9

    # end to end: X host -> device, forward, Y device -> host
    e2e_steps = max(3, min(100, args.steps // 10))
    hx = X.cpu().pin_memory()
    hy = torch.empty_like(Y, device="cpu").pin_memory()
    dx = torch.empty_like(X)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(e2e_steps):
        dx.copy_(hx, non_blocking=True)
        step(i, dx)
        hy.copy_(Y, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    hbm, _, _, peak_src = _peaks()
    achieved = packed / (kern_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy N(0,std) rounded to bf16)",
        "config": {"workload": f"small-M forward: W {N}x{K} NF4+DQ, {M} tokens, LoRA r={r} alpha={case.alpha}",
                   "M": M, "N": N, "K": K, "r": r, "parallelism": f"replicas x{world} (no shard)",
                   "step": "forward (X·A, then the dequant GEMM with the adapter term)",
                   "l2": f"{ncopy} resident weight copies used in rotation ({ncopy * packed / 1e6:.0f} MB > L2)"},
        "kernels": {"smallm_gemm_ms": round(kern_ms, 5)},
        "roofline": {"kernel": "small-M dequant GEMM", "bound": "hbm", "achieved": round(achieved, 1),
                     "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                     "peak_source": f"{peak_src} HBM copy",
                     "traffic": (SMALLM_TRAFFIC.get((N, M))
                                 if SMALLM_TRAFFIC["sources_sha1"] == kernel_sources_sha1(SMALLM_SOURCES) else None),
                     "traffic_unit": "bytes per launch (ncu dram read+write)"},
        "e2e": {"value": round(packed / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": X.numel() * 2, "d2h_bytes_per_step": Y.numel() * 2, "steps": e2e_steps},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_smallm(case)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


ADAMW_SHAPES = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]  # (name, N out, K in)
ADAMW_BYTES_PER_PARAM = 4 * 4 + 3 * 4 + 2  # read p, g, m, v; write p, m, v and the bfloat16 copy


def run_adamw(args):
    """The adapter optimiser step for one LLaMA-7B decoder layer (r = 64)."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from bit_nf4_quantised_codebook_b200 import api

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    api.lib()
    dev = torch.device("cuda", local)
    r = 64
    gen = torch.Generator(device=dev).manual_seed(0)
    tensors, host_g, dev_g = [], [], []
    for _, n_out, k_in in ADAMW_SHAPES:
        for shape in ((k_in, r), (r, n_out)):  # A = L1 [K, r], B = L2 [r, N]
            p = torch.randn(shape, generator=gen, device=dev) * 0.01
            g = torch.randn(shape, generator=gen, device=dev)
            tensors.append((p, torch.empty(shape, dtype=torch.bfloat16, device=dev), g,
                            torch.zeros(shape, device=dev), torch.zeros(shape, device=dev)))
            dev_g.append(g)
            host_g.append(g.cpu().pin_memory())
    nparam = sum(t[0].numel() for t in tensors)
    step_bytes = nparam * ADAMW_BYTES_PER_PARAM
    group = api.AdamwGroup(tensors)  # marshalled once; each step is the C call alone

    def step(i):
        group.step(2e-4, 0.9, 0.999, 1e-8, 0.01, i + 1)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = api.qlora_kernel_launch_count()
    sampler.mark_start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        step(args.warmup + i)
    t1.record()
    torch.cuda.synchronize()
    sampler.mark_end()
    launches = api.qlora_kernel_launch_count() - launches0
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1)
    if world > 1:
        ms = max_over_ranks(ms, dev)
    ms_step = ms / args.steps
    value = whole_job_rate(step_bytes, world, ms_step * 1e-3) / 1e9

    # end to end: the gradients host -> device, the step, the bfloat16 parameters device -> host
    e2e_steps = max(3, min(50, args.steps // 10))
    host_b = [torch.empty_like(t[1], device="cpu").pin_memory() for t in tensors]
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(e2e_steps):
        for hg, dg in zip(host_g, dev_g):
            dg.copy_(hg, non_blocking=True)
        step(args.warmup + args.steps + i)
        for hb, t in zip(host_b, tensors):
            hb.copy_(t[1], non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if world > 1:
        e2e_ms = max_over_ranks(e2e_ms, dev)

    hbm, _, _, peak_src = _peaks()
    achieved = step_bytes / (ms_step * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded torch normal)",
        "config": {"workload": "AdamW step on the r=64 adapters of one LLaMA-7B decoder layer (14 tensors)",
                   "params": nparam, "parallelism": f"replicas x{world} (no shard)",
                   "step": "one fused launch: decay, moments, bias-corrected update, bfloat16 copy",
                   "l2": f"working set {step_bytes / 1e6:.0f} MB > L2"},
        "roofline": {"kernel": "k_adamw", "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
                     "unit": "GB/s", "frac": round(achieved / hbm, 4), "peak_source": f"{peak_src} HBM copy",
                     "traffic": (ADAMW_TRAFFIC["bytes"] if ADAMW_TRAFFIC["sources_sha1"] ==
                                 kernel_sources_sha1(ADAMW_SOURCES) else None),
                     "traffic_unit": "bytes per launch (ncu dram read+write)"},
        "e2e": {"value": round(step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": nparam * 4, "d2h_bytes_per_step": nparam * 2, "steps": e2e_steps},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_adamw()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


MERGE_SHAPES = ADAMW_SHAPES  # the seven linears of one LLaMA-7B decoder layer
# ncu DRAM read + write of the merge-and-code kernel over one step's seven launches
# (profiles/merge_requantize_llama7b_layer.md), valid for the sources it was taken from.
MERGE_SOURCES = ["merge.cu", "nf4_decode.cuh", "nf4_quant.cuh", "ptx.cuh", "launch.cuh"]
MERGE_TRAFFIC = {"sources_sha1": "4e714f616c7e4e56f4c0d477b522210425681dd2", "bytes_per_step": 117_096_000}


def merge_bytes(N: int, K: int, r: int) -> int:
    """Algorithmic bytes of one merge: the stored weight read and written once
    (codes, E4M3 constants, group scales, mean) and the adapter read once."""
    nb = N * K // 64
    packed = N * K // 2 + nb + 4 * (-(-nb // 256)) + 4
    return 2 * packed + 2 * r * (K + N)


def merge_kernel_bytes(N: int, K: int, r: int) -> int:
    """Algorithmic bytes of the merge-and-code kernel: old codes and constants
    in, the adapter in, new codes and the float32 block absmax out."""
    nb = N * K // 64
    return N * K // 2 + nb + 4 * (-(-nb // 256)) + 4 + 2 * r * (K + N) + N * K // 2 + 4 * nb


def run_merge(args):
    """Merge the r = 64 adapters of one LLaMA-7B layer into its NF4 weights and
    requantise them: a step is the seven merges."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from bit_nf4_quantised_codebook_b200 import api, inputs

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    api.lib()
    dev = torch.device("cuda", local)
    r, alpha = 64, 16.0
    s = alpha / r
    ncopy = 2  # two resident copies of the layer (each > 200 MB read + written per step) in rotation
    mats, adapters, outs = [], [], []
    for j, (_, N, K) in enumerate(MERGE_SHAPES):
        W = api.bits_to_tensor(inputs.weight_bf16(N, K, 0.02, 10 * j, 0.001), dev)
        mats.append([api.qlora_quantize(W) for _ in range(ncopy)])
        outs.append([api.alloc_weight(N, K, dev) for _ in range(ncopy)])
        del W
        adapters.append((api.bits_to_tensor(inputs.normal_bf16((K, r), 0.01, 10 * j + 2), dev),
                         api.bits_to_tensor(inputs.normal_bf16((r, N), 0.01, 10 * j + 3), dev)))
    ws = torch.empty(max(api.qlora_workspace_size(api.QLORA_OP_MERGE, 0, N, K, r) for _, N, K in MERGE_SHAPES),
                     dtype=torch.uint8, device=dev)
    err = api.new_error_word(dev)
    step_bytes = sum(merge_bytes(N, K, r) for _, N, K in MERGE_SHAPES)
    kern_bytes = sum(merge_kernel_bytes(N, K, r) for _, N, K in MERGE_SHAPES)

    def step(i, hooks=None):
        c = i % ncopy
        for j in range(len(MERGE_SHAPES)):
            if hooks is not None:
                api.qlora_set_timing_events(hooks[j][0], hooks[j][1])
            A, B = adapters[j]
            api.qlora_merge_requantize(mats[j][c], A, B, s, out=outs[j][c], ws=ws, dev_err=err)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    nj = len(MERGE_SHAPES)
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(nj)] for _ in range(args.steps)]
    for row in ev:  # torch creates the CUDA event at its first record; the library records them afterwards
        for pair in row:
            for e in pair:
                e.record()
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = api.qlora_kernel_launch_count()
    sampler.mark_start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        step(i)
    t1.record()
    torch.cuda.synchronize()
    sampler.mark_end()
    launches = api.qlora_kernel_launch_count() - launches0
    # the merge-and-code kernels alone, events around each (a separate loop: the
    # events end the programmatic overlap between the kernels of a merge)
    for i in range(args.steps):
        step(i, ev[i])
    torch.cuda.synchronize()
    api.qlora_set_timing_events()
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1)
    kern_ms = sum(a.elapsed_time(b) for row in ev for a, b in row) / args.steps
    if world > 1:
        ms = max_over_ranks(ms, dev)
    if int(err[0].item()) != 0:
        raise RuntimeError(f"device error word {int(err[0].item())}")
    ms_step = ms / args.steps
    value = whole_job_rate(step_bytes, world, ms_step * 1e-3) / 1e9

    # end to end: each weight's stored form and its adapter host -> device, merge,
    # the new stored form device -> host
    e2e_steps = max(3, min(20, args.steps // 10))
    host_in, host_out, h2d, d2h = [], [], 0, 0
    for j in range(nj):
        q, o = mats[j][0], outs[j][0]
        A, B = adapters[j]
        host_in.append([t.cpu().pin_memory() for t in (q.codes, q.c2q, q.c1, q.mean, A, B)])
        host_out.append([torch.empty_like(t, device="cpu").pin_memory() for t in (o.codes, o.c2q, o.c1, o.mean)])
        h2d += sum(t.numel() * t.element_size() for t in host_in[-1])
        d2h += sum(t.numel() * t.element_size() for t in host_out[-1])
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        for j in range(nj):
            q, o = mats[j][0], outs[j][0]
            A, B = adapters[j]
            for dst, src in zip((q.codes, q.c2q, q.c1, q.mean, A, B), host_in[j]):
                dst.copy_(src, non_blocking=True)
            api.qlora_merge_requantize(q, A, B, s, out=o, ws=ws, dev_err=err)
            for dst, src in zip(host_out[j], (o.codes, o.c2q, o.c1, o.mean)):
                dst.copy_(src, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    hbm, _, _, peak_src = _peaks()
    achieved = kern_bytes / (kern_ms * 1e-3) / 1e9
    line = {
        "metric": "merge + requantise throughput (stored weight read and written, adapter read)",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded numpy N(0,std) rounded to bf16; W with 0.1% t(3) outliers)",
        "config": {"workload": f"adapter merge + NF4 requantisation of one LLaMA-7B layer's 7 linears, "
                               f"LoRA r={r} alpha={alpha}",
                   "shapes": [f"{nm} {N}x{K}" for nm, N, K in MERGE_SHAPES], "r": r,
                   "parallelism": f"replicas x{world} (no shard)",
                   "step": "7 x qlora_merge_requantize (merge-and-code kernel, group sums, mean, E4M3 codes)",
                   "l2": f"{ncopy} copies of the layer in rotation; each step reads and writes "
                         f"{step_bytes / 1e6:.0f} MB (> L2)"},
        "kernels": {"merge_kernel_ms_per_step": round(kern_ms, 5)},
        "roofline": {"kernel": "k_merge_quant (7 launches per step)", "bound": "hbm", "achieved": round(achieved, 1),
                     "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                     "peak_source": f"{peak_src} HBM copy",
                     "traffic": (MERGE_TRAFFIC["bytes_per_step"] if MERGE_TRAFFIC["sources_sha1"] ==
                                 kernel_sources_sha1(MERGE_SOURCES) else None),
                     "traffic_unit": "bytes per step, 7 launches (ncu dram read+write)"},
        "e2e": {"value": round(step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_merge()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def cpu_baseline_merge(min_seconds: float = 10.0) -> dict:
    """The oracle's merge + requantisation on a 256-row slice of the 4096 x 4096
    q projection, repeated; GB/s counted as on the GPU."""
    from bit_nf4_quantised_codebook_b200 import inputs
    from oracle import merge, nf4
    rows, K, r = 256, 4096, 64
    q = nf4.quantize_nf4(inputs.weight_bf16(4096, K, 0.02, 0, 0.001)[:rows])
    A = inputs.normal_bf16((K, r), 0.01, 2)
    B = inputs.normal_bf16((r, 4096), 0.01, 3)[:, :rows]
    tot_t, n = 0.0, 0
    while tot_t < min_seconds or n == 0:
        t = time.perf_counter()
        merge.merge_requantize(q, A, B, 0.25)
        tot_t += time.perf_counter() - t
        n += 1
    return {"value": round(n * merge_bytes(rows, K, r) / tot_t / 1e9, 6), "unit": "GB/s", "cores": os.cpu_count(),
            "kind": "oracle", "sample": f"{n} x merge + requantise of {rows} of the 4096 rows of the 4096x4096 "
                                        f"q projection (float64 numpy); {tot_t:.1f} s"}


FORMAT_CODEBOOKS = ("nf4", "int4", "fp4_e2m1", "fp4_e3m0")
FORMAT_BLOCKS = (32, 64, 128, 256)
FORMAT_DQ = ("none", "e4m3", "int8")


def format_stored_bytes(n: int, k: int, block: int, dq: str) -> int:
    nb = n * k // block
    return n * k // 2 + (4 * nb if dq == "none" else nb + 4 * (-(-nb // 256)) + 4)


def format_step_bytes(n: int, k: int, block: int, dq: str) -> int:
    """Algorithmic bytes of one study point: quantise (read W, write the stored
    form), dequantise (read it, write W_hat), error (read W and W_hat)."""
    st = format_stored_bytes(n, k, block, dq)
    return (2 * n * k + st) + (st + 2 * n * k) + 4 * n * k


def run_formats(args):
    """The format study: the 4096 x 4096 weight (N(0, 0.02) with 0.1% t(3)
    outliers) quantised, dequantised and measured in every code book x block
    size x constant treatment; a step is the 48 round trips."""
    import itertools
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from bit_nf4_quantised_codebook_b200 import api, inputs

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    api.lib()
    dev = torch.device("cuda", local)
    N = K = 4096
    wbits = inputs.weight_bf16(N, K, 0.02, 0, 0.001)
    ncopy = 4  # 4 x 33.5 MB of W in rotation (> L2)
    Ws = [api.bits_to_tensor(wbits, dev) for _ in range(ncopy)]
    fmts = list(itertools.product(FORMAT_CODEBOOKS, FORMAT_BLOCKS, FORMAT_DQ))
    outs = [api.alloc_format_weight(N, K, cb, b, dq, dev) for cb, b, dq in fmts]
    what = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
    stats = torch.empty(len(fmts), 3, dtype=torch.float64, device=dev)
    ws = torch.empty(1 << 24, dtype=torch.uint8, device=dev)
    err = api.new_error_word(dev)
    step_bytes = sum(format_step_bytes(N, K, b, dq) for _, b, dq in fmts)

    def step(i, W=None):
        W = Ws[i % ncopy] if W is None else W
        for j, (cb, b, dq) in enumerate(fmts):
            api.qlora_quantize_format(W, cb, b, dq, out=outs[j], ws=ws, dev_err=err)
            api.qlora_dequantize_format(outs[j], what)
            api.qlora_quant_error(W, what, stats[j])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = api.qlora_kernel_launch_count()
    sampler.mark_start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        step(i)
    t1.record()
    torch.cuda.synchronize()
    sampler.mark_end()
    launches = api.qlora_kernel_launch_count() - launches0
    # the NF4 / 64 / E4M3 quantisation alone (block kernel + second quantisation)
    j0 = fmts.index(("nf4", 64, "e4m3"))
    q_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        q_ev[i][0].record()
        api.qlora_quantize_format(Ws[i % ncopy], "nf4", 64, "e4m3", out=outs[j0], ws=ws, dev_err=err)
        q_ev[i][1].record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1)
    q_ms = sum(a.elapsed_time(b) for a, b in q_ev) / args.steps
    if world > 1:
        ms = max_over_ranks(ms, dev)
    if int(err[0].item()) != 0:
        raise RuntimeError(f"device error word {int(err[0].item())}")
    ms_step = ms / args.steps
    value = whole_job_rate(step_bytes, world, ms_step * 1e-3) / 1e9
    st = stats.cpu().numpy()
    curves = []
    for j, (cb, b, dq) in enumerate(fmts):
        curves.append({"codebook": cb, "block": b, "dq": dq,
                       "bits_per_weight": round(8 * format_stored_bytes(N, K, b, dq) / (N * K), 4),
                       "rel_fro": round(float((st[j, 0] / st[j, 1]) ** 0.5), 5), "max_abs": float(st[j, 2])})

    # end to end: W host -> device, the 48 round trips, the statistics device -> host
    e2e_steps = max(3, min(20, args.steps // 10))
    hw = Ws[0].cpu().pin_memory()
    hs = torch.empty_like(stats, device="cpu").pin_memory()
    dw = torch.empty_like(Ws[0])
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(e2e_steps):
        dw.copy_(hw, non_blocking=True)
        step(i, dw)
        hs.copy_(stats, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    hbm, _, _, peak_src = _peaks()
    q_bytes = 2 * N * K + format_stored_bytes(N, K, 64, "e4m3")
    achieved = q_bytes / (q_ms * 1e-3) / 1e9
    line = {
        "metric": "format study throughput (quantise + dequantise + error, all formats)",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded numpy N(0,0.02) with 0.1% 0.2*t(3) outliers, rounded to bf16)",
        "config": {"workload": "NF4 / Int4 / FP4 E2M1 / FP4 E3M0 x blocks 32-256 x constants float32/E4M3/int8 "
                               "on a 4096x4096 weight", "formats": len(fmts),
                   "parallelism": f"replicas x{world} (no shard)",
                   "l2": f"{ncopy} copies of W in rotation ({ncopy * 2 * N * K / 1e6:.0f} MB > L2)"},
        "curves": curves,
        "kernels": {"quantize_nf4_64_e4m3_ms": round(q_ms, 5)},
        "roofline": {"kernel": "k_quant_format<64> + second quantisation (NF4, E4M3)", "bound": "hbm",
                     "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                     "peak_source": f"{peak_src} HBM copy", "traffic": None,
                     "traffic_unit": "bytes per launch (ncu dram read+write)"},
        "e2e": {"value": round(step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": 2 * N * K, "d2h_bytes_per_step": stats.numel() * 8, "steps": e2e_steps},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_formats(wbits[:256])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def cpu_baseline_formats(wbits, min_seconds: float = 10.0) -> dict:
    """The oracle's round trip in every format on a slice of the weight."""
    import itertools
    from oracle import formats as F
    n, k = wbits.shape
    fmts = list(itertools.product(FORMAT_CODEBOOKS, FORMAT_BLOCKS, FORMAT_DQ))
    tot_t, reps = 0.0, 0
    while tot_t < min_seconds or reps == 0:
        t = time.perf_counter()
        for cb, b, dq in fmts:
            F.error_stats(wbits, F.dequantize_q(F.quantize(wbits, cb, b, dq)))
        tot_t += time.perf_counter() - t
        reps += 1
    by = reps * sum(format_step_bytes(n, k, b, dq) for _, b, dq in fmts)
    return {"value": round(by / tot_t / 1e9, 6), "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{reps} x the 48 round trips on {n} of the 4096 rows (float64 numpy); {tot_t:.1f} s"}


def cpu_baseline_adamw(min_seconds: float = 10.0) -> dict:
    """The oracle's AdamW step on 2^20 parameters, repeated; bytes as on the GPU."""
    import numpy as np
    from oracle import adamw
    rng = np.random.default_rng(0)
    n = 1 << 20
    p, m, v = rng.normal(size=n) * 0.01, np.zeros(n), np.zeros(n)
    g = rng.normal(size=n)
    tot_t, k = 0.0, 0
    while tot_t < min_seconds or k == 0:
        t = time.perf_counter()
        p, m, v = adamw.adamw_step(p, g, m, v, k + 1, 2e-4, 0.9, 0.999, 1e-8, 0.01)
        tot_t += time.perf_counter() - t
        k += 1
    return {"value": round(k * n * ADAMW_BYTES_PER_PARAM / tot_t / 1e9, 4), "unit": "GB/s", "cores": os.cpu_count(),
            "kind": "oracle", "sample": f"{k} AdamW steps on 2^20 parameters (float64 numpy); {tot_t:.1f} s"}


def cpu_baseline_smallm(case, min_seconds: float = 10.0) -> dict:
    """The oracle on a slice of the small-M forward: quantise `rows` W rows and run
    the forward for all tokens through them; GB/s of packed weight per host second."""
    from oracle import linear, nf4
    rows = 256
    W, X, A, B = case.W()[:rows], case.X(), case.A(), case.B()[:, :rows]
    tot_t, n = 0.0, 0
    while tot_t < min_seconds or n == 0:
        t = time.perf_counter()
        what = nf4.dequantize_nf4(nf4.quantize_nf4(W))
        linear.forward(X, what, A, B, case.s)
        tot_t += time.perf_counter() - t
        n += 1
    packed = rows * case.K // 2 + rows * case.K // 64
    return {"value": round(n * packed / tot_t / 1e9, 6), "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{n} x (quantise + dequantise {rows} of the {case.N} W rows, forward for all {case.M} "
                      f"tokens through them); {tot_t:.1f} s"}


def _oracle_sample(rows: int, qrows: int | None = None):
    """The oracle on a bounded sample of the workload: quantise + dequantise
    `qrows` rows of the 4096 x 4096 weight (all of it by default), then forward +
    backward for `rows` token rows through that (sub-)layer."""
    from bit_nf4_quantised_codebook_b200 import inputs
    from oracle import linear, nf4

    case = inputs.proj_7b()
    n = case.N if qrows is None else qrows
    W, X, A, B, dY = case.W()[:n], case.X()[:rows], case.A(), case.B()[:, :n], case.dY()[:rows, :n]
    t = time.perf_counter()
    q = nf4.quantize_nf4(W)
    what = nf4.dequantize_nf4(q)
    linear.forward(X, what, A, B, case.s)
    linear.backward(X, dY, what, A, B, case.s)
    dt = time.perf_counter() - t
    c = inputs.LinearCase(case.name, rows, n, case.K, case.r, case.alpha, case.w_std, case.a_std, case.b_std)
    return dt, c.flops_fwd() + c.flops_bwd()


def cpu_baseline(min_seconds: float = 10.0) -> dict:
    """The oracle as it stands on the full workload (quantise + dequantise the
    4096 x 4096 W, forward + backward on all 4096 token rows), repeated until
    `min_seconds` of host time have passed."""
    tot_t, tot_f, n = 0.0, 0.0, 0
    while tot_t < min_seconds or n == 0:
        dt, fl = _oracle_sample(4096)
        tot_t += dt
        tot_f += fl
        n += 1
    return {"value": round(tot_f / tot_t / 1e12, 6), "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{n} x the full step on the host (quantise + dequantise the 4096x4096 W, fwd + bwd on "
                      f"4096 tokens; float64 numpy, BLAS threads = cores); {tot_t:.1f} s"}


def run_reference(args):
    """The oracle as the reference arm: every step is a bounded sample of the
    workload (a slice of `n` weight rows and `n` token rows), sized so that the
    whole --steps/--warmup run takes about two minutes of host time."""
    world, rank, _ = _dist()
    if rank != 0:
        return
    # host seconds for the whole run (about two minutes; a test shortens it)
    budget = float(os.environ.get("QLORA_REFERENCE_SECONDS", "120")) / max(1, args.steps + args.warmup)
    n = 16
    dt, _ = _oracle_sample(n, n)
    while n < 1024 and dt * 2.2 < budget:
        n *= 2
        dt, _ = _oracle_sample(n, n)
    for _ in range(args.warmup):
        _oracle_sample(n, n)
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = _oracle_sample(n, n)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded numpy N(0,std) rounded to bf16)",
        "config": {"workload": WORKLOAD, "M": 4096, "N": 4096, "K": 4096, "r": 64, "alpha": 16.0,
                   "global_batch": 4, "seq_len": 1024, "parallelism": "cpu oracle"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"per step: quantise+dequantise {n} weight rows (K=4096), fwd+bwd on {n} "
                                   f"token rows through them"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["proj7b", "smallm", "adamw", "merge", "formats"], default="proj7b")
    ap.add_argument("--n", type=int, default=8192, help="smallm: W rows (8192 or 28672)")
    ap.add_argument("--m", type=int, default=16, help="smallm: tokens (1..64)")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "smallm":
        run_smallm(args)
    elif args.workload == "adamw":
        run_adamw(args)
    elif args.workload == "merge":
        run_merge(args)
    elif args.workload == "formats":
        run_formats(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
