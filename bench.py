"""Benchmark of the QLoRA frozen-NF4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload shapes_65b | llama7b_layer | proj7b | smallm --n N --m M
                                | adamw | merge | formats] [--no-sub] [--no-cpu-baseline]

Default workload: the 65B-class shapes.  The seven linears of one decoder
layer with hidden size 8192 and FFN 22016 (q, k, v, o 8192 x 8192; gate, up
22016 x 8192; down 8192 x 22016), weights N(0, 0.015) with 0.1% Student-t(3)
outliers, quantised to NF4 + double quantisation once at load (the weights
stay resident); 8192 tokens (batch 4 x seq 2048); LoRA r = 64, alpha = 16.
One step = the forward of the seven linears (T = X·A, fused dequant GEMM
Y = X·W_hatᵀ + sT·B) followed by their backward in reverse order (U = dY·Bᵀ,
fused dequant GEMM dX = dY·W_hat + sU·Aᵀ, dA, dB).
value = algorithmic fwd+bwd flops per step / device time (TFLOP/s).

The default line also carries sub-records, each measured the same way: the
single 7B-class projection (4096^3, r = 64), the LLaMA-7B decoder layer's
seven linears at 4096 tokens, the decode-sized forward (packed-weight GB/s
and the fraction of HBM bandwidth of the small-M kernel) on 8192 x 8192 and
28672 x 8192 at 1 and 16 tokens, and the quantiser (load-time cost) on the
22016 x 8192 weight.

--workload smallm: the decode-sized forward alone (K = 8192, N = 8192 or 28672
W rows, M = 1..64 tokens, r = 64).  --workload adamw / merge / formats: the
optimiser step on the adapters, the adapter merge with requantisation and the
storage-format study (see their functions).

Multi-GPU: data parallel over tokens.  Every rank runs the step on its own
8192-token shard (its own seeds for X and dY; the same weights and adapters);
the adapter gradients of all seven linears, one float32 bucket, are summed
over the ranks by one NCCL all-reduce per step.  value sums the ranks' work
over the slowest rank's time (weak scaling).  Rank 0 prints one JSON line.
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
WORKLOADS = {
    "shapes_65b": "65B-class shapes: q/k/v/o 8192x8192, gate/up 22016x8192, down 8192x22016, NF4+DQ, "
                  "8192 tokens (4x2048), LoRA r=64 alpha=16, fwd+bwd of all 7",
    "llama7b_layer": "LLaMA-7B decoder layer linears: q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008, "
                     "NF4+DQ, 4096 tokens (2x2048), LoRA r=64 alpha=16, fwd+bwd of all 7",
    "proj7b": "single 7B-class projection: W 4096x4096 NF4+DQ, X 4096 tokens (4x1024), LoRA r=64 alpha=16, "
              "fwd+bwd",
}
BATCH = {"shapes_65b": (4, 2048), "llama7b_layer": (2, 2048), "proj7b": (4, 1024)}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# DRAM traffic (ncu dram__bytes_read.sum + dram__bytes_write.sum) of the dominant
# kernels, from one-pass ncu launch-list captures, reported only while the kernel
# sources hash to the build each capture was taken of (otherwise null).
# Source hashes below were renewed once without a new capture, after the GEMMs'
# launches switched to plain stream order: a host-side launch attribute, with the
# kernels, their grids and tiles unchanged, so the bytes per launch are too.
# Fused dequant GEMMs, bytes per launch, keyed by (layer set, N, K, "fwd" | "bwd"):
# `ncu --metrics gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum
# --clock-control none -k regex:gemm_pair -s 6 -c 2` over `bench.py --linear <name>
# --no-cpu-baseline --steps 3 --warmup 3` (one linear per step; the capture is the
# first timed step's forward and backward launch), one run per weight shape of the
# set (q, gate and down: k, v and o share q's shape, up shares gate's).  A set's
# figure is the sum over its linears.  The 7B projection's two entries come from
# the launch list of `bench.py --workload proj7b --no-sub --no-cpu-baseline
# --steps 2 --warmup 3` (the same metrics, `-s 21 -c 6`: one step after the load
# and warm-up launches).
KERNEL_SOURCES = ["gemm_pair.cuh", "gemm.cuh", "nf4_decode.cuh", "ptx.cuh", "launch.cuh", "linear.cu"]
TRAFFIC_CAPTURE = {"sources_sha1": "b40d0bee28beb57f87da184c3853be6494423554",
                   ("shapes_65b", 8192, 8192, "fwd"): 539_570_944,
                   ("shapes_65b", 8192, 8192, "bwd"): 535_533_824,
                   ("shapes_65b", 22016, 8192, "fwd"): 1_105_506_048,
                   ("shapes_65b", 22016, 8192, "bwd"): 1_421_735_680,
                   ("shapes_65b", 8192, 22016, "fwd"): 1_415_080_704,
                   ("shapes_65b", 8192, 22016, "bwd"): 1_208_976_128,
                   ("llama7b_layer", 4096, 4096, "fwd"): 46_345_472,
                   ("llama7b_layer", 4096, 4096, "bwd"): 44_085_248,
                   ("llama7b_layer", 11008, 4096, "fwd"): 118_707_968,
                   ("llama7b_layer", 11008, 4096, "bwd"): 197_318_912,
                   ("llama7b_layer", 4096, 11008, "fwd"): 196_402_176,
                   ("llama7b_layer", 4096, 11008, "bwd"): 117_616_896,
                   ("proj7b", 4096, 4096, "fwd"): 44_851_200,
                   ("proj7b", 4096, 4096, "bwd"): 45_932_288}
# The small-M kernel, bytes per launch, per (N, M): the same three metrics with
# `-k regex:smallm -s 3 -c 1` over `bench.py --workload smallm --n N --m M --steps 5
# --warmup 3 --no-cpu-baseline`.
SMALLM_SOURCES = ["gemm_smallm.cuh", "gemm.cuh", "nf4_decode.cuh", "ptx.cuh", "launch.cuh", "linear.cu"]
SMALLM_TRAFFIC = {"sources_sha1": "a8228d129df7c1a36e47db167baba47c3046508d",
                  (8192, 1): 35_737_856, (8192, 16): 35_979_264,
                  (28672, 1): 128_225_536, (28672, 16): 128_480_768}
# The AdamW kernel, bytes per launch: `-k regex:adamw -s 3 -c 1` over `bench.py --workload adamw
# --steps 3 --warmup 3 --no-cpu-baseline` (the 150 MB working set is only a little larger than
# L2, so part of the writes stay in L2).
ADAMW_SOURCES = ["adamw.cu", "ptx.cuh", "launch.cuh"]
ADAMW_TRAFFIC = {"sources_sha1": "4fff1a2cc2a9bff24c7253a43f3cd653498792f8", "bytes": 97_109_760}


def kernel_sources_sha1(files=None) -> str:
    h = hashlib.sha1()
    for f in files or KERNEL_SOURCES:
        with open(os.path.join(ROOT, "bit_nf4_quantised_codebook_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _traffic(table, files, key):
    if table.get("sources_sha1") and table["sources_sha1"] == kernel_sources_sha1(files):
        return table.get(key)
    return None


def fused_traffic(name: str, cases, dom: str, table=None, files=None):
    """DRAM bytes of the fused GEMM launches (forward or backward) of `cases`:
    the sum of the per-shape captures, or None if any shape is missing or the
    kernel sources have changed since the capture."""
    table = TRAFFIC_CAPTURE if table is None else table
    vals = [_traffic(table, files or KERNEL_SOURCES, (name, c.N, c.K, dom)) for c in cases]
    return None if not vals or any(v is None for v in vals) else int(sum(vals))


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


def _gpu_sampler(local):
    import torch
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    s = ClockSampler(gpu_id)
    s.start()
    return s


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _init_dist(world, local):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))


def max_over_ranks(x: float, device) -> float:
    """The slowest rank's value (device time), so every rank reports the same job time."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(work_per_replica: float, world: int, seconds: float) -> float:
    """Every rank does the same amount of work (its own shard or replica), so the job does `world` times it."""
    return work_per_replica * world / seconds


def grad_bucket(shapes, device):
    """One float32 bucket holding the adapter gradients dA [K, r] and dB [r, N]
    of every linear, so that a data-parallel step sums them with one
    all-reduce.  shapes = [(K, r, N), ...]; returns (bucket, [(dA, dB), ...])."""
    import torch
    total = sum(k * r + r * n for k, r, n in shapes)
    bucket = torch.zeros(total, dtype=torch.float32, device=device)
    views, off = [], 0
    for k, r, n in shapes:
        dA = bucket[off:off + k * r].view(k, r)
        off += k * r
        dB = bucket[off:off + r * n].view(r, n)
        off += r * n
        views.append((dA, dB))
    return bucket, views


def allreduce_grads(bucket) -> None:
    """The exchange step of data parallelism: dA and dB are sums over tokens, so
    the ranks' shard gradients add up to the whole batch's (one sum all-reduce)."""
    import torch.distributed as dist
    dist.all_reduce(bucket)


# ---------------------------------------------------------------- inputs
def _gen_tensor(kind: str, fields: dict):
    """One seeded input tensor (bfloat16 bits) of a linear; runs in a worker process."""
    from bit_nf4_quantised_codebook_b200 import inputs
    return getattr(inputs.LinearCase(**fields), kind)()


def _fields(c) -> dict:
    return dict(name=c.name, M=c.M, N=c.N, K=c.K, r=c.r, alpha=c.alpha, w_std=c.w_std, a_std=c.a_std,
                b_std=c.b_std, outlier_frac=c.outlier_frac, seed=c.seed)


def tensor_key(kind: str, c) -> tuple:
    """Inputs that the seeded recipe makes identical (same generator seed, shape
    and distribution) share one key and are generated once."""
    if kind == "W":
        return ("W", c.N, c.K, c.w_std, c.outlier_frac, c.seed)
    if kind == "X":
        return ("X", c.M, c.K, c.seed)
    if kind == "A":
        return ("A", c.K, c.r, c.a_std, c.seed)
    if kind == "B":
        return ("B", c.r, c.N, c.b_std, c.seed)
    return ("dY", c.M, c.N, c.seed)


def generate(requests, workers: int) -> dict:
    """requests = {key: (kind, case)} -> {key: bfloat16 bits}; independent tensors
    are drawn in parallel worker processes (spawned, so safe beside CUDA)."""
    specs = {k: (kind, _fields(c)) for k, (kind, c) in requests.items()}
    if workers > 1 and len(specs) > 1:
        import multiprocessing as mp
        from concurrent.futures import ProcessPoolExecutor
        with ProcessPoolExecutor(max_workers=min(workers, len(specs)), mp_context=mp.get_context("spawn")) as ex:
            futs = {k: ex.submit(_gen_tensor, *v) for k, v in specs.items()}
            return {k: f.result() for k, f in futs.items()}
    return {k: _gen_tensor(*v) for k, v in specs.items()}


def _workers(world: int) -> int:
    return max(1, min(8, (os.cpu_count() or 1) // max(1, world)))


def shard_case(c, rank: int):
    """The case whose X and dY are rank `rank`'s token shard (other seeds); rank 0 keeps the configuration's."""
    from bit_nf4_quantised_codebook_b200 import inputs
    return c if rank == 0 else inputs.LinearCase(c.name, c.M, c.N, c.K, c.r, c.alpha, c.w_std, c.a_std, c.b_std,
                                                 c.outlier_frac, c.seed + 1000 * rank)


def fused_bytes(c) -> tuple[int, int]:
    """Algorithmic bytes of the two fused dequant GEMM launches of one linear: the
    activation read, the stored weight read once, the adapter operands, the output
    written (forward: X, W_nf4, sT, B, Y; backward: dY, W_nf4, sU, A, dX)."""
    nb = c.N * c.K // 64
    packed = c.N * c.K // 2 + nb + 4 * (-(-nb // 256)) + 4
    return (2 * c.M * c.K + packed + 2 * c.M * c.r + 2 * c.r * c.N + 2 * c.M * c.N,
            2 * c.M * c.N + packed + 2 * c.M * c.r + 2 * c.K * c.r + 2 * c.M * c.K)


def fused_flops(c) -> tuple[float, float]:
    """Algorithmic flops of the two fused dequant GEMM launches of one linear:
    forward X·W_hatᵀ + sT·B and backward dY·W_hat + sU·Aᵀ."""
    return (2.0 * c.M * c.N * c.K + 2.0 * c.M * c.r * c.N, 2.0 * c.M * c.N * c.K + 2.0 * c.M * c.r * c.K)


# ---------------------------------------------------------------- layer sets (fwd + bwd)
class LayerSet:
    """The linears of one workload on the device: weights quantised once and
    resident, every linear's own input, output and gradient buffers, and one
    training step over them (forwards in order, backwards in reverse)."""

    def __init__(self, cases, dev, rank: int = 0, world: int = 1):
        import torch
        from bit_nf4_quantised_codebook_b200 import api
        self.api = api
        self.cases = list(cases)
        self.dev = dev
        xcases = [shard_case(c, rank) for c in self.cases]
        req = {}
        for c, xc in zip(self.cases, xcases):
            for kind in ("W", "A", "B"):
                req[tensor_key(kind, c)] = (kind, c)
            for kind in ("X", "dY"):
                req[tensor_key(kind, xc)] = (kind, xc)
        host = generate(req, _workers(world))
        self.err = api.new_error_word(dev)
        ws_q = torch.empty(max(api.qlora_workspace_size(api.QLORA_OP_QUANTIZE, 0, c.N, c.K, 0) for c in self.cases),
                           dtype=torch.uint8, device=dev)
        self.ws_f = torch.empty(max(16, max(api.qlora_workspace_size(api.QLORA_OP_FORWARD, c.M, c.N, c.K, c.r)
                                            for c in self.cases)), dtype=torch.uint8, device=dev)
        self.ws_b = torch.empty(max(16, max(api.qlora_workspace_size(api.QLORA_OP_BACKWARD, c.M, c.N, c.K, c.r)
                                            for c in self.cases)), dtype=torch.uint8, device=dev)
        self.bucket, views = grad_bucket([(c.K, c.r, c.N) for c in self.cases], dev)
        self.lin = []
        for c, xc, (dA, dB) in zip(self.cases, xcases, views):
            W = api.bits_to_tensor(host[tensor_key("W", c)], dev)
            q = api.qlora_quantize(W, ws=ws_q, dev_err=self.err)
            del W
            L = {"case": c, "q": q, "dA": dA, "dB": dB,
                 "X": api.bits_to_tensor(host[tensor_key("X", xc)], dev),
                 "dY": api.bits_to_tensor(host[tensor_key("dY", xc)], dev),
                 "A": api.bits_to_tensor(host[tensor_key("A", c)], dev),
                 "B": api.bits_to_tensor(host[tensor_key("B", c)], dev),
                 "Y": torch.empty(c.M, c.N, dtype=torch.bfloat16, device=dev),
                 "sT": torch.empty(c.M, c.r, dtype=torch.bfloat16, device=dev),
                 "dX": torch.empty(c.M, c.K, dtype=torch.bfloat16, device=dev)}
            self.lin.append(L)
        del host, ws_q
        torch.cuda.synchronize()
        self.check("quantisation at load")

    def check(self, what: str) -> None:
        import torch
        torch.cuda.synchronize()
        if int(self.err[0].item()) != 0:
            raise RuntimeError(f"device error word {int(self.err[0].item())} during {what}")

    def flops(self) -> float:
        return sum(c.flops_fwd() + c.flops_bwd() for c in self.cases)

    def packed_bytes(self) -> int:
        return sum(L["q"].nbytes() for L in self.lin)

    def step(self, ev=None) -> None:
        api = self.api
        for j, L in enumerate(self.lin):
            if ev is not None:
                api.qlora_set_timing_events(*ev[j])
            api.qlora_linear_forward(L["q"], L["X"], L["A"], L["B"], L["case"].s, Y=L["Y"], T_save=L["sT"],
                                     ws=self.ws_f, dev_err=self.err)
        for j in reversed(range(len(self.lin))):
            L = self.lin[j]
            if ev is not None:
                api.qlora_set_timing_events(*ev[j])
            api.qlora_linear_backward(L["q"], L["X"], L["dY"], L["A"], L["B"], L["case"].s, T_saved=L["sT"],
                                      dX=L["dX"], dA=L["dA"], dB=L["dB"], ws=self.ws_b, dev_err=self.err)
        if ev is not None:
            api.qlora_set_timing_events()

    def e2e(self, e2e_steps: int, world: int) -> tuple[float, int, int]:
        """Device time of `e2e_steps` training steps with every input copied in from
        pinned host memory and every output copied back, the copies on their own
        streams so that they overlap the compute and each other (host-to-device and
        device-to-host run on separate copy engines).  X, dY, Y and dX are double
        buffered by step parity; event waits keep every buffer from being refilled
        before its last reader is done.  Returns (ms, h2d bytes, d2h bytes) per step."""
        import torch
        nl = len(self.lin)
        h_in = [{k: torch.empty_like(L[k], device="cpu").pin_memory() for k in ("X", "dY")} for L in self.lin]
        for h, L in zip(h_in, self.lin):
            for k in h:
                h[k].copy_(L[k])
        h_out = [{k: torch.empty_like(L[k], device="cpu").pin_memory() for k in ("Y", "dX")} for L in self.lin]
        h_grad = torch.empty_like(self.bucket, device="cpu").pin_memory()
        h2d = sum(t.numel() * t.element_size() for h in h_in for t in h.values())
        d2h = sum(t.numel() * t.element_size() for h in h_out for t in h.values()) + h_grad.numel() * 4
        bufs = [[{k: L[k] for k in ("X", "dY", "Y", "dX")} for L in self.lin],
                [{k: torch.empty_like(L[k]) for k in ("X", "dY", "Y", "dX")} for L in self.lin]]
        main = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

        def events():
            return [torch.cuda.Event() for _ in range(nl)]

        # per parity: inputs landed, forward done, backward done, outputs copied out
        in_x, in_dy, fwd_done, bwd_done, out_y, out_dx = ([events(), events()] for _ in range(6))
        grad_out = torch.cuda.Event()
        api = self.api
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(main)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for st in range(e2e_steps):
            p, old = st % 2, st >= 2  # `old`: the buffers of parity p were used two steps ago
            B = bufs[p]
            with torch.cuda.stream(s_in):
                for i in range(nl):
                    if old:
                        s_in.wait_event(bwd_done[p][i])  # the last reader of X_i and dY_i
                    B[i]["X"].copy_(h_in[i]["X"], non_blocking=True)
                    in_x[p][i].record(s_in)
                for i in reversed(range(nl)):
                    B[i]["dY"].copy_(h_in[i]["dY"], non_blocking=True)
                    in_dy[p][i].record(s_in)
            for i, L in enumerate(self.lin):
                main.wait_event(in_x[p][i])
                if old:
                    main.wait_event(out_y[p][i])  # Y_i of two steps ago has been copied out
                api.qlora_linear_forward(L["q"], B[i]["X"], L["A"], L["B"], L["case"].s, Y=B[i]["Y"],
                                         T_save=L["sT"], ws=self.ws_f, dev_err=self.err)
                fwd_done[p][i].record(main)
            if st >= 1:
                main.wait_event(grad_out)  # the previous step's gradients have been copied out
            for i in reversed(range(nl)):
                L = self.lin[i]
                main.wait_event(in_dy[p][i])
                if old:
                    main.wait_event(out_dx[p][i])
                api.qlora_linear_backward(L["q"], B[i]["X"], B[i]["dY"], L["A"], L["B"], L["case"].s,
                                          T_saved=L["sT"], dX=B[i]["dX"], dA=L["dA"], dB=L["dB"], ws=self.ws_b,
                                          dev_err=self.err)
                bwd_done[p][i].record(main)
            if world > 1:
                allreduce_grads(self.bucket)
            grads_ready = torch.cuda.Event()
            grads_ready.record(main)
            with torch.cuda.stream(s_out):
                for i in range(nl):
                    s_out.wait_event(fwd_done[p][i])
                    h_out[i]["Y"].copy_(B[i]["Y"], non_blocking=True)
                    out_y[p][i].record(s_out)
                for i in reversed(range(nl)):
                    s_out.wait_event(bwd_done[p][i])
                    h_out[i]["dX"].copy_(B[i]["dX"], non_blocking=True)
                    out_dx[p][i].record(s_out)
                s_out.wait_event(grads_ready)
                h_grad.copy_(self.bucket, non_blocking=True)
                grad_out.record(s_out)
        done_in, done_out = torch.cuda.Event(), torch.cuda.Event()
        done_in.record(s_in)
        done_out.record(s_out)
        main.wait_event(done_in)
        main.wait_event(done_out)
        e1.record(main)
        torch.cuda.synchronize()
        # the overlapped copies must not have changed the result: the outputs copied out
        # should equal the device step's (both buffer sets hold the same inputs); the
        # outcome is reported in the line rather than raised
        differ = [f"{k}{i}" for i, L in enumerate(self.lin) for k in ("Y", "dX")
                  if not torch.equal(h_out[i][k], L[k].cpu())]
        if not torch.equal(h_grad, self.bucket.cpu()):
            differ.append("grads")
        self.e2e_differ = differ
        return e0.elapsed_time(e1), h2d, d2h

    def measure(self, steps: int, warmup: int, world: int, local: int, e2e_steps: int = 3) -> dict:
        """Warm-up, K timed steps (barrier + synchronize on both sides, max over
        ranks), a second loop with events around every fused dequant GEMM, and
        the end-to-end loop through pinned host buffers."""
        import torch
        import torch.distributed as dist
        api = self.api

        def one(ev=None):
            self.step(ev)
            if world > 1:
                allreduce_grads(self.bucket)

        for _ in range(warmup):
            one()
        self.check("warm-up")
        sampler = _gpu_sampler(local)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        launches0 = api.qlora_kernel_launch_count()
        sampler.mark_start()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(steps):
            one()
        t1.record()
        torch.cuda.synchronize()
        sampler.mark_end()
        launches = api.qlora_kernel_launch_count() - launches0
        if world > 1:
            dist.barrier()
        clocks = sampler.stop()
        ms = t0.elapsed_time(t1)
        if world > 1:
            ms = max_over_ranks(ms, self.dev)
        self.check("timing")

        # the fused dequant GEMMs alone: events the library records around each launch
        # (a separate loop, since an event between two kernels ends their programmatic overlap)
        ksteps = max(1, min(steps, 10))
        nl = len(self.lin)
        ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nl)] for _ in range(ksteps)]
        for row in ev:  # torch creates a CUDA event at its first record; the library records them afterwards
            for quad in row:
                for e in quad:
                    e.record()
        for i in range(ksteps):
            one(ev[i])
        torch.cuda.synchronize()
        fwd_ms = [sum(ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(ksteps)) / ksteps for j in range(nl)]
        bwd_ms = [sum(ev[i][j][2].elapsed_time(ev[i][j][3]) for i in range(ksteps)) / ksteps for j in range(nl)]

        # end to end through the public API: every linear's X and dY in from pinned
        # host memory, the step, Y, dX and the adapter gradients back out
        e2e_ms, h2d, d2h = self.e2e(e2e_steps, world)
        if world > 1:
            e2e_ms = max_over_ranks(e2e_ms, self.dev)
        self.check("the end-to-end loop")
        return {"ms_step": ms / steps, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "launches": int(launches),
                "clocks": clocks, "e2e_ms_step": e2e_ms / e2e_steps, "e2e_steps": e2e_steps, "h2d": h2d,
                "d2h": d2h, "e2e_differ": self.e2e_differ}


def layer_record(name: str, ls: LayerSet, m: dict, world: int, steps: int, warmup: int) -> dict:
    """The JSON record of one layer-set measurement (the main line's fields)."""
    hbm, bf16_burst, bf16_sus, peak_src = _peaks()
    flops = ls.flops()
    value = whole_job_rate(flops, world, m["ms_step"] * 1e-3) / 1e12
    ff = [fused_flops(c) for c in ls.cases]
    fwd_f, bwd_f = sum(f for f, _ in ff), sum(b for _, b in ff)
    fwd_t, bwd_t = sum(m["fwd_ms"]), sum(m["bwd_ms"])
    # dominant kernel: the fused dequant GEMM variant (forward or backward) with the larger share of the step;
    # achieved = its algorithmic flops over the seven launches / their summed event time
    dom = "bwd" if bwd_t >= fwd_t else "fwd"
    dom_f, dom_t = (bwd_f, bwd_t) if dom == "bwd" else (fwd_f, fwd_t)
    achieved = dom_f / (dom_t * 1e-3) / 1e12
    c0 = ls.cases[0]
    batch, seq = BATCH.get(name, (1, c0.M))
    packed = ls.packed_bytes()
    per = [{"linear": c.name.split("_")[1] if name != "proj7b" else "proj", "N": c.N, "K": c.K,
            "fwd_fused_ms": round(f, 5), "bwd_fused_ms": round(b, 5),
            "fwd_fused_tflops": round(fused_flops(c)[0] / (f * 1e-3) / 1e12, 1),
            "bwd_fused_tflops": round(fused_flops(c)[1] / (b * 1e-3) / 1e12, 1)}
           for c, f, b in zip(ls.cases, m["fwd_ms"], m["bwd_ms"])]
    nlin = len(ls.cases)
    return {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": round(m["ms_step"], 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy N(0,std) rounded to bf16" +
                ("; W with 0.1% 0.2*t(3) outliers)" if c0.outlier_frac else ")"),
        "config": {"workload": WORKLOADS[name], "M": c0.M, "r": c0.r, "alpha": c0.alpha,
                   "shapes": [f"{c.name.split('_')[1] if name != 'proj7b' else 'proj'} {c.N}x{c.K}"
                              for c in ls.cases],
                   "global_batch": batch * world, "seq_len": seq,
                   "parallelism": (f"data parallel x{world}: a {c0.M}-token shard per rank, the adapter gradients "
                                   f"summed by one NCCL all-reduce per step" if world > 1 else "one GPU"),
                   "step": (f"forward of the {nlin} linears, then their backward in reverse order; the weights are "
                            f"quantised once at load (the quantiser is reported on its own)" if nlin > 1 else
                            "forward + backward; the weight is quantised once at load"),
                   "l2": f"inputs larger than L2: a step reads {(packed + sum(2 * c.M * (c.K + c.N) for c in ls.cases)) / 1e9:.2f} GB"},
        "packed_weight_gbs": round(2 * packed / (m["ms_step"] * 1e-3) / 1e9, 2),
        "kernels": {"fwd_fused_ms": round(fwd_t, 5), "bwd_fused_ms": round(bwd_t, 5), "per_linear": per},
        "roofline": {"kernel": f"fused dequant GEMM ({dom}, {nlin} launch{'es' if nlin > 1 else ''} per step)",
                     "bound": "tensor", "achieved": round(achieved, 2), "peak": bf16_burst, "unit": "TFLOP/s",
                     "frac": round(achieved / bf16_burst, 4),
                     "frac_of_sustained": round(achieved / bf16_sus, 4) if bf16_sus else None,
                     "peak_source": f"{peak_src} bf16 burst",
                     "traffic": fused_traffic(name, ls.cases, dom),
                     "traffic_unit": f"bytes per step over the {nlin} {dom} launches (ncu dram read+write, "
                                     f"one capture per weight shape)",
                     "algorithmic_bytes": sum(fused_bytes(c)[0 if dom == "fwd" else 1] for c in ls.cases)},
        "e2e": {"value": round(whole_job_rate(flops, world, m["e2e_ms_step"] * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": m["h2d"], "d2h_bytes_per_step": m["d2h"], "steps": m["e2e_steps"],
                "copies": "overlapped with the compute on two copy streams",
                "outputs_equal_device_step": not m["e2e_differ"],
                **({"outputs_differing": m["e2e_differ"]} if m["e2e_differ"] else {})},
        "gpu_launches": m["launches"],
        "clocks": m["clocks"],
    }


def layer_cases(name: str):
    from bit_nf4_quantised_codebook_b200 import inputs
    return {"shapes_65b": inputs.shapes_65b, "llama7b_layer": inputs.llama7b_layer,
            "proj7b": lambda: [inputs.proj_7b()]}[name]()


def measure_layer_set(name: str, steps: int, warmup: int, world: int, rank: int, local: int,
                      only: str | None = None) -> dict:
    import torch
    dev = torch.device("cuda", local)
    cases = layer_cases(name)
    if only:  # one linear of the set (for a profiler capture of a single shape)
        cases = [c for c in cases if c.name.split("_")[1] == only][:1]
        if not cases:
            raise SystemExit(f"--linear {only}: no such linear in {name}")
    ls = LayerSet(cases, dev, rank, world)
    m = ls.measure(steps, warmup, world, local, e2e_steps=max(4, min(10, steps // 2)))
    rec = layer_record(name, ls, m, world, steps, warmup)
    del ls
    torch.cuda.empty_cache()
    return rec


# ---------------------------------------------------------------- decode-sized forward
def measure_smallm(n: int, m_tok: int, steps: int, warmup: int, world: int, local: int,
                   e2e_steps: int | None = None) -> dict:
    """Forward at decode batch sizes: T = X·A, then the small-M dequant GEMM.
    The weight is quantised once and kept resident, rotated over enough copies
    that no forward finds it in L2."""
    import torch
    import torch.distributed as dist
    from bit_nf4_quantised_codebook_b200 import api, inputs
    dev = torch.device("cuda", local)
    case = inputs.small_m(n, m_tok)
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

    def step(i, Xin=None, Yout=None):
        api.qlora_linear_forward(qs[i % ncopy], X if Xin is None else Xin, A, B, s, Y=Y if Yout is None else Yout,
                                 T_save=sT, ws=ws, dev_err=err)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for pair in ev:
        for e in pair:
            e.record()
    sampler = _gpu_sampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = api.qlora_kernel_launch_count()
    sampler.mark_start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(steps):
        step(i)
    t1.record()
    torch.cuda.synchronize()
    sampler.mark_end()
    launches = api.qlora_kernel_launch_count() - launches0
    # the small-M kernel alone: events around it (they end the programmatic overlap
    # with the X·A kernel, so this loop is timed separately from the step loop)
    for i in range(steps):
        api.qlora_set_timing_events(ev[i][0], ev[i][1])
        step(i)
    torch.cuda.synchronize()
    api.qlora_set_timing_events()
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1)
    kern_ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    if world > 1:
        ms = max_over_ranks(ms, dev)
    if int(err[0].item()) != 0:
        raise RuntimeError(f"device error word {int(err[0].item())}")
    ms_step = ms / steps

    # end to end: X host -> device, forward, Y device -> host, every step.  The copies
    # run on one stream of their own, so they overlap the forwards around them; X and
    # Y are double buffered by step parity.  Per step i the copy stream waits for
    # forward i, copies Y_i out and X_{i+2} in (into forward i's X buffer), so forward
    # i+2 (which waits for that X) also finds Y_i's buffer copied out.  Two event
    # records and two waits per step keep the host's share of a step small.
    e2e_steps = e2e_steps or max(3, min(100, steps // 10))
    hx = X.cpu().pin_memory()
    hy = torch.empty_like(Y, device="cpu").pin_memory()
    dxs = [torch.empty_like(X) for _ in range(2)]
    dys = [torch.empty_like(Y) for _ in range(2)]
    main = torch.cuda.current_stream()
    s_copy = torch.cuda.Stream()
    x_in = [torch.cuda.Event() for _ in range(e2e_steps)]  # X of step i landed
    fwd = [torch.cuda.Event() for _ in range(e2e_steps)]   # forward of step i done
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(main)
    s_copy.wait_event(e0)
    with torch.cuda.stream(s_copy):
        for i in range(min(2, e2e_steps)):
            dxs[i].copy_(hx, non_blocking=True)
            x_in[i].record(s_copy)
    for i in range(e2e_steps):
        p = i % 2
        main.wait_event(x_in[i])
        step(i, dxs[p], dys[p])
        fwd[i].record(main)
        s_copy.wait_event(fwd[i])
        with torch.cuda.stream(s_copy):
            hy.copy_(dys[p], non_blocking=True)
            if i + 2 < e2e_steps:
                dxs[p].copy_(hx, non_blocking=True)
                x_in[i + 2].record(s_copy)
    done = torch.cuda.Event()
    done.record(s_copy)
    main.wait_event(done)
    e1.record(main)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_equal = torch.equal(hy, Y.cpu())  # the copied-out Y equals the device loop's
    del qs
    torch.cuda.empty_cache()

    hbm, _, _, peak_src = _peaks()
    achieved = packed / (kern_ms * 1e-3) / 1e9
    return {
        "metric": METRIC, "value": round(whole_job_rate(packed, world, ms_step * 1e-3) / 1e9, 2), "unit": "GB/s",
        "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded numpy N(0,std) rounded to bf16; W with 0.1% 0.2*t(3) outliers)",
        "config": {"workload": f"small-M forward: W {N}x{K} NF4+DQ, {M} tokens, LoRA r={r} alpha={case.alpha}",
                   "M": M, "N": N, "K": K, "r": r, "parallelism": f"replicas x{world} (no shard)",
                   "step": "forward (X·A, then the dequant GEMM with the adapter term)",
                   "l2": f"{ncopy} resident weight copies used in rotation ({ncopy * packed / 1e6:.0f} MB > L2)"},
        "packed_weight_bytes": packed,
        "kernels": {"smallm_gemm_ms": round(kern_ms, 5)},
        "roofline": {"kernel": "small-M dequant GEMM", "bound": "hbm", "achieved": round(achieved, 1),
                     "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                     "peak_source": f"{peak_src} HBM copy",
                     "traffic": _traffic(SMALLM_TRAFFIC, SMALLM_SOURCES, (N, M)),
                     "traffic_unit": "bytes per launch (ncu dram read+write)"},
        "e2e": {"value": round(packed / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": X.numel() * 2, "d2h_bytes_per_step": Y.numel() * 2, "steps": e2e_steps,
                "copies": "overlapped with the compute on one copy stream", "outputs_equal_device_step": e2e_equal},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }


# ---------------------------------------------------------------- quantiser (load time)
def measure_quantiser(n: int, k: int, steps: int, local: int, w_std: float = 0.015, outliers: float = 0.001) -> dict:
    """qlora_quantize (block kernel, mean, E4M3 constants) timed alone with events
    around each call, a buffer larger than L2 written before each call so that W
    comes from HBM."""
    import torch
    from bit_nf4_quantised_codebook_b200 import api, inputs
    dev = torch.device("cuda", local)
    W = api.bits_to_tensor(inputs.weight_bf16(n, k, w_std, 0, outliers), dev)
    wq = api.alloc_weight(n, k, dev)
    ws = torch.empty(api.qlora_workspace_size(api.QLORA_OP_QUANTIZE, 0, n, k, 0), dtype=torch.uint8, device=dev)
    err = api.new_error_word(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        api.qlora_quantize(W, out=wq, ws=ws, dev_err=err)
    qev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        qev[i][0].record()
        api.qlora_quantize(W, out=wq, ws=ws, dev_err=err)
        qev[i][1].record()
    torch.cuda.synchronize()
    if int(err[0].item()) != 0:
        raise RuntimeError(f"device error word {int(err[0].item())}")
    q_ms = sum(a.elapsed_time(b) for a, b in qev) / steps
    hbm, _, _, peak_src = _peaks()
    by = 2 * n * k + wq.nbytes()
    del W, flush
    torch.cuda.empty_cache()
    return {"shape": f"{n}x{k}", "ms": round(q_ms, 5), "params_per_s": round(n * k / (q_ms * 1e-3), 1),
            "gbs": round(by / (q_ms * 1e-3) / 1e9, 1), "hbm_frac": round(by / (q_ms * 1e-3) / 1e9 / hbm, 4),
            "peak_source": f"{peak_src} HBM copy",
            "bytes": "bf16 W read + stored weight written, per call (3 kernels), L2 flushed before each"}


def run_quantiser(args):
    """--workload quantiser: qlora_quantize alone on one weight (--n rows x --k
    columns, default the 65B gate/up weight 22016 x 8192, N(0, 0.015) with 0.1%
    outliers), L2 flushed before every call; GB/s of bf16 weight read plus stored
    weight written."""
    import torch
    import torch.distributed as dist
    from bit_nf4_quantised_codebook_b200 import api, inputs
    world, rank, local = _dist()
    _init_dist(world, local)
    api.lib()
    n, k = args.n, args.k
    sampler = _gpu_sampler(local)
    sampler.mark_start()
    q = measure_quantiser(n, k, args.steps, local)
    sampler.mark_end()
    clocks = sampler.stop()
    by = 2 * n * k + api.alloc_weight(n, k).nbytes()
    dev = torch.device("cuda", local)
    # end to end: the bf16 weight host -> device, quantise, the stored weight device ->
    # host, every call; the copies on two streams of their own, overlapping the calls
    # around them, with the device weight and its stored form double buffered
    hw = api.bits_to_tensor(inputs.weight_bf16(n, k, 0.015, 0, 0.001), dev).cpu().pin_memory()
    Ws = [torch.empty_like(hw, device=dev) for _ in range(2)]
    wqs = [api.alloc_weight(n, k, dev) for _ in range(2)]
    ws = torch.empty(api.qlora_workspace_size(api.QLORA_OP_QUANTIZE, 0, n, k, 0), dtype=torch.uint8, device=dev)
    outs = [torch.empty_like(t, device="cpu").pin_memory() for t in (wqs[0].codes, wqs[0].c2q, wqs[0].c1, wqs[0].mean)]
    e2e_steps = 5
    main = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    w_in, q_done, q_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    launches0 = api.qlora_kernel_launch_count()
    e0.record(main)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(e2e_steps):
        p = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(q_done[p])  # the call two back has read this weight buffer
            Ws[p].copy_(hw, non_blocking=True)
            w_in[p].record(s_in)
        main.wait_event(w_in[p])
        if i >= 2:
            main.wait_event(q_out[p])  # the stored weight of two calls back has been copied out
        api.qlora_quantize(Ws[p], out=wqs[p], ws=ws)
        q_done[p].record(main)
        with torch.cuda.stream(s_out):
            s_out.wait_event(q_done[p])
            for h, d in zip(outs, (wqs[p].codes, wqs[p].c2q, wqs[p].c1, wqs[p].mean)):
                h.copy_(d, non_blocking=True)
            q_out[p].record(s_out)
    done = torch.cuda.Event()
    done.record(s_out)
    main.wait_event(done)
    e1.record(main)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    wq = wqs[(e2e_steps - 1) % 2]
    other = wqs[e2e_steps % 2]  # the same weight quantised by another call (two calls back)
    e2e_equal = all(torch.equal(h, d.cpu()) for h, d in zip(outs, (other.codes, other.c2q, other.c1, other.mean)))
    launches = (api.qlora_kernel_launch_count() - launches0) // e2e_steps * args.steps
    hbm, _, _, peak_src = _peaks()
    line = {
        "metric": "NF4 + double quantisation throughput (bf16 weight read, stored weight written)",
        "value": round(whole_job_rate(by, world, q["ms"] * 1e-3) / 1e9, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": 3, "ms_per_step": q["ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded numpy N(0,0.015) with 0.1% 0.2*t(3) outliers, rounded to bf16)",
        "config": {"workload": f"qlora_quantize on a {n}x{k} weight", "parallelism": f"replicas x{world}",
                   "step": "one qlora_quantize call (block kernel, mean, E4M3 constants)",
                   "l2": "a 256 MB buffer written before every call"},
        "params_per_s": q["params_per_s"],
        "roofline": {"kernel": "qlora_quantize (3 kernels)", "bound": "hbm", "achieved": q["gbs"], "peak": hbm,
                     "unit": "GB/s", "frac": q["hbm_frac"], "peak_source": f"{peak_src} HBM copy", "traffic": None,
                     "traffic_unit": "bytes per call (ncu dram read+write)"},
        "e2e": {"value": round(by / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": 2 * n * k,
                "d2h_bytes_per_step": wq.nbytes(), "steps": e2e_steps,
                "copies": "overlapped with the compute on two copy streams", "outputs_equal_device_step": e2e_equal},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_quantiser(n, k)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def cpu_baseline_quantiser(n: int, k: int, min_seconds: float = 10.0) -> dict:
    """The oracle's quantiser on 256 rows of the weight, repeated; GB/s counted as on the GPU."""
    from bit_nf4_quantised_codebook_b200 import inputs
    from oracle import nf4
    rows = 256
    W = inputs.LinearCase("q", 1, rows, k, 8, 16.0, 0.015, 0.01, 0.01, 0.001, 0).W()
    tot_t, reps = 0.0, 0
    while tot_t < min_seconds or reps == 0:
        t = time.perf_counter()
        nf4.quantize_nf4(W)
        tot_t += time.perf_counter() - t
        reps += 1
    by = reps * (2 * rows * k + nf4.storage_bytes(rows, k))
    return {"value": round(by / tot_t / 1e9, 6), "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{reps} x quantise {rows} rows x {k} drawn from the same recipe (float64/float32 numpy); "
                      f"{tot_t:.1f} s"}


# ---------------------------------------------------------------- the default line
def run_ours(args):
    import torch
    import torch.distributed as dist
    from bit_nf4_quantised_codebook_b200 import api

    world, rank, local = _dist()
    _init_dist(world, local)
    api.lib()
    name = args.workload
    line = measure_layer_set(name, args.steps, args.warmup, world, rank, local, args.linear)
    if args.linear:
        line["config"]["linear"] = args.linear
    if name == "shapes_65b" and world == 1 and not args.linear:
        line["quantiser"] = measure_quantiser(22016, 8192, 20, local)
    if name == "shapes_65b" and world == 1 and not args.no_sub and not args.linear:
        sub_steps = max(args.steps, 20)
        line["subrecords"] = {
            "proj7b": measure_layer_set("proj7b", max(args.steps, 50), max(args.warmup, 5), 1, 0, local),
            "llama7b_layer": measure_layer_set("llama7b_layer", sub_steps, max(args.warmup, 3), 1, 0, local),
            "smallm": [measure_smallm(n, m, 500, 20, 1, local, e2e_steps=20)
                       for n in (8192, 28672) for m in (1, 16)],
        }
    if world == 1 and rank == 0 and not args.no_cpu_baseline and not args.linear:
        line["cpu_baseline"] = cpu_baseline_layers(name)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_smallm(args):
    """--workload smallm: the decode-sized forward alone."""
    import torch.distributed as dist
    from bit_nf4_quantised_codebook_b200 import api, inputs
    world, rank, local = _dist()
    _init_dist(world, local)
    api.lib()
    line = measure_smallm(args.n, args.m, args.steps, args.warmup, world, local)
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_smallm(inputs.small_m(args.n, args.m))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


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


# ---------------------------------------------------------------- the oracle on a sample
def oracle_sample(name: str, tok: int, wrows: int):
    """A bounded sample of a layer set for the CPU oracle: for every linear, `tok`
    token rows through `wrows` output features (full K, the same r, scale,
    distributions and outliers), drawn from the workload's recipe as a layer of
    that size.  The oracle quantises and dequantises the sample's weights
    before the clock starts (the step keeps its weights resident too).
    Returns (run, flops): run() is one forward + backward of every linear."""
    from bit_nf4_quantised_codebook_b200 import inputs
    from oracle import linear, nf4
    prepared = {}
    jobs = []
    for c in layer_cases(name):
        sc = inputs.LinearCase(c.name, tok, min(wrows, c.N), c.K, c.r, c.alpha, c.w_std, c.a_std, c.b_std,
                               c.outlier_frac, c.seed)
        key = (sc.N, sc.K)
        if key not in prepared:
            prepared[key] = (sc, nf4.dequantize_nf4(nf4.quantize_nf4(sc.W())), sc.X(), sc.A(), sc.B(), sc.dY())
        jobs.append(prepared[key])
    flops = sum(sc.flops_fwd() + sc.flops_bwd() for sc, *_ in jobs)

    def run():
        for sc, wh, X, A, B, dY in jobs:
            linear.forward(X, wh, A, B, sc.s)
            linear.backward(X, dY, wh, A, B, sc.s)

    return run, flops


def cpu_baseline_layers(name: str, min_seconds: float = 10.0) -> dict:
    """The oracle as it stands (float64 numpy, BLAS on all host cores) on a
    bounded sample of the layer set, repeated until `min_seconds` have passed."""
    tok, wrows = 256, 256
    run, flops = oracle_sample(name, tok, wrows)
    tot_t, n = 0.0, 0
    while tot_t < min_seconds or n == 0:
        t = time.perf_counter()
        run()
        tot_t += time.perf_counter() - t
        n += 1
    nlin = len(layer_cases(name))
    return {"value": round(n * flops / tot_t / 1e12, 6), "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{n} x fwd + bwd of the {nlin} linears on {tok} token rows through {wrows} output features "
                      f"each (full K, r=64; float64 numpy); {tot_t:.1f} s"}


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
# ncu DRAM read + write of the merge-and-code kernel over one step's seven launches (a one-pass
# `--metrics gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum -k regex:merge
# -s 21 -c 7` capture of `bench.py --workload merge --steps 3 --warmup 3 --no-cpu-baseline`),
# valid for the sources it was taken from.
MERGE_SOURCES = ["merge.cu", "nf4_decode.cuh", "nf4_quant.cuh", "ptx.cuh", "launch.cuh"]
MERGE_TRAFFIC = {"sources_sha1": "e700d8e13803ffca02afa8d12ef8424109bd85c8", "bytes_per_step": 117_138_432}


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




def run_reference(args):
    """The oracle as the reference arm, on the same workload, metric and unit as
    our line: every step is a bounded sample of the layer set (every linear,
    `tok` token rows through `tok` output features), sized so that the whole
    --steps/--warmup run takes about two minutes of host time.  Under torchrun
    rank 0 alone runs it."""
    world, rank, _ = _dist()
    if rank != 0:
        return
    name = args.workload if args.workload in WORKLOADS else "shapes_65b"
    budget = float(os.environ.get("QLORA_REFERENCE_SECONDS", "120")) / max(1, args.steps + args.warmup)
    n = 16
    run, flops = oracle_sample(name, n, n)
    t = time.perf_counter()
    run()
    dt = time.perf_counter() - t
    while n < 1024 and dt * 2.2 < budget:
        n *= 2
        run, flops = oracle_sample(name, n, n)
        t = time.perf_counter()
        run()
        dt = time.perf_counter() - t
    for _ in range(args.warmup):
        run()
    tot_t = 0.0
    for _ in range(args.steps):
        t = time.perf_counter()
        run()
        tot_t += time.perf_counter() - t
    value = args.steps * flops / tot_t / 1e12
    cases = layer_cases(name)
    c0 = cases[0]
    batch, seq = BATCH[name]
    sample = (f"per step: fwd + bwd of the {len(cases)} linears on {n} token rows through {n} output features each "
              f"(full K, r={c0.r}), weights quantised and dequantised by the oracle before the clock starts")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded numpy N(0,std) rounded to bf16)",
        "config": {"workload": WORKLOADS[name], "M": c0.M, "r": c0.r, "alpha": c0.alpha,
                   "shapes": [f"{c.N}x{c.K}" for c in cases], "global_batch": batch, "seq_len": seq,
                   "parallelism": "cpu oracle on the host cores (rank 0)",
                   "sample": sample, "sample_tokens": n, "sample_output_features": n},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub", action="store_true", help="main line only (no sub-records)")
    ap.add_argument("--workload", choices=list(WORKLOADS) + ["smallm", "quantiser", "adamw", "merge", "formats"],
                    default="shapes_65b")
    ap.add_argument("--n", type=int, default=None, help="smallm: W rows (8192 or 28672); quantiser: rows (22016)")
    ap.add_argument("--k", type=int, default=8192, help="quantiser: columns")
    ap.add_argument("--linear", default=None, help="layer sets: run only this linear (q, k, v, o, gate, up, down)")
    ap.add_argument("--m", type=int, default=16, help="smallm: tokens (1..64)")
    args = ap.parse_args()
    if args.impl == "ours":
        args.warmup = max(3, args.warmup)  # at least three untimed steps before any timing
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "smallm":
        args.n = args.n or 8192
        run_smallm(args)
    elif args.workload == "quantiser":
        args.n = args.n or 22016
        run_quantiser(args)
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
