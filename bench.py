#!/usr/bin/env python3
"""Attention forward + backward throughput on B200, one JSON line.

A step is one pass of the whole hot path over one batch of the workload:
fa_fwd (O, LSE) then fa_bwd (preprocess D_i and zero the dQ accumulator, the
fused backward kernel, the dQ conversion), all through the C ABI of
libfa_b200.so. Inputs are seeded
synthetic Gaussians resident in HBM before the timed region starts.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the float64 CPU oracle arm)

A decode workload (``--workload bf16_decode_...``) times the split-KV decode
path instead: a step is one fa_decode call (split partials + merge) of the
q_len newest tokens of every sequence against its KV cache, resident in HBM;
the metric is the KV-cache bytes it must read per second.

``--workload fp8_fwd_causal_b2_h16_n8192_d128`` times the FP8 (E4M3)
forward on that workload's inputs: a step is pass 1 (fa_fp8_quantize of Q and
of K) plus pass 2 (fa_fwd_fp8); the metric is forward TFLOP/s.

With N > 1 (launched by torch.distributed.run) every rank runs its own
independently seeded batch of the same shape (the (batch, head) units are
independent; no collective on the data path): weak scaling, timed as the
max over ranks of CUDA-event time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOP/s (bf16, device-timed) and % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "bf16_gqa_causal_b1_h32_kv8_n16384_d128"
# A timed region shorter than this runs at the burst clock (the driver's
# default 20 steps take well under a second); a longer one settles under the
# power cap, where the sustained figure is the fair denominator.
SUSTAINED_AFTER_S = 1.0
L2_BYTES = 126 * 1024 * 1024
FP8_METRIC = "attention forward TFLOP/s, FP8 E4M3 Q K^T (two-pass, device-timed)"
# FP8 workloads run the two passes on the inputs of the named bf16 workload.
FP8_WORKLOADS = {"fp8_fwd_causal_b2_h16_n8192_d128": "bf16_causal_b2_h16_n8192_d128"}
DECODE_METRIC = "split-KV decode attention, KV-cache GB/s read (bf16, device-timed)"
DECODE_UNIT = "GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------ host logic ---

def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def tensor_peak(peaks: dict, timed_s: float) -> tuple:
    """(peak TFLOP/s, kind) for a kernel timed inside a region of ``timed_s``
    seconds: the burst figure for a short region, the sustained one for a
    region long enough to reach the power cap."""
    if timed_s < SUSTAINED_AFTER_S:
        return peaks["bf16_tflops"], "burst"
    return peaks["bf16_tflops_sustained"], "sustained"


def step_flops(lengths, H: int, D: int, causal: bool) -> tuple:
    """Algorithmic FLOPs: forward 4*H*sum(L^2)*D, backward 2.5x, causal halves."""
    from exact_io_aware_tmem_b200.workloads import flops
    return flops(lengths, H, D, causal)


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own batch: same shape, independent values."""
    return seed + 1000 * rank


def aggregate(units_per_rank: float, world: int, times_s: list) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / max(times_s)


def reduce_max(value: float, device=None) -> float:
    """Max over ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def source_sha(*names) -> str:
    """Hash of the code in the named csrc files: ``//`` comments and blank
    lines are left out, so editing a comment does not orphan a capture."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "exact_io_aware_tmem_b200", "csrc", n)) as f:
            for line in f:
                if line.lstrip().startswith("//"):
                    continue
                code = line.split("//", 1)[0].rstrip() if '"' not in line else line.rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


KERNEL_SOURCES = {"fwd_pair_kernel": ("fwd_pair.cu", "common.cuh", "params.h"),
                  "fwd_d64_kernel": ("fwd_d64.cu", "fwd_d64.h", "ex2_fma.cuh", "common.cuh", "params.h"),
                  "bwd_fused_kernel": ("bwd_fused.cu", "ex2_fma.cuh", "common.cuh", "params.h"),
                  "bwd_dkdv_kernel": ("bwd_bf16.cu", "common.cuh", "params.h"),
                  "bwd_dq_kernel": ("bwd_bf16.cu", "common.cuh", "params.h"),
                  "decode": ("decode_split.cu", "common.cuh", "params.h"),
                  "decode_t": ("decode_t.cu", "decode_t.h", "common.cuh", "params.h"),
                  "fp8_fwd": ("fwd_pair.cu", "common.cuh", "params.h"),
                  "fp8_quantize_kernel": ("fp8.cu", "common.cuh", "params.h")}


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu capture of this kernel on this
    workload (one record, or a list of records, per kernel), if the kernel is
    unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            recs = json.load(f)[kernel]
    except (OSError, KeyError, ValueError):
        return None
    for rec in recs if isinstance(recs, list) else [recs]:
        if rec.get("workload") == workload and \
                rec.get("source_sha") == source_sha(*KERNEL_SOURCES[kernel]):
            return rec.get("bytes_per_launch")
    return None


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.out = None

    def start(self):
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        text = self.out.read()
        os.unlink(self.out.name)
        return parse_clock_rows(text)


def parse_clock_rows(text: str) -> dict:
    """Median SM clock, max clock and the throttle reasons seen in the samples."""
    sm, smax, power, reasons = [], [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in text.strip().splitlines():
        r = [x.strip() for x in line.split(",")]
        try:
            sm.append(float(r[0]))
            smax.append(float(r[1]))
            power.append(float(r[2]))
        except (ValueError, IndexError):
            continue
        for n, v in zip(names, r[3:7]):
            if v.lower() == "active":
                reasons.add(n)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(smax) if smax else None,
            "power_w_max": max(power) if power else None,
            "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- oracle ---

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w, n_tokens: int):
    """Forward + backward of one query head of the workload, truncated to
    ``n_tokens`` positions, with the float64 oracle. Returns (seconds, flops)."""
    import torch
    from exact_io_aware_tmem_b200.workloads import random_case
    from oracle import attention as oa
    inp = random_case(w.seed, dtype=w.dtype, lengths=[n_tokens], H=1, H_kv=1, D=w.D, varlen=False,
                      std=w.qk_mult)
    q = inp.q[:, 0].to(torch.float64).numpy()
    k = inp.k[:, 0].to(torch.float64).numpy()
    v = inp.v[:, 0].to(torch.float64).numpy()
    do = inp.do[:, 0].to(torch.float64).numpy()
    t0 = time.perf_counter()
    oa.head_forward(q, k, v, w.scale, w.causal)
    if w.backward:
        oa.head_backward(q, k, v, do, w.scale, w.causal)
    dt = time.perf_counter() - t0
    fwd, bwd = step_flops([n_tokens], 1, w.D, w.causal)
    return dt, fwd + (bwd if w.backward else 0.0)


def oracle_tokens_for(w, seconds: float) -> int:
    """Sequence length of the oracle sample that takes about ``seconds``."""
    n0 = 512
    t0, _ = oracle_sample(w, n0)
    n = int(n0 * math.sqrt(max(seconds, 0.05) / max(t0, 1e-3)))
    n = max(128, min(w.N, n // 128 * 128))
    return n


def cpu_baseline(w, seconds: float = 15.0) -> dict:
    n = oracle_tokens_for(w, seconds)
    dt, fl = oracle_sample(w, n)
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "seconds": round(dt, 3),
            "sample": f"float64 numpy oracle, {config_of(w)['pass']} of one query head of "
                      f"{w.name} truncated to N={n} (causal={w.causal}, D={w.D}); FLOPs by the "
                      f"same formula as the GPU line"}


def run_reference(args, w) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = max(0.5, 150.0 / max(1, args.steps + args.warmup))
    n = oracle_tokens_for(w, per_step)
    for _ in range(args.warmup):
        oracle_sample(w, n)
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = oracle_sample(w, n)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    sample = (f"float64 numpy oracle, one query head of {w.name} truncated to N={n}, "
              f"{config_of(w)['pass']} per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(w) -> dict:
    from exact_io_aware_tmem_b200.workloads import make_inputs  # noqa: F401
    return {"workload": w.name, "B": w.B, "H": w.H, "H_kv": w.H_kv, "N": w.N, "D": w.D,
            "causal": w.causal, "varlen": w.varlen is not None,
            "pass": "fwd+bwd" if w.backward else "fwd",
            "seed": w.seed}


# -------------------------------------------------------------- GPU arm ---

def pipelined_e2e(torch, dev, host_in, dev_in, dev_out, run_step, steps: int) -> float:
    """End-to-end device time (ms) of ``steps`` steps through the public API.

    Every step copies its inputs host -> device from pinned memory, runs, and
    reads its outputs back into pinned memory; all of it inside the timed
    region. The copies of neighbouring steps overlap the computation, as a
    serving or training loop would arrange: two sets of device buffers, one
    stream per direction plus the compute stream, and events so that a
    buffer set is refilled only after the step two back has finished with it
    (inputs) and been read out (outputs).
    """
    sets_in = [dev_in, [torch.empty_like(t) for t in dev_in]]
    sets_out = [dev_out, [torch.empty_like(t) for t in dev_out]]
    host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in dev_out]
                for _ in range(2)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()  # noqa: E731
    e_in, e_cmp, e_out = ([ev() for _ in range(steps)] for _ in range(3))
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    start.record()
    for st_ in (s_in, s_cmp, s_out):
        st_.wait_event(start)
    for i in range(steps):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(e_cmp[i - 2])      # step i-2 no longer reads set b
            for dst, src in zip(sets_in[b], host_in):
                dst.copy_(src, non_blocking=True)
            e_in[i].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(e_in[i])
            if i >= 2:
                s_cmp.wait_event(e_out[i - 2])     # step i-2's outputs have been read out
            run_step(sets_in[b], sets_out[b])
            e_cmp[i].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(e_cmp[i])
            for dst, src in zip(host_out[b], sets_out[b]):
                dst.copy_(src, non_blocking=True)
            e_out[i].record(s_out)
    cur = torch.cuda.current_stream(dev)
    for e in (e_in[-1], e_cmp[-1], e_out[-1]):
        cur.wait_event(e)
    end.record()
    torch.cuda.synchronize(dev)
    return start.elapsed_time(end)

def run_ours(args, w) -> None:
    import torch
    import torch.distributed as dist

    import exact_io_aware_tmem_b200 as fa
    from exact_io_aware_tmem_b200.workloads import Workload, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)
    peaks = load_peaks()

    # Baseline on the host first (rank 0, one GPU only), before any GPU work.
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_seconds)

    wr = Workload(**{**w.__dict__, "seed": rank_seed(w.seed, rank)})
    inp = make_inputs(wr)
    B = len(inp.cu_seqlens) - 1
    lengths = inp.cu_seqlens.diff().tolist()
    fwd_fl, bwd_fl = step_flops(lengths, w.H, w.D, w.causal)
    T = inp.q.shape[0]

    def to_dev(t):
        t = t.to(dev)
        return t if inp.varlen else t.view(B, w.N, t.shape[1], w.D)

    q, k, v, do = (to_dev(t) for t in (inp.q, inp.k, inp.v, inp.do))
    kw = dict(causal=w.causal, scale=w.scale)
    if inp.varlen:
        kw.update(cu_seqlens=inp.cu_seqlens.to(dev), max_seqlen=inp.max_seqlen)
    o = torch.empty_like(q)
    lse = torch.empty((B, w.H, w.N) if not inp.varlen else (w.H, T), device=dev,
                      dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(fa.workspace_size(T, w.H, w.D, q.dtype),
                         fa.workspace_size(T, w.H, w.D, q.dtype, fa.BWD_SPLIT)),
                     dtype=torch.uint8, device=dev)
    # The backward's three kernels: preprocess (+ accumulator zeroing), fused
    # kernel, dQ conversion; or, with --bwd split, preprocess, dK / dV kernel,
    # dQ kernel (the reproducible split backward).
    split = getattr(args, "bwd", "fused") == "split"
    ph_steps = (0x01, 0x02, 0x04) if split else (0x01, 0x08, 0x10)
    bwd_names = (("bwd_preprocess", "bwd_dkdv_kernel", "bwd_dq_kernel") if split else
                 ("bwd_preprocess", "bwd_fused_kernel", "dq_convert"))
    # Forward-only workloads (the B4 N2048 D64 configuration) time the
    # forward alone: their step is one fa_fwd.
    do_bwd = w.backward
    ins = (q, k, v, do) if do_bwd else (q, k, v)
    bytes_in = sum(t.numel() * t.element_size() for t in ins)
    fwd_name = "fwd_pair_kernel" if w.D == 128 else "fwd_d64_kernel"

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        fa.fwd(q, k, v, out=o, lse=lse, **kw)
        if ev is not None:
            ev[1].record()
        if not do_bwd:
            return
        for i, ph in enumerate(ph_steps):
            fa.bwd(do, q, k, v, o, lse, workspace=ws, dq=dq, dk=dk, dv=dv, phases=ph, **kw)
            if ev is not None:
                ev[2 + i].record()

    for _ in range(args.warmup):
        step()
    st, where = fa.check_device_error(dev)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where:#x} during warm-up")

    gpu_uuid = ""
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
        gpu_uuid = gpu_uuid if gpu_uuid.startswith("GPU-") else "GPU-" + gpu_uuid
    except Exception:
        pass
    sampler = ClockSampler(gpu_uuid)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    start.record()
    for i in range(args.steps):
        step(evs[i])
    end.record()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    st, where = fa.check_device_error(dev)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where:#x} in the timed region")
    elapsed_ms = start.elapsed_time(end)
    max_ms = reduce_max(elapsed_ms, dev)
    spans = {fwd_name: (0, 1)}
    if do_bwd:
        spans.update({name: (1 + i, 2 + i) for i, name in enumerate(bwd_names)})
    k_ms = {name: statistics.mean(e[a].elapsed_time(e[b]) for e in evs)
            for name, (a, b) in spans.items()}
    k_ms = {n: reduce_max(t, dev) for n, t in k_ms.items()}

    # End to end through the public API with host buffers: pinned H2D of the
    # step's inputs, forward + backward, D2H of every output, pipelined.
    e2e_steps = max(3, min(args.steps, 20))
    host_in = [t.cpu().pin_memory() for t in ins]
    outs = [o, lse, dq, dk, dv] if do_bwd else [o, lse]
    bytes_out = sum(t.numel() * t.element_size() for t in outs)

    def e2e_step(ins_, outs_):
        qq, kk, vv = ins_[:3]
        fa.fwd(qq, kk, vv, out=outs_[0], lse=outs_[1], **kw)
        if do_bwd:
            gq, gk, gv = outs_[2:]
            fa.bwd(ins_[3], qq, kk, vv, outs_[0], outs_[1], workspace=ws, dq=gq, dk=gk, dv=gv,
                   phases=fa.BWD_SPLIT if split else fa.BWD_FUSED, **kw)

    if world > 1:
        dist.barrier()
    e2e_ms = reduce_max(pipelined_e2e(torch, dev, host_in, list(ins), outs, e2e_step,
                                      e2e_steps), dev)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    if not do_bwd:
        bwd_fl = 0.0
    per_step_fl = fwd_fl + bwd_fl
    value = aggregate(per_step_fl * args.steps, world, [max_ms / 1e3]) / 1e12
    fwd_tf = fwd_fl / (k_ms[fwd_name] / 1e3) / 1e12
    bwd_tf = None
    if do_bwd:
        bwd_ms = sum(k_ms[n] for n in bwd_names)
        bwd_tf = bwd_fl / (bwd_ms / 1e3) / 1e12
    # Dominant kernel: the one with the largest share of the step. FLOPs per
    # launch: the forward's two products (4 N^2 D per head) and the fused
    # backward's five (S, dP, dV, dK, dQ: 10 N^2 D, the method's 2.5x), causal
    # halving each; the split backward's kernels count the products they run
    # (dK / dV kernel: S, dP, dV, dK; dQ kernel: S, dP, dQ).
    kernel_fl = {fwd_name: fwd_fl}
    if do_bwd and split:
        kernel_fl.update({"bwd_dkdv_kernel": 2.0 * fwd_fl, "bwd_dq_kernel": 1.5 * fwd_fl})
    elif do_bwd:
        kernel_fl["bwd_fused_kernel"] = bwd_fl
    dom = max(kernel_fl, key=lambda n: k_ms[n])
    dom_fl = kernel_fl[dom]
    achieved = dom_fl / (k_ms[dom] / 1e3) / 1e12
    peak, peak_kind = tensor_peak(peaks, max_ms / 1e3)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_of(w), parallelism=f"replicas{world}" if world > 1 else "none",
                       backward=("split (dK / dV kernel + dQ kernel)" if split else "fused")
                       if do_bwd else None,
                       l2=f"not flushed: every step reads and writes "
                          f"{(bytes_in + bytes_out) / 2**20:.0f} MiB > {L2_BYTES >> 20} MiB L2",
                       ranks="each rank its own seeded batch of this shape"),
        "fwd_tflops": fwd_tf, "bwd_tflops": bwd_tf,
        "fwd_frac_of_peak": fwd_tf / peak,
        "bwd_frac_of_peak": None if bwd_tf is None else bwd_tf / peak,
        "peak_tflops": {"burst": peaks["bf16_tflops"], "sustained": peaks["bf16_tflops_sustained"],
                        "source": peaks["source"]},
        "kernel_ms": {n: round(t, 4) for n, t in k_ms.items()},
        "roofline": {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_kind": f"{peaks['source']} {peak_kind} bf16 (timed region "
                                  f"{max_ms / 1e3:.2f} s)",
                     "frac_of_burst": achieved / peaks["bf16_tflops"],
                     "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                     "traffic": recorded_traffic(dom, w.name)},
        "cpu_baseline": cpu,
        "e2e": {"value": per_step_fl * e2e_steps * world / (e2e_ms / 1e3) / 1e12, "unit": UNIT,
                "steps": e2e_steps, "h2d_bytes_per_step": bytes_in,
                "d2h_bytes_per_step": bytes_out,
                "how": "public API, pinned host buffers, copies of neighbouring steps "
                       "overlapping the computation (double-buffered, three streams)"},
        "gpu_launches": (4 if do_bwd else 1) * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- FP8 arm ---

def fp8_oracle_sample(w, n_tokens: int):
    """Pass 1 + pass 2 of the FP8 forward with the float64 oracle on one head
    of the workload truncated to ``n_tokens``. Returns (seconds, FLOPs)."""
    from exact_io_aware_tmem_b200.workloads import random_case
    from oracle import fp8 as of
    inp = random_case(w.seed, dtype=w.dtype, lengths=[n_tokens], H=1, H_kv=1, D=w.D, varlen=False,
                      std=w.qk_mult)
    t0 = time.perf_counter()
    of.fp8_forward(inp.q, inp.k, inp.v, 1, n_tokens, w.causal, w.scale)
    dt = time.perf_counter() - t0
    fwd, _ = step_flops([n_tokens], 1, w.D, w.causal)
    return dt, fwd


def fp8_cpu_baseline(w, seconds: float) -> dict:
    n = 512
    t0, _ = fp8_oracle_sample(w, n)
    n = max(128, min(w.N, int(n * math.sqrt(max(seconds, 0.05) / max(t0, 1e-3))) // 128 * 128))
    dt, fl = fp8_oracle_sample(w, n)
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "seconds": round(dt, 3),
            "sample": f"float64 numpy FP8 oracle (block quantisation + attention on the "
                      f"dequantised Q, K), one head of {w.name} truncated to N={n}"}


def run_fp8_reference(args, name, w) -> None:
    if int(os.environ.get("RANK", "0")) != 0:
        return
    n = 1024
    for _ in range(args.warmup):
        fp8_oracle_sample(w, n)
    tot_t = tot_f = 0.0
    for _ in range(args.steps):
        dt, fl = fp8_oracle_sample(w, n)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    sample = f"float64 numpy FP8 oracle, one head of {w.name} truncated to N={n} per step"
    line = {"impl": "reference", "metric": FP8_METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(config_of(w), **{"workload": name, "pass": "fp8 fwd"}),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_fp8(args, name, w) -> None:
    import torch
    import torch.distributed as dist

    import exact_io_aware_tmem_b200 as fa
    from exact_io_aware_tmem_b200.workloads import Workload, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)
    peaks = load_peaks()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = fp8_cpu_baseline(w, args.cpu_seconds)
    wr = Workload(**{**w.__dict__, "seed": rank_seed(w.seed, rank)})
    inp = make_inputs(wr)
    B, N = w.B, w.N
    fwd_fl, _ = step_flops([N] * B, w.H, w.D, w.causal)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    q8, qs = fa.fp8_quantize(q, B, N)
    k8, ks = fa.fp8_quantize(k, B, N)
    o = torch.empty_like(q)
    lse = torch.empty((B, w.H, N), device=dev, dtype=torch.float32)

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        fa.fp8_quantize(q, B, N, out=q8, scale=qs)
        fa.fp8_quantize(k, B, N, out=k8, scale=ks)
        if ev is not None:
            ev[1].record()
        fa.fwd_fp8(q8, k8, v, qs, ks, B=B, N=N, causal=w.causal, scale=w.scale, out=o, lse=lse)
        if ev is not None:
            ev[2].record()

    for _ in range(args.warmup):
        step()
    st, where = fa.check_device_error(dev)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where:#x} during warm-up")
    gpu_uuid = ""
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
        gpu_uuid = gpu_uuid if gpu_uuid.startswith("GPU-") else "GPU-" + gpu_uuid
    except Exception:
        pass
    sampler = ClockSampler(gpu_uuid)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    start.record()
    for i in range(args.steps):
        step(evs[i])
    end.record()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    st, where = fa.check_device_error(dev)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where:#x} in the timed region")
    max_ms = reduce_max(start.elapsed_time(end), dev)
    q_ms = reduce_max(statistics.mean(e[0].elapsed_time(e[1]) for e in evs), dev)
    f_ms = reduce_max(statistics.mean(e[1].elapsed_time(e[2]) for e in evs), dev)
    # End to end: bf16 Q, K, V in from pinned host memory, both passes, O and
    # LSE out, pipelined.
    e2e_steps = max(3, min(args.steps, 20))
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
    d2h = o.numel() * o.element_size() + lse.numel() * 4

    def e2e_step(ins, outs_):
        qq, kk, vv = ins
        oo, ll = outs_
        fa.fp8_quantize(qq, B, N, out=q8, scale=qs)
        fa.fp8_quantize(kk, B, N, out=k8, scale=ks)
        fa.fwd_fp8(q8, k8, vv, qs, ks, B=B, N=N, causal=w.causal, scale=w.scale, out=oo, lse=ll)

    if world > 1:
        dist.barrier()
    e2e_ms = reduce_max(pipelined_e2e(torch, dev, [t.cpu().pin_memory() for t in (q, k, v)],
                                      [q, k, v], [o, lse], e2e_step, e2e_steps), dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    value = aggregate(fwd_fl * args.steps, world, [max_ms / 1e3]) / 1e12
    # Pass 2's two products: Q K^T at the E4M3 rate (twice bf16, the nominal
    # ratio) and P V in bf16, half of the FLOPs each, so its tensor-core floor
    # is 0.75 of the bf16 time: peak = measured bf16 / 0.75 (burst or sustained
    # by the length of the timed region).
    bf16_peak, peak_kind = tensor_peak(peaks, max_ms / 1e3)
    peak = bf16_peak / 0.75
    p1_bytes = sum(3 * t.numel() + 4 * s_.numel() for t, s_ in ((q, qs), (k, ks)))
    achieved = fwd_fl / (f_ms / 1e3) / 1e12
    line = {
        "metric": FP8_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 Q K^T, bf16 P V",
        "data": "synthetic",
        "config": dict(config_of(w), **{"workload": name, "base_workload": w.name,
                                         "pass": "fp8 fwd (quantise Q, K + forward)"},
                       parallelism=f"replicas{world}" if world > 1 else "none",
                       l2="not flushed: every step reads and writes > 200 MiB > 126 MiB L2",
                       ranks="each rank its own seeded batch of this shape"),
        "kernel_ms": {"fp8_quantize_kernel (Q and K)": round(q_ms, 4),
                      "fwd_pair_kernel<128, e4m3>": round(f_ms, 4)},
        "roofline": {"kernel": "fwd_pair_kernel<128, e4m3>", "bound": "tensor",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "peak_kind": f"{peaks['source']} {peak_kind} bf16 / 0.75 (E4M3 Q K^T at the "
                                  f"nominal 2x rate, bf16 P V)",
                     "traffic": recorded_traffic("fp8_fwd", name)},
        # Pass 1 is HBM-bound: it reads bf16 Q and K once and writes their
        # E4M3 codes and steps.
        "pass1_roofline": {"kernel": "fp8_quantize_kernel (Q and K)", "bound": "hbm",
                           "achieved": p1_bytes / (q_ms / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": p1_bytes / (q_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                           "algorithmic_bytes": p1_bytes,
                           # one launch quantises one of the two tensors
                           "traffic": (lambda t: None if t is None else 2 * t)(
                               recorded_traffic("fp8_quantize_kernel", name))},
        "cpu_baseline": cpu,
        "e2e": {"value": fwd_fl * e2e_steps * world / (e2e_ms / 1e3) / 1e12, "unit": UNIT,
                "steps": e2e_steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "how": "public API, pinned host buffers, copies of neighbouring steps "
                       "overlapping the computation (double-buffered, three streams)"},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- decode arm ---

def decode_config(w) -> dict:
    lengths = w.lengths()
    return {"workload": w.name, "B": w.B, "q_len": w.q_len, "H": w.H, "H_kv": w.H_kv, "D": w.D,
            "causal": w.causal, "cache": f"paged, {w.page_size} rows per page, shuffled blocks"
            if w.page_size else "contiguous", "cache_len_range": [w.len_lo, w.len_hi],
            "cache_tokens": int(sum(lengths)), "pass": "decode", "seed": w.seed}


def decode_oracle_case(w, n_seq: int):
    """Seeded inputs of the first ``n_seq`` sequences of a decode workload."""
    from exact_io_aware_tmem_b200.workloads import decode_case
    return decode_case(w.seed, dtype=w.dtype, lengths=w.lengths()[:n_seq], q_len=w.q_len,
                       H=w.H, H_kv=w.H_kv, D=w.D, page_size=w.page_size)


def decode_oracle_sample(w, n_seq: int, c=None):
    """The float64 decode oracle on the first ``n_seq`` sequences of the
    workload (``c``: their inputs, drawn if not given). Returns (seconds, KV
    bytes, FLOPs)."""
    from exact_io_aware_tmem_b200.workloads import decode_bytes, decode_flops
    from oracle import decode as od
    lengths = w.lengths()[:n_seq]
    if c is None:
        c = decode_oracle_case(w, n_seq)
    t0 = time.perf_counter()
    od.decode_forward(c.q, c.k_cache, c.v_cache, c.cache_seqlens, q_len=w.q_len, scale=w.scale,
                      causal=w.causal, stride=c.page_size, page_size=c.page_size,
                      block_table=c.block_table)
    dt = time.perf_counter() - t0
    return dt, decode_bytes(lengths, w.H_kv, w.D), decode_flops(lengths, w.q_len, w.H, w.D)


def decode_cpu_baseline(w) -> dict:
    n = max(1, w.B // 4)
    dt, by, _ = decode_oracle_sample(w, n)
    return {"value": by / dt / 1e9, "unit": DECODE_UNIT, "cores": blas_threads(),
            "kind": "oracle", "seconds": round(dt, 3),
            "sample": f"float64 numpy decode oracle on the first {n} of the {w.B} sequences of "
                      f"{w.name}; bytes by the same formula as the GPU line"}


def run_decode_reference(args, w) -> None:
    if int(os.environ.get("RANK", "0")) != 0:
        return
    # About 150 s of oracle work over all steps: the sample is drawn once and
    # is as many leading sequences as fit one step's share.
    per_step = max(0.2, 150.0 / max(1, args.steps + args.warmup))
    c1 = decode_oracle_case(w, 1)
    t1, _, _ = decode_oracle_sample(w, 1, c1)
    n = max(1, min(w.B, int(per_step / max(t1, 1e-3))))
    c = c1 if n == 1 else decode_oracle_case(w, n)
    for _ in range(args.warmup):
        decode_oracle_sample(w, n, c)
    tot_t = tot_b = 0.0
    for _ in range(args.steps):
        dt, by, _ = decode_oracle_sample(w, n, c)
        tot_t += dt
        tot_b += by
    value = tot_b / tot_t / 1e9
    sample = f"float64 numpy decode oracle, first {n} of {w.B} sequences of {w.name} per step"
    line = {"impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": DECODE_UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(w),
            "cpu_baseline": {"value": value, "unit": DECODE_UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": DECODE_UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_decode(args, w) -> None:
    import torch
    import torch.distributed as dist

    import exact_io_aware_tmem_b200 as fa
    from exact_io_aware_tmem_b200.workloads import (DecodeWorkload, decode_bytes, decode_flops,
                                                    make_decode_inputs)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)
    peaks = load_peaks()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = decode_cpu_baseline(w)

    wr = DecodeWorkload(**{**w.__dict__, "seed": rank_seed(w.seed, rank)})
    c = make_decode_inputs(wr)
    lengths = c.cache_seqlens.tolist()
    max_len = max(lengths)
    kv_bytes = decode_bytes(lengths, w.H_kv, w.D)
    fl = decode_flops(lengths, w.q_len, w.H, w.D)
    q = c.q.to(dev)
    kc, vc = c.k_cache.to(dev), c.v_cache.to(dev)
    lens = c.cache_seqlens.to(dev)
    table = None if c.block_table is None else c.block_table.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((q.shape[0], w.H), device=dev, dtype=torch.float32)
    n_split = fa.decode_num_splits(w.B, w.H_kv, max_len)
    balanced = fa.decode_balanced(w.D, w.q_len, w.H, w.H_kv)
    ws = torch.empty(max(1, fa.decode_workspace_size(w.B, w.q_len, w.H, w.H_kv, w.D, max_len)),
                     dtype=torch.uint8, device=dev)
    alg_bytes = kv_bytes + 2 * q.numel() * q.element_size() + lse.numel() * 4

    def step():
        fa.decode(q, kc, vc, lens, q_len=w.q_len, max_seqlen_k=max_len, block_table=table,
                  page_size=c.page_size, causal=w.causal, scale=w.scale, out=o, lse=lse,
                  workspace=ws)

    for _ in range(args.warmup):
        step()
    st, where = fa.check_device_error(dev)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where:#x} during warm-up")
    gpu_uuid = ""
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
        gpu_uuid = gpu_uuid if gpu_uuid.startswith("GPU-") else "GPU-" + gpu_uuid
    except Exception:
        pass
    sampler = ClockSampler(gpu_uuid)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    start.record()
    for i in range(args.steps):
        evs[i][0].record()
        step()
        evs[i][1].record()
    end.record()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    st, where = fa.check_device_error(dev)
    if st != 0:
        raise RuntimeError(f"device error {st} at {where:#x} in the timed region")
    max_ms = reduce_max(start.elapsed_time(end), dev)
    call_ms = reduce_max(statistics.mean(e[0].elapsed_time(e[1]) for e in evs), dev)

    # End to end: the step's new tokens (Q, and the cache lengths) go host ->
    # device from pinned memory and O, LSE come back, pipelined with the
    # neighbouring steps; the KV cache is the state a decode step reads in
    # place, resident as in serving.
    e2e_steps = max(3, min(args.steps, 50))
    h2d = q.numel() * q.element_size() + lens.numel() * 4
    d2h = o.numel() * o.element_size() + lse.numel() * 4

    def e2e_step(ins, outs_):
        qq, ll = ins
        oo, ss = outs_
        fa.decode(qq, kc, vc, ll, q_len=w.q_len, max_seqlen_k=max_len, block_table=table,
                  page_size=c.page_size, causal=w.causal, scale=w.scale, out=oo, lse=ss,
                  workspace=ws)

    if world > 1:
        dist.barrier()
    e2e_ms = reduce_max(pipelined_e2e(torch, dev, [q.cpu().pin_memory(), lens.cpu().pin_memory()],
                                      [q, lens], [o, lse], e2e_step, e2e_steps), dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    value = aggregate(kv_bytes * args.steps, world, [max_ms / 1e3]) / 1e9
    achieved = alg_bytes / (call_ms / 1e3) / 1e9
    peak = peaks["hbm_gbs"]
    line = {
        "metric": DECODE_METRIC, "value": value, "unit": DECODE_UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(decode_config(w),
                       partition=("balanced: equal key-tile ranges over one persistent CTA "
                                  "per SM" if balanced else f"{n_split} splits per sequence"),
                       parallelism=f"replicas{world}" if world > 1 else "none",
                       l2=f"not flushed: every step reads {kv_bytes / 2**20:.0f} MiB of cache "
                          f"> {L2_BYTES >> 20} MiB L2",
                       ranks="each rank its own seeded batch of this shape"),
        "tflops": fl / (call_ms / 1e3) / 1e12,
        "kernel_ms": {"fa_decode (partials + merge)": round(call_ms, 4)},
        "roofline": {"kernel": ("decode_t_kernel + decode_t_merge_kernel" if balanced else
                                "decode_split_kernel + decode_combine_kernel") +
                               " (one fa_decode)",
                     "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": f"{peaks['source']} HBM copy",
                     "algorithmic_bytes": alg_bytes,
                     "traffic": recorded_traffic("decode_t" if balanced else "decode", w.name)},
        "cpu_baseline": cpu,
        "e2e": {"value": kv_bytes * e2e_steps * world / (e2e_ms / 1e3) / 1e9,
                "unit": DECODE_UNIT, "steps": e2e_steps, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "how": "public API, pinned host buffers, copies of neighbouring steps "
                       "overlapping the computation (double-buffered, three streams)"},
        "gpu_launches": (2 if balanced or n_split > 1 else 1) * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bwd", choices=["fused", "split"], default="fused",
                    help="backward path of the attention step (default: the fused kernel)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args(argv)
    from exact_io_aware_tmem_b200.workloads import DECODE_WORKLOADS, WORKLOADS
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload in FP8_WORKLOADS:
        w = WORKLOADS[FP8_WORKLOADS[args.workload]]
        if args.impl == "reference":
            run_fp8_reference(args, args.workload, w)
        else:
            run_fp8(args, args.workload, w)
        return 0
    if args.workload in DECODE_WORKLOADS:
        w = DECODE_WORKLOADS[args.workload]
        if args.impl == "reference":
            run_decode_reference(args, w)
        else:
            run_decode(args, w)
        return 0
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)
    return 0


if __name__ == "__main__":
    sys.exit(main())
