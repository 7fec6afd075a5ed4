"""Throughput of the TTT trunk+branch attention, forward + backward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one forward and one backward (every kernel of the path) over one batch
of the workload, inputs resident in HBM; the algorithmic work is 14*D flops per
visible (query, trunk key) pair per query head and pass plus the branch keys.
Prints one JSON line (rank 0).  Under torchrun each rank runs its own copy of the
workload (independent batches, no collective): weak scaling.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (one sequence and one KV head group), scaled to the metric's unit.
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import ttt_inputs  # noqa: E402

METRIC = "TTT attention fwd+bwd TFLOP/s and tokens/s at 1 B200; % of bf16 tensor peak"
DEFAULT_WORKLOAD = "qwen3_8b_4k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings (the job is as slow as its slowest rank)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_tflops(flops_per_rank_step, world, ms_per_step):
    """Aggregate throughput: the work of all ranks over the (max-over-ranks) step time."""
    return flops_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


class ClockSampler:
    """SM clock and throttle-reason samples while the timed steps run.

    Reads NVML directly from a background thread every ``period_s`` (5 ms by default),
    so that a timed region of a few tens of milliseconds still gets several samples;
    the NVML device is the one behind the CUDA device (mapped by torch, which honours
    CUDA_VISIBLE_DEVICES).  Falls back to ``nvidia-smi -lms 100`` when NVML cannot be
    used.  Samples outside [t_begin, t_end] are dropped, except that a region shorter
    than the sampling period keeps the one sample nearest to each of its ends."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")

    def __init__(self, cuda_index: int, period_s: float = 0.005):
        self.cuda_index = cuda_index
        self.period = period_s
        self.samples = []  # (time, sm_mhz, sm_max_mhz, set of active reasons)
        self.source = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            idx = torch.cuda._get_nvml_device_index(self.cuda_index)
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._nv = pynvml
            self.smax = float(pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM))
            self.source = "nvml"
            self._thread = threading.Thread(target=self._poll_nvml, daemon=True)
        except Exception:
            try:
                idx = torch.cuda._get_nvml_device_index(self.cuda_index)
            except Exception:
                idx = self.cuda_index
            try:
                self._proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(idx), f"--query-gpu={self.SMI_FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except (FileNotFoundError, OSError):
                return
            self.source = "nvidia-smi"
            self._thread = threading.Thread(target=self._read_smi, daemon=True)
        self._thread.start()

    def _poll_nvml(self):
        nv, h = self._nv, self._h
        while not self._stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
            except Exception:
                break
            self.samples.append((time.time(), sm, self.smax, {n for n, b in self.REASONS if bits & b}))
            self._stop.wait(self.period)

    def _read_smi(self):
        for line in self._proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 6:
                continue
            try:
                sm, smax = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            act = {n for (n, _), v in zip(self.REASONS, parts[2:6]) if v.lower().startswith("active")}
            self.samples.append((time.time(), sm, smax, act))

    def mark(self, name):
        setattr(self, name, time.time())

    def stop(self):
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no NVML and no nvidia-smi"], "samples": 0}
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self._proc.kill()
        if self._thread:
            self._thread.join(timeout=2)
        t0 = getattr(self, "t_begin", 0.0)
        t1 = getattr(self, "t_end", float("inf"))
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        kept = "inside the timed region"
        if not inside and self.samples:
            before = [s for s in self.samples if s[0] < t0]
            after = [s for s in self.samples if s[0] > t1]
            inside = ([before[-1]] if before else []) + ([after[0]] if after else [])
            kept = "nearest to the ends of a timed region shorter than the sampling period"
        sm = [s[1] for s in inside]
        reasons = sorted(set().union(*[s[3] for s in inside])) if inside else []
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(s[2] for s in inside) if inside else None,
                "reasons": reasons, "samples": len(sm), "source": self.source, "kept": kept,
                "period_ms": self.period * 1e3 if self.source == "nvml" else 100.0}


def applicable_peak(peaks, peak_src, timed_s):
    """Dense bf16 peak that a kernel timed over ``timed_s`` seconds is held to: the burst
    figure for a region shorter than a second (the GPU is still at its top clock), the
    sustained figure (seconds-long loop under the power cap) otherwise."""
    if timed_s < 1.0:
        return peaks["bf16_tflops"], f"{peak_src} bf16_tflops (burst: timed region {timed_s:.3f} s < 1 s)"
    return peaks["bf16_tflops_sustained"], \
        f"{peak_src} bf16_tflops_sustained (timed region {timed_s:.2f} s >= 1 s)"


# ----------------------------------------------------------------------------- ours

class Job:
    """One workload's step on the device: `step(events)` runs every kernel of the path once
    over resident inputs; `host_in` / `dev_in` / `outputs` serve the end-to-end leg."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def ttt_job(args, w, device, rank):
    from attention_pass_rope_b200 import ops
    # every rank draws its own batch (weak scaling); the sizes are the workload's
    inp = ttt_inputs.make_inputs(w, seed=w.seed + rank)

    def dev(t):
        t = t.to(device)
        if w.dense:
            t = t.view(t.shape[0], len(w.lengths), w.lengths[0], *t.shape[2:])
        return t.contiguous()

    q, k, v, do = dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.do)
    cu = None if w.dense else torch.tensor(w.cu_seqlens, dtype=torch.int32, device=device)
    kw = dict(theta=w.theta, cu_seqlens=cu, max_seqlen=None if w.dense else w.max_seqlen)
    lay = ops._layout(q, k, v, cu, kw["max_seqlen"])
    ws = ops.alloc_workspace(max(ops.workspace_bytes(lay, w.theta), ops.workspace_bytes(lay, w.theta, for_backward=True)),
                             device)
    o = torch.empty_like(q)
    lse = torch.empty(lay.lse_shape, dtype=torch.float32, device=device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def step(events=None):
        # one workspace for both calls: the backward reuses the forward's rotated q~ / k~
        ops.ttt_attn_fwd(q, k, v, workspace=ws, out=(o, lse), events=events, **kw)
        ops.ttt_attn_bwd(q, k, v, o, lse, do, workspace=ws, out=(dq, dk, dv), events=events,
                         rotated_in_workspace=True, **kw)

    desc = (f"{w.name}: B={len(w.lengths)} S={w.lengths[0]} P={w.P} H={w.H}/{w.Hkv} D={w.D} theta={w.theta:g}"
            if w.dense else
            f"{w.name}: THD nseq={w.nseq} T={w.T} P={w.P} H={w.H}/{w.Hkv} D={w.D} theta={w.theta:g}")
    return Job(step=step, ws=ws, host_src=(inp.q, inp.k, inp.v, inp.do), dev_in=(q, k, v, do),
               outputs=(o, lse, dq, dk, dv), flops=w.flops_fwd_bwd(), flops_12d=w.flops_fwd_bwd(per_pair=12),
               query_tokens=w.P * w.T,
               trunk_bwd_flops=10 * w.D * w.trunk_pairs * w.H * w.P, tokens=w.T, desc=desc,
               launches=5, unit_note="tokens = B*S (or T) positions, each carrying P passes", name=w.name)


def block_job(args, w, device, rank):
    from attention_pass_rope_b200 import ops
    inp = ttt_inputs.make_block_inputs(dataclasses.replace(w, seed=w.seed + rank))
    B, S, nblk = w.nseq, w.ctx_lengths[0], w.nblocks[0]

    def dev(t, shape):
        return t.to(device).view(*shape).contiguous()

    k_ctx, v_ctx = dev(inp.k_ctx, (B, S, w.Hkv, w.D)), dev(inp.v_ctx, (B, S, w.Hkv, w.D))
    qb, do = dev(inp.qb, (B, nblk, w.Bs, w.H, w.D)), dev(inp.do, (B, nblk, w.Bs, w.H, w.D))
    kb, vb = dev(inp.kb, (B, nblk, w.Bs, w.Hkv, w.D)), dev(inp.vb, (B, nblk, w.Bs, w.Hkv, w.D))
    anchors = inp.anchors.to(device).view(B, nblk).contiguous()
    lay = ops._block_layout(k_ctx, v_ctx, qb, kb, vb, anchors, None, None, None, None)
    ws = ops.alloc_workspace(ops.block_workspace_bytes(lay, anchors, w.theta, for_backward=True), device)
    o = torch.empty_like(qb)
    lse = torch.empty(lay.lse_shape, dtype=torch.float32, device=device)
    grads = tuple(torch.empty_like(t) for t in (k_ctx, v_ctx, qb, kb, vb))
    args_ = (k_ctx, v_ctx, qb, kb, vb, anchors)

    def step(events=None):
        ops.block_attn_fwd(*args_, theta=w.theta, workspace=ws, out=(o, lse), events=events)
        ops.block_attn_bwd(*args_, o, lse, do, theta=w.theta, workspace=ws, out=grads, events=events,
                           rotated_in_workspace=True)

    a = inp.anchors.tolist()
    trunk_pairs = sum((x + 1) * w.Bs for x in a)  # per query head
    desc = (f"{w.name}: block-draft B={B} context S={S} blocks={nblk} x Bs={w.Bs} H={w.H}/{w.Hkv} D={w.D} "
            f"theta={w.theta:g}, anchors sorted uniform")
    return Job(step=step, ws=ws, host_src=(inp.k_ctx, inp.v_ctx, inp.qb, inp.kb, inp.vb, inp.do),
               dev_in=(k_ctx, v_ctx, qb, kb, vb, do), outputs=(o, lse) + grads, flops=w.flops_fwd_bwd(a),
               flops_12d=w.flops_fwd_bwd(a, per_pair=12),
               trunk_bwd_flops=10 * w.D * trunk_pairs * w.H, tokens=w.NB * w.Bs, desc=desc, launches=6,
               unit_note="tokens = block tokens", name=w.name)


SOFTCE_METRIC = "TTT draft soft cross-entropy loss fwd+bwd TFLOP/s at 1 B200; % of bf16 tensor peak"
SOFTCE_KERNELS = {0: "rows", 1: "logits", 2: "combine", 4: "dz", 5: "dh", 6: "dw"}


def softce_job(args, w, device, rank):
    from attention_pass_rope_b200 import softce as ce
    inp = ttt_inputs.make_softce_inputs(dataclasses.replace(w, seed=w.seed + rank))
    h, W, y, m = (t.to(device).contiguous() for t in (inp.h, inp.W, inp.y, inp.mask))
    cu = torch.tensor(w.cu_seqlens, dtype=torch.int32, device=device)
    chunk = args.chunk or 4096
    R = w.P * w.T
    nch = (R + chunk - 1) // chunk
    need = ce.workspace_bytes(ce.make_desc(h, W, y, cu, m, token_chunk_size=chunk), 2)
    ws = torch.empty(need, dtype=torch.uint8, device=device)
    loss = torch.empty(w.P + 1, dtype=torch.float32, device=device)
    rows = torch.empty(w.P, w.T, dtype=torch.float32, device=device)
    lse = torch.empty(2, w.P, w.T, dtype=torch.float32, device=device)
    dh = torch.empty_like(h)
    dW = torch.zeros(w.V, w.d, dtype=torch.float32, device=device)

    def step(events=None):
        # the loss's forward and backward in one sweep (upstream gradient 1); the gradient of
        # the head is accumulated across steps, as over micro-batches
        ce.softce_fwd_bwd(h, W, y, cu_seqlens=cu, loss_mask=m, token_chunk_size=chunk, dW=dW, dh=dh,
                          out=(loss, rows, lse), workspace=ws, events=events)

    desc = (f"{w.name}: P={w.P} passes x T={w.T} tokens ({len(w.lengths)} sequences of {w.lengths[0]}), "
            f"d={w.d}, V={w.V}, fused forward + backward in chunks of {chunk} rows ({nch} chunks), "
            f"loss mask keep {w.mask_keep}; work = logits, dh and dW GEMMs")
    return Job(step=step, ws=ws, host_src=(inp.h, inp.W, inp.y, inp.mask), dev_in=(h, W, y, m),
               outputs=(loss, rows, lse, dh, dW), flops=w.flops_fwd_bwd(), tokens=w.T, desc=desc,
               launches=2 + 5 * nch, unit_note="tokens = positions, each carrying P draft rows", name=w.name,
               metric=SOFTCE_METRIC, kernel_names=SOFTCE_KERNELS, status=ce.device_status,
               # dominant kernel: the dW GEMM (the largest share of the step); its per-launch
               # work is one chunk's 2 * rows * V * d, timed at the first chunk
               dom_kernel="dw", dom_flops=2.0 * min(chunk, R) * w.V * w.d)


def run_ours(args, rank, world, local):
    from attention_pass_rope_b200 import _lib, ops

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    if args.workload in ttt_inputs.block_workloads():
        job = block_job(args, ttt_inputs.block_workloads()[args.workload], device, rank)
    elif args.workload in ttt_inputs.softce_workloads():
        job = softce_job(args, ttt_inputs.softce_workloads()[args.workload], device, rank)
    else:
        job = ttt_job(args, workload(args), device, rank)
    step, ws = job.step, job.ws
    names = getattr(job, "kernel_names", None) or {i: n for i, n in enumerate(_lib.KERNELS)
                                                    if not n.startswith("unused")}
    status = getattr(job, "status", None) or ops.device_status

    # per-kernel CUDA events, recorded by the library on the launching stream
    K = args.steps
    evs = [_lib.TTTEvents() for _ in range(K)]
    ev_objs = []
    for e in evs:
        objs = {}
        for kk in names:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()  # torch creates the CUDA event on first use; the library re-records it
            b.record()
            e.start[kk] = a.cuda_event
            e.stop[kk] = b.cuda_event
            objs[kk] = (a, b)
        ev_objs.append(objs)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, word = status(ws)
    if st != _lib.TTT_OK:
        raise RuntimeError(f"device status after warm-up: {st} {word:#x}")

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark("t_begin")
    t0.record()
    for i in range(K):
        step(evs[i])
    t1.record()
    torch.cuda.synchronize()
    sampler.mark("t_end")
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1)
    per_kernel = {}
    for kk, name in names.items():
        per_kernel[name] = sum(ev_objs[i][kk][0].elapsed_time(ev_objs[i][kk][1]) for i in range(K)) / K
    st, word = status(ws)
    if st != _lib.TTT_OK:
        raise RuntimeError(f"device status after timing: {st} {word:#x}")

    # end to end: pinned host inputs -> device, fwd+bwd, results back to pinned host memory
    host_in = [t.pin_memory() for t in job.host_src]
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in job.outputs]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)

    def e2e_step():
        for hsrc, dst in zip(host_in, job.dev_in):
            dst.view(-1).copy_(hsrc.view(-1), non_blocking=True)
        step()
        for src, hdst in zip(job.outputs, host_out):
            hdst.copy_(src, non_blocking=True)

    E = max(1, min(K, 5))
    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(E):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / E

    if world > 1:
        ms, e2e_ms = max_over_ranks([ms, e2e_ms], device)

    ms_step = ms / K
    flops = job.flops
    tflops = whole_job_tflops(flops, world, ms_step)
    peaks, peak_src = load_peaks()
    peak, peak_kind = applicable_peak(peaks, peak_src, ms * 1e-3)
    # dominant kernel (tensor bound) and its algorithmic flops per launch: the trunk
    # backward's 10*D per visible trunk pair per query head (and pass), or the job's own
    dom = getattr(job, "dom_kernel", "trunk_bwd")
    dom_flops = getattr(job, "dom_flops", None) or job.trunk_bwd_flops
    achieved = dom_flops / (per_kernel[dom] * 1e-3) / 1e12
    traffic = read_traffic(dom, job.name)
    line = {
        "metric": getattr(job, "metric", METRIC),
        "value": round(tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": job.desc, "tokens_per_step": job.tokens, "tokens": job.unit_note,
                   "flops_per_step": flops, "parallelism": f"replicas{world}",
                   "l2": "inputs per step (%.0f MB) exceed L2 (126 MB)" % (h2d / 1e6)},
        "tokens_per_s": round(job.tokens * world / (ms_step * 1e-3), 1),
        # the stricter count without the backward's recomputed Q K^T (12*D per pair), and
        # P*B*S query-tokens/s (every position carries P passes)
        **({"tflops_12d": round(whole_job_tflops(job.flops_12d, world, ms_step), 2)}
           if getattr(job, "flops_12d", None) else {}),
        **({"query_tokens_per_s": round(job.query_tokens * world / (ms_step * 1e-3), 1)}
           if getattr(job, "query_tokens", None) else {}),
        "pct_of_peak": round(100.0 * tflops / world / peak, 2),
        "peak": {"tflops": peak, "source": peak_kind, "pct_of_burst": round(100.0 * tflops / world / peaks["bf16_tflops"], 2),
                 "pct_of_sustained": round(100.0 * tflops / world / peaks["bf16_tflops_sustained"], 2)},
        "kernel_ms": {k_: round(v_, 4) for k_, v_ in per_kernel.items()},
        "roofline": {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": peak_kind,
                     "frac_of_burst": round(achieved / peaks["bf16_tflops"], 4),
                     "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                     "traffic": traffic},
        "e2e": {"value": round(flops * world / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": job.launches * K,
        "clocks": clocks,
    }
    if rank == 0 and not args.no_cpu_baseline:
        if args.workload in ttt_inputs.block_workloads():
            line["cpu_baseline"] = block_cpu_baseline(ttt_inputs.block_workloads()[args.workload])
        elif args.workload in ttt_inputs.softce_workloads():
            line["cpu_baseline"] = softce_cpu_baseline(ttt_inputs.softce_workloads()[args.workload])
        else:
            line["cpu_baseline"] = cpu_baseline(workload(args), budget_s=args.cpu_budget)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def workload(args):
    w = ttt_inputs.workloads()[args.workload]
    if args.batch and w.dense:
        # a smaller batch of the same sequences (profiling captures)
        w = ttt_inputs.dense(f"{w.name}_b{args.batch}", args.batch, w.lengths[0], w.P, w.H, w.Hkv, w.D, w.theta,
                             w.scale, w.seed)
    return w


def read_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu record of the kernel, or None when
    there is none or the kernel's source changed since the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        with open(os.path.join(ROOT, d["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != d["source_sha256"]:
                return None
        return d.get("dram_bytes_per_launch")
    except (OSError, ValueError, KeyError):
        return None


# ----------------------------------------------------------------------------- oracle

def oracle_sample(w, n_groups=1):
    """The bounded sample: sequence 0, KV heads 0..n_groups-1 (all their query heads
    and passes), fwd + bwd.  Returns (seconds, flops of the sample)."""
    import numpy as np
    from oracle import ttt_oracle as orc

    inp = ttt_inputs.make_inputs(w)
    a, b = w.cu_seqlens[0], w.cu_seqlens[1]
    g = w.H // w.Hkv
    kvs = list(range(n_groups))
    heads = [h for kv in kvs for h in range(kv * g, (kv + 1) * g)]
    q = inp.q[:, a:b].double().numpy()
    k = inp.k[:, a:b].double().numpy()
    v = inp.v[:, a:b].double().numpy()
    do = inp.do[:, a:b].double().numpy()
    t0 = time.perf_counter()
    O, lse = orc.forward_twopart(q, k, v, w.theta, heads=heads)
    orc.backward_twopart(q, k, v, do, lse, w.theta, kv_heads=kvs)
    dt = time.perf_counter() - t0
    L = b - a
    sub = ttt_inputs.thd("sample", [L], w.P, len(heads), n_groups, w.D, w.theta)
    return dt, sub.flops_fwd_bwd(), np


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 0) for i in threadpool_info()), default=None)
    except Exception:
        return None


def cpu_baseline(w, budget_s=30.0):
    dt, fl, _ = oracle_sample(w)
    cores = blas_threads() or len(os.sched_getaffinity(0))
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 NumPy oracle, fwd+bwd of sequence 0 and KV head 0 ({w.H // w.Hkv} query heads x "
                      f"{w.P} passes x {w.lengths[0]} positions) = 1/{w.nseq * w.Hkv} of the workload, {dt:.1f} s",
            "seconds": round(dt, 2)}


def block_cpu_baseline(w):
    """The fp64 block-draft oracle on one sequence and one KV-head group of the workload."""
    import numpy as np
    from oracle import block_draft_oracle as bd
    inp = ttt_inputs.make_block_inputs(w)
    g = w.H // w.Hkv
    b1 = w.cu_blocks[1]
    f64 = lambda x: x.float().numpy().astype(np.float64)
    c = dict(k_ctx=f64(inp.k_ctx[:w.cu_ctx[1], :1]), v_ctx=f64(inp.v_ctx[:w.cu_ctx[1], :1]),
             anchors=inp.anchors[:b1].tolist(), qb=f64(inp.qb[:b1, :, :g]), kb=f64(inp.kb[:b1, :, :1]),
             vb=f64(inp.vb[:b1, :, :1]))
    t0 = time.perf_counter()
    O, lse = bd.forward_twopart(theta=w.theta, rope_round="bf16", **c)
    bd.backward_twopart(do=f64(inp.do[:b1, :, :g]), O=O, lse=lse, theta=w.theta, rope_round="bf16", **c)
    dt = time.perf_counter() - t0
    sub = dataclasses.replace(w, H=g, Hkv=1, ctx_lengths=w.ctx_lengths[:1], nblocks=w.nblocks[:1])
    fl = sub.flops_fwd_bwd(inp.anchors[:b1].tolist())
    cores = blas_threads() or len(os.sched_getaffinity(0))
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 block-draft oracle, fwd+bwd of sequence 0 and KV head 0 = 1/{w.nseq * w.Hkv} of the "
                      f"workload, {dt:.1f} s", "seconds": round(dt, 2)}


def softce_cpu_baseline(w, n_rows=8):
    """The fp64 soft-CE oracle on n_rows draft rows of the workload (pass 0, the first valid
    rows): their losses and dh, i.e. three 2*V*d passes per row (logits, logits again, dz W)."""
    from oracle import softce_oracle as sco
    inp = ttt_inputs.make_softce_inputs(w)
    m = inp.mask.numpy().astype(bool)
    idx = sco.teacher_index(w.cu_seqlens[:2], 1, m[:w.cu_seqlens[1]])
    ts = [t for t in range(idx.shape[1]) if idx[0, t] >= 0][:n_rows]
    hr = inp.h[0, ts]
    yr = inp.y[[int(idx[0, t]) for t in ts]]
    t0 = time.perf_counter()
    sco.rows_forward(hr, inp.W, yr)
    sco.rows_dh(hr, inp.W, yr, [1.0] * len(ts))
    dt = time.perf_counter() - t0
    fl = 3 * 2.0 * len(ts) * w.V * w.d
    cores = blas_threads() or len(os.sched_getaffinity(0))
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 soft-CE oracle, loss and dh of {len(ts)} draft rows (of {w.P * w.T}), {dt:.1f} s",
            "seconds": round(dt, 2)}


def run_reference(args, rank, world):
    if rank != 0:
        return
    metric = METRIC
    sample = f"sequence 0, KV head 0 of {args.workload} per step"
    if args.workload in ttt_inputs.block_workloads():
        wb = ttt_inputs.block_workloads()[args.workload]
        runs = [block_cpu_baseline(wb) for _ in range(args.steps)]
        dt = sum(r["seconds"] for r in runs) / len(runs)
        value = sum(r["value"] for r in runs) / len(runs)
    elif args.workload in ttt_inputs.softce_workloads():
        ws_ = ttt_inputs.softce_workloads()[args.workload]
        runs = [softce_cpu_baseline(ws_) for _ in range(args.steps)]
        dt = sum(r["seconds"] for r in runs) / len(runs)
        value = sum(r["value"] for r in runs) / len(runs)
        metric = SOFTCE_METRIC
        sample = runs[0]["sample"] + " per step"
    else:
        w = workload(args)
        # the oracle has no warm-up state; one untimed sample warms the BLAS pool
        oracle_sample(ttt_inputs.thd("warm", [256], w.P, w.H // w.Hkv, 1, w.D, w.theta))
        times, fl = [], None
        for _ in range(args.steps):
            dt, fl, _ = oracle_sample(w)
            times.append(dt)
        dt = sum(times) / len(times)
        value = fl / dt / 1e12
    cores = blas_threads() or len(os.sched_getaffinity(0))
    line = {
        "impl": "reference",
        "metric": metric,
        "value": round(value, 6),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": args.workload, "parallelism": "cpu oracle, rank 0 only"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(ttt_inputs.workloads()) + sorted(ttt_inputs.block_workloads()) +
                    sorted(ttt_inputs.softce_workloads()))
    ap.add_argument("--chunk", type=int, default=0,
                    help="soft-CE backward: draft rows per chunk (0: the pages' default, 4096)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=30.0)
    ap.add_argument("--batch", type=int, default=0, help="override B of a dense workload (profiling)")
    args = ap.parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
