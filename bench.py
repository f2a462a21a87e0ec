"""Benchmark: radial block-sparse attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wan] [--impl ours|reference]

One step = the whole hot path on one synthetic problem already resident in
HBM: radial block-list build (count, scan, fill; asynchronous, into
preallocated buffers), the longest-row-first work order, and the tcgen05
attention kernel. Each GPU (one process per GPU under torchrun) runs its own
independent problem, so per-GPU work is fixed as N grows (weak scaling) and
no collective touches the data path; the only collectives are the timing
barrier and the max over ranks.

Prints one JSON line on rank 0. ``value`` is effective TFLOP/s on computed
blocks over all ranks: 4 * D * sum over listed (query block, key block) of
valid rows x valid cols, per head, divided by the slowest rank's time.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "block-sparse attn fwd ms & effective TFLOP/s vs bf16 peak at 32k–120k tokens"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CSRC = "block_sparse_attention_radial_b200/csrc/"
KERNEL_SOURCES = {
    "fwd": (CSRC + "attn_fwd_pair_sm100.cuh", CSRC + "attn_fwd_sm100.cuh", CSRC + "ptx_sm100.cuh",
            CSRC + "rowgen.cuh"),
    "bwd": (CSRC + "attn_bwd_sm100.cuh", CSRC + "attn_fwd_sm100.cuh", CSRC + "ptx_sm100.cuh"),
}
TRAFFIC_FILES = {"fwd": "attn_fwd_pair_sm100_{}_traffic.json", "bwd": "attn_bwd_sm100_{}_traffic.json"}


def _code_only(text: str) -> str:
    """C++ source without comments and blank lines: what the compiler sees."""
    import re

    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_source_hash(which: str = "fwd") -> str:
    """Hash of the kernels' source code (comments excluded), recorded with an
    ncu capture so that a changed kernel invalidates its traffic figure."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[which]:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def load_traffic(workload: str, which: str = "fwd"):
    """DRAM bytes per launch (per backward call for ``which="bwd"``) of the
    timed kernels from a committed ncu summary, or None when the summary is
    missing or was taken on different kernel source."""
    path = os.path.join(ROOT, "profiles", TRAFFIC_FILES[which].format(workload))
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_source_hash") != kernel_source_hash(which):
        return None
    return d.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks ---

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid: str | None):
        self.proc = None
        self.path = os.path.join("/tmp", f"bsa_clocks_{os.getpid()}.csv")
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "200"]
        if device_uuid:
            cmd += ["-i", device_uuid]
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    rows.append((float(parts[0]), float(parts[1]), parts[3:]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        max_mhz = max(r[1] for r in rows)
        loaded = [r for r in rows if r[0] > 0.5 * max_mhz] or rows
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2][1:5])
                          if v.strip().lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max_mhz,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------- helpers ---

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import datetime

    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank float over all ranks (identity at world size 1)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ------------------------------------------------------------ CPU oracle ---

def oracle_sample_rate(w, lists_host, q, k, v, budget_s: float, head: int = 0):
    """Time the CPU oracle on query rows of one head; returns (TFLOP/s, seconds,
    rows, flops). Rows are a contiguous run around the middle of the sequence,
    sized by a short calibration run to take about ``budget_s``."""
    import numpy as np

    import oracle

    rp, ci = lists_host
    D = w.head_dim
    qh, kh, vh = (t[:, head:head + 1].cpu() for t in (q, k, v))
    valid = np.minimum(w.block, w.n - np.arange(w.nqb) * w.block)

    def flops_of(rows):
        f = 0
        for r in rows:
            qb = r // w.block
            f += 4 * D * int(valid[ci[rp[qb]:rp[qb + 1]]].sum())
        return f

    start = (w.n // 2) // w.block * w.block
    cal = np.arange(start, min(w.n, start + 256))
    for _ in range(2):  # the first call pays one-time costs
        t0 = time.perf_counter()
        oracle.masked_attention_fp64(qh, kh, vh, rp, ci, 1, w.block, rows=cal)
        t_cal = max(time.perf_counter() - t0, 1e-3)
    # a contiguous run centred on the middle of the sequence (all of head 0
    # at most)
    nrows = int(min(w.n, max(64, cal.size * budget_s / t_cal)))
    first = max(0, min(w.n - nrows, w.n // 2 - nrows // 2))
    rows = np.arange(first, first + nrows)
    t0 = time.perf_counter()
    oracle.masked_attention_fp64(qh, kh, vh, rp, ci, 1, w.block, rows=rows)
    dt = time.perf_counter() - t0
    fl = flops_of(rows)
    return fl / dt / 1e12, dt, rows, fl


# ------------------------------------------------------------------ main ---

def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, as it stands, on the host cores."""
    if rank != 0:
        return 0
    import numpy as np
    import torch

    import oracle
    from workloads import WORKLOADS, make_qkv

    w = WORKLOADS[args.workload]
    q, k, v = make_qkv(w, "cpu", heads=1)
    rp_all, ci_all, _ = host_lists(w)
    rp, ci = rp_all[:w.nqb + 1], ci_all[:rp_all[w.nqb]]   # head 0's list
    per_step = max(0.2, min(2.0, 150.0 / max(1, args.steps + args.warmup)))
    rate, dt, rows, fl = oracle_sample_rate(w, (rp, ci), q, k, v, per_step)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.masked_attention_fp64(q, k, v, rp, ci, 1, w.block, rows=rows)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = fl * len(times) / total / 1e12
    cores = blas_threads()
    sample = (f"head 0, query rows {int(rows[0])}..{int(rows[-1])} ({rows.size} rows) of the "
              f"{w.name} problem per step; fp64 NumPy oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total / len(times) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, nnz=int(rp_all[-1])),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, nnz):
    if w.radial:
        text = f" + {w.text_tokens} text tokens" if w.text_tokens else ""
        desc = (f"{w.name}: B={w.batch} H={w.heads} D={w.head_dim} "
                f"{w.frames}x{w.tokens_per_frame} tokens{text} (n={w.n}), radial "
                f"{w.block}x{w.block} blocks")
    else:
        desc = (f"{w.name}: B={w.batch} H={w.heads} D={w.head_dim} n={w.n}, one seeded tile "
                f"pattern per head (diagonal, multi-diagonal, stripes, dual window), "
                f"{w.block}x{w.block} blocks")
    return {"workload": desc,
            "global_batch": w.batch, "heads": w.heads, "head_dim": w.head_dim, "seq_len": w.n,
            "frames": w.frames, "tokens_per_frame": w.tokens_per_frame, "block": w.block,
            ("nnz_blocks_per_head" if w.radial else "nnz_blocks_all_heads"): nnz,
            "parallelism": "independent problem per GPU",
            "l2": "inputs larger than L2 (Q, K, V per problem exceed 126 MB); no flush"}


def host_lists(w):
    """The workload's block lists on the host from the oracle: ``(row_ptr,
    col_idx, num_lists)`` (head 0's list first)."""
    import oracle

    if w.radial:
        rp, ci = oracle.joint_block_lists(w.frames, w.tokens_per_frame, w.text_tokens, w.block)
        return rp, ci, 1
    from workloads import generic_tile_patterns

    rp, ci = oracle.tile_pattern_lists(generic_tile_patterns(w.heads, w.nqb), w.nqb)
    return rp, ci, w.heads


def _gpu_uuid(dev):
    import torch

    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid).replace("GPU-", "")
    except Exception:
        return None


class FwdProblem:
    """One forward workload resident on the device: inputs, lists, outputs and
    the step that rebuilds the lists and runs the attention."""

    def __init__(self, w, dev, stream, generated: bool = False):
        import torch

        import block_sparse_attention_radial_b200 as bsa
        from workloads import make_qkv

        self.w, self.dev, self.stream, self.bsa = w, dev, stream, bsa
        self.generated = generated
        self.q, self.k, self.v = make_qkv(w, dev)
        if w.radial:
            self.num_lists = 1
            self.lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block, device=dev,
                                                text_tokens=w.text_tokens)
        else:  # per-head tile patterns, expanded on the GPU
            from workloads import generic_tile_patterns

            self.num_lists = w.heads
            pats = generic_tile_patterns(w.heads, w.nqb)
            self.pat_raw, self.pat_cols = bsa.pack_tile_patterns(pats, dev)
            self.lists = bsa.tile_pattern_block_lists(pats, w.nqb, w.block, device=dev)
        self.rp_h = self.lists.row_ptr.cpu().numpy()
        self.ci_h = self.lists.col_idx.cpu().numpy()
        self.flops = bsa.computed_flops(self.rp_h, self.ci_h, w.n, w.block, w.head_dim, w.batch,
                                        w.heads, self.num_lists)
        self.dense_flops = 4 * w.head_dim * w.batch * w.heads * w.n * w.n
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty((w.batch, w.heads, w.n), dtype=torch.float32, device=dev)
        self.ws = torch.empty(max(bsa.bsa_attn_fwd_workspace_bytes(w.batch, w.heads, self.lists),
                                  16), dtype=torch.uint8, device=dev)
        self.launches_per_step = 5  # list count, scan, fill; work order; attention
        if generated:  # rows generated in the kernel: count, scan, work order, attention
            self.launches_per_step = 4
            if w.radial:
                nbytes = bsa._lib.load().bsa_attn_fwd_radial_workspace_bytes(
                    w.frames, w.tokens_per_frame, w.text_tokens)
            else:
                self.pat_raw, self.pat_cols = bsa.pack_tile_patterns(pats, dev)
                nbytes = bsa._lib.load().bsa_attn_fwd_patterns_workspace_bytes(w.heads, w.nqb)
            self.gws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)

    def build_lists(self):
        w, l, bsa = self.w, self.lists, self.bsa
        if w.radial:
            bsa.bsa_joint_mask_build(w.frames, w.tokens_per_frame, w.text_tokens, w.block,
                                     l.row_ptr, l.col_idx, l.col_idx.numel(), want_nnz=False,
                                     stream=self.stream)
        else:
            bsa.bsa_tile_pattern_lists_build(w.heads, w.nqb, self.pat_raw, self.pat_cols,
                                             l.row_ptr, l.col_idx, l.col_idx.numel(),
                                             want_nnz=False, stream=self.stream)

    def step(self, ev=None):
        w, bsa = self.w, self.bsa
        if self.generated:
            # the whole entry is timed: row lengths, work order and attention
            if ev is not None:
                ev[0].record(self.stream)
            if w.radial:
                bsa.bsa_attn_fwd_radial(self.q, self.k, self.v, w.frames, w.tokens_per_frame,
                                        self.out, self.lse, w.text_tokens, self.gws, 0.0,
                                        self.stream)
            else:
                bsa.bsa_attn_fwd_patterns(self.q, self.k, self.v, self.pat_raw, self.pat_cols,
                                          self.out, self.lse, None, self.gws, 0.0, self.stream)
            if ev is not None:
                ev[1].record(self.stream)
            return
        self.build_lists()
        if ev is not None:
            ev[0].record(self.stream)
        bsa.bsa_attn_fwd(self.q, self.k, self.v, self.lists, self.out, self.lse, self.ws,
                         0.0, self.stream)
        if ev is not None:
            ev[1].record(self.stream)

    def timed(self, steps, warmup, rank):
        """W untimed steps, then K steps bracketed by a barrier and a device
        synchronisation, with the clocks sampled meanwhile. Returns (ms over
        all K steps, max over ranks; mean attention-kernel ms; clocks)."""
        import numpy as np
        import torch

        bsa, dev, stream = self.bsa, self.dev, self.stream
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize(dev)
        status = bsa.bsa_get_device_status()
        if status != 0:
            raise SystemExit(f"device status {status} after warm-up")
        sampler = ClockSampler(_gpu_uuid(dev)) if rank == 0 else None
        if sampler is not None:
            time.sleep(0.4)   # let the sampler start before the timed region
        kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(dev)
        torch.cuda.synchronize(dev)
        t_start.record(stream)
        for i in range(steps):
            self.step(kev[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        barrier(dev)
        clocks = sampler.stop() if sampler is not None else None
        ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
        kernel_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
        status = bsa.bsa_get_device_status()
        if status != 0:
            raise SystemExit(f"device status {status} after the timed region")
        # the lists rebuilt inside every step are the ones the FLOPs were counted on
        if not self.generated and not (np.array_equal(self.lists.row_ptr.cpu().numpy(), self.rp_h)
                and np.array_equal(self.lists.col_idx.cpu().numpy(), self.ci_h)):
            raise SystemExit("lists rebuilt in the timed steps differ from the counted lists")
        return ms, kernel_ms, clocks

    def roofline(self, kernel_ms, peaks, peak_kind):
        peak = float(peaks["bf16_tflops"])
        achieved = self.flops / (kernel_ms * 1e-3) / 1e12
        kernel = ("attn_fwd_pair_sm100_kernel<128> (+ work-order prepass)" if not self.generated
                  else "attn_fwd_pair_sm100_kernel<128>, rows generated in the kernel "
                       "(+ row-length count, scan and work order, all timed)")
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "traffic": None if self.generated else load_traffic(self.w.name),
                "peak_kind": f"{peak_kind} bf16 burst",
                "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                "kernel": kernel, "kernel_ms": kernel_ms, "flops_per_launch": self.flops}


# The other configurations of the metric's 32k-131k token range, timed in the
# same default run after the headline one (one GPU only).
PER_CONFIG = ("hunyuan", "long4x", "generic")


def per_config_records(args, dev, stream, rank, peaks, peak_kind):
    import torch

    from workloads import WORKLOADS

    recs = {}
    steps, warmup = max(3, min(args.steps, args.per_config_steps)), 3
    for name in PER_CONFIG:
        prob = FwdProblem(WORKLOADS[name], dev, stream)
        ms, kernel_ms, clocks = prob.timed(steps, warmup, rank)
        recs[name] = {
            "value": prob.flops * steps / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": ms / steps, "steps": steps, "warmup": warmup,
            "config": workload_config(prob.w, nnz=int(prob.rp_h[-1])),
            "roofline": prob.roofline(kernel_ms, peaks, peak_kind),
            "gpu_launches": prob.launches_per_step * steps,
            "dense_equivalent_tflops": prob.dense_flops * steps / (ms * 1e-3) / 1e12,
            "clocks": clocks,
        }
        del prob
        torch.cuda.empty_cache()
    return recs


def run_ours(args, world, rank, local):
    import torch

    import block_sparse_attention_radial_b200 as bsa
    from workloads import WORKLOADS

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the library has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    w = WORKLOADS[args.workload]
    stream = torch.cuda.current_stream(dev)
    prob = FwdProblem(w, dev, stream, generated=args.rows == "generated")
    q, k, v, lists = prob.q, prob.k, prob.v, prob.lists
    rp_h, ci_h, flops = prob.rp_h, prob.ci_h, prob.flops
    ms, kernel_ms, clocks = prob.timed(args.steps, args.warmup, rank)

    # ---- end to end through the C ABI on host buffers: bsa_attn_fwd_host copies
    # pinned q, k, v in and out / lse back, pipelined with the kernels by head group
    e2e_steps = max(3, min(args.steps, 10))
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty(prob.out.shape, dtype=prob.out.dtype).pin_memory()
    lh = torch.empty(prob.lse.shape, dtype=prob.lse.dtype).pin_memory()
    ws_host = torch.empty(bsa.bsa_attn_fwd_host_workspace_bytes(w.batch, w.heads, w.n,
                                                                w.head_dim, lists),
                          dtype=torch.uint8, device=dev)

    def e2e_step():
        prob.build_lists()
        bsa.bsa_attn_fwd_host(qh, kh, vh, lists, oh, lh, ws_host, 0.0, stream)

    e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        head0 = (rp_h[:w.nqb + 1], ci_h[:rp_h[w.nqb]])
        rate, dt, rows, fl = oracle_sample_rate(w, head0, q, k, v, args.cpu_seconds)
        cpu_baseline = {"value": rate, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                        "sample": f"head 0, {rows.size} query rows ({int(rows[0])}..{int(rows[-1])}) "
                                  f"of the {w.name} problem, {dt:.1f} s, fp64 NumPy"}
    del qh, kh, vh, oh, lh, ws_host

    peaks, peak_kind = load_peaks()
    roofline = prob.roofline(kernel_ms, peaks, peak_kind)
    dense_flops, launches_per_step = prob.dense_flops, prob.launches_per_step
    per_config = None
    if world == 1 and args.workload == "wan" and args.rows == "lists" and args.per_config_steps > 0:
        del prob, q, k, v, lists
        torch.cuda.empty_cache()
        per_config = per_config_records(args, dev, stream, rank, peaks, peak_kind)
    if rank == 0:
        line = {
            "metric": METRIC,
            "value": flops * world * args.steps / (ms * 1e-3) / 1e12,
            "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, nnz=int(rp_h[-1])),
            "roofline": roofline,
            "e2e": {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches_per_step * args.steps,
            "dense_equivalent_tflops": dense_flops * world * args.steps / (ms * 1e-3) / 1e12,
            "clocks": clocks,
            "cpu_baseline": cpu_baseline,
            "per_config": per_config,
        }
        line["config"]["rows"] = ("generated in the kernel" if args.rows == "generated"
                                  else "block lists rebuilt every step")
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


METRIC_BWD = "block-sparse attn bwd ms & effective TFLOP/s (2.5x forward FLOPs) at 32k-120k tokens"


def run_ours_bwd(args, world, rank, local):
    """The backward pass (bsa_attn_bwd) on the same workload: a step is one
    backward call from resident Q, K, V, O, dO and lse (the forward runs once
    before timing). value counts the algorithmic backward FLOPs, 2.5 x the
    forward's; the kernels execute 3.5 x (dQ recomputes S and dP), which the
    roofline uses. --bwd-kernel one_pass times bsa_attn_bwd_one_pass instead
    (one kernel, 2.5 x executed, dQ parts added in row order)."""
    import numpy as np
    import torch

    import block_sparse_attention_radial_b200 as bsa
    from workloads import WORKLOADS, make_qkv

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the library has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    w = WORKLOADS[args.workload]
    q, k, v = make_qkv(w, dev)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 1000)
    do = torch.randn(q.shape, generator=g, device=dev).to(torch.bfloat16)
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block, device=dev,
                                  text_tokens=w.text_tokens)
    rp_h, ci_h = lists.row_ptr.cpu().numpy(), lists.col_idx.cpu().numpy()
    fwd_flops = bsa.computed_flops(rp_h, ci_h, w.n, w.block, w.head_dim, w.batch, w.heads, 1)
    one_pass = args.bwd_kernel == "one_pass"
    flops, exec_flops = 2.5 * fwd_flops, (2.5 if one_pass else 3.5) * fwd_flops
    out, lse = bsa.attention(q, k, v, lists)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = (bsa.bsa_attn_bwd_one_pass_workspace_bytes if one_pass else
                bsa.bsa_attn_bwd_workspace_bytes)(w.batch, w.heads, w.n, lists)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    # prep, transposed-list count, scan, fill; dK/dV and dQ (or the one-pass
    # kernel and its initialisation)
    launches_per_step = 6
    bwd_call = bsa.bsa_attn_bwd_one_pass if one_pass else bsa.bsa_attn_bwd

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        bwd_call(q, k, v, out, do, lse, lists, dq, dk, dv, ws, 0.0, stream)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if bsa.bsa_get_device_status() != 0:
        raise SystemExit("device status after warm-up")
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid).replace("GPU-", "")
    except Exception:
        pass
    sampler = ClockSampler(uuid) if rank == 0 else None
    if sampler is not None:
        time.sleep(0.4)
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    t_start.record(stream)
    for i in range(args.steps):
        step(kev[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    clocks = sampler.stop() if sampler is not None else None
    ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
    kernel_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
    if bsa.bsa_get_device_status() != 0:
        raise SystemExit("device status after the timed region")

    # end to end through the C ABI on host buffers: bsa_attn_bwd_host copies
    # pinned q, k, v, out, dout, lse in and dq, dk, dv back, pipelined with the
    # kernels by head group
    e2e_steps = max(3, min(args.steps, 10))
    host_in = [t.cpu().pin_memory() for t in (q, k, v, out, do, lse)]
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (dq, dk, dv)]
    ws_host = torch.empty(bsa.bsa_attn_bwd_host_workspace_bytes(w.batch, w.heads, w.n,
                                                                w.head_dim, lists),
                          dtype=torch.uint8, device=dev)

    def e2e_step():
        bsa.bsa_attn_bwd_host(*host_in, lists, *host_out, ws_host, 0.0, stream)

    e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        qh, kh, vh, dh = (t[:, :1].cpu() for t in (q, k, v, do))
        start = (w.n // 2) // w.block * w.block
        cal = np.arange(start, min(w.n, start + 256))
        for _ in range(2):  # the first call pays one-time costs
            t0 = time.perf_counter()
            oracle.masked_attention_dq_rows(qh, kh, vh, dh, rp_h, ci_h, 1, w.block, 0, 0, cal)
            t_cal = max(time.perf_counter() - t0, 1e-3)
        # a contiguous run centred on the middle of the sequence, sized to
        # take about --cpu-seconds, in chunks of 1024 rows (bounded memory)
        nrows = int(min(w.n, max(256, cal.size * args.cpu_seconds / t_cal)))
        first = max(0, min(w.n - nrows, w.n // 2 - nrows // 2))
        rows = np.arange(first, first + nrows)
        t0 = time.perf_counter()
        for c0 in range(0, rows.size, 1024):
            oracle.masked_attention_dq_rows(qh, kh, vh, dh, rp_h, ci_h, 1, w.block, 0, 0,
                                            rows[c0:c0 + 1024])
        dt = time.perf_counter() - t0
        valid = np.minimum(w.block, w.n - np.arange(w.nqb) * w.block)
        rf = sum(4 * w.head_dim * int(valid[ci_h[rp_h[r // w.block]:rp_h[r // w.block + 1]]].sum())
                 for r in rows)
        cpu_baseline = {"value": 2 * rf / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
                        "kind": "oracle",
                        "sample": f"dQ of head 0, query rows {int(rows[0])}..{int(rows[-1])} "
                                  f"({rows.size} rows; 2x their forward FLOPs), {dt:.1f} s, fp64 NumPy"}

    if rank == 0:
        peaks, peak_kind = load_peaks()
        peak = float(peaks["bf16_tflops"])
        achieved = exec_flops / (kernel_ms * 1e-3) / 1e12
        line = {
            "metric": METRIC_BWD,
            "value": flops * world * args.steps / (ms * 1e-3) / 1e12,
            "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(w, nnz=int(rp_h[-1])), bwd_kernel=args.bwd_kernel),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak,
                         "traffic": None if one_pass else load_traffic(w.name, "bwd"),
                         "peak_kind": f"{peak_kind} bf16 burst",
                         "kernel": ("attn_bwd_fused_kernel<128> (+ prep, transposed lists, "
                                    "counter initialisation)" if one_pass else
                                    "attn_bwd_dkdv_kernel<128> + attn_bwd_dq_kernel<128> "
                                    "(+ prep and transposed lists)"),
                         "kernel_ms": kernel_ms, "flops_per_launch": exec_flops},
            "e2e": {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu_baseline,
        }
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


METRIC_MODULE = ("radial attention module fwd (q/k/v projection, block-sparse attention, "
                 "out projection) ms & effective TFLOP/s at 32k-120k tokens")
METRIC_MODULE_BWD = ("radial attention module bwd (dx, dW, db of the four projections through the "
                     "block-sparse attention backward) ms & effective TFLOP/s at 32k-120k tokens")


def run_ours_module(args, world, rank, local, backward=False):
    """Time bsa_attn_module_fwd: the RadialAttention module forward of the
    skill page (one stacked q/k/v projection GEMM, the attention on strided
    views of its output, the output projection GEMM), with random-init
    weights of the workload's width (C = heads x head_dim). value counts the
    two GEMMs' FLOPs plus the attention's computed-block FLOPs.

    With ``backward``, time bsa_attn_module_bwd instead (after one forward
    that fills the saved q/k/v, attention output and lse): four GEMMs
    (16 n C^2 FLOPs), the attention backward (counted as 2.5 x the forward's
    computed-block FLOPs; it executes 3.5 x) and two column sums."""
    import numpy as np
    import torch

    import block_sparse_attention_radial_b200 as bsa
    from workloads import WORKLOADS, make_module_inputs

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the library has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    w = WORKLOADS[args.workload]
    H, D, n = w.heads, w.head_dim, w.n
    x, wqkv, bqkv, wo, bo = make_module_inputs(w.batch, n, H, D, w.seed, device=dev)
    lists = bsa.radial_block_lists(w.frames, w.tokens_per_frame, w.block, device=dev,
                                  text_tokens=w.text_tokens)
    rp_h, ci_h = lists.row_ptr.cpu().numpy(), lists.col_idx.cpu().numpy()
    att_flops = bsa.computed_flops(rp_h, ci_h, n, w.block, D, w.batch, H, 1)
    flops = bsa.module_flops(w.batch, n, H, D, att_flops)
    exec_flops = flops
    y = torch.empty_like(x)
    ws = torch.empty(bsa.bsa_attn_module_workspace_bytes(w.batch, n, H, D, lists),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = 4  # q/k/v GEMM, work order, attention, out GEMM
    if backward:
        C = H * D
        flops = 16 * w.batch * n * C * C + 2.5 * att_flops
        exec_flops = 16 * w.batch * n * C * C + 3.5 * att_flops
        g = torch.Generator(device=dev)
        g.manual_seed(w.seed + 2000)
        dy = torch.randn(x.shape, generator=g, device=dev).to(torch.bfloat16)
        grads = (torch.empty_like(x), torch.empty_like(wqkv),
                 torch.empty(3 * C, dtype=x.dtype, device=dev), torch.empty_like(wo),
                 torch.empty(C, dtype=x.dtype, device=dev))
        bws = torch.empty(bsa.bsa_attn_module_bwd_workspace_bytes(w.batch, n, H, D, lists),
                          dtype=torch.uint8, device=dev)
        bsa.bsa_attn_module_fwd(x, wqkv, bqkv, wo, bo, H, lists, y, ws, 0.0, stream)
        # four GEMMs; attention backward: prep, transposed-list count, scan,
        # fill, dK/dV, dQ; two column-sum passes for each bias gradient
        launches_per_step = 4 + 6 + 4

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if backward:
            bsa.bsa_attn_module_bwd(x, wqkv, wo, dy, H, lists, ws, *grads, bws, 0.0, stream)
        else:
            bsa.bsa_attn_module_fwd(x, wqkv, bqkv, wo, bo, H, lists, y, ws, 0.0, stream)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if bsa.bsa_get_device_status() != 0:
        raise SystemExit("device status after warm-up")
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid).replace("GPU-", "")
    except Exception:
        pass
    sampler = ClockSampler(uuid) if rank == 0 else None
    if sampler is not None:
        time.sleep(0.4)
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    torch.cuda.synchronize(dev)
    t_start.record(stream)
    for i in range(args.steps):
        step(kev[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    clocks = sampler.stop() if sampler is not None else None
    ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
    kernel_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)
    if bsa.bsa_get_device_status() != 0:
        raise SystemExit("device status after the timed region")

    # end to end: x (backward: dy) from pinned host memory in, y (backward:
    # every gradient) back to the host
    e2e_steps = max(3, min(args.steps, 10))
    if backward:
        x_host = dy.cpu().pin_memory()
        x_dev = torch.empty_like(dy)
        out_dev = grads
    else:
        x_host = x.cpu().pin_memory()
        x_dev = torch.empty_like(x)
        out_dev = (y,)
    out_host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in out_dev]

    def e2e_step():
        x_dev.copy_(x_host, non_blocking=True)
        if backward:
            bsa.bsa_attn_module_bwd(x, wqkv, wo, x_dev, H, lists, ws, *grads, bws, 0.0, stream)
        else:
            bsa.bsa_attn_module_fwd(x_dev, wqkv, bqkv, wo, bo, H, lists, y, ws, 0.0, stream)
        for h_, d_ in zip(out_host, out_dev):
            h_.copy_(d_, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    h2d = x_host.numel() * x_host.element_size()
    d2h = sum(t.numel() * t.element_size() for t in out_host)

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not backward:
        import oracle

        C = H * D
        xc, wqc, bqc, woc, boc = (t.cpu() for t in (x, wqkv, bqkv, wo, bo))
        rows = np.arange(n // 2, min(n, n // 2 + 64))
        valid = np.minimum(w.block, n - np.arange(w.nqb) * w.block)
        att_row = sum(4 * D * int(valid[ci_h[rp_h[r // w.block]:rp_h[r // w.block + 1]]].sum())
                      for r in rows)

        def sample_flops(h):  # K, V projections of h heads, Q rows, attention rows, out_proj
            return h * (4 * n * C * D + 2 * rows.size * C * D + att_row + 2 * rows.size * D * C)

        for _ in range(2):  # the first call pays one-time costs
            t0 = time.perf_counter()
            oracle.radial_attention_module_rows(xc, wqc, bqc, woc, boc, H, rp_h, ci_h, 1,
                                                w.block, 0, rows, heads_used=[0])
            t_one = max(time.perf_counter() - t0, 1e-3)
        hs = int(max(1, min(H, args.cpu_seconds / t_one)))
        t0 = time.perf_counter()
        oracle.radial_attention_module_rows(xc, wqc, bqc, woc, boc, H, rp_h, ci_h, 1, w.block, 0,
                                            rows, heads_used=list(range(hs)))
        dt = time.perf_counter() - t0
        cpu_baseline = {"value": sample_flops(hs) / dt / 1e12, "unit": "TFLOP/s",
                        "cores": blas_threads(), "kind": "oracle",
                        "sample": f"module output rows {int(rows[0])}..{int(rows[-1])} of batch 0 "
                                  f"through heads 0..{hs - 1} (their k/v projections of all "
                                  f"{n} tokens, q rows, attention rows, out_proj columns), "
                                  f"{dt:.1f} s, fp64 NumPy"}

    if rank == 0:
        peaks, peak_kind = load_peaks()
        peak = float(peaks["bf16_tflops"])
        achieved = exec_flops / (kernel_ms * 1e-3) / 1e12
        cfg = workload_config(w, nnz=int(rp_h[-1]))
        cfg["hidden"] = H * D
        cfg["l2"] = ("x and the q/k/v projection output exceed L2 (126 MB) many times over; "
                     "no flush")
        line = {
            "metric": METRIC_MODULE_BWD if backward else METRIC_MODULE,
            "value": flops * world * args.steps / (ms * 1e-3) / 1e12,
            "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (random-init weights)",
            "config": cfg,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None,
                         "peak_kind": f"{peak_kind} bf16 burst",
                         "kernel": ("whole module backward: four gemm_bf16_sm100 GEMMs + attention "
                                    "backward (attn_bwd_dkdv/dq_kernel<128>) + column sums")
                         if backward else
                         ("whole module: gemm_bf16_sm100 q/k/v GEMM + work order + "
                          "attn_fwd_pair_sm100_kernel<128> + gemm_bf16_sm100 out GEMM"),
                         "kernel_ms": kernel_ms, "flops_per_launch": exec_flops},
            "e2e": {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu_baseline,
        }
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


METRIC_GEMM = "bf16 GEMM ms & TFLOP/s of the module's linear layers (Wan width)"
GEMM_SHAPES = {  # name: (m, n, k, A MN-major, B MN-major), rows = 21 x 1560 tokens, C = 5120
    "qkv": (32760, 15360, 5120, False, False),
    "out": (32760, 5120, 5120, False, False),
    "dattn": (32760, 5120, 5120, False, True),
    "dw_out": (5120, 5120, 32760, True, True),
    "dw_qkv": (15360, 5120, 32760, True, True),
    "dx": (32760, 5120, 15360, False, True),
}


def run_gemm(args, world, rank, local):
    """The module's six GEMM shapes (forward projections and backward
    products) through bsa_gemm_bf16, each timed with CUDA events; with
    --gemm-vs-torch also torch.matmul on the same operands, for context."""
    import torch

    import block_sparse_attention_radial_b200 as bsa

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the library has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    names = list(GEMM_SHAPES) if args.gemm_shape == "all" else [args.gemm_shape]
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    res = {}
    for name in names:
        m, n, k, amn, bmn = GEMM_SHAPES[name]
        a = torch.randn((k, m) if amn else (m, k), generator=g, device=dev).to(torch.bfloat16)
        b = torch.randn((k, n) if bmn else (n, k), generator=g, device=dev).to(torch.bfloat16)
        out = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        arms = [("ours", lambda: bsa.bsa_gemm_bf16(a, b, out, None, amn, bmn))]
        if args.gemm_vs_torch:
            arms.append(("torch_matmul", lambda: torch.matmul(a.t() if amn else a,
                                                              b if bmn else b.t(), out=out)))
        r = {"m": m, "n": n, "k": k, "a_mn_major": amn, "b_mn_major": bmn}
        for tag, fn in arms:
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize(dev)
            ts = []
            for _ in range(args.steps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize(dev)
                ts.append(e0.elapsed_time(e1))
            ms = statistics.median(ts)
            r[tag] = {"ms": ms, "tflops": 2 * m * n * k / ms / 1e9}
        if bsa.bsa_get_device_status() != 0:
            raise SystemExit("device status after the GEMMs")
        res[name] = r
        del a, b, out
        torch.cuda.empty_cache()
    head = names[0]
    achieved = res[head]["ours"]["tflops"]
    if rank == 0:
        print(json.dumps({
            "metric": METRIC_GEMM, "value": achieved, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic", "config": {"workload": f"gemm {head}"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "peak_kind": f"{peak_kind} bf16 burst",
                         "kernel": "gemm_bf16_sm100_kernel"},
            "shapes": res}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="wan",
                    choices=("wan", "hunyuan", "long4x", "tiny", "hunyuan_text", "generic",
                             "wan_b64"),
                    help="generic: per-head tile patterns built on the GPU (forward only)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--per-config-steps", type=int, default=10,
                    help="timed steps for each of the other forward configurations recorded "
                         "under per_config in the default (wan, one GPU) run; 0 skips them")
    ap.add_argument("--bwd-kernel", choices=("two", "one_pass"), default="two",
                    help="--pass bwd: bsa_attn_bwd (dK/dV + dQ kernels) or bsa_attn_bwd_one_pass")
    ap.add_argument("--rows", choices=("lists", "generated"), default="lists",
                    help="forward: read the block lists (default), or generate every row's key "
                         "blocks inside the attention kernel from the radial geometry / the "
                         "tile patterns (bsa_attn_fwd_radial / bsa_attn_fwd_patterns)")
    ap.add_argument("--gemm-shape", default="all", choices=("all",) + tuple(GEMM_SHAPES),
                    help="--pass gemm: one of the module's GEMM shapes, or all six")
    ap.add_argument("--gemm-vs-torch", action="store_true",
                    help="--pass gemm: also time torch.matmul on the same operands")
    ap.add_argument("--pass", dest="which",
                    choices=("fwd", "bwd", "module", "module_bwd", "gemm"),
                    default="fwd",
                    help="time the forward (default, the headline), the backward pass, the "
                         "whole module forward / backward (projections + attention), or the "
                         "module's GEMMs alone")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.workload == "generic" and args.which != "fwd":
        ap.error("the generic workload is timed for the forward pass only")
    if args.impl == "reference" and args.which != "fwd":
        ap.error("the reference arm times the forward oracle only (the backward and module "
                 "passes report their own oracle samples as cpu_baseline)")
    world, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.which == "bwd":
        return run_ours_bwd(args, world, rank, local)
    if args.which in ("module", "module_bwd"):
        return run_ours_module(args, world, rank, local, backward=args.which == "module_bwd")
    if args.which == "gemm":
        return run_gemm(args, world, rank, local)
    return run_ours(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
