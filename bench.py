#!/usr/bin/env python
"""Benchmark of the BA-Att forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload sweep_32k] [--keep 0.5] [--no-cpu-baseline]
                    [--no-extras]

One step is one pass of the whole hot path over one batch of synthetic input
already resident in HBM: block statistics -> corrected scores + top-k
(ba_att_selector) -> block-sparse attention over the kept blocks
(ba_att_sparse_fwd). Workloads whose recipe splits the keys (the 128K case)
run the split form instead: the kept lists are split at a seeded key-block
boundary, the first span is attended into an fp32 partial and the second is
attended and merged with it in its epilogue (FlashBlock Eq. 5 and Eq. 9).
The default workload is the 32K-token diffusion-LM case (B=1, 32 query /
8 KV heads, d=128, block 128, bf16, keep 0.5), single pass. Prints one JSON
line (rank 0).

Beside the timed K steps, rank 0 of a one-GPU run also reports: the same
step repeated for at least two seconds (`sustained`), the other full-size
workloads (`by_workload`, 128K with the split and merge included), the
end-to-end call from pinned host buffers (`e2e`), the GPU's own keep = 1 run,
the selector timed alone, the standalone merge and the CPU oracle on a
bounded sample (`cpu_baseline`).

With N > 1 (torchrun), every rank runs an independent replica of the
workload (the attention calls are independent units; nothing is exchanged),
so scaling is weak and `value` sums over ranks using the slowest rank's time.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import shutil
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "BA-Att fwd ms/call and kept-block TFLOP/s @50% keep, N=32K–128K; % of roofline"
UNIT = "TFLOP/s (kept-block FLOPs)"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SUSTAINED_SECONDS = 2.0
EXTRA_WORKLOADS = ("extreme_128k", "dlm_16k", "video_32k", "sweep_32k")


# --------------------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    return int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(x: float, device=None) -> float:
    """The slowest rank's value (all ranks call it; identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, flops_per_rank_step: float, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes its own replica of the step."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def kept_flops(cnt_total: int, block: int, d: int) -> float:
    """Two GEMMs (Q K^T and P V) per kept (query block, key block) pair."""
    return 4.0 * block * block * d * cnt_total


def selector_bytes(w, k: int) -> int:
    """Algorithmic selector traffic: read Q and K once, write the index lists."""
    e = 2 if w.dtype == "bf16" else 4
    qk = (w.B * w.Hq + w.B * w.Hkv) * w.N * w.d * e
    lists = w.B * w.Hq * w.nb * (k + 1) * 4
    return qk + lists


# kernels launched by one step: stats_warp, select_feat, topk_rows_lm, attn_tc (+ split_lists and a
# second attn_tc in the split form)
LAUNCHES_PER_STEP = {False: 4, True: 6}


def kernel_sources_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "block_sparse_attention_ba_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_from_profile(sha: str, step_key: str):
    """DRAM bytes of the step's attention launches from the committed ncu
    summary, if it was taken on the current kernel source for this step."""
    p = os.path.join(ROOT, "profiles", "attn_tc_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    entry = d.get("steps", {}).get(step_key)
    if not entry or entry.get("source_sha") != sha:
        return None
    return entry.get("dram_bytes_per_step")


def smi_gpu_id(props) -> str:
    """The nvidia-smi --id of a CUDA device: its PCI bus id. nvidia-smi counts
    GPUs by physical index and ignores CUDA_VISIBLE_DEVICES, so the CUDA
    ordinal would name another GPU whenever only some GPUs are visible."""
    return f"{int(props.pci_domain_id):08X}:{int(props.pci_bus_id):02X}:{int(props.pci_device_id):02X}.0"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons of one GPU (by PCI bus id),
    sampled every 50 ms with their timestamps; stop() summarises the samples
    taken inside a wall-clock window (the timed region)."""

    FIELDS = ("timestamp,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = os.path.join("/tmp", f"ba_att_clocks_{os.getpid()}_{id(self)}.csv")

    def command(self):
        return ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                "-lms", "50"]

    def start(self):
        self.proc = None
        if shutil.which("nvidia-smi") is None:
            return
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(self.command(), stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            self.fh.close()
            os.unlink(self.path)
            return
        # nvidia-smi is sampling once its first line is out (bounded wait)
        t0 = time.time()
        while time.time() - t0 < 3.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.05)

    def stop(self, window=None):
        """Stop sampling; summarise the samples inside window = (t0, t1) in
        seconds since the epoch (all samples when none fall inside)."""
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        out = self.summarise(lines, window)
        if out is not None:
            out["gpu"] = self.gpu
        return out

    @classmethod
    def summarise(cls, lines, window=None):
        import datetime
        rows = []
        for line in lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                ts = None
            rows.append((ts, parts[1:]))
        if not rows:
            return None
        inside = [r for ts, r in rows if window is not None and ts is not None and window[0] <= ts <= window[1]]
        use = inside if inside else [r for _, r in rows]

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [v for v in (num(r[1]) for r in use) if v is not None]
        smax = [v for v in (num(r[2]) for r in use) if v is not None]
        reasons = sorted({cls.REASONS[k] for r in use for k in range(4) if r[5 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(use), "in_timed_region": bool(inside),
                "bus_ids": sorted({r[0] for r in use})}


# --------------------------------------------------------------------------- CPU oracle arms

def oracle_sample(w, Q, K, V, keep, seed, n_blocks, n_sel_heads):
    """Time the oracle (float32, all host cores) on a bounded sample of one
    step: the selector for `n_sel_heads` query heads (with their KV heads)
    and masked attention for `n_blocks` query blocks; extrapolate linearly
    to the full step. Returns (seconds per full step, description)."""
    import oracle as O
    rng = np.random.default_rng(seed)
    s = w.d ** -0.5
    k = O.keep_count(keep, w.nb)
    G = w.Hq // w.Hkv
    heads = sorted(rng.choice(w.Hq, size=n_sel_heads, replace=False).tolist())
    t0 = time.perf_counter()
    kv_heads = sorted({h // G for h in heads})
    qm, qv, _ = O.block_stats(Q[:, heads], w.N, w.block, dtype=np.float32)
    km, kv, kc = O.block_stats(K[:, kv_heads], w.N, w.block, dtype=np.float32)
    # corrected_scores maps query head -> KV head by position; lay the
    # sampled KV heads out so that each sampled query head finds its own
    kmap = [kv_heads.index(h // G) for h in heads]
    S = O.corrected_scores(qm, qv, km[:, kmap], kv[:, kmap], kc, s, dtype=np.float32)
    idx, cnt = O.select_topk(S, k)
    t_sel = time.perf_counter() - t0
    blocks = [(0, heads[int(rng.integers(len(heads)))], int(rng.integers(w.nb))) for _ in range(n_blocks)]
    idx_full = np.zeros((w.B, w.Hq, w.nb, k), dtype=np.int32)
    cnt_full = np.full((w.B, w.Hq, w.nb), k, dtype=np.int32)
    for hi, h in enumerate(heads):
        idx_full[:, h] = idx[:, hi]
    t1 = time.perf_counter()
    O.masked_attention(Q, K, V, idx_full, cnt_full, w.N, w.block, s, query_blocks=blocks, dtype=np.float32)
    t_att = time.perf_counter() - t1
    per_step = t_sel * (w.Hq / n_sel_heads) + t_att * (w.B * w.Hq * w.nb / n_blocks)
    desc = (f"oracle float32 on host cores: selector for {n_sel_heads}/{w.Hq} query heads, masked attention for "
            f"{n_blocks}/{w.B * w.Hq * w.nb} query blocks; extrapolated linearly to one full step")
    return per_step, desc, t_sel + t_att


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# --------------------------------------------------------------------------- our arm

def step_config(w, keep: float, k: int, split_block, world: int) -> dict:
    """The JSON `config` of a step on workload w; both arms report the same one."""
    in_mib = (w.B * w.Hq + 2 * w.B * w.Hkv) * w.N_alloc * w.d * 2 / 2**20
    form = (f"selector(stats+scores+top-k)+split(block {split_block})+sparse_fwd+sparse_fwd_merge"
            if split_block is not None else "selector(stats+scores+top-k)+sparse_fwd")
    cfg = {"workload": f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} d={w.d} block={w.block} "
                       f"bf16 keep={keep}; step = {form}",
           "keep": keep, "kept_blocks_per_query_block": k,
           "parallelism": f"{world} independent replica(s)",
           "l2": f"inputs {in_mib:.0f} MiB > L2 126 MiB; no flush"}
    if split_block is not None:
        cfg["split_block"] = split_block
    return cfg


class Step:
    """One pass of the hot path on device-resident inputs, every buffer
    allocated once. split_block None: selector -> sparse_fwd; otherwise
    selector -> split_lists -> sparse_fwd (fp32 partial) -> sparse_fwd_merge."""

    def __init__(self, w, keep, Qd, Kd, Vd, split_block, dev):
        import torch
        from block_sparse_attention_ba_b200 import api
        self.api, self.w, self.keep, self.dev = api, w, keep, dev
        self.Qd, self.Kd, self.Vd = Qd, Kd, Vd
        self.split_block = split_block
        self.shape = shape = api.Shape.of(Qd, Kd, w.N, w.block)
        self.k = k = api.keep_count(shape, keep)
        nb = shape.nb
        self.stats_buf = (torch.empty((w.B, w.Hq, nb, w.d), device=dev),
                          torch.empty((w.B, w.Hq, nb, w.d), device=dev),
                          torch.empty((w.B, w.Hkv, nb, w.d), device=dev),
                          torch.empty((w.B, w.Hkv, nb, w.d), device=dev))
        self.idx = torch.empty((w.B, w.Hq, nb, k), device=dev, dtype=torch.int32)
        self.cnt = torch.empty((w.B, w.Hq, nb), device=dev, dtype=torch.int32)
        # the score map is not asked for: ba_att_selector keeps it in its workspace
        self.sel_ws = torch.empty(api.selector_workspace_bytes(shape), device=dev, dtype=torch.uint8)
        self.O = torch.empty_like(Qd)
        self.L = torch.empty((w.B, w.Hq, w.N_alloc), device=dev)
        if split_block is not None:
            self.lists = (torch.empty_like(self.idx), torch.empty_like(self.cnt), torch.empty_like(self.idx),
                          torch.empty_like(self.cnt))
            # the first span's partial stays in fp32 so the merged output is rounded to bf16 once
            self.O1 = torch.empty(Qd.shape, device=dev, dtype=torch.float32)
            self.L1 = torch.empty((w.B, w.Hq, w.N_alloc), device=dev)
            self.names = ("selector", "split", "sparse_lo", "sparse_hi_merge")
            self.attention = ("sparse_lo", "sparse_hi_merge")
        else:
            self.names = ("selector", "sparse")
            self.attention = ("sparse",)
        self.stream = torch.cuda.current_stream(dev)

    def __call__(self, events=None):
        api = self.api

        def mark(i):
            if events is not None:
                events[i].record(self.stream)
        mark(0)
        api.selector(self.Qd, self.Kd, self.shape, self.keep, kmax=self.k,
                     out=(self.stats_buf, self.idx, self.cnt, None), workspace=self.sel_ws)
        mark(1)
        if self.split_block is None:
            api.sparse_fwd(self.Qd, self.Kd, self.Vd, self.idx, self.cnt, self.shape, out=(self.O, self.L))
            mark(2)
            return
        api.split_lists(self.idx, self.cnt, self.shape, self.split_block, out=self.lists)
        mark(2)
        api.sparse_fwd(self.Qd, self.Kd, self.Vd, self.lists[0], self.lists[1], self.shape, out=(self.O1, self.L1))
        mark(3)
        # second span, merged with the first in its epilogue (FlashBlock Eq. 9)
        api.sparse_fwd_merge(self.Qd, self.Kd, self.Vd, self.lists[2], self.lists[3], self.shape, self.O1, self.L1,
                             out=(self.O, self.L))
        mark(4)


def timed_steps(step, steps, clock_id, barrier=None):
    """Run exactly `steps` steps between CUDA events on the launching stream,
    synchronised (and barriered) on both sides, with per-stage events and the
    nvidia-smi clocks of that window."""
    import torch
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(step.names) + 1)] for _ in range(steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(clock_id)
    clocks.start()                                  # returns once nvidia-smi is sampling
    if barrier:
        barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    t_start.record(step.stream)
    for s_i in range(steps):
        step(ev[s_i])
    t_end.record(step.stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    if barrier:
        barrier()
    time.sleep(0.06)                                # the sample that covers the region's end
    clk = clocks.stop(window=(wall0, wall1))
    per = {n: [ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps)] for i, n in enumerate(step.names)}
    return {"elapsed_ms": t_start.elapsed_time(t_end), "clocks": clk,
            "stage_ms": {n: float(np.mean(v)) for n, v in per.items()},
            # the first timed step starts on an idle GPU, so its first stage also
            # holds the host's launch latency; the median over steps leaves that out
            "stage_ms_median": {n: float(np.median(v)) for n, v in per.items()},
            "step_ms": [ev[s][0].elapsed_time(ev[s][-1]) for s in range(steps)]}


def check_device(api, when):
    st, word = api.get_device_error()
    if st != 0:
        raise RuntimeError(f"device error word {word:#x} {when}")


def attention_kernel_name(w):
    """The attention kernel the library runs for this workload's shape."""
    if w.dtype != "bf16" or w.block not in (64, 128, 256) or w.d not in (64, 128):
        return "attn_simt_kernel"
    return "attn_tc2_kernel (256-row blocks on a CTA pair)" if (w.block == 256 and w.d == 128) else "attn_tc_kernel"


def attention_roofline(step, t, flops, peaks, peak_src, traffic=None):
    att_ms = sum(t["stage_ms"][n] for n in step.attention)
    achieved = flops / (att_ms * 1e-3) / 1e12
    return {"bound": "tensor",
            "kernel": attention_kernel_name(step.w) + (" (both span launches of a step; the second also merges the first "
                                          "span's fp32 partial in its epilogue)" if step.split_block is not None
                                          else " (one launch per step)"),
            "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(achieved / peaks["bf16_tflops"], 4),
            "frac_vs_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
            "peak_source": f"{peak_src} (dense bf16 burst; of measured)" if peak_src == "measured"
            else f"{peak_src} (dense bf16 burst; of fallback)",
            "traffic": traffic, "ms": round(att_ms, 4),
            "units": f"{int(step.cnt.sum().item())} kept (query block, key block) pairs x 4*b^2*d FLOP"}


def selector_entry(step, t, peaks):
    w, k = step.w, step.k
    sel_bytes = selector_bytes(w, k)
    frac = lambda byts, ms: round(byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)
    sel_ms = t["stage_ms_median"]["selector"]
    return {"bound": "hbm", "call": "ba_att_selector (stats, scores, top-k)",
            "achieved": round(sel_bytes / (sel_ms * 1e-3) / 1e9, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": frac(sel_bytes, sel_ms), "bytes": sel_bytes, "ms": round(sel_ms, 4),
            "timing": "in the step, median over steps",
            "frac_mean_over_steps": frac(sel_bytes, t["stage_ms"]["selector"])}


def run_ours(args):
    import torch
    import torch.distributed as dist

    from block_sparse_attention_ba_b200 import api
    from block_sparse_attention_ba_b200.workloads import WORKLOADS, make_inputs

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    api.load_library()
    dev = torch.device("cuda", local)
    clock_id = smi_gpu_id(torch.cuda.get_device_properties(dev))
    barrier = dist.barrier if world > 1 else None

    w = WORKLOADS[args.workload]
    if args.block:
        w = w.with_(block=args.block)
    keep = args.keep
    Q, K, V, meta = make_inputs(w)
    split_block = meta.get("split_block") if w.split else None
    Qd = torch.from_numpy(Q).to(torch.bfloat16).to(dev)
    Kd = torch.from_numpy(K).to(torch.bfloat16).to(dev)
    Vd = torch.from_numpy(V).to(torch.bfloat16).to(dev)
    step = Step(w, keep, Qd, Kd, Vd, split_block, dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    check_device(api, "during warm-up")
    cnt_total = int(step.cnt.sum().item())
    flops = kept_flops(cnt_total, w.block, w.d)

    t = timed_steps(step, args.steps, clock_id, barrier)
    check_device(api, "during timing")
    elapsed_ms = max_over_ranks(t["elapsed_ms"], dev)
    ms_per_step = elapsed_ms / args.steps
    value = job_tflops(world, flops, ms_per_step)

    result = None
    if rank == 0:
        peaks, peak_src = load_peaks()
        step_key = f"{w.name}/b{w.block}/{'split' if split_block is not None else 'single'}/keep{keep}"
        traffic = traffic_from_profile(kernel_sources_sha(["attn_tc.cuh", "common.cuh"]), step_key)
        result = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": step_config(w, keep, step.k, split_block, world),
            "roofline": attention_roofline(step, t, flops, peaks, peak_src, traffic),
            "selector": selector_entry(step, t, peaks),
            "stages_ms": {n: round(v, 4) for n, v in t["stage_ms"].items()},
            "stages_ms_median": {n: round(v, 4) for n, v in t["stage_ms_median"].items()},
            "gpu_launches": LAUNCHES_PER_STEP[split_block is not None] * args.steps, "clocks": t["clocks"],
        }
    return result, dict(Qd=Qd, Kd=Kd, Vd=Vd, shape=step.shape, keep=keep, w=w, Q=Q, K=K, V=V,
                        split_block=split_block, step=step, flops=flops, world=world, rank=rank, dev=dev,
                        clock_id=clock_id, ms_per_step=ms_per_step)


def run_sustained(ctx, seconds=SUSTAINED_SECONDS):
    """The same step repeated back to back for at least `seconds` of GPU time
    (per-step CUDA events, median step), with the clocks of that window: a
    steadier figure than the K-step region under the power cap."""
    import torch
    step = ctx["step"]
    n = max(10, int(math.ceil(seconds * 1e3 / ctx["ms_per_step"])))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    clocks = ClockSampler(ctx["clock_id"])
    clocks.start()
    torch.cuda.synchronize()
    wall0 = time.time()
    ev[0].record(step.stream)
    for i in range(n):
        step()
        ev[i + 1].record(step.stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    clk = clocks.stop(window=(wall0, wall1))
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(n)]
    med = float(np.median(per))
    return {"steps": n, "seconds": round(ev[0].elapsed_time(ev[-1]) * 1e-3, 3), "ms_per_step_median": round(med, 4),
            "value_median_step": round(job_tflops(1, ctx["flops"], med), 2),
            "ms_per_step_p10_p90": [round(float(np.percentile(per, 10)), 4), round(float(np.percentile(per, 90)), 4)],
            "clocks": clk}


def run_e2e(ctx, steps, warmup):
    """Same step through the public host-buffer entry point (ba_att_forward_host):
    per step, the H2D copy of Q, K, V from pinned host memory, the selector,
    the sparse attention (split + fused merge where the workload splits), and
    the D2H copy of O and LSE, all inside the timed region. The library
    pipelines the copies against the compute in chunks of KV heads."""
    import torch
    from block_sparse_attention_ba_b200 import api

    dev = ctx["dev"]
    w = ctx["w"]
    Qh = torch.from_numpy(ctx["Q"]).to(torch.bfloat16).pin_memory()
    Kh = torch.from_numpy(ctx["K"]).to(torch.bfloat16).pin_memory()
    Vh = torch.from_numpy(ctx["V"]).to(torch.bfloat16).pin_memory()
    Oh = torch.empty(Qh.shape, dtype=torch.bfloat16).pin_memory()
    Lh = torch.empty(Qh.shape[:3], dtype=torch.float32).pin_memory()
    split = ctx["split_block"] if ctx["split_block"] is not None else -1
    ws = torch.empty(api.forward_host_workspace_bytes(ctx["shape"], ctx["keep"], split), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def e2e_step():
        api.forward_host(Qh, Kh, Vh, w.N, w.block, ctx["keep"], split_block=split, workspace=ws, out=(Oh, Lh),
                         device=dev)

    for _ in range(warmup):
        e2e_step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    check_device(api, "in e2e")
    ms = max_over_ranks(a.elapsed_time(b) / steps, dev)
    h2d = (Qh.numel() + Kh.numel() + Vh.numel()) * 2
    d2h = (Oh.numel() * 2 + Lh.numel() * 4) * w.N // w.N_alloc
    return {"value": round(job_tflops(ctx["world"], ctx["flops"], ms), 2), "unit": UNIT,
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "api": "ba_att_forward_host (pinned host buffers, copies pipelined per chunk of KV heads)"}


def run_selector_isolated(step, reps=20):
    """The selector on its own, back to back: ba_att_selector, then the
    two-call form (ba_att_stats, ba_att_select). The launches are queued
    behind a GPU sleep so that no host launch latency falls inside the timed
    intervals. Q and K exceed L2, so each pass streams them from HBM."""
    import torch
    api, shape, keep, w = step.api, step.shape, step.keep, step.w
    stats_buf, idx, cnt = step.stats_buf, step.idx, step.cnt
    scores = torch.empty((w.B, w.Hq, w.nb, w.nb), device=step.dev, dtype=torch.float32)   # the two-call form's map
    one_call = lambda: api.selector(step.Qd, step.Kd, shape, keep, kmax=step.k, out=(stats_buf, idx, cnt, None),
                                    workspace=step.sel_ws)
    one_call()
    api.stats(step.Qd, step.Kd, shape, out=stats_buf)
    api.select(stats_buf, shape, keep, out=(idx, cnt, scores))
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(reps)]
    torch.cuda._sleep(100_000_000)                 # ~50 ms of GPU time while the host queues the reps
    for r in range(reps):
        ev[r][0].record(step.stream)
        one_call()
        ev[r][1].record(step.stream)
        api.stats(step.Qd, step.Kd, shape, out=stats_buf)
        ev[r][2].record(step.stream)
        api.select(stats_buf, shape, keep, out=(idx, cnt, scores))
        ev[r][3].record(step.stream)
    torch.cuda.synchronize()
    med = lambda a, b: float(np.median([e[a].elapsed_time(e[b]) for e in ev]))
    o_ms, s_ms, l_ms = med(0, 1), med(1, 2), med(2, 3)
    byts = selector_bytes(w, step.k)
    stats_bytes = byts - w.B * w.Hq * w.nb * (step.k + 1) * 4
    peaks, _ = load_peaks()
    fr = lambda b, ms: round(b / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)
    return {"ms": round(o_ms, 4), "bytes": byts, "achieved_gbs": round(byts / (o_ms * 1e-3) / 1e9, 1),
            "frac": fr(byts, o_ms),
            "two_calls": {"stats_ms": round(s_ms, 4), "select_ms": round(l_ms, 4), "frac": fr(byts, s_ms + l_ms),
                          "stats_frac": fr(stats_bytes, s_ms)},
            "timing": f"ba_att_selector, then ba_att_stats + ba_att_select, back to back, median of {reps}, "
                      "launches queued ahead"}


def run_merge_standalone(ctx, steps=5):
    """ba_att_merge_lse on its own: the kept lists split at the middle key
    block, each span attended into an fp32 partial, the two partials merged
    into bf16 (HBM-bound)."""
    import torch
    from block_sparse_attention_ba_b200 import api

    step, shape = ctx["step"], ctx["shape"]
    lo_i, lo_c, hi_i, hi_c = api.split_lists(step.idx, step.cnt, shape, shape.nk // 2)
    O1, L1 = api.sparse_fwd(ctx["Qd"], ctx["Kd"], ctx["Vd"], lo_i, lo_c, shape, out_dtype=torch.float32)
    O2, L2 = api.sparse_fwd(ctx["Qd"], ctx["Kd"], ctx["Vd"], hi_i, hi_c, shape, out_dtype=torch.float32)
    Ox, Lx = torch.empty_like(ctx["Qd"]), torch.empty_like(L1)
    api.merge_lse(O1, L1, O2, L2, out=(Ox, Lx))
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(ctx["dev"])
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        api.merge_lse(O1, L1, O2, L2, out=(Ox, Lx))
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    byts = (O1.numel() + O2.numel()) * 4 + (L1.numel() + L2.numel()) * 4 + Ox.numel() * 2 + Lx.numel() * 4
    peaks, _ = load_peaks()
    gbs = byts / (ms * 1e-3) / 1e9
    del O1, O2, L1, L2, Ox, Lx
    return {"ms": round(ms, 4), "bytes": byts, "achieved_gbs": round(gbs, 1),
            "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4)}


def run_dense(step, steps=3):
    """The GPU path's own dense run: keep = 1.0, single pass (stats, select, sparse_fwd)."""
    import torch
    api, shape, w = step.api, step.shape, step.w
    st = api.stats(step.Qd, step.Kd, shape)
    idx, cnt, sc1 = api.select(st, shape, 1.0, with_scores=True)
    O, L = api.sparse_fwd(step.Qd, step.Kd, step.Vd, idx, cnt, shape)
    torch.cuda.synchronize()
    a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    a.record(step.stream)
    for _ in range(steps):
        api.stats(step.Qd, step.Kd, shape, out=st)
        api.select(st, shape, 1.0, out=(idx, cnt, sc1))
    b.record(step.stream)
    for _ in range(steps):
        api.sparse_fwd(step.Qd, step.Kd, step.Vd, idx, cnt, shape, out=(O, L))
    c.record(step.stream)
    torch.cuda.synchronize()
    sel_ms = a.elapsed_time(b) / steps
    att_ms = b.elapsed_time(c) / steps
    fl = kept_flops(int(cnt.sum().item()), w.block, w.d)
    return {"keep": 1.0, "ms_per_call": round(sel_ms + att_ms, 4), "sparse_fwd_ms": round(att_ms, 4),
            "tflops": round(fl / ((sel_ms + att_ms) * 1e-3) / 1e12, 1),
            "sparse_fwd_tflops": round(fl / (att_ms * 1e-3) / 1e12, 1)}


def run_workload_entry(name, keep, dev, clock_id, steps=5, warmup=3, block=0):
    """A full-size workload timed like the headline (its own recipe's step
    form: single pass, or split + fused merge for the 128K case), with inputs
    drawn on the device (timing only; parity at full size is in the tests)."""
    import torch
    from block_sparse_attention_ba_b200 import api
    from block_sparse_attention_ba_b200.workloads import WORKLOADS, make_inputs_device

    w = WORKLOADS[name]
    if block:
        w = w.with_(block=block)
    Qd, Kd, Vd, meta = make_inputs_device(w, dev)
    split_block = meta.get("split_block") if w.split else None
    step = Step(w, keep, Qd, Kd, Vd, split_block, dev)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    check_device(api, f"in {name}")
    flops = kept_flops(int(step.cnt.sum().item()), w.block, w.d)
    t = timed_steps(step, steps, clock_id)
    check_device(api, f"in {name}")
    peaks, peak_src = load_peaks()
    ms = t["elapsed_ms"] / steps
    sel = selector_entry(step, t, peaks)
    sel["isolated"] = run_selector_isolated(step, reps=10)
    out = {"config": step_config(w, keep, step.k, split_block, 1), "steps": steps, "warmup": warmup,
           "ms_per_step": round(ms, 4), "value": round(job_tflops(1, flops, ms), 2), "unit": UNIT,
           "roofline": attention_roofline(step, t, flops, peaks, peak_src),
           "selector": sel, "stages_ms_median": {n: round(v, 4) for n, v in t["stage_ms_median"].items()},
           "clocks": t["clocks"], "inputs": "drawn on the device with the workload's recipe (make_inputs_device)"}
    del step, Qd, Kd, Vd
    torch.cuda.empty_cache()
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="sweep_32k")
    ap.add_argument("--keep", type=float, default=0.5)
    ap.add_argument("--block", type=int, default=0,
                    help="query and key block size in place of the workload's (0: the workload's own)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="only the timed K steps (no sustained loop, other workloads, e2e, dense, merge)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, _ = dist_env()

    if args.impl == "reference":
        if rank != 0:
            return
        run_reference(args)
        return

    result, ctx = run_ours(args)
    if not args.no_extras:
        # every rank takes the same collective steps: the e2e run reduces its time over ranks
        e2e = run_e2e(ctx, max(3, args.steps // 2), 3)
        if rank == 0:
            result["e2e"] = e2e
    if rank == 0 and not args.no_extras and world == 1:
        result["sustained"] = run_sustained(ctx)
        result["selector"]["isolated"] = run_selector_isolated(ctx["step"])
        result["dense_keep1"] = run_dense(ctx["step"])
        result["merge_lse_standalone"] = run_merge_standalone(ctx)
        by = {}
        for name in EXTRA_WORKLOADS if not args.block else ():
            if name != args.workload:
                by[name] = run_workload_entry(name, args.keep, ctx["dev"], ctx["clock_id"])
        if not args.block and args.workload == "sweep_32k":
            # the rest of the 32K keep sweep, and 64- and 256-row query blocks at keep 0.5
            by["sweep_32k@keep0.25"] = run_workload_entry("sweep_32k", 0.25, ctx["dev"], ctx["clock_id"])
            by["sweep_32k@block64"] = run_workload_entry("sweep_32k", args.keep, ctx["dev"], ctx["clock_id"],
                                                         block=64)
            by["sweep_32k@block256"] = run_workload_entry("sweep_32k", args.keep, ctx["dev"], ctx["clock_id"],
                                                          block=256)
        result["by_workload"] = by
    if rank == 0:
        if not args.no_cpu_baseline:
            per_step, desc, spent = oracle_sample(ctx["w"], ctx["Q"], ctx["K"], ctx["V"], ctx["keep"], 0,
                                                  n_blocks=768, n_sel_heads=8)
            result["cpu_baseline"] = {"value": round(ctx["flops"] / per_step / 1e12, 6), "unit": UNIT,
                                      "cores": cpu_cores(), "kind": "oracle", "sample": desc,
                                      "sample_seconds": round(spent, 1)}
        print(json.dumps(result), flush=True)
    if ctx["world"] > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def run_reference(args):
    """The oracle as it stands, timed on the host cores on bounded samples of
    the same workload; each step is one sample, extrapolated to a full step."""
    from block_sparse_attention_ba_b200.workloads import WORKLOADS, make_inputs
    import oracle as O

    w = WORKLOADS[args.workload]
    if args.block:
        w = w.with_(block=args.block)
    Q, K, V, meta = make_inputs(w)
    split_block = meta.get("split_block") if w.split else None
    k = O.keep_count(args.keep, w.nb)
    flops = kept_flops(w.B * w.Hq * w.nb * k, w.block, w.d)
    for i in range(args.warmup):
        oracle_sample(w, Q, K, V, args.keep, 1000 + i, n_blocks=2, n_sel_heads=1)
    per = []
    t0 = time.perf_counter()
    for i in range(args.steps):
        ps, desc, _ = oracle_sample(w, Q, K, V, args.keep, i, n_blocks=192, n_sel_heads=2)
        per.append(ps)
    wall = time.perf_counter() - t0
    ms = float(np.mean(per)) * 1e3
    value = flops / (ms * 1e-3) / 1e12
    out = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": 1,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
           "config": step_config(w, args.keep, k, split_block, dist_env()[0]),
           "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                            "sample": desc + "; one sample per step", "wall_seconds": round(wall, 1)},
           "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           "gpu_launches": 0}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
