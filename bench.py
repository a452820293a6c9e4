#!/usr/bin/env python
"""Benchmark of adaptive block-sparse spatiotemporal attention on B200.

Metric: sparse-attention forward ms and effective TFLOP/s at the Wan-480p
latent (20x32x52 = 33,280 tokens, 40 heads, d=128, bf16, top-p 0.95,
k_min 8).  One step = one ``fvattn_forward`` call: pool/select, schedule and
the block-sparse fine stage over one batch of synthetic input (the tile
reorder and its inverse are fused into the loads and stores).  Effective
FLOPs = 4 * 64 * 64 * d per selected (query tile, key tile) pair.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fvattn|reference]

Multi-GPU: one process per GPU (torchrun); every rank runs an independent
replica of the workload (heads shard with no exchange), the time is the max
over ranks and ``value`` counts the work of all ranks ("scaling": "weak").
``--impl reference`` times the CPU oracle on a bounded sample instead.
A single-GPU line also carries ``secondary``: the same forward, device-timed,
on the 720p latent (20x48x80 = 76,800 tokens, 3D Hilbert order, RoPE in the
loads) with its own stage times, roofline and CTA load balance.
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
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_spatiotemporal_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "sparse-attn fwd ms & effective TFLOP/s (33k tok, 40 heads, d=128, top-p .95)"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def pair_flops(d: int) -> float:
    return 4.0 * 64 * 64 * d


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    # the kernel and the work-list order it runs (which decides its L2 reuse)
    for rel in ("block_sparse_spatiotemporal_b200/csrc/fine_tc.cu",
                "block_sparse_spatiotemporal_b200/csrc/fvattn_internal.cuh",
                "block_sparse_spatiotemporal_b200/csrc/schedule.cu",
                "block_sparse_spatiotemporal_b200/csrc/api.cu"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """dram bytes per fine-kernel launch from the committed ncu summary, or
    None when the summary is absent or was taken on another kernel source."""
    path = os.path.join(ROOT, "profiles", f"fine_tc_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpus):
        self.gpus = set(gpus)
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.12)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9 or not f[0].isdigit() or int(f[0]) not in self.gpus:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle arm (bounded sample of the same workload)
# ---------------------------------------------------------------------------
def oracle_sample(wl, q, k, v, budget_s: float, seed: int = 0, gpu_lists=None):
    """Time the oracle as it stands on a bounded sample: the coarse stage
    (pool, scores, top-p selection) head by head, then the fine stage of
    randomly drawn (head, query tile) rows until the budget is spent.  With
    ``gpu_lists`` = (counts, idx) host arrays [B, H, nT(, cap)] the coarse
    stage runs on every head and each head's GPU lists are checked against
    the oracle's (oracle/list_check.py) on every row.

    Returns a dict: est_s (the whole workload, scaled by heads and by
    selected pairs), flops, stage_s (coarse: measured, scaled by heads;
    fine: scaled by selected pairs), desc, threads, and parity (or None)."""
    from oracle import fvattn_oracle as O
    from oracle.list_check import check_lists, merge
    rope = dict(dims=wl.rope_dims, base=wl.rope_base) if wl.rope else None
    pos = O.positions(wl.grid, wl.order)
    scale = O.default_scale(wl.head_dim)
    t0 = time.perf_counter()
    coarse = []
    coarse_heads = 0
    parity = None
    t_check = 0.0
    for h in range(wl.heads):
        coarse.append(O.coarse_head(O.as_f64(q[0, h], wl.dtype), O.as_f64(k[0, h], wl.dtype), wl.grid, wl.order,
                                    wl.top_p, wl.k_min, scale, rope, pos))
        coarse_heads += 1
        if gpu_lists is not None:
            tc = time.perf_counter()
            one = check_lists(coarse[-1], gpu_lists[0][0, h], gpu_lists[1][0, h], wl.top_p, wl.k_min)
            one["bad_rows"] = [(h, r) for r in one["bad_rows"]]
            parity = merge(parity or {}, one)
            t_check += time.perf_counter() - tc
        elif time.perf_counter() - t0 > budget_s / 2 and h < wl.heads - 1:
            break
    t_coarse = time.perf_counter() - t0 - t_check
    pairs_per_head = [int(r["counts"].sum()) for r in coarse]
    est_pairs_total = sum(pairs_per_head) * wl.heads / coarse_heads
    rng = np.random.default_rng(seed)
    t1 = time.perf_counter()
    done_pairs = 0
    rows = 0
    vt_cache = {}
    while time.perf_counter() - t1 < budget_s / 2 or rows == 0:
        h = int(rng.integers(coarse_heads))
        i = int(rng.integers(wl.num_tiles))
        r = coarse[h]
        if h not in vt_cache:
            qt, kt = O.fine_operands(O.as_f64(q[0, h], wl.dtype), O.as_f64(k[0, h], wl.dtype), wl.grid, wl.dtype,
                                     rope, pos)
            vt_cache = {h: (qt, kt, O.to_tiled(O.as_f64(v[0, h], wl.dtype), pos))}
        qt, kt, vt = vt_cache[h]
        O.fine_tile(qt[i * 64:(i + 1) * 64], kt, vt, r["idx"][i, :r["counts"][i]], scale)
        done_pairs += int(r["counts"][i])
        rows += 1
    t_fine = time.perf_counter() - t1
    coarse_s = t_coarse * wl.heads / coarse_heads
    fine_s = t_fine * est_pairs_total / max(done_pairs, 1)
    desc = (f"oracle (numpy fp64) coarse stage of {coarse_heads}/{wl.heads} heads + fine stage of {rows} random "
            f"(head, query tile) rows ({done_pairs} selected pairs of ~{int(est_pairs_total)}), scaled to the full "
            f"workload by heads and by selected pairs")
    return dict(est_s=coarse_s + fine_s, flops=est_pairs_total * pair_flops(wl.head_dim),
                stage_s={"coarse": coarse_s, "fine": fine_s}, desc=desc, threads=_threads(), parity=parity)


def _threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((x.get("num_threads", 1) for x in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def workload_config(wl, args, world: int = 1) -> dict:
    """The workload as both arms name it (no measured figures)."""
    qk_bytes = 2 * wl.heads * wl.tokens * wl.head_dim * 2
    return {"workload": wl.name, "grid": list(wl.grid), "tokens": wl.tokens, "heads": wl.heads,
            "head_dim": wl.head_dim, "top_p": wl.top_p, "k_min": wl.k_min, "order": wl.order, "rope": wl.rope,
            "scoring": "sub-block 2x2x2" if getattr(args, "subblock", False) else "tile mean",
            "l2": "inputs larger than L2 (q+k+v = %.0f MB)" % (3 * qk_bytes / 2 / 1e6),
            "parallelism": f"replica x{world}"}


def oracle_tiny_single_core() -> dict:
    """The oracle's whole path (coarse stage and fine stage of every head)
    on the tiny fp32 workload (8x16x16 tokens, 2 heads, d=64) on one core."""
    from oracle import fvattn_oracle as O
    wl1 = WORKLOADS["tiny_fp32"]
    q, k, v = make_inputs(wl1)
    try:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(1)
    except Exception:
        limit = None
    t0 = time.perf_counter()
    for h in range(wl1.heads):
        O.forward_head(q[0, h], k[0, h], v[0, h], wl1.grid, wl1.order, wl1.top_p, wl1.k_min, wl1.dtype)
    ms = (time.perf_counter() - t0) * 1e3
    if limit is not None:
        limit.unregister()
    return {"workload": wl1.name, "ms": ms, "cores": 1}


def cpu_baseline_of(res: dict) -> dict:
    return {"value": res["flops"] / res["est_s"] / 1e12, "unit": UNIT, "cores": res["threads"],
            "nproc": os.cpu_count(), "kind": "oracle", "sample": res["desc"],
            "est_ms_per_step": res["est_s"] * 1e3,
            "stage_ms": {k: v * 1e3 for k, v in res["stage_s"].items()},
            "ms_is": "estimate: the sample's time scaled to the whole workload"}


def sm_imbalance(F, shape, ws, rope=None) -> dict:
    """Load balance of the last profiled fine-stage launch on `ws`: busy time
    (set-up done to last item finished) of every persistent CTA; the ratio
    max / mean is the single-GPU counterpart of the per-rank imbalance ratio
    the load balancing targets."""
    t = F.profile_cta_times(shape, ws, rope)
    if len(t) == 0:
        return None
    busy = (t[:, 1] - t[:, 0]).astype(np.float64)
    span = float(t[:, 1].max() - t[:, 0].min())
    return {"ctas": int(len(t)), "max_over_mean": float(busy.max() / busy.mean()),
            "mean_busy_us": float(busy.mean() / 1e3), "max_busy_us": float(busy.max() / 1e3),
            "min_busy_us": float(busy.min() / 1e3), "launch_span_us": span / 1e3,
            "what": "per-CTA busy time of the persistent fine stage in the last timed step (globaltimer)"}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    q, k, v = make_inputs(wl)
    per_step = max(0.5, 150.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(wl, q, k, v, min(per_step, 2.0), seed=1)
    secs, res = [], None
    for s in range(args.steps):
        res = oracle_sample(wl, q, k, v, per_step, seed=100 + s)
        secs.append(res["est_s"])
    ms = 1000.0 * statistics.mean(secs)
    value = res["flops"] / (ms / 1000.0) / 1e12
    desc, cores = res["desc"], res["threads"]
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "ms_per_step_is": "an estimate: each step times the oracle on a bounded sample of the workload "
                              "(about %.1f s of CPU work) and scales it to the whole workload" % per_step,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, args, int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": dict(cpu_baseline_of(res), value=value),
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
SECONDARY = "wan720p_hilbert_rope"


def run_secondary(args, dev, name: str = SECONDARY, steps: int = 5, warmup: int = 3) -> dict:
    """The forward on a second workload (720p, 3D Hilbert order, RoPE applied in
    the loads), device-timed like the main line: its own stage times, the
    fine kernel's roofline, the CTA load balance and the workspace it needs."""
    import torch
    from block_sparse_spatiotemporal_b200 import fvattn as F
    wl = WORKLOADS[name]
    q, k, v = make_inputs(wl)
    as_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    qd, kd, vd = as_dev(q), as_dev(k), as_dev(v)
    del q, k, v
    shape = F.make_shape(wl.batch, wl.heads, wl.head_dim, wl.grid, dtype=F.BF16,
                         order=F.HILBERT if wl.order == "hilbert" else F.RASTER_CUBE)
    rope = F.make_rope(wl.rope_dims, wl.rope_base) if wl.rope else None
    ws = F.workspace(shape, rope, device=dev)
    cache, counts, idx = F.new_cache(shape, device=dev)
    out = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:-1], dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        F.forward(shape, qd, kd, vd, ws, wl.top_p, wl.k_min, rope=rope, cache=cache, out=out, lse=lse)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    if F.device_status(ws) != 0:
        raise RuntimeError("device status set during the second workload's warm-up")
    pairs = int(counts.sum().item())
    flops_step = pairs * pair_flops(wl.head_dim)
    F.profile_read()
    F.profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    F.profile_enable(False)
    stages = F.profile_read()
    imbalance = sm_imbalance(F, shape, ws, rope)
    if F.device_status(ws) != 0:
        raise RuntimeError("device status set during the second workload's timed steps")
    ms = e0.elapsed_time(e1) / steps
    pk, pk_kind = peaks()
    fine_ms, fine_n = stages["fine"]
    achieved = flops_step / (fine_ms / max(fine_n, 1) / 1e3) / 1e12
    return {"workload": wl.name, "config": workload_config(wl, args), "steps": steps, "warmup": warmup,
            "ms_per_step": ms, "value": flops_step / (ms / 1e3) / 1e12, "unit": UNIT,
            "selected_pairs": pairs, "density": pairs / (wl.heads * wl.num_tiles ** 2),
            "stage_ms": {n: round(v[0] / steps, 4) for n, v in stages.items() if v[1]},
            "roofline": {"kernel": "fine_tc_kernel", "bound": "tensor", "achieved": achieved,
                         "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                         "peak_source": f"{pk_kind} bf16 burst"},
            "sm_imbalance": imbalance, "gpu_launches": sum(n for _, n in stages.values()),
            "workspace_mib": F.workspace_size(shape, rope) / 2 ** 20}

def max_over_ranks(ms: float, device, world: int) -> float:
    """The slowest rank's time: every rank takes part (a collective), so the
    job's time is the max.  A single rank returns its own time."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world: int, units_per_rank: float, ms_max: float) -> float:
    """Weak scaling: every rank processes the same units; value = all ranks'
    units / the slowest rank's time (per second), in 1e12 units."""
    return world * units_per_rank / (ms_max / 1e3) / 1e12


def run_gpu(args, wl):
    import torch
    import torch.distributed as dist
    from block_sparse_spatiotemporal_b200 import fvattn as F

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    q, k, v = make_inputs(wl)
    as_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    qd, kd, vd = as_dev(q), as_dev(k), as_dev(v)
    shape = F.make_shape(wl.batch, wl.heads, wl.head_dim, wl.grid, dtype=F.BF16,
                         order=F.HILBERT if wl.order == "hilbert" else F.RASTER_CUBE)
    rope = F.make_rope(wl.rope_dims, wl.rope_base) if wl.rope else None
    ws = F.workspace(shape, rope, device=dev, subblock=args.subblock)
    cache, counts, idx = F.new_cache(shape, device=dev)
    out = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:-1], dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(qx=qd, kx=kd, vx=vd, o=None):
        o = out if o is None else o
        if args.subblock:   # sub-block scoring, then the fine stage on its lists
            F.pool_select_subblock(shape, qx, kx, ws, wl.top_p, wl.k_min, rope=rope, blocks=(counts, idx, cache.blocks))
            F.block_sparse_fwd(shape, qx, kx, vx, counts, idx, ws, rope=rope, out=o, lse=lse)
        else:
            F.forward(shape, qx, kx, vx, ws, wl.top_p, wl.k_min, rope=rope, cache=cache, out=o, lse=lse)

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize(dev)
    if F.device_status(ws) != 0:
        raise RuntimeError("device status set during warm-up")
    pairs = int(counts.sum().item())
    flops_step = pairs * pair_flops(wl.head_dim)

    # ---- timed region (device time, CUDA events on the launch stream)
    sampler = ClockSampler(range(world)) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    F.profile_read()
    F.profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    F.profile_enable(False)
    stages = F.profile_read()
    imbalance = None if args.subblock else sm_imbalance(F, shape, ws, rope)
    clocks = sampler.stop() if sampler else None
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1) / args.steps
    if F.device_status(ws) != 0:
        raise RuntimeError("device status set during the timed region")
    ms_max = max_over_ranks(ms, dev, world)

    # ---- end to end through the public API: pinned host in, host out.  A
    # serving loop's pipeline: step i's inputs go up on one copy stream while
    # step i-1 computes and step i-2's output comes down on another (PCIe is
    # full duplex); device inputs and outputs are double-buffered, and events
    # keep a buffer from being refilled before the step reading it is done.
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in (q, k, v))
        ohs = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        ins = [(torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)) for _ in range(2)]
        outs = [torch.empty_like(out) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

        def pipelined(n):
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(s_in)
            for i in range(n):
                b = i % 2
                if i >= 2:
                    s_in.wait_event(ev_comp[b])       # step i-2 has read ins[b]
                with torch.cuda.stream(s_in):
                    for dst, src in zip(ins[b], (qh, kh, vh)):
                        dst.copy_(src, non_blocking=True)
                ev_in[b].record(s_in)
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])      # step i-2's output has left outs[b]
                step(*ins[b], o=outs[b])
                ev_comp[b].record(stream)
                s_out.wait_event(ev_comp[b])
                with torch.cuda.stream(s_out):
                    ohs[b].copy_(outs[b], non_blocking=True)
                ev_out[b].record(s_out)
            t1.record(s_out)
            return t0, t1

        pipelined(3)
        torch.cuda.synchronize(dev)
        n_e2e = max(3, min(args.steps, 20))
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        s0, s1 = pipelined(n_e2e)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(s0.elapsed_time(s1) / n_e2e, dev, world)
        h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh))
        d2h = ohs[0].numel() * ohs[0].element_size()
        e2e = {"value": whole_job_value(world, flops_step, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipeline": "inputs of step i up (copy stream) while step i-1 computes and step i-2's output "
                           "comes down (second copy stream); double-buffered device inputs and outputs"}
        del ins, outs

    # ---- the tile reorder as its own pass (the forward folds it into its loads): q, k, v to
    # tiled layout and out back, 2 bytes moved per byte
    tmp = torch.empty_like(qd)
    for _ in range(2):
        F.tile_reorder(shape, qd, ws, out=tmp)
    torch.cuda.synchronize(dev)
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_reo = 5
    r0.record(stream)
    for _ in range(n_reo):
        for x in (qd, kd, vd):
            F.tile_reorder(shape, x, ws, out=tmp)
        F.tile_reorder(shape, out, ws, inverse=True, out=tmp)
    r1.record(stream)
    torch.cuda.synchronize(dev)
    reorder_ms = r0.elapsed_time(r1) / n_reo
    reorder_bytes = 4 * 2 * qd.numel() * qd.element_size()
    del tmp

    if rank == 0:
        pk, pk_kind = peaks()
        fine_ms, fine_n = stages["fine"]
        fine_avg = fine_ms / max(fine_n, 1)
        achieved = flops_step / (fine_avg / 1e3) / 1e12
        peak = pk["bf16_tflops"]
        traffic = profiled_traffic(wl.name)
        stage_ms = {name: round(v[0] / max(args.steps, 1), 4) for name, v in stages.items() if v[1]}
        pool_select_ms = (stages["pool"][0] + stages["select"][0]) / args.steps
        qk_bytes = 2 * wl.heads * wl.tokens * wl.head_dim * 2
        line = {
            "metric": METRIC,
            "value": whole_job_value(world, flops_step, ms_max),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_max,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(wl, args, world),
            "selected_pairs": pairs,
            "density": pairs / (wl.heads * wl.num_tiles ** 2),
            "stage_ms": stage_ms,
            "pool_select": {"ms": pool_select_ms, "gbs": qk_bytes / (pool_select_ms / 1e3) / 1e9,
                            "frac_of_hbm": qk_bytes / (pool_select_ms / 1e3) / 1e9 / pk["hbm_gbs"]},
            "reorder": {"ms": reorder_ms, "gbs": reorder_bytes / (reorder_ms / 1e3) / 1e9,
                        "frac_of_hbm": reorder_bytes / (reorder_ms / 1e3) / 1e9 / pk["hbm_gbs"],
                        "note": "q, k, v to tiled and out back; not part of the forward, which gathers tiles "
                                "in its loads"},
            "roofline": {"kernel": "fine_tc_kernel", "bound": "tensor", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{pk_kind} bf16 burst",
                         "peak_sustained": pk.get("bf16_tflops_sustained"),
                         "frac_sustained": achieved / pk["bf16_tflops_sustained"]
                         if pk.get("bf16_tflops_sustained") else None},
            "gpu_launches": sum(n for _, n in stages.values()),
            "sm_imbalance": imbalance,
            "clocks": clocks,
            "e2e": e2e,
        }
        if world == 1 and not args.no_secondary and not args.subblock and wl.name != SECONDARY:
            line["secondary"] = run_secondary(args, dev)
        if world == 1 and not args.no_cpu_baseline:
            # the oracle leg: its coarse stage runs on every head and checks the GPU's lists row by row
            lists = None if args.subblock else (counts.cpu().numpy(), idx.cpu().numpy())
            res = oracle_sample(wl, q, k, v, budget_s=args.cpu_budget, gpu_lists=lists)
            line["cpu_baseline"] = cpu_baseline_of(res)
            line["cpu_baseline"]["tiny_single_core"] = oracle_tiny_single_core()
            if res["parity"] is not None:
                line["parity"] = dict(res["parity"], what="block lists of the timed forward vs the oracle, every "
                                      "row of every head; borderline / near-tie rows that differ must be valid "
                                      "lists")
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_sweep(args):
    """The 480p sweep (seed 4): at every (top_p, k_min) point -- top-p 0.5 ..
    1.0 with k_min 8 and fixed top-k 8 / 32 / 128 -- the forward's ms,
    effective TFLOP/s and density, the informational error of its output
    against the dense output (top_p = 1) of the same inputs, and cached-mask
    mode: the point's step-0 lists reused on the ten perturbed steps
    (Q, K += 0.05 N(0,1) per step, V fixed), each step timed.  One JSON line."""
    import torch
    from block_sparse_spatiotemporal_b200 import fvattn as F
    from block_sparse_spatiotemporal_b200.inputs import perturb_steps, sweep_points

    wl = WORKLOADS["wan480p_sweep"]
    dev = torch.device("cuda", 0)
    q, k, v, masters = make_inputs(wl, keep_f32_masters=True)
    as_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    qd, kd, vd = as_dev(q), as_dev(k), as_dev(v)
    perturbed = [(as_dev(qt), as_dev(kt)) for qt, kt in perturb_steps(wl, masters)]
    shape = F.make_shape(wl.batch, wl.heads, wl.head_dim, wl.grid, dtype=F.BF16)
    ws = F.workspace(shape, device=dev)
    cache, counts, _ = F.new_cache(shape, device=dev)
    out = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:-1], dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    F.forward(shape, qd, kd, vd, ws, 1.0, 1, cache=cache, out=out, lse=lse)
    dense = out.float().clone()
    fl = pair_flops(wl.head_dim)
    total = wl.heads * wl.num_tiles ** 2

    def timed(fn, n):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        F.profile_read()
        F.profile_enable(True)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        F.profile_enable(False)
        st = F.profile_read()
        if F.device_status(ws) != 0:
            raise RuntimeError("device status set in the sweep")
        return e0.elapsed_time(e1) / n, st["fine"][0] / max(st["fine"][1], 1)

    points = []
    for top_p, k_min in sweep_points():
        ms, fine = timed(lambda: F.forward(shape, qd, kd, vd, ws, top_p, k_min, cache=cache, out=out, lse=lse),
                         args.steps)
        pairs = int(counts.sum().item())      # the cache holds this point's step-0 lists
        err = (out.float() - dense).abs()
        cached_ms = []
        for qx, kx in perturbed:
            cms, _ = timed(lambda: F.forward(shape, qx, kx, vd, ws, top_p, k_min, cache=cache, reuse_mask=True,
                                             out=out, lse=lse), max(3, args.steps // 4))
            cached_ms.append(cms)
        points.append({"top_p": top_p, "k_min": k_min, "ms": ms, "fine_ms": fine,
                       "tflops": pairs * fl / (ms / 1e3) / 1e12, "fine_tflops": pairs * fl / (fine / 1e3) / 1e12,
                       "density": pairs / total, "selected_pairs": pairs,
                       "err_vs_dense": {"max_abs": float(err.max().item()), "mean_abs": float(err.mean().item())},
                       "cached_mask": {"steps": len(cached_ms), "ms_per_step": cached_ms,
                                       "ms_mean": statistics.mean(cached_ms),
                                       "tflops_mean": pairs * fl / (statistics.mean(cached_ms) / 1e3) / 1e12}})
    line = {"metric": METRIC, "unit": UNIT, "workload": wl.name, "steps": args.steps, "warmup": args.warmup,
            "dtype": "bf16", "data": "synthetic",
            "dense_reference": "the forward at top_p = 1 (every key tile) on the same step-0 inputs",
            "sweep": points}
    print(json.dumps(line), flush=True)
    return 0


def run_prologue(args, wl):
    """The attention prologue at the workload's shape: X [1, N, C = H*d] and a
    linear layer W [3*H*d, C] (+ bias) projected to Q, K, V with the 3D RoPE
    on Q and K, written in the workload's tiled order.  One JSON line; cuBLAS
    time of the bare X W^T product (no bias, rotation or reorder) beside it."""
    import torch
    from block_sparse_spatiotemporal_b200 import fvattn as F
    from block_sparse_spatiotemporal_b200.inputs import make_projection_inputs

    dev = torch.device("cuda", 0)
    B, N, H, d = wl.batch, wl.tokens, wl.heads, wl.head_dim
    C = H * d
    x, w, b = make_projection_inputs(B, N, C, H, d, wl.seed)
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
    wd = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).to(dev)
    bd = torch.from_numpy(b).to(dev)
    shape = F.make_shape(B, H, d, wl.grid, dtype=F.BF16,
                         order=F.HILBERT if wl.order == "hilbert" else F.RASTER_CUBE, layout=F.TILED)
    rope = F.make_rope(wl.rope_dims, wl.rope_base)
    ws = torch.empty(F.workspace_size_qkv(shape, rope), dtype=torch.uint8, device=dev)
    out = tuple(torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev) for _ in range(3))
    stream = torch.cuda.current_stream(dev)
    flops = 2.0 * B * N * C * 3 * H * d

    def step(xx=xd):
        F.qkv_rope(shape, xx, wd, ws, bias=bd, rope=rope, t_offset=0, out=out)

    def timed(fn, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if F.device_status(ws) != 0:
        raise RuntimeError("device status set during warm-up")
    sampler = ClockSampler([0])
    sampler.start()
    time.sleep(0.3)
    F.profile_read()
    F.profile_enable(True)
    ms = timed(step, args.steps)
    F.profile_enable(False)
    stages = F.profile_read()
    clocks = sampler.stop()
    if F.device_status(ws) != 0:
        raise RuntimeError("device status set during the timed region")
    k_ms, k_n = stages["prologue"]
    kernel_ms = k_ms / max(k_n, 1)

    x2 = xd.view(B * N, C)
    for _ in range(3):
        torch.matmul(x2, wd.t())
    cublas_ms = timed(lambda: torch.matmul(x2, wd.t()), max(3, min(args.steps, 20)))

    # end to end: pinned host X in, q, k, v back to pinned host buffers
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    oh = tuple(torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory() for _ in range(3))
    xb = torch.empty_like(xd)

    def e2e_step():
        xb.copy_(xh, non_blocking=True)
        step(xb)
        for o, hst in zip(out, oh):
            hst.copy_(o, non_blocking=True)
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    e2e_ms = timed(e2e_step, max(3, min(args.steps, 10)))

    pk, pk_kind = peaks()
    achieved = flops / (kernel_ms / 1e3) / 1e12
    line = {
        "metric": "QKV projection + 3D RoPE prologue ms & TFLOP/s", "value": flops / (ms / 1e3) / 1e12,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"prologue_{wl.name}", "grid": list(wl.grid), "tokens": N, "channels": C,
                   "heads": H, "head_dim": d, "order": wl.order, "rope": list(wl.rope_dims), "bias": True,
                   "layout": "tiled", "l2": "inputs larger than L2 (X = %.0f MB, W = %.0f MB)"
                   % (xd.numel() * 2 / 1e6, wd.numel() * 2 / 1e6)},
        "stage_ms": {k: round(v[0] / args.steps, 4) for k, v in stages.items() if v[1]},
        "roofline": {"kernel": "qkv_rope_kernel", "bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"], "traffic": None,
                     "peak_source": f"{pk_kind} bf16 burst"},
        "cublas_gemm": {"ms": cublas_ms, "tflops": flops / (cublas_ms / 1e3) / 1e12,
                        "note": "torch.matmul(X, W^T) alone: no bias, rotation or tiled scatter"},
        "gpu_launches": sum(n for _, n in stages.values()),
        "clocks": clocks,
        "e2e": {"value": flops / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": xh.numel() * 2, "d2h_bytes_per_step": sum(o.numel() * 2 for o in oh)},
    }
    if not args.no_cpu_baseline:
        from oracle import fvattn_oracle as O
        rng = np.random.default_rng(0)
        orope = dict(dims=wl.rope_dims, base=wl.rope_base)
        n_tok, t0 = 0, time.perf_counter()
        wf, bf = O.as_f64(w, "bf16"), b.astype(np.float64)
        while time.perf_counter() - t0 < args.cpu_budget / 2 or n_tok == 0:
            toks = np.sort(rng.choice(N, 64, replace=False))
            O.qkv_rope(O.as_f64(x[:, toks], "bf16"), wf, bf, wl.grid, H, d, orope, tokens=toks, gathered=True)
            n_tok += 64
        el = time.perf_counter() - t0
        est = el * (B * N) / n_tok
        line["cpu_baseline"] = {"value": flops / est / 1e12, "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
                                "sample": f"oracle (numpy fp64) prologue of {n_tok} random tokens, scaled to "
                                          f"{B * N} tokens", "est_ms_per_step": est * 1e3}
    print(json.dumps(line), flush=True)
    return 0


def run_backward(args, wl):
    """The fine-stage backward at the workload's shape: lists from the
    library's own selection, out / lse from its forward, a seeded dout, all
    in the tiled layout; one step = one fvattn_block_sparse_bwd call (both
    schedules, D, the dK/dV and dQ kernels).  Effective FLOP/s counts the five
    products of the gradient, 5 * 2 * 64 * 64 * d per selected pair."""
    import torch
    from block_sparse_spatiotemporal_b200 import fvattn as F
    from block_sparse_spatiotemporal_b200.inputs import f32_to_bf16_bits

    dev = torch.device("cuda", 0)
    B, H, N, d = wl.batch, wl.heads, wl.tokens, wl.head_dim
    q, k, v = make_inputs(wl)
    g = f32_to_bf16_bits(np.random.default_rng(wl.seed + 77).standard_normal((B, H, N, d), dtype=np.float32))
    as_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    order = F.HILBERT if wl.order == "hilbert" else F.RASTER_CUBE
    nat = F.make_shape(B, H, d, wl.grid, dtype=F.BF16, order=order, layout=F.NATURAL)
    shape = F.make_shape(B, H, d, wl.grid, dtype=F.BF16, order=order, layout=F.TILED)
    rope = F.make_rope(wl.rope_dims, wl.rope_base) if wl.rope else None
    ws = torch.empty(max(F.workspace_size(shape, rope), F.workspace_size_bwd(shape)), dtype=torch.uint8, device=dev)
    qt, kt, vt = (F.tile_reorder(nat, as_dev(x), ws) for x in (q, k, v))
    gd = as_dev(g)
    counts, idx = F.pool_select(shape, qt, kt, ws, wl.top_p, wl.k_min, rope=rope)
    if rope is not None:   # the backward takes the rotated q, k the fine stage consumed
        raise SystemExit("--backward takes workloads without RoPE")
    out, lse = F.block_sparse_fwd(shape, qt, kt, vt, counts, idx, ws)
    grads = tuple(torch.empty_like(qt) for _ in range(3))
    stream = torch.cuda.current_stream(dev)
    pairs = int(counts.sum().item())
    flops = 5.0 * 2 * 64 * 64 * d * pairs

    def step():
        F.block_sparse_bwd(shape, qt, kt, vt, out, gd, lse, counts, idx, ws, grads=grads)

    def timed(fn, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if F.device_status(ws) != 0:
        raise RuntimeError("device status set during warm-up")
    sampler = ClockSampler([0])
    sampler.start()
    time.sleep(0.3)
    F.profile_read()
    F.profile_enable(True)
    ms = timed(step, args.steps)
    F.profile_enable(False)
    stages = F.profile_read()
    clocks = sampler.stop()
    if F.device_status(ws) != 0:
        raise RuntimeError("device status set during the timed region")
    per = {k: v[0] / max(v[1], 1) for k, v in stages.items() if v[1]}
    kv_ms, q_ms = per["bwd_kv"], per["bwd_q"]
    unit_flop = 2.0 * 64 * 64 * d * pairs           # one 64x64xd product per selected pair
    pk, pk_kind = peaks()
    kv_ach = 4 * unit_flop / (kv_ms / 1e3) / 1e12   # S^T, dP^T, dV, dK
    q_ach = 3 * unit_flop / (q_ms / 1e3) / 1e12     # S, dP, dQ

    # end to end: q, k, v, out, dout, lse and the lists from pinned host, dq, dk, dv back
    hosts = [x.cpu().pin_memory() for x in (qt, kt, vt, out, gd, lse, counts, idx)]
    devs = [torch.empty_like(x) for x in (qt, kt, vt, out, gd, lse, counts, idx)]
    ghost = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in grads]

    def e2e_step():
        for hst, dv_ in zip(hosts, devs):
            dv_.copy_(hst, non_blocking=True)
        F.block_sparse_bwd(shape, *devs[:6], devs[6], devs[7], ws, grads=grads)
        for gr, hst in zip(grads, ghost):
            hst.copy_(gr, non_blocking=True)
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    e2e_ms = timed(e2e_step, max(3, min(args.steps, 10)))
    big = kv_ms >= q_ms
    line = {
        "metric": "fine-stage backward ms & effective TFLOP/s", "value": flops / (ms / 1e3) / 1e12,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"backward_{wl.name}", "grid": list(wl.grid), "tokens": N, "heads": H, "head_dim": d,
                   "top_p": wl.top_p, "k_min": wl.k_min, "order": wl.order, "layout": "tiled",
                   "selected_pairs": pairs, "density": pairs / (H * wl.num_tiles ** 2),
                   "l2": "inputs larger than L2 (q, k, v, out, dout = %.0f MB)" % (5 * qt.numel() * 2 / 1e6)},
        "stage_ms": {k: round(v[0] / args.steps, 4) for k, v in stages.items() if v[1]},
        "kernels": {"bwd_kv": {"ms": kv_ms, "tflops": kv_ach, "products_per_pair": 4},
                    "bwd_q": {"ms": q_ms, "tflops": q_ach, "products_per_pair": 3}},
        "roofline": {"kernel": "bwd_tc_kernel<true>" if big else "bwd_tc_kernel<false>", "bound": "tensor",
                     "achieved": kv_ach if big else q_ach, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": (kv_ach if big else q_ach) / pk["bf16_tflops"], "traffic": None,
                     "peak_source": f"{pk_kind} bf16 burst"},
        "gpu_launches": sum(n for _, n in stages.values()),
        "clocks": clocks,
        "e2e": {"value": flops / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in hosts),
                "d2h_bytes_per_step": sum(x.numel() * x.element_size() for x in ghost)},
    }
    if not args.no_cpu_baseline:
        from oracle import fvattn_oracle as O
        rng = np.random.default_rng(0)
        ch, ih = counts.cpu().numpy()[0], idx.cpu().numpy()[0]
        pos = O.positions(wl.grid, wl.order)
        t0 = time.perf_counter()
        done, rows, cache = 0, 0, {}
        scale = O.default_scale(d)
        while time.perf_counter() - t0 < args.cpu_budget or rows == 0:
            h = int(rng.integers(H))
            i = int(rng.integers(wl.num_tiles))
            if h not in cache:   # the head in tiled order (dout is drawn tiled)
                cache = {h: [O.to_tiled(O.as_f64(x[0, h], "bf16"), pos) for x in (q, k, v)]
                         + [O.as_f64(g[0, h], "bf16")]}
            qh, kh, vh, gh = cache[h]
            sl = slice(64 * i, 64 * i + 64)
            O.fine_tile_backward(qh[sl], kh, vh, gh[sl], ih[h, i, :ch[h, i]], scale)
            done += int(ch[h, i])
            rows += 1
        el = time.perf_counter() - t0
        est = el * pairs / max(done, 1)
        line["cpu_baseline"] = {"value": flops / est / 1e12, "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
                                "sample": f"oracle (numpy fp64) backward of {rows} random (head, query tile) rows "
                                          f"({done} selected pairs), scaled by selected pairs",
                                "est_ms_per_step": est * 1e3}
    print(json.dumps(line), flush=True)
    return 0


def run_augment(args, wl):
    """Slack-aware augmentation at the workload's shape: the plain path
    (selection, schedule, fine stage) against selection, augmentation to one
    CTA per SM and the fine stage on the kept work list; then the kept work
    list on the plain lists ("kept"), whose last step's per-CTA busy times
    size a second augmentation ("measured": slack = measured idle time, at
    --fill percent); one JSON line with every arm's times, the selected pairs
    and the fine-stage times."""
    import torch
    from block_sparse_spatiotemporal_b200 import fvattn as F

    dev = torch.device("cuda", 0)
    q, k, v = make_inputs(wl)
    as_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)  # noqa: E731
    qd, kd, vd = as_dev(q), as_dev(k), as_dev(v)
    shape = F.make_shape(wl.batch, wl.heads, wl.head_dim, wl.grid, dtype=F.BF16,
                         order=F.HILBERT if wl.order == "hilbert" else F.RASTER_CUBE)
    rope = F.make_rope(wl.rope_dims, wl.rope_base) if wl.rope else None
    ws = F.workspace(shape, rope, device=dev)
    G = torch.cuda.get_device_properties(dev).multi_processor_count
    base = F.new_blocks(shape, dev)
    aug = F.new_blocks(shape, dev)
    out = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:-1], dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def plain():
        F.pool_select(shape, qd, kd, ws, wl.top_p, wl.k_min, rope=rope, blocks=base)
        F.block_sparse_fwd(shape, qd, kd, vd, base[0], base[1], ws, rope=rope, out=out, lse=lse)

    def augmented():
        F.pool_select(shape, qd, kd, ws, wl.top_p, wl.k_min, rope=rope, blocks=base)
        _, _, wlist = F.augment_lists(shape, qd, kd, ws, base[0], base[1], num_ctas=G, rope=rope,
                                      out=(aug[0], aug[1]))
        F.block_sparse_fwd_worklist(shape, qd, kd, vd, aug[0], aug[1], wlist, ws, num_ctas=G, rope=rope,
                                    out=out, lse=lse)

    wkept = None      # the kept work list of the plain lists, built before the "kept" arm
    meas = F.new_blocks(shape, dev)
    busy_ns = []

    def kept():
        F.pool_select(shape, qd, kd, ws, wl.top_p, wl.k_min, rope=rope, blocks=base)
        F.block_sparse_fwd_worklist(shape, qd, kd, vd, base[0], base[1], wkept, ws, num_ctas=G, rope=rope,
                                    out=out, lse=lse)

    def measured():
        F.pool_select(shape, qd, kd, ws, wl.top_p, wl.k_min, rope=rope, blocks=base)
        _, _, wlist = F.augment_lists(shape, qd, kd, ws, base[0], base[1], num_ctas=G, rope=rope,
                                      out=(meas[0], meas[1]), cta_busy_ns=busy_ns, fill_percent=args.fill)
        F.block_sparse_fwd_worklist(shape, qd, kd, vd, meas[0], meas[1], wlist, ws, num_ctas=G, rope=rope,
                                    out=out, lse=lse)

    # the arms alternate step by step (clock and thermal drift fall on all of
    # them alike); "measured" always follows "kept" and takes its slack from
    # that step's per-CTA busy times, as a diffusion step would from the last
    arms = (("plain", plain), ("augmented", augmented), ("kept", kept), ("measured", measured))
    F.pool_select(shape, qd, kd, ws, wl.top_p, wl.k_min, rope=rope, blocks=base)
    wkept = F.build_worklist(shape, base[0], base[1], ws)   # the selection is deterministic: same lists each step
    acc = {name: {"ms": 0.0, "fine": 0.0, "stages": {}} for name, _ in arms}
    imb = {}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for step in range(args.warmup + args.steps):
        for name, fn in arms:
            if name == "measured":
                t = F.profile_cta_times(shape, ws, rope)   # the "kept" step just run
                busy_ns[:] = (t[:, 1] - t[:, 0]).tolist()
            torch.cuda.synchronize(dev)
            F.profile_read()
            F.profile_enable(True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            F.profile_enable(False)
            st = F.profile_read()
            if step >= args.warmup:
                a = acc[name]
                a["ms"] += e0.elapsed_time(e1)
                a["fine"] += st["fine"][0]
                for k2, v2 in st.items():
                    if v2[1]:
                        a["stages"][k2] = a["stages"].get(k2, 0.0) + v2[0]
                imb[name] = sm_imbalance(F, shape, ws, rope)
    if F.device_status(ws) != 0:
        raise RuntimeError("device status set")
    res = {name: {"ms": a["ms"] / args.steps, "fine_ms": a["fine"] / args.steps,
                  "stage_ms": {k2: round(v2 / args.steps, 4) for k2, v2 in a["stages"].items()},
                  "sm_imbalance": imb[name]} for name, a in acc.items()}
    pairs = int(base[0].sum().item())
    apairs = int(aug[0].sum().item())
    mpairs = int(meas[0].sum().item())
    fl = pair_flops(wl.head_dim)
    line = {"metric": "slack-aware augmentation: sparse-attn fwd ms & effective TFLOP/s", "unit": UNIT,
            "value": apairs * fl / (res["augmented"]["ms"] / 1e3) / 1e12, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["augmented"]["ms"], "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"augment_{wl.name}", "grid": list(wl.grid), "heads": wl.heads,
                       "top_p": wl.top_p, "k_min": wl.k_min, "ctas": G},
            "selected_pairs": {"plain": pairs, "augmented": apairs, "added": apairs - pairs,
                               "measured": mpairs, "added_measured": mpairs - pairs},
            "plain": res["plain"], "augmented": res["augmented"], "kept": res["kept"],
            "measured": dict(res["measured"], fill_percent=args.fill,
                             extra_fine_vs_kept=res["measured"]["fine_ms"] / res["kept"]["fine_ms"] - 1.0,
                             added_pairs_frac=(mpairs - pairs) / pairs),
            "fine_tflops": {"plain": pairs * fl / (res["plain"]["fine_ms"] / 1e3) / 1e12,
                            "augmented": apairs * fl / (res["augmented"]["fine_ms"] / 1e3) / 1e12,
                            "kept": pairs * fl / (res["kept"]["fine_ms"] / 1e3) / 1e12,
                            "measured": mpairs * fl / (res["measured"]["fine_ms"] / 1e3) / 1e12}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("fvattn", "reference"), default="fvattn")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="wan480p")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the 720p Hilbert + RoPE forward the single-GPU line also reports")
    ap.add_argument("--sweep", action="store_true", help="the 480p top-p / top-k / cached-mask sweep (one JSON line)")
    ap.add_argument("--subblock", action="store_true",
                    help="hierarchical sub-block scoring (pool_select_subblock + block_sparse_fwd)")
    ap.add_argument("--prologue", action="store_true",
                    help="the fused QKV projection + 3D RoPE prologue at the workload's shape (one JSON line)")
    ap.add_argument("--backward", action="store_true",
                    help="the fine-stage backward (dq, dk, dv) at the workload's shape (one JSON line)")
    ap.add_argument("--augment", action="store_true",
                    help="slack-aware augmentation against the plain path at the workload's shape (one JSON line)")
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--fill", type=int, default=50,
                    help="--augment: percent of the measured idle time the measured-slack arm fills")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.workload]
    if args.sweep:
        return run_sweep(args)
    if args.prologue:
        return run_prologue(args, wl)
    if args.backward:
        return run_backward(args, wl)
    if args.augment:
        return run_augment(args, wl)
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_gpu(args, wl)


if __name__ == "__main__":
    sys.exit(main())
