#!/usr/bin/env python
"""Benchmark of the Prism sparse video self-attention layer (fwd + bwd) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2k] [--dense]
    python bench.py --impl reference      # the fp64 CPU oracle on a bounded sample
    python bench.py --forward-only        # inference: the forward stages, no backward state
    python bench.py --bwd-ds              # backward with the dS handoff (no e2e figure)

One step = one pass of the whole hot path over the configured synthetic layer:
zone indicator -> shapes/permutation -> permute Q,K,V -> pooled block
probabilities -> hybrid selection -> sparse attention forward -> unpermute O ->
permute dO -> sparse attention backward -> unpermute dQ, dK, dV.
``value`` is TFLOP/s on the selected blocks (algorithmic FLOPs 3.5 * F_fwd,
F_fwd = 4 d sum_h sum_i sum_{j in S_i} |B_i||B_j|) over the device time of the
sparse attention forward + backward calls, summed over ranks (each rank runs
its own layer: weak scaling, no data-path collective).  Prints one JSON line
on rank 0.  With --forward-only a step ends at the unpermuted O, the layer holds
no backward buffers, and ``value`` is F_fwd over the forward call's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dynamic_block_sparse_macro_b200 import inputs  # noqa: E402
from dynamic_block_sparse_macro_b200.configs import get_config  # noqa: E402

METRIC = "sparse attn fwd+bwd ms/layer & TFLOP/s on selected blocks, 2K grid (295k tok)"
METRIC_FWD = "sparse attn fwd ms/layer & TFLOP/s on selected blocks, 2K grid (295k tok), inference"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) of one backward call, by (config, heads), from an ncu capture of
# the backward kernels (profiles/attn_kernels_2k_4heads.md: 4 heads scaled by 6, plus the
# Delta kernel's algorithmic 5.5 GB)
BWD_DRAM_BYTES = {("2k", 24): 33.2e9}


def metric_name(cfg, fwd_only):
    """The headline metric names the 2K grid; other grids get the same metric on their own size."""
    m = METRIC_FWD if fwd_only else METRIC
    if cfg.name != "2k":
        m = m.replace("2K grid (295k tok)", f"{cfg.name} grid {cfg.T}x{cfg.H}x{cfg.W} ({cfg.n_tokens / 1e3:.0f}k tok)")
    return m


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.t = None
        self.t0 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()
        # the first sample must precede the timed region: a short region would otherwise end
        # before nvidia-smi prints anything
        t_end = time.monotonic() + 5.0
        while not self.lines and time.monotonic() < t_end and self.proc.poll() is None:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def mark(self):
        """Start of the timed region: samples before it only stand in when none falls inside."""
        self.t0 = time.monotonic()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        # a region shorter than the 200 ms period: take the first sample after it (the clocks
        # right after the load) rather than the idle one before it
        t_end = time.monotonic() + 1.0
        while (self.t0 is not None and not any(t >= self.t0 for t, _ in self.lines)
               and time.monotonic() < t_end):
            time.sleep(0.01)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        inside = [ln for t, ln in self.lines if self.t0 is None or t >= self.t0]
        n_inside = len(inside)
        for ln in inside:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "samples_from_region_start": n_inside}


# ---------------------------------------------------------------- helpers
# ---------------------------------------------------------------- ranks
def max_over_ranks(values, device):
    """Element-wise max of per-rank timings over all ranks (identity with one rank).

    Every rank must call it at the same point (it is a collective)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return [float(v) for v in values]
    if torch.distributed.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_tflops(world, flops_per_rank, ms):
    """Whole-job throughput: every rank runs one replica of the layer in `ms` (the max over ranks)."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def unpack_sel_dev(words: torch.Tensor, nb: int) -> torch.Tensor:
    """[h, MB, SW] int32 bitmask -> bool [h, nb, nb] on the device."""
    w = words[:, :nb, :].to(torch.int64) & 0xFFFFFFFF
    sh = torch.arange(32, device=words.device, dtype=torch.int64)
    b = ((w.unsqueeze(-1) >> sh) & 1).reshape(w.shape[0], nb, -1)
    return b[..., :nb].bool()


def _popcount_rows(words: torch.Tensor) -> torch.Tensor:
    """Set bits per row of an int32 [..., SW] bitmask (int64)."""
    w = words.to(torch.int64) & 0xFFFFFFFF
    cnt = torch.zeros(w.shape[:-1], dtype=torch.int64, device=w.device)
    for s in range(32):
        cnt += ((w >> s) & 1).sum(-1)
    return cnt


def selected_flops(mod, rows_per_chunk=1024) -> dict:
    """F_fwd = 4 d sum_h sum_i |B_i| sum_{j in S_i} |B_j| and density figures.

    Works one head and a bounded chunk of selection rows at a time, so that it
    fits beside the layer at every grid size."""
    nb = mod.num_blocks()
    bs = mod.blk_start[: nb + 1].to(torch.int64)
    sz = (bs[1:] - bs[:-1]).to(torch.float64)
    keys_per_row = torch.empty((mod.heads, nb), dtype=torch.float64, device=sz.device)
    n_sel = torch.empty((mod.heads, nb), dtype=torch.float64, device=sz.device)
    for hh in range(mod.heads):
        for r0 in range(0, nb, rows_per_chunk):
            r1 = min(nb, r0 + rows_per_chunk)
            w = mod.sel[hh, r0:r1].to(torch.int64) & 0xFFFFFFFF
            sh = torch.arange(32, device=w.device, dtype=torch.int64)
            bits = ((w.unsqueeze(-1) >> sh) & 1).reshape(r1 - r0, -1)[:, :nb].to(torch.float64)
            keys_per_row[hh, r0:r1] = bits @ sz
            n_sel[hh, r0:r1] = bits.sum(-1)
    f_fwd = 4.0 * mod.d * float((keys_per_row * sz).sum().item())
    dense = 4.0 * mod.d * mod.heads * float(sz.sum().item()) ** 2
    vol = {int(v): int((sz == v).sum().item()) for v in (64, 128, 256)}
    # work per 128-row tile of the attention kernels: union of its granules' selections
    q = torch.tensor([0.5, 0.99, 1.0], dtype=torch.float64, device=sz.device)
    tile_gran = torch.cat([_popcount_rows(mod.gsel[hh, 0::2] | mod.gsel[hh, 1::2]) for hh in range(mod.heads)])
    tq = torch.quantile(tile_gran.double(), q).tolist()
    kq = None
    if mod.gselT is not None:
        key_gran = torch.cat([_popcount_rows(mod.gselT[hh, 0::2] | mod.gselT[hh, 1::2]) for hh in range(mod.heads)])
        kq = torch.quantile(key_gran.double(), q).tolist()
    return {"F_fwd": f_fwd, "F_dense_fwd": dense, "n_blk": nb, "density": f_fwd / dense,
            "mean_sel_blocks": float(n_sel.mean().item()), "max_sel_blocks": float(n_sel.max().item()),
            "mean_sel_tokens": float(keys_per_row.mean().item()), "block_volumes": vol,
            "tile_key_granules_p50_p99_max": tq, "tile_query_granules_p50_p99_max": kq}


class StepTimer:
    """CUDA events around the stages of one step (on the launching stream)."""
    NAMES = ("plan_select", "attn_fwd", "unpermute_o", "permute_do", "attn_bwd", "unpermute_grads")

    def __init__(self):
        self.ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(self.NAMES) + 1)]

    def times(self):
        return {n: self.ev[i].elapsed_time(self.ev[i + 1]) for i, n in enumerate(self.NAMES)}


def run_step(mod, x, out, grads, timer=None, ds=None):
    """One layer step; ds: a dS handoff buffer for the backward (None: S and dP
    are recomputed for dQ)."""
    from dynamic_block_sparse_macro_b200 import _abi
    ev = timer.ev if timer else None
    rec = (lambda i: ev[i].record()) if ev else (lambda i: None)
    rec(0)
    mod.plan(x["V"], x["hhat"])
    if mod.raster:                            # no blocked copies: the kernels read and write raster
        mod.select_raster(x["Q"], x["K"])
        rec(1)
        mod.attend_raster(x["Q"], x["K"], x["V"], out)
        rec(2)
        rec(3)
    else:
        mod.select(x["Q"], x["K"], x["V"])
        rec(1)
        mod.attend()
        rec(2)
        _abi.prism_unpermute(mod.prob, mod.Op, mod.perm, out)
        rec(3)
    if not mod.with_backward:                 # inference: the step ends with O
        for i in (4, 5, 6):
            rec(i)
        return
    if mod.raster:
        rec(4)
        if ds is None:
            mod.attend_backward_raster(x["Q"], x["K"], x["V"], x["dO"], *grads)
        else:
            _abi.prism_sparse_attn_bwd_raster_ds(mod.prob, x["Q"], x["K"], x["V"], mod.Of32, x["dO"], mod.lse,
                                                 mod.perm, mod.shape_id, mod.gsel, mod.gselT, mod.scale, *grads,
                                                 mod.dev_status, mod.ws_bwd, ds)
        rec(5)
        rec(6)
        return
    _abi.prism_permute(mod.prob, x["dO"], mod.perm, mod.dOp)
    rec(4)
    if ds is None:
        _abi.prism_sparse_attn_bwd(mod.prob, mod.Qp, mod.Kp, mod.Vp, mod.Op, mod.Of32, mod.dOp, mod.lse,
                                   mod.gsel, mod.gselT, mod.scale, mod.dQp, mod.dKp, mod.dVp, mod.dev_status,
                                   mod.ws_bwd)
    else:
        _abi.prism_sparse_attn_bwd_ds(mod.prob, mod.Qp, mod.Kp, mod.Vp, mod.Op, mod.Of32, mod.dOp, mod.lse,
                                      mod.gsel, mod.gselT, mod.scale, mod.dQp, mod.dKp, mod.dVp, mod.dev_status,
                                      mod.ws_bwd, ds)
    rec(5)
    for src, dst in zip((mod.dQp, mod.dKp, mod.dVp), grads):
        _abi.prism_unpermute(mod.prob, src, mod.perm, dst)
    rec(6)


# ---------------------------------------------------------------- CPU oracle sample
def oracle_sample(cfg, host, target_s=15.0, max_blocks=None, seed=0, forward_only=False):
    """Time the fp64 oracle's sparse attention fwd+bwd (or fwd alone) on a bounded
    sample of query blocks of head 0, under the given selection.  Returns a dict."""
    import oracle as orc
    from threadpoolctl import threadpool_info
    Qb, Kb, Vb, dOb, bs, sel = (host[k] for k in ("Qb", "Kb", "Vb", "dOb", "bs", "sel"))
    nb = len(bs) - 1
    rng = np.random.default_rng(seed)
    order = rng.permutation(nb)
    sizes = np.diff(bs)
    done, flops, t_used = 0, 0.0, 0.0
    step = 2
    while t_used < target_s and done < nb and (max_blocks is None or done < max_blocks):
        blocks = sorted(order[done:done + step].tolist())
        t0 = time.perf_counter()
        orc.sparse_attention_fwd(Qb, Kb, Vb, bs, sel, heads=[0], q_blocks=blocks)
        if not forward_only:
            orc.sparse_attention_bwd(Qb, Kb, Vb, dOb, bs, sel, heads=[0], q_blocks=blocks)
        t_used += time.perf_counter() - t0
        mult = 1.0 if forward_only else 3.5
        for i in blocks:
            flops += mult * 4.0 * Qb.shape[-1] * sizes[i] * float(sizes[sel[0, i]].sum())
        done += len(blocks)
        step = min(step * 2, 64)
    threads = 1
    for lib in threadpool_info():
        threads = max(threads, int(lib.get("num_threads", 1)))
    return {"tflops": flops / t_used / 1e12, "seconds": t_used, "blocks": done, "flops": flops,
            "threads": threads}


def make_host_sample(mod, x):
    """fp64 host copies of head 0's blocked tensors and the GPU's selection (for the oracle)."""
    nb = mod.num_blocks()
    sel = unpack_sel_dev(mod.sel[:1], nb).cpu().numpy()
    bs = mod.blk_start[: nb + 1].cpu().numpy().astype(np.int64)
    f = lambda t: t[:1].float().cpu().double().numpy()
    from dynamic_block_sparse_macro_b200 import _abi
    if mod.Qp is None:                        # raster layer: gather head 0 through the permutation
        perm = mod.perm.long()
        g = lambda t: t[perm, :1].permute(1, 0, 2).float().cpu().double().numpy()
        dOb = g(x["dO"]) if mod.with_backward else None
        return {"Qb": g(x["Q"]), "Kb": g(x["K"]), "Vb": g(x["V"]), "dOb": dOb, "bs": bs, "sel": sel}
    dOb = None
    if mod.with_backward:
        _abi.prism_permute(mod.prob, x["dO"], mod.perm, mod.dOp)
        torch.cuda.synchronize()
        dOb = f(mod.dOp)
    return {"Qb": f(mod.Qp), "Kb": f(mod.Kp), "Vb": f(mod.Vp), "dOb": dOb, "bs": bs, "sel": sel}


# ---------------------------------------------------------------- arms
def bench_prism(args, cfg, rank, world, local_rank):
    from dynamic_block_sparse_macro_b200 import _abi
    from dynamic_block_sparse_macro_b200.layer import PrismSparseAttention
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    x = inputs.make_inputs(cfg, dev)
    torch.cuda.synchronize()
    fwd_only = bool(args.forward_only)
    if fwd_only:
        del x["dO"]
    torch.cuda.reset_peak_memory_stats(dev)
    mod = PrismSparseAttention(cfg.T, cfg.H, cfg.W, cfg.heads, cfg.head_dim, cfg.audio_dim, cfg.dtype,
                               cfg.top_k, cfg.top_p if not args.dense else 1.0, device=dev,
                               with_backward=not fwd_only, raster=bool(args.raster))
    out = torch.empty_like(x["Q"])
    grads = [] if fwd_only else [torch.empty_like(x["Q"]) for _ in range(3)]
    ds = None
    if args.bwd_ds and not fwd_only:
        # dS handoff: a buffer for every selected (query granule, key granule) pair of
        # this selection (the inputs are fixed, so the selection is the same each step)
        run_step(mod, x, out, grads)
        pairs = int(sum(_popcount_rows(mod.gsel[hh]).sum().item() for hh in range(mod.heads)))
        ds = torch.empty(_abi.prism_attn_bwd_ds_bytes(mod.prob, max(1, pairs)), dtype=torch.uint8, device=dev)
    for _ in range(max(args.warmup, 1)):
        run_step(mod, x, out, grads, ds=ds)
    torch.cuda.synchronize()
    fl = selected_flops(mod)

    timers = [StepTimer() for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    n0 = _abi.launch_count()
    clocks.mark()
    start.record()
    for t in timers:
        run_step(mod, x, out, grads, t, ds=ds)
    stop.record()
    torch.cuda.synchronize()
    launches = _abi.launch_count() - n0
    clk = clocks.stop()
    total_ms = start.elapsed_time(stop)
    per = [t.times() for t in timers]
    stage_ms = {n: float(np.mean([p[n] for p in per])) for n in StepTimer.NAMES}
    attn_ms = stage_ms["attn_fwd"] + stage_ms["attn_bwd"]
    status = mod.status()
    total_ms, attn_ms = max_over_ranks([total_ms, attn_ms], dev)
    ms_step = total_ms / args.steps
    # fwd: 2 contractions of 2 d |B_i||B_j| flops each; bwd adds 5 at half the weight each (2.5x)
    attn_flops = (1.0 if fwd_only else 3.5) * fl["F_fwd"]
    tflops = job_tflops(world, attn_flops, attn_ms)
    memory = mod.memory_report()
    memory["inputs_outputs"] = int(sum(t.numel() * t.element_size() for t in list(x.values()) + [out] + grads))
    if ds is not None:
        memory["ds_handoff"] = int(ds.numel())
    memory["peak_allocated"] = int(torch.cuda.max_memory_allocated(dev))

    # end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e and ds is None:        # the host-buffer step runs the layer's own backward
        e2e = bench_e2e(args, cfg, mod, x, dev, world, attn_flops)

    peaks = load_peaks()
    # F_fwd already counts both forward contractions (4 d |B_i||B_j| per selected pair)
    fwd_ach = fl["F_fwd"] / (stage_ms["attn_fwd"] * 1e-3) / 1e12
    bwd_ach = 2.5 * fl["F_fwd"] / (stage_ms["attn_bwd"] * 1e-3) / 1e12
    dom = "attn_bwd" if stage_ms["attn_bwd"] >= stage_ms["attn_fwd"] else "attn_fwd"
    ach = bwd_ach if dom == "attn_bwd" else fwd_ach
    # the capture is of the blocked-operand kernels: none for the raster ones
    traffic = (BWD_DRAM_BYTES.get((cfg.name, cfg.heads))
               if dom == "attn_bwd" and not args.dense and not args.raster and ds is None else None)
    # the attention kernels run at 1.85-1.97 GHz (clocks below): the burst peak is the fair
    # denominator; the sustained one (measured at ~1.33 GHz under the power cap) is reported beside it
    peak = peaks["bf16_tflops"]
    peak_sus = peaks.get("bf16_tflops_sustained")
    res = {
        "metric": metric_name(cfg, fwd_only), "value": round(tflops, 3), "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "attn_ms_per_layer": round(attn_ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "config": {"workload": f"prism {cfg.name} layer " + ("fwd (inference)" if fwd_only else "fwd+bwd")
                               + (", raster operands (no blocked copies)" if args.raster else ""),
                   "grid": [cfg.T, cfg.H, cfg.W],
                   "tokens": cfg.n_tokens, "heads": cfg.heads, "head_dim": cfg.head_dim,
                   "top_k": cfg.top_k, "top_p": 1.0 if args.dense else cfg.top_p,
                   "all_blocks_dense": bool(args.dense), "global_batch": world,
                   "backward": "dS handoff" if ds is not None else "recompute S, dP for dQ",
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs larger than L2 (126 MB): no flush"},
        "stage_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "selection": {k: (round(v, 6) if isinstance(v, float) else v) for k, v in fl.items()},
        "roofline": {"kernel": ("prism_sparse_attn_bwd" + ("_ds" if ds is not None else "")) if dom == "attn_bwd"
                     else "prism_sparse_attn_fwd",
                     "bound": "tensor", "achieved": round(ach, 3), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(ach / peak, 4), "traffic": traffic,
                     "peak_source": f"{peaks['source']} bf16_tflops (burst)",
                     "frac_of_sustained": round(ach / peak_sus, 4) if peak_sus else None,
                     "traffic_source": "ncu dram__bytes_read+write, profiles/attn_kernels_2k_4heads.md"
                     if traffic else None},
        "gpu_launches": int(launches),
        "memory_bytes": memory,
        "clocks": clk,
        "dev_status": status,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        host = make_host_sample(mod, x)
        cs = oracle_sample(cfg, host, target_s=args.cpu_seconds, forward_only=fwd_only)
        res["cpu_baseline"] = {"value": round(cs["tflops"], 6), "unit": "TFLOP/s", "cores": cs["threads"],
                               "kind": "oracle",
                               "sample": f"fp64 numpy oracle, head 0, {cs['blocks']} random query blocks "
                                         f"({'fwd' if fwd_only else 'fwd+bwd'} under the GPU's selection), "
                                         f"{cs['seconds']:.1f} s"}
    return res


def bench_e2e(args, cfg, mod, x, dev, world, attn_flops):
    """The same metric end to end through the library's host-buffer step
    (prism_layer_step_host): every step uploads its inputs from page-locked host
    memory, runs the layer and downloads its outputs, one cudaMemcpyAsync per
    tensor on two copy streams beside the compute stream.  Timed from an event
    on the compute stream before the first step to one on the download stream
    after the last, where every step's work ends."""
    names = ("Q", "K", "V", "hhat", "dO") if mod.with_backward else ("Q", "K", "V", "hhat")
    hin = {k: torch.empty(x[k].shape, dtype=x[k].dtype, pin_memory=True) for k in names}
    for k in names:
        hin[k].copy_(x[k])
    dx = {k: torch.empty_like(x[k]) for k in names}
    n_out = 4 if mod.with_backward else 1
    hout = [torch.empty(x["Q"].shape, dtype=x["Q"].dtype, pin_memory=True) for _ in range(n_out)]
    douts = [torch.empty_like(x["Q"]) for _ in range(n_out)]
    mod.attach_io(dx["Q"], dx["K"], dx["V"], dx["hhat"], douts[0], dx.get("dO"), *(douts[1:] + [None] * (4 - n_out)))
    compute, h2d, d2h = (torch.cuda.Stream(device=dev) for _ in range(3))
    # steady state: the first step's uploads and the last one's downloads overlap
    # nothing, so more steps show the pipelined rate (each ~0.2 s at 2K)
    steps = max(1, min(args.steps, 8))
    hargs = [hin["Q"], hin["K"], hin["V"], hin["hhat"], hin.get("dO")] + hout + [None] * (4 - n_out)

    def one():
        mod.step_host(*hargs, compute, h2d, d2h)

    one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(compute)
    for _ in range(steps):
        one()
    b.record(d2h)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    ms = max_over_ranks([ms], dev)[0]
    h2d_b = sum(hin[k].numel() * hin[k].element_size() for k in names)
    d2h_b = sum(h.numel() * h.element_size() for h in hout)
    return {"value": round(job_tflops(world, attn_flops, ms), 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 3), "h2d_bytes_per_step": int(h2d_b), "d2h_bytes_per_step": int(d2h_b),
            "steps": steps, "api": "prism_layer_step_host (C ABI, host buffers, three streams)",
            "note": "selected-block FLOPs over the whole layer step incl. host copies"}


def bench_reference(args, cfg):
    """The fp64 oracle as it stands, on host cores: each step is a bounded sample
    (query blocks of head 0) of the same workload's attention fwd+bwd."""
    import oracle as orc
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = inputs.make_inputs(cfg, dev)
    V = inputs.to_f64(x["V"])
    hh = inputs.to_f64(x["hhat"])
    ind = orc.zone_indicator(V, hh, cfg.T, cfg.H, cfg.W)
    del V
    shp = orc.assign_shapes(ind["g"], ind["rho"])
    perm, bs = orc.build_permutation(shp["shape_id"], cfg.T, cfg.H, cfg.W)
    q0 = lambda t: inputs.to_f64(t[:, :1, :])
    Qb, Kb, Vb, dOb = (orc.permute(q0(x[k]), perm) for k in ("Q", "K", "V", "dO"))
    _, _, P = orc.block_pool_score(Qb, Kb, bs)
    sel = orc.block_select(P, cfg.top_k, cfg.top_p)["sel"]
    host = {"Qb": Qb, "Kb": Kb, "Vb": Vb, "dOb": dOb, "bs": bs, "sel": sel}
    per_step = max(2.0, args.cpu_seconds / max(1, args.steps + args.warmup))
    fo = bool(args.forward_only)
    for w in range(args.warmup):
        oracle_sample(cfg, host, target_s=per_step, seed=1000 + w, forward_only=fo)
    res = [oracle_sample(cfg, host, target_s=per_step, seed=s, forward_only=fo) for s in range(args.steps)]
    what = "fwd" if fo else "fwd+bwd"
    fl = sum(r["flops"] for r in res)
    sec = sum(r["seconds"] for r in res)
    v = fl / sec / 1e12
    blocks = sum(r["blocks"] for r in res)
    return {"metric": metric_name(cfg, fo), "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * sec / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": f"prism {cfg.name} layer " + ("fwd (inference)" if fo else "fwd+bwd")
                                   + " (oracle sample)",
                       "grid": [cfg.T, cfg.H, cfg.W], "tokens": cfg.n_tokens, "heads": cfg.heads,
                       "head_dim": cfg.head_dim, "top_k": cfg.top_k, "top_p": cfg.top_p},
            "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": res[0]["threads"],
                             "kind": "oracle",
                             "sample": f"fp64 numpy oracle sparse attention {what}, head 0, {blocks} query "
                                       f"blocks over {args.steps} steps, selection by the oracle's own stages"},
            "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="prism", choices=["prism", "reference"])
    ap.add_argument("--config", default="2k")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the config's head count (smaller profiling captures)")
    ap.add_argument("--dense", action="store_true", help="select every block (all-blocks dense run)")
    ap.add_argument("--forward-only", action="store_true",
                    help="inference: the forward stages alone, no backward buffers (value = forward TFLOP/s)")
    ap.add_argument("--raster", action="store_true",
                    help="the attention reads Q, K, V, dO and writes O, dQ, dK, dV in the raster layout")
    ap.add_argument("--bwd-ds", action="store_true",
                    help="backward through prism_sparse_attn_bwd_ds (dS handoff) instead of recomputing S, dP")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--out", default=None, help="also append the JSON line to this file")
    args = ap.parse_args()
    cfg = get_config(args.config, **({"heads": args.heads} if args.heads else {}))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        res = bench_reference(args, cfg)
    else:
        if world > 1:
            import datetime
            torch.cuda.set_device(local_rank)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                                 device_id=torch.device("cuda", local_rank))
        res = bench_prism(args, cfg, rank, world, local_rank)
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
    if rank == 0:
        line = json.dumps(res)
        print(line, flush=True)
        if args.out:
            with open(args.out, "a") as f:
                f.write(line + "\n")
    return 0


if __name__ == "__main__":
    sys.exit(main())
