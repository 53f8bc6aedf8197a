#!/usr/bin/env python
"""Benchmark of the causal alpha-entmax attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

A step is one full forward pass over the workload's synthetic batch, with the inputs already
resident in HBM: the tau pass, which also writes the output of every query tile whose rows'
supports its candidate buffers held, then the tile output pass over the query tiles left
pending (those whose candidates overflowed).  The same step on the tile path (tau pass, then
the output pass over every query tile's active key tiles) is timed beside it.  The metric is effective TFLOP/s: 4 d FLOPs per
causally valid (query, key) pair inside the active 128 x 128 tiles (recomputed scores + p V),
summed over heads and batch, divided by the step time; tokens/s and the fraction of the
measured bf16 dense tensor-core peak ride along.  Rank 0 prints one JSON line.

Multi-GPU (torchrun): every (batch, kv-head group) is independent, so each rank runs its own
full-size problem (weak scaling, no collective on the data path); the step time is the max over
ranks.  --impl reference times the fp64 CPU oracle instead, on a bounded sample of whole query
tiles of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from adaptive_sparse_attention_b200 import api as ea  # noqa: E402
from adaptive_sparse_attention_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

DEFAULT_WORKLOAD = "t128k_gqa4_bf16_d128_a1.5"
METRIC = "effective TFLOP/s and tokens/s of entmax attention fwd; % of bf16 TC peak"
TILE = 128
L2_BYTES = 126 * 2**20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------------------ work counts --

def pair_matrix(L: int, causal: bool) -> np.ndarray:
    """[nqt, nkt] number of valid (query, key) pairs of each tile of one sequence of length L."""
    nt = (L + TILE - 1) // TILE
    rows = np.minimum(TILE, L - np.arange(nt) * TILE)
    if not causal:
        return np.outer(rows, rows).astype(np.int64)
    m = np.zeros((nt, nt), dtype=np.int64)
    for qt in range(nt):
        m[qt, :qt] = rows[qt] * rows[:qt]
        r = rows[qt]
        m[qt, qt] = r * (r + 1) // 2  # diagonal tile: keys <= own position
    return m


def count_pairs(w, bits, cu):
    """(pairs inside active tiles, all valid pairs) summed over batch and heads."""
    table = ea.tile_slot_table(w.B, w.T, None if cu is None else cu.tolist())
    act = dense = 0
    nb = 1 if cu is not None else w.B
    for b in range(nb):
        seqs = range(len(table)) if cu is not None else [b]
        for s in seqs:
            slot0, nqt, start, L = table[s]
            if nqt == 0:
                continue
            pm = pair_matrix(L, w.causal)
            blk = bits[b, :, slot0:slot0 + nqt, :pm.shape[1]]  # [Hq, nqt, nkt]
            act += int((blk * pm[None]).sum())
            dense += int(pm.sum()) * w.Hq
    return act, dense


# --------------------------------------------------------------------------------- helpers --

# DRAM bytes (read + write) per launch from one ncu capture of the dominant kernel, with the
# hash of the kernel sources at capture time: reported only while the sources are unchanged.
NCU_TRAFFIC = {
    # (workload, pass): (bytes per launch, sources hash, capture)
    ("b2_t16k_gqa4_bf16_d128_a2", "tau_pass"): (768.7e6, "02415218cf5ab321",
                                                "tau_tc_kernel, ncu --metrics dram__bytes_*"),
    ("t128k_gqa4_bf16_d128_a1.5", "tau_pass"): (1529.2e6, "02415218cf5ab321",
                                                "tau_tc_kernel, ncu --metrics dram__bytes_*"),
}


def _code_only(src: str) -> str:
    """C++ source without its comments and blank space: what the compiler sees of it."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_sources_hash() -> str:
    """Hash of the tau kernel's sources, comments and layout left out (a comment edit does not
    invalidate a capture)."""
    import hashlib
    h = hashlib.sha256()
    for f in ("tc.cu", "common.cuh", "tcgen05.cuh"):
        with open(os.path.join(ROOT, "adaptive_sparse_attention_b200", "csrc", f)) as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, kernel: str):
    rec = NCU_TRAFFIC.get((workload, kernel))
    if rec is None or rec[1] != kernel_sources_hash():
        return None
    return rec[0]


def _alpha_f32(alpha: float) -> float:
    """alpha as the fp32 value the kernels receive (the C ABI takes a float)."""
    return float(np.float32(alpha))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        if not self.lines:
            return None
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            try:
                sm.append(float(f[1]))
                smax = max(smax, float(f[2]))
            except (ValueError, IndexError):
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        loaded = [x for x in sm if x > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def _reduce(x: float, world: int, op: str, device: str) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The largest of the ranks' x (times: the job ends with its slowest rank)."""
    return _reduce(x, world, "max", device)


def sum_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The sum of the ranks' x (work: each rank solves its own problem)."""
    return _reduce(x, world, "sum", device)


def job_rate(units_per_rank: float, ms_per_rank: float, world: int, device: str = "cuda") -> float:
    """Whole-job throughput in units per second: the units of all ranks over the slowest rank's
    time (weak scaling: every rank runs a full problem of its own)."""
    units = sum_over_ranks(units_per_rank, world, device)
    ms = max_over_ranks(ms_per_rank, world, device)
    return units / (ms * 1e-3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------------- oracle sampling --

def oracle_tile_sample(w, inputs, budget_s: float, seed: int = 0):
    """Times the oracle on whole query tiles of the workload until about budget_s seconds of
    CPU work; returns (effective flops, rows, seconds, n tiles, threads)."""
    from oracle import oracle
    q, k, v, cu = inputs
    alpha = oracle.alpha_as_float32(w.alpha)
    table = ea.tile_slot_table(w.B, w.T, None if cu is None else cu.tolist())
    rng = np.random.default_rng(seed)
    nb = 1 if cu is not None else w.B
    # candidate tiles: (b, h, s, qt) drawn uniformly over all query tiles
    all_t = [(b, h, s, qt) for b in range(nb) for h in range(w.Hq)
             for s in (range(len(table)) if cu is not None else [b]) for qt in range(table[s][1])]
    order = rng.permutation(len(all_t))
    flops = rows_done = 0
    spent = 0.0
    ntiles = 0
    batch = 1
    threads = oracle.host_threads()
    for i0 in range(0, len(order)):
        if spent >= budget_s or ntiles >= len(order):
            break
        pick = [all_t[j] for j in order[ntiles:ntiles + batch]]
        rows, meta = [], []
        for b, h, s, qt in pick:
            slot0, nqt, start, L = table[s]
            pos = np.arange(qt * TILE, min((qt + 1) * TILE, L))
            r = ((b * w.Hq + h) * w.T + pos) if cu is None else (h * w.T + start + pos)
            rows.append(r)
            meta.append((L, qt, pos.size))
        rr = np.concatenate(rows)
        t0 = time.perf_counter()
        res = oracle.attention_rows(q, k, v, alpha, w.causal, cu, rr, nthreads=threads)
        dt = time.perf_counter() - t0
        spent += dt
        off = 0
        for (L, qt, n) in meta:
            active = (res["maxp"][off:off + n] > 0).any(axis=0)
            pm = pair_matrix(L, w.causal)[qt]
            flops += 4 * w.d * int((active[:pm.size] * pm).sum())
            off += n
        rows_done += rr.size
        ntiles += len(pick)
        batch = max(1, min(64, int(batch * 2))) if dt < budget_s / 8 else batch
    return flops, rows_done, spent, ntiles, threads


# -------------------------------------------------------------------------------- arms --

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    inputs = make_inputs(w, seed=0)
    per_step = max(1.0, min(20.0, 150.0 / (args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_tile_sample(w, inputs, per_step, seed=1)
    vals, times, rows, tiles = [], [], 0, 0
    threads = 0
    for i in range(args.steps):
        fl, nr, dt, nt, threads = oracle_tile_sample(w, inputs, per_step, seed=100 + i)
        vals.append(fl / dt / 1e12)
        times.append(dt)
        rows += nr
        tiles += nt
    value = float(np.mean(vals))
    sample = (f"{tiles} whole 128-row query tiles drawn uniformly over (batch, head, tile) "
              f"({rows} rows) across {args.steps} steps of ~{per_step:.0f} s")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * float(np.mean(times)), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, world):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "T": w.T, "d": w.d,
            "alpha": w.alpha, "n_iter": w.n_iter, "causal": w.causal, "input_dtype": w.dtype,
            "seqlens": list(w.seqlens) if w.seqlens else None,
            "spikes": f"{w.spike_frac:g} of keys x{w.spike_scale:g}" if w.spike_frac else None,
            "tile": "128x128", "parallelism": f"dp{world} (independent per-rank problems)"}


def launches_per_step(w, mode: str = "fused") -> int:
    """Kernels of one step on the library's full workspace: the tau kernel, the overflow kernel
    and the tile output kernel; for bf16 problems with at least 1024 keys the key-norm and
    warm-up selection kernels of the tau pass; on the support path with bf16 inputs the kernel
    that computes o from the supports; with the FP8 screen its two prep kernels and its sweep."""
    bf16 = w.dtype == "bf16"
    return (3 + (2 if bf16 and w.T >= 1024 else 0)
            + (1 if bf16 and mode in ("fused", "screen") else 0)
            + (3 if mode == "screen" else 0))  # the screen's two prep kernels and its sweep


# The forward pass, three ways through the C ABI's two-pass entry points:
#   fused    with ENTMAX_ATTN_FLAG_SUPPORT: the tau pass (tau, mask, lists, and the support of
#            every row whose candidates it held), then the output pass (o from the supports, the
#            tile pass over the other query tiles): the path entmax_attn_fwd takes, and the step
#            this benchmark times;
#   tile     without the flag: the output pass over every query tile's active key tiles (o
#            recomputed tile by tile on the tensor cores), reported beside it;
#   nomask   the variant without block mask (--no-block-mask);
#   screen   the fused step with the FP8-screened tau pass (--fp8-screen).
MODES = ("fused", "tile", "nomask", "screen")


class Problem:
    """Device copies of one workload's inputs, outputs and workspace."""

    def __init__(self, w, rank, local):
        self.w = w
        self.dev = torch.device("cuda", local)
        self.host = make_inputs(w, seed=rank)
        q, k, v, cu = self.host
        self.in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
        self.q, self.k, self.v = q.to(self.dev), k.to(self.dev), v.to(self.dev)
        self.cu = cu.to(self.dev) if cu is not None else None
        self.alpha = _alpha_f32(w.alpha)
        self.stream = torch.cuda.current_stream(self.dev)
        self.out, self.tau, self.mask = ea.alloc_outputs(self.q, self.k, self.cu)
        self.ws = ea.alloc_workspace(self.q, self.k, self.cu)
        self.screen = None

    def step(self, mode, ev=None):
        from adaptive_sparse_attention_b200 import _native
        w, s = self.w, self.stream
        a = (self.q, self.k)
        if ev:
            ev[0].record(s)
        flags = {"fused": _native.FLAG_SUPPORT, "tile": 0, "screen": _native.FLAG_SUPPORT,
                 "nomask": _native.FLAG_NO_BLOCK_MASK}[mode]
        if mode == "screen":
            if self.screen is None:
                self.screen = ea.alloc_screen(self.q, self.k, self.cu)
            ea.tau_pass_screened(*a, self.tau, self.mask, self.ws, self.screen, self.alpha,
                                 w.n_iter, w.causal, self.cu, flags=flags, stream=s)
        else:
            ea.tau_pass(*a, self.tau, self.mask, self.ws, self.alpha, w.n_iter, w.causal, self.cu,
                        flags=flags, stream=s)
        if ev:
            ev[1].record(s)
        ea.out_pass(*a, self.v, self.tau, self.ws, self.out, self.alpha, w.causal, self.cu,
                    flags=flags, stream=s)
        if ev:
            ev[2].record(s)

    def time(self, mode, steps, warmup, world, sampler=None):
        """(ms per step of this rank, per-step tau-pass ms, per-step output-pass ms, overflow
        tiles), CUDA events on the launching stream, barrier + synchronize on both sides."""
        for _ in range(warmup):
            self.step(mode)
        torch.cuda.synchronize()
        assert ea.status(self.stream) == 0
        nfb = ea.fallback_tiles(self.ws, self.stream)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        with (sampler if sampler is not None else _NullCtx()):
            start.record(self.stream)
            for i in range(steps):
                self.step(mode, evs[i])
            stop.record(self.stream)
            torch.cuda.synchronize()
        barrier(world)
        st = ea.status(self.stream)
        assert st == 0, f"device status {st}"
        return (start.elapsed_time(stop) / steps, [e[0].elapsed_time(e[1]) for e in evs],
                [e[1].elapsed_time(e[2]) for e in evs], nfb)

    def time_e2e(self, steps, world):
        """ms per call of entmax_attn_fwd_host on pinned host copies of the inputs and outputs
        (CUDA events on the stream the call completes on), after two untimed calls."""
        w, q, k, v, cu = self.w, *self.host
        qh, kh, vh = (t.pin_memory() for t in (q, k, v))
        outh = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        tauh = torch.empty(self.tau.shape, dtype=self.tau.dtype).pin_memory()
        maskh = torch.empty(self.mask.shape, dtype=self.mask.dtype).pin_memory()

        def call():
            ea.entmax_attn_fwd_host(qh, kh, vh, self.alpha, w.n_iter, w.causal, cu, out=outh,
                                    tau=tauh, block_mask=maskh, stream=self.stream,
                                    synchronize=False)

        for _ in range(2):
            call()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for _ in range(steps):
            call()
        e1.record(self.stream)
        torch.cuda.synchronize()
        assert ea.status(self.stream) == 0
        return e0.elapsed_time(e1) / steps

    def screen_kept(self):
        """(key tiles the FP8 screen kept, all causally valid key tiles) of the last screened
        tau pass, from the documented order of the screen buffer's sections."""
        w, cu = self.w, self.host[3]
        up = lambda x: (x + 255) // 256 * 256  # noqa: E731
        nb = 1 if cu is not None else w.B
        slots, _ = ea.mask_layout(w.B, w.Hq, w.T, cu is not None)
        nkt = -(-w.T // TILE)
        tiles = nb * w.Hq * slots
        off = (up(nb * w.Hq * w.T * 128) + up(nb * w.Hq * w.T * 16) + up(nb * w.Hkv * w.T * 128)
               + up(nb * w.Hkv * slots * 16) + up(4 * tiles * nkt))
        kept = int(self.screen[off:off + 4 * tiles].view(torch.int32).sum().item())
        total = 0
        for slot0, nq, start, L in ea.tile_slot_table(w.B, w.T, None if cu is None else
                                                      cu.tolist()):
            total += (nq * (nq + 1) // 2 if w.causal else nq * nq) * w.Hq
        return kept, total

    def pair_counts(self):
        """(pairs inside active tiles, all causally valid pairs) from the last masked tau pass."""
        w = self.w
        bits = ea.decode_block_mask(self.mask.cpu().numpy(), w.B, w.Hq, w.T, self.host[3])
        return count_pairs(w, bits, self.host[3])


class _NullCtx:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def secondary(args):
    """The other target workload measured in the same run (16K with 128K and back)."""
    if args.also == "none":
        return []
    if args.also != "auto":
        return [n for n in args.also.split(",") if n and n != args.workload]
    pair = ("t128k_gqa4_bf16_d128_a1.5", "b2_t16k_gqa4_bf16_d128_a2")
    if args.workload in pair and not args.no_block_mask:
        return [pair[1] if args.workload == pair[0] else pair[0]]
    return []


def run_native(args, rank, world, local):
    w = WORKLOADS[args.workload]
    pb = Problem(w, rank, local)
    nm = args.no_block_mask
    mode = "nomask" if nm else ("screen" if args.fp8_screen else "fused")
    clk = ClockSampler(local)  # samples the clocks during the timed region only
    ms_one, t_tau, t_out, nfb = pb.time(mode, args.steps, args.warmup, world, sampler=clk)
    ms_step = max_over_ranks(ms_one, world)

    if nm:  # the mask, for the effective FLOP count only: one masked tau pass, not timed
        pb.step("tile")
        torch.cuda.synchronize()
    act_pairs, dense_pairs = pb.pair_counts()
    eff_flops = 4 * w.d * act_pairs
    tau_flops = 2 * w.d * dense_pairs
    q, k, v, cu = pb.host
    tokens = w.B * w.T * w.Hq if cu is None else w.T * w.Hq  # query rows (token x head)
    tokens_seq = w.B * w.T if cu is None else w.T
    value = job_rate(eff_flops, ms_one, world) / 1e12
    dense_rate = job_rate(4 * w.d * dense_pairs, ms_one, world)

    # the tile path (every query tile's output recomputed over its active key tiles on the
    # tensor cores), on the same inputs, for comparison: same warm-up, same step count
    tile = None
    if not nm and not args.step_only:
        ms_t, tt_tau, tt_out, _ = pb.time("tile", args.steps, args.warmup, world)
        ms_t = max_over_ranks(ms_t, world)
        out_tile = float(np.mean(tt_out))
        tile = {"ms_per_step": ms_t, "value": job_rate(eff_flops, ms_t, world) / 1e12,
                "ms_tau_pass": float(np.mean(tt_tau)), "ms_out_pass": out_tile,
                "out_pass_tflops": eff_flops / (out_tile * 1e-3) / 1e12}

    # end to end through the C ABI: inputs and outputs in pinned host memory, every step.  The
    # masked path goes through entmax_attn_fwd_host (the library streams (batch row, kv head)
    # chunks: copies in and out overlap the computation); the variant without block mask
    # copies with torch around entmax_attn_fwd_no_block_mask.
    qd, kd, vd, cud, out, tau, mask, stream = (pb.q, pb.k, pb.v, pb.cu, pb.out, pb.tau, pb.mask,
                                               pb.stream)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    outh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    tauh = torch.empty(tau.shape, dtype=tau.dtype).pin_memory()
    maskh = torch.empty(mask.shape, dtype=mask.dtype).pin_memory()

    def fwd_e2e():
        if nm:
            qd.copy_(qh, non_blocking=True)
            kd.copy_(kh, non_blocking=True)
            vd.copy_(vh, non_blocking=True)
            ea.entmax_attn_fwd_no_block_mask(qd, kd, vd, pb.alpha, w.n_iter, w.causal, cud, out,
                                             tau, stream=stream)
            outh.copy_(out, non_blocking=True)
        else:
            ea.entmax_attn_fwd_host(qh, kh, vh, pb.alpha, w.n_iter, w.causal, cu, out=outh,
                                    tau=tauh, block_mask=maskh, stream=stream, synchronize=False)

    e2e_steps = 0 if args.step_only else max(2, min(args.steps, 5))
    for _ in range(2 if e2e_steps else 0):
        fwd_e2e()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        fwd_e2e()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_one = e0.elapsed_time(e1) / e2e_steps if e2e_steps else float("nan")
    e2e_ms = max_over_ranks(e2e_one, world)
    e2e_rate = job_rate(eff_flops, e2e_one, world)
    assert ea.status(stream) == 0
    d2h_bytes = out.numel() * out.element_size() + (0 if nm else tau.numel() * 4
                                                    + mask.numel() * 4)

    others = []
    for name in ([] if args.step_only else secondary(args)):
        w2 = WORKLOADS[name]
        p2 = Problem(w2, rank, local)
        ms2, t2_tau, t2_out, nfb2 = p2.time("fused", args.steps, args.warmup, world)
        a2, d2 = p2.pair_counts()
        ms2_max = max_over_ranks(ms2, world)
        v2 = job_rate(4 * w2.d * a2, ms2, world) / 1e12
        e2 = p2.time_e2e(max(2, min(args.steps, 5)), world)
        others.append({"workload": name, "value": v2, "unit": "TFLOP/s", "ms_per_step": ms2_max,
                       "frac_of_bf16_peak": None, "ms_tau_pass": float(np.mean(t2_tau)),
                       "ms_out_pass": float(np.mean(t2_out)),
                       "active_tile_pair_fraction": a2 / d2, "overflow_tiles": nfb2,
                       "tau_pass_tflops": 2 * w2.d * d2 / (float(np.mean(t2_tau)) * 1e-3) / 1e12,
                       "e2e": {"value": job_rate(4 * w2.d * a2, e2, world) / 1e12,
                               "unit": "TFLOP/s", "ms_per_step": max_over_ranks(e2, world),
                               "entry": "entmax_attn_fwd_host (pinned host buffers)"}})
        del p2
        torch.cuda.empty_cache()

    if rank != 0:
        return 0
    peaks, peak_src = load_peaks()
    tc = w.dtype == "bf16"
    mean_tau = float(np.mean(t_tau))
    mean_out = float(np.mean(t_out))
    dom_tau = mean_tau >= mean_out
    timed_s = ms_one * args.steps * 1e-3
    sustained = timed_s > 1.0
    peak_key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    if tc:
        bound, unit, peak = "tensor", "TFLOP/s", float(peaks[peak_key])
        peak_note = f"{peak_src} {peak_key}"
    else:
        # fp32 on the CUDA cores: 148 SMs x 128 FMA/clk x 2 FLOP x max SM clock
        bound, unit = "alu", "TFLOP/s"
        peak = 148 * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12
        peak_note = "fp32 FMA: 148 SMs x 128 lanes x 2 x max SM clock"
    out_flops = 4 * w.d * (dense_pairs if nm else act_pairs)
    achieved = (tau_flops / (mean_tau * 1e-3) if dom_tau else out_flops / (mean_out * 1e-3)) / 1e12
    kname = "tau_pass" if dom_tau else "out_pass"
    traffic = ncu_traffic(w.name, kname)
    roofline = {"kernel": kname, "bound": bound,
                "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                "traffic": traffic, "peak_source": peak_note,
                "algorithmic": ("2 d flops per causally valid pair (dense scores)" if dom_tau
                                else ("4 d flops per causally valid pair (every tile)" if nm
                                      else "4 d flops per valid pair inside active tiles"))}

    cpu = None
    if world == 1 and not args.no_cpu_baseline and not args.step_only:
        fl, nr, dt, nt, thr = oracle_tile_sample(w, pb.host, args.cpu_budget)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
               "sample": f"{nt} whole 128-row query tiles ({nr} rows) drawn uniformly, "
                         f"{dt:.1f} s of fp64 oracle work"}

    bf16_peak = float(peaks["bf16_tflops"])
    for o in others:
        o["frac_of_bf16_peak"] = o["value"] / world / bf16_peak
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype if w.dtype == "bf16" else "f32", "data": "synthetic",
        "config": dict(workload_config(w, world),
                       variant="no_block_mask" if nm else "block_mask",
                       path=("tau pass + output pass over every causal tile" if nm else
                             ("FP8 screen of the key tiles, then " if mode == "screen" else "")
                             + "tau pass recording each row's support + output from the "
                             "supports (tile output pass for query tiles without one)"),
                       l2=f"inputs {pb.in_bytes / 2**20:.0f} MiB vs {L2_BYTES / 2**20:.0f} MiB "
                          f"L2; no flush" if pb.in_bytes > L2_BYTES
                       else "inputs fit in L2; no flush"),
        "tokens_per_s": world * tokens_seq / (ms_step * 1e-3),
        "query_rows_per_s": world * tokens / (ms_step * 1e-3),
        "frac_of_bf16_peak": value / world / bf16_peak,
        "dense_equiv_tflops": dense_rate / 1e12,
        "active_tile_pair_fraction": act_pairs / dense_pairs,
        "ms_tau_pass": mean_tau, "ms_out_pass": mean_out,
        "tau_pass_hbm_gbs": (q.numel() * q.element_size() + k.numel() * k.element_size()
                             + tau.numel() * 4 + mask.numel() * 4) / (mean_tau * 1e-3) / 1e9,
        "overflow_tiles": nfb,
        "fp8_screen_kept_tiles": (dict(zip(("kept", "causal"), pb.screen_kept()))
                                  if mode == "screen" else None),
        "tile_path": tile,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": None if args.step_only else {"value": e2e_rate / 1e12, "unit": "TFLOP/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": pb.in_bytes,
                "d2h_bytes_per_step": d2h_bytes,
                "entry": ("entmax_attn_fwd_no_block_mask + torch copies" if nm
                          else "entmax_attn_fwd_host (pinned host buffers)")},
        "gpu_launches": launches_per_step(w, mode) * args.steps,
        "clocks": clk.summary(),
        "other_workloads": others,
    }
    print(json.dumps(line), flush=True)
    return 0


BWD_METRIC = "effective TFLOP/s of the entmax attention backward pass (dq, dk, dv)"


def run_backward(args, rank, world, local):
    """The backward pass (entmax_attn_bwd) of the workload, after one forward pass (with
    ENTMAX_ATTN_FLAG_SUPPORT) whose tau, compact lists and support lists it reuses.  A step is
    one backward call with the same flag over resident inputs and upstream gradient: the rows
    with a recorded support from their supports (bwd_support_kernel), the other query tiles over
    their listed key tiles on the CUDA cores.  Effective FLOPs: 10 d per valid pair inside
    active tiles, the work of the pages' tile-based backward (recomputed scores, dout v^T, and
    the dq, dk, dv products), a fixed count per workload.  The support kernel is a gather and
    scatter bound by memory, so its roofline counts the bytes the step must move (q, dout, k, v
    read once; dq, dk, dv and delta written once) against the measured HBM bandwidth.  The tile
    path (every query tile over its listed key tiles) is timed beside it where it takes under a
    few seconds per step."""
    from adaptive_sparse_attention_b200 import _native
    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    q, k, v, cu = make_inputs(w, seed=rank)
    gen = torch.Generator().manual_seed(1000 + rank)
    g = torch.randn(q.shape, generator=gen).to(q.dtype)
    qd, kd, vd, gd = q.to(dev), k.to(dev), v.to(dev), g.to(dev)
    cud = cu.to(dev) if cu is not None else None
    alpha = _alpha_f32(w.alpha)
    stream = torch.cuda.current_stream(dev)
    out, tau, mask = ea.alloc_outputs(qd, kd, cud)
    ws = ea.alloc_workspace(qd, kd, cud)
    sup = _native.FLAG_SUPPORT
    ea.tau_pass(qd, kd, tau, mask, ws, alpha, w.n_iter, w.causal, cud, flags=sup, stream=stream)
    ea.out_pass(qd, kd, vd, tau, ws, out, alpha, w.causal, cud, flags=sup, stream=stream)

    def bwd(flags):
        return ea.entmax_attn_bwd(qd, kd, vd, gd, tau, ws, alpha, w.causal, cud, flags=flags,
                                  stream=stream)

    for _ in range(args.warmup):
        grads = bwd(sup)
    torch.cuda.synchronize()
    assert ea.status(stream) == 0
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for _ in range(args.steps):
            grads = bwd(sup)
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    total_ms = start.elapsed_time(stop)
    ms_one = total_ms / args.steps
    ms_step = max_over_ranks(ms_one, world)
    assert ea.status(stream) == 0
    nfb = ea.fallback_tiles(ws, stream)
    bits = ea.decode_block_mask(mask.cpu().numpy(), w.B, w.Hq, w.T, cu)
    act_pairs, _ = count_pairs(w, bits, cu)
    eff_flops = 10 * w.d * act_pairs
    value = job_rate(eff_flops, ms_one, world) / 1e12
    peaks, peak_src = load_peaks()
    esz = q.element_size()
    bytes_step = (2 * q.numel() * esz + 2 * k.numel() * esz   # q, dout, k, v read
                  + q.numel() * 4 + 2 * k.numel() * 4          # dq, dk, dv written (fp32)
                  + tau.numel() * 4)                           # delta written
    achieved = bytes_step / (ms_one * 1e-3) / 1e9
    roofline = {"kernel": "entmax_attn_bwd (bwd_support_kernel)", "bound": "hbm",
                "achieved": achieved, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                "frac": achieved / float(peaks["hbm_gbs"]), "traffic": None,
                "peak_source": f"{peak_src} hbm_gbs",
                "algorithmic": "q, dout, k, v read once; dq, dk, dv (fp32) and delta written "
                               "once"}

    tile = None
    tile_steps = 0 if (args.step_only or w.T > 32768) else min(args.steps, 3)
    if tile_steps:
        bwd(0)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(tile_steps):
            bwd(0)
        t1.record(stream)
        torch.cuda.synchronize()
        ms_t = max_over_ranks(t0.elapsed_time(t1) / tile_steps, world)
        tile = {"ms_per_step": ms_t, "value": job_rate(eff_flops, ms_t, world) / 1e12,
                "steps": tile_steps}

    # end to end: H2D of the upstream gradient from pinned memory, the backward call, D2H of
    # dq, dk and dv, every step (forward state resident)
    gh = g.pin_memory()
    dq, dk, dv, _ = grads
    hosts = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (dq, dk, dv)]
    e2e_steps = 0 if args.step_only else max(2, min(args.steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        gd.copy_(gh, non_blocking=True)
        res = bwd(sup)
        for hst, dev_t in zip(hosts, res[:3]):
            hst.copy_(dev_t, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world) if e2e_steps else None

    cpu = None
    if world == 1 and not args.no_cpu_baseline and not args.step_only:
        from oracle import backward as obwd  # the timed CPU baseline only
        import time
        # a bounded sample: the oracle backward of the workload's first (batch, head) over a
        # prefix of its rows, grown until it takes about the budget
        nrow, spent, done_flops = 128, 0.0, 0
        per_pair = 10 * w.d
        while spent < args.cpu_budget / 3 and nrow <= w.T:
            if cu is None:
                qs, ks_, vs_, gs = (t[:1, :1, :nrow] for t in (q, k, v, g))
            else:
                qs, ks_, vs_, gs = (t[:1, :nrow] for t in (q, k, v, g))
                qs, ks_, vs_, gs = qs[None], ks_[None], vs_[None], gs[None]
            t0 = time.perf_counter()
            obwd.attention_backward(qs, ks_, vs_, gs, alpha, w.causal, None)
            spent = time.perf_counter() - t0
            pairs = nrow * (nrow + 1) // 2 if w.causal else nrow * nrow
            done_flops = per_pair * pairs
            sample = f"oracle backward of one head over its first {nrow} rows"
            nrow *= 2
        cpu = {"value": done_flops / spent / 1e12, "unit": "TFLOP/s", "cores": 1,
               "kind": "oracle", "sample": sample + f", {spent:.1f} s (numpy fp64, one thread; "
               "all valid pairs counted)"}

    line = {
        "metric": BWD_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": dict(workload_config(w, world), variant="backward",
                       grads="fp32 dq, dk, dv",
                       path="rows with a recorded support from their supports; other query "
                            "tiles over their listed key tiles"),
        "active_tile_pair_fraction": None,
        "overflow_tiles": nfb,
        "tile_path": tile,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": None if e2e_ms is None else {
            "value": job_rate(eff_flops, e2e_ms, world) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": e2e_ms, "h2d_bytes_per_step": g.numel() * g.element_size(),
            "d2h_bytes_per_step": sum(t.numel() * 4 for t in (dq, dk, dv))},
        "gpu_launches": (3 if w.dtype == "bf16" else 2) * args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


ROUTE_METRIC = "query rows/s of entmax block routing over chunk summaries"
ROUTE_CHUNK = 64  # tokens per chunk (the routing entry point's default)


def run_routing(args, rank, world, local):
    """Entmax block routing (DashAttention page, "How it works", stage 2): every query row of
    the workload's q scored against the summaries of the chunks it may see (the chunks before
    its own plus its own, estimate_diagonal), then alpha-entmax over those scores, giving the
    routing priors pi and tau.  The summaries are synthetic: the mean of each 64-key chunk of the
    workload's keys (the page builds them with learned weights).  A step is one
    entmax_attn_route_chunks call over resident inputs (the score kernel on the tensor cores,
    then the row search, which keeps each row's scores in its row of pi between steps).  Its
    roofline counts the bytes the call must move -- q and the summaries read once, pi (fp32) and
    tau written once -- against the measured HBM bandwidth."""
    w = WORKLOADS[args.workload]
    if w.T > 32768 or w.seqlens:
        raise SystemExit("--routing takes a fixed-length workload of at most 32K tokens")
    dev = torch.device("cuda", local)
    q, k, _, _ = make_inputs(w, seed=rank)
    nc = -(-w.T // ROUTE_CHUNK)
    kp = torch.nn.functional.pad(k.float(), (0, 0, 0, nc * ROUTE_CHUNK - w.T))
    sig = kp.view(w.B, w.Hkv, nc, ROUTE_CHUNK, w.d).mean(dim=3).to(q.dtype).contiguous()
    qd, sd = q.to(dev), sig.to(dev)
    alpha = _alpha_f32(w.alpha)
    stream = torch.cuda.current_stream(dev)

    def step():
        return ea.route_chunks(qd, sd, alpha, ROUTE_CHUNK, w.n_iter, w.causal, True, 1.0,
                               stream=stream)

    for _ in range(args.warmup):
        pi, tau = step()
    torch.cuda.synchronize()
    assert ea.status(stream) == 0
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for _ in range(args.steps):
            pi, tau = step()
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_one = start.elapsed_time(stop) / args.steps
    ms_step = max_over_ranks(ms_one, world)
    assert ea.status(stream) == 0
    rows = w.B * w.Hq * w.T
    value = job_rate(rows, ms_one, world)
    peaks, peak_src = load_peaks()
    bytes_step = (q.numel() * q.element_size() + sig.numel() * sig.element_size()
                  + pi.numel() * 4 + tau.numel() * 4)
    achieved = bytes_step / (ms_one * 1e-3) / 1e9
    roofline = {"kernel": "entmax_attn_route_chunks (route_scores_kernel + route_chunks_kernel)",
                "bound": "hbm", "achieved": achieved, "peak": float(peaks["hbm_gbs"]),
                "unit": "GB/s", "frac": achieved / float(peaks["hbm_gbs"]), "traffic": None,
                "peak_source": f"{peak_src} hbm_gbs",
                "algorithmic": "q and the summaries read once; pi (fp32) and tau written once"}

    # end to end: q and the summaries in from pinned memory, pi and tau out, every step
    qh, sh = q.pin_memory(), sig.pin_memory()
    pih = torch.empty(pi.shape, dtype=pi.dtype).pin_memory()
    tauh = torch.empty(tau.shape, dtype=tau.dtype).pin_memory()
    e2e_steps = 0 if args.step_only else max(2, min(args.steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        qd.copy_(qh, non_blocking=True)
        sd.copy_(sh, non_blocking=True)
        pi, tau = step()
        pih.copy_(pi, non_blocking=True)
        tauh.copy_(tau, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world) if e2e_steps else None

    cpu = None
    if world == 1 and not args.no_cpu_baseline and not args.step_only:
        from oracle import routing as orout  # the timed CPU baseline only
        import time
        # a bounded sample: the oracle over the first rows of the first (batch, head), grown
        # until it takes about a third of the budget (a causal row prefix sees the same chunks)
        n, spent = 256, 0.0
        while spent < args.cpu_budget / 3 and n <= w.T:
            t0 = time.perf_counter()
            orout.route_chunks(q[:1, :1, :n], sig[:1, :1, :-(-n // ROUTE_CHUNK)], alpha,
                               ROUTE_CHUNK, w.causal, True, 1.0)
            spent = time.perf_counter() - t0
            done = n
            n *= 2
        cpu = {"value": done / spent, "unit": "rows/s", "cores": 1, "kind": "oracle",
               "sample": f"oracle routing of one head's first {done} rows, {spent:.1f} s "
                         "(numpy fp64 per row, one thread)"}

    line = {
        "metric": ROUTE_METRIC, "value": value, "unit": "rows/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if w.dtype == "fp32" else "bf16 scores, f32 search", "data": "synthetic",
        "config": dict(workload_config(w, world), variant="routing", chunk_size=ROUTE_CHUNK,
                       chunks=nc, estimate_diagonal=True,
                       summaries="mean of each chunk's keys"),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": None if e2e_ms is None else {
            "value": job_rate(rows, e2e_ms, world), "unit": "rows/s", "ms_per_step": e2e_ms,
            "h2d_bytes_per_step": q.numel() * q.element_size() + sig.numel() * sig.element_size(),
            "d2h_bytes_per_step": pi.numel() * 4 + tau.numel() * 4},
        "gpu_launches": (2 if w.dtype == "bf16" and w.d in (64, 128) else 1) * args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


ROWS_METRIC = "rows/s of row-wise alpha-entmax"
ROWS_SHAPE = (8192, 16384)  # rows x row length: 8192 score rows of a 16K context


def run_rows(args, rank, world, local):
    """The standalone row-wise alpha-entmax ("Triton Entmax" section of the AdaSplash page) of a
    bf16 matrix of 8192 rows of 16384 scores (standard normal, so a row's support is a few keys
    above its max minus 1 / (alpha - 1)), alpha 1.5, 10 search steps.  A step is one
    entmax_attn_rows call over the resident matrix.  Its roofline counts the bytes the call must
    move -- x read once, p (bf16) and tau written once -- against the measured HBM bandwidth."""
    dev = torch.device("cuda", local)
    n_rows, n = ROWS_SHAPE
    gen = torch.Generator().manual_seed(2000 + rank)
    x = torch.randn(n_rows, n, generator=gen).to(torch.bfloat16)
    xd = x.to(dev)
    alpha, n_iter = _alpha_f32(1.5), 10
    stream = torch.cuda.current_stream(dev)
    p_out = torch.empty_like(xd)
    t_out = torch.empty(n_rows, dtype=torch.float32, device=dev)

    def step():
        return ea.entmax_rows(xd, alpha, n_iter, out=p_out, tau=t_out, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert ea.status(stream) == 0
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for _ in range(args.steps):
            step()
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms_one = start.elapsed_time(stop) / args.steps
    ms_step = max_over_ranks(ms_one, world)
    assert ea.status(stream) == 0
    value = job_rate(n_rows, ms_one, world)
    peaks, peak_src = load_peaks()
    bytes_step = 2 * x.numel() * 2 + n_rows * 4
    achieved = bytes_step / (ms_one * 1e-3) / 1e9
    roofline = {"kernel": "entmax_attn_rows (entmax_rows_kernel)", "bound": "hbm", "achieved": achieved,
                "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                "frac": achieved / float(peaks["hbm_gbs"]), "traffic": None,
                "peak_source": f"{peak_src} hbm_gbs",
                "algorithmic": "x read once; p (bf16) and tau written once"}

    xh = x.pin_memory()
    ph = torch.empty(x.shape, dtype=x.dtype).pin_memory()
    th = torch.empty(n_rows, dtype=torch.float32).pin_memory()
    e2e_steps = 0 if args.step_only else max(2, min(args.steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        xd.copy_(xh, non_blocking=True)
        step()
        ph.copy_(p_out, non_blocking=True)
        th.copy_(t_out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world) if e2e_steps else None

    cpu = None
    if world == 1 and not args.no_cpu_baseline and not args.step_only:
        from oracle import oracle as orc  # the timed CPU baseline only
        import time
        xs = x.float().numpy()
        done, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < args.cpu_budget / 3 and done < n_rows:
            orc.entmax_vec(xs[done], alpha)
            done += 1
        spent = time.perf_counter() - t0
        cpu = {"value": done / spent, "unit": "rows/s", "cores": 1, "kind": "oracle",
               "sample": f"oracle entmax of the first {done} rows, {spent:.1f} s (fp64 C, exact "
                         "tau by sort, one thread)"}

    line = {
        "metric": ROWS_METRIC, "value": value, "unit": "rows/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 in/out, f32 search", "data": "synthetic",
        "config": {"workload": f"rows_{n_rows}x{n}_bf16_a1.5", "rows": n_rows, "row_length": n,
                   "alpha": 1.5, "n_iter": n_iter, "values": "standard normal",
                   "parallelism": f"dp{world} (independent per-rank problems)"},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": None if e2e_ms is None else {
            "value": job_rate(n_rows, e2e_ms, world), "unit": "rows/s", "ms_per_step": e2e_ms,
            "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": x.numel() * 2 + n_rows * 4},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the cpu_baseline figure")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (entmax_attn_bwd) instead of the forward pass")
    ap.add_argument("--rows", action="store_true",
                    help="time the standalone row-wise alpha-entmax (entmax_attn_rows) of an "
                         "8192 x 16384 bf16 matrix")
    ap.add_argument("--routing", action="store_true",
                    help="time entmax block routing over chunk summaries of the workload "
                         "(entmax_attn_route_chunks; fixed length, at most 32K tokens)")
    ap.add_argument("--also", default="auto",
                    help="other workloads timed in the same run (comma list, 'none'; 'auto': "
                         "the 16K workload beside the 128K one and back)")
    ap.add_argument("--step-only", action="store_true",
                    help="time the step only (no tile-path comparison, e2e, cpu baseline or "
                         "second workload): for profiler launch lists")
    ap.add_argument("--fp8-screen", action="store_true",
                    help="time the step with the FP8-screened tau pass (bf16, d = 128)")
    ap.add_argument("--no-block-mask", action="store_true",
                    help="time the variant without block mask (output pass over every causal "
                         "tile); the effective FLOPs keep counting active tiles only")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "native":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        return run_reference(args, rank, world)
    rank, world, local = dist_setup(args)
    try:
        if args.backward:
            return run_backward(args, rank, world, local)
        if args.routing:
            return run_routing(args, rank, world, local)
        if args.rows:
            return run_rows(args, rank, world, local)
        return run_native(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
