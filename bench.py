#!/usr/bin/env python
"""Benchmark of the block-sparse video self-attention path on B200.

One step = one pass of the whole hot path over one batch of synthetic input,
on the SPADE adaptive workload (1 x 24 heads, grid 32x48x80, S = 122880,
D = 128, bf16, candidate tiles (1,8,16), (2,8,8), (4,4,8), 10 % top-k budget):
per-head tiling choice -> block summaries -> block scores -> top-k + sink +
diagonal lists -> block-sparse attention.  The permutation to each head's
tile-contiguous order and back is done inside the summaries and attention
kernels (TMA boxes in, token rows out); the explicit permute -> ... ->
unpermute composition is timed beside it as a secondary line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  `value` is the effective TFLOP/s on the
computed blocks (4 * 128 * 128 * D FLOPs per listed block pair) over the whole
step, all ranks together (each rank runs its own batch: weak scaling).
`--impl reference` times the fp64 CPU oracle on a bounded sample instead.
"""

from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, make_qkv  # noqa: E402

METRIC = "sparse-attn ms/call & effective TFLOP/s on computed blocks (frac of B200 peak)"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "spade_adaptive_s122880"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("attention_pp.cu", "common.cuh"):
        h.update(open(os.path.join(ROOT, "block_sparse_self_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per attention launch from a committed ncu summary, if the
    kernel source has not changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "attention_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(workload)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", uuid, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[3:7]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "power_w_max": max(r[2] for r in rows)}


# --------------------------------------------------------------------------
# the GPU step
# --------------------------------------------------------------------------

PHASES = ("select_tiling", "permute", "summaries", "scores", "topk", "attention", "unpermute")
TILED_PHASES = ("select_tiling", "summaries", "scores", "topk", "attention")


class SpadeStep:
    """The SPADE path on preallocated device buffers (inputs resident in HBM).

    tiled=True: summaries and attention read T-major Q/K/V through each head's
    tiling and attention writes T-major O (no permuted copies); tiled=False:
    explicit permute / unpermute around the same kernels."""

    def __init__(self, w, q, k, v, tiled: bool = True):
        import block_sparse_self_b200 as vsa
        self.vsa, self.w = vsa, w
        self.q, self.k, self.v = q, k, v
        self.tiles = list(w.tiles)
        self.block = w.tiles[0][0] * w.tiles[0][1] * w.tiles[0][2]
        self.kk = w.k
        self.tiled = tiled and self.block == 128 and vsa.tiled_supported(self.tiles)
        self.phases = TILED_PHASES if self.tiled else PHASES
        self.events = []

    def launches(self) -> int:
        sel = 2 if len(self.tiles) > 1 else 0
        if self.tiled:
            return sel + 2 + 1 + 1 + 1
        return sel + 3 + 2 + 1 + 1 + 1 + 1

    def __call__(self, record: bool):
        vsa, w = self.vsa, self.w
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(self.phases) + 1)] if record else None
        n = [0]

        def mark():
            if record:
                ev[n[0]].record()
            n[0] += 1

        mark()
        choice = vsa.select_tiling(self.q, w.grid, self.tiles) if len(self.tiles) > 1 else None
        mark()
        if self.tiled:
            qmax, qmin = vsa.block_summaries_tiled(self.q, w.grid, self.tiles, choice, self.block)
            kmax, kmin = vsa.block_summaries_tiled(self.k, w.grid, self.tiles, choice, self.block)
        else:
            qp, kp, vp = (vsa.permute(x, w.grid, self.tiles, choice) for x in (self.q, self.k, self.v))
            mark()
            qmax, qmin = vsa.block_summaries(qp, self.block)
            kmax, kmin = vsa.block_summaries(kp, self.block)
        mark()
        scores = vsa.block_scores(qmax, qmin, kmax, kmin)
        mark()
        idx, cnt = vsa.topk_block_mask(scores, self.kk, w.n_sink_blocks, w.diag_halfwidth)
        mark()
        if self.tiled:
            o = vsa.block_sparse_attention_tiled(self.q, self.k, self.v, w.grid, self.tiles, choice, idx, cnt)
            mark()
        else:
            op = vsa.block_sparse_attention(qp, kp, vp, idx, cnt, self.block)
            mark()
            o = vsa.unpermute(op, w.grid, self.tiles, choice)
            mark()
        if record:
            self.events.append(ev)
        self.last = dict(cnt=cnt, o=o, scores=scores, idx=idx)
        return o

    def phase_ms(self):
        out = {p: [] for p in self.phases}
        for ev in self.events:
            for i, p in enumerate(self.phases):
                out[p].append(ev[i].elapsed_time(ev[i + 1]))
        return {p: float(np.mean(v)) for p, v in out.items() if v}


def computed_flops(cnt: torch.Tensor, block: int, D: int) -> float:
    return float(cnt.to(torch.int64).sum().item()) * 4.0 * block * block * D


def mask_pipeline_bytes(w, BH: int) -> float:
    """Algorithmic HBM bytes of summaries + scores + top-k (no re-reads)."""
    S, D, nb = w.S, w.D, w.nb
    cap = min(nb, w.k + w.n_sink_blocks + (2 * w.diag_halfwidth + 1 if w.diag_halfwidth >= 0 else 0))
    summ = 2 * BH * S * D * 2 + 4 * BH * nb * D * 2
    scores = 4 * BH * nb * D * 2 + BH * nb * nb * 4
    topk = BH * nb * nb * 4 + BH * nb * (cap + 1) * 4
    return float(summ + scores + topk)


def rank_workload(w, rank: int):
    """Each rank's own batch of heads (weak scaling): the same shapes, its own
    seeded inputs, no data exchanged between ranks."""
    from dataclasses import replace
    return replace(w, seed_base=w.seed_base + 100 * rank)


def reduce_over_ranks(x: float, op: str, dist_on: bool, device) -> float:
    """MAX (times) or SUM (work) of a per-rank number over all ranks."""
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if dist_on:
        ops = {"max": torch.distributed.ReduceOp.MAX, "sum": torch.distributed.ReduceOp.SUM}
        torch.distributed.all_reduce(t, op=ops[op])
    return float(t.item())


def time_steps(fn, steps: int, warmup: int, dist_on: bool):
    for _ in range(warmup):
        fn(False)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        fn(True)
    e.record()
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    return s.elapsed_time(e) / steps


def run_e2e(w, step, q, k, v, steps: int, groups: int = 8):
    """Same metric through the public API with host buffers: spade_attention_host
    takes Q, K, V in pinned host memory and returns O there; every step's H2D
    copies and D2H copy are inside the timed region (the call overlaps the
    copies of one group of heads with the kernels of another)."""
    import block_sparse_self_b200 as vsa
    qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    kw = dict(topk=w.k, n_sink_blocks=w.n_sink_blocks, diag_halfwidth=w.diag_halfwidth)

    def once():
        vsa.spade_attention_host(qh, kh, vh, w.grid, list(w.tiles), out=oh, chunks=groups, **kw)

    once()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        once()
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    # the host path computes the same output as the device step
    ref = step(False)
    torch.cuda.synchronize()
    assert torch.equal(oh, ref.cpu()), "host-buffer path differs from the device step"
    h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size()
    return ms, h2d, d2h


# --------------------------------------------------------------------------
# the fp64 oracle on the host (CPU baseline / reference arm)
# --------------------------------------------------------------------------

def oracle_sample(w, qh, kh, vh, n_query_blocks: int, seed: int = 0):
    """Time the oracle on one head: the mask pipeline in full, attention on a
    few query blocks.  Returns (mask_seconds, attn_seconds, sampled_pairs,
    mean_list_length)."""
    import oracle
    t0 = time.perf_counter()
    tiles = list(w.tiles)
    choice = oracle.select_tiling(qh, w.grid, tiles)[0] if len(tiles) > 1 else 0
    tile = tiles[choice]
    block = tile[0] * tile[1] * tile[2]
    perm = oracle.tile_permutation(w.grid, tile)
    qp, kp, vp = (oracle.permute_rows(x, perm) for x in (qh, kh, vh))
    qmax, qmin = oracle.block_minmax(qp, block)
    kmax, kmin = oracle.block_minmax(kp, block)
    score = oracle.block_scores(qmax, qmin, kmax, kmin)
    idx, cnt = oracle.topk_block_list(score, w.k, w.n_sink_blocks, w.diag_halfwidth)
    t1 = time.perf_counter()
    rng = np.random.default_rng(seed)
    blocks = np.sort(rng.choice(w.nb, n_query_blocks, replace=False))
    rows = np.concatenate([np.arange(b * block, (b + 1) * block) for b in blocks])
    t2 = time.perf_counter()
    oracle.block_sparse_attention(qp, kp, vp, idx, cnt, block, 0, None, rows)
    t3 = time.perf_counter()
    return t1 - t0, t3 - t2, int(cnt[blocks].sum()), float(cnt.mean())


def cpu_estimate(w, BH, total_pairs, mask_s, attn_s, pairs, mean_cnt):
    if total_pairs is None:
        total_pairs = mean_cnt * w.nb * BH
    est_s = mask_s * BH + attn_s * (total_pairs / max(pairs, 1))
    flops = total_pairs * 4.0 * w.block * w.block * w.D
    return flops / est_s / 1e12, est_s


def host_head(w, head: int = 0):
    """One head of the workload's inputs generated on the host."""
    q, k, v = make_qkv(w, device="cpu", B=1, heads=head + 1)
    return tuple(x[0, head].float().numpy() for x in (q, k, v))


# --------------------------------------------------------------------------
# arms
# --------------------------------------------------------------------------

def workload_config(w, BH_rank: int, n: int):
    return {"workload": w.name, "B": w.B, "heads": w.heads, "grid": list(w.grid), "S": w.S, "D": w.D,
            "block": w.block, "tiles": [list(t) for t in w.tiles], "topk": w.k,
            "budget": w.budget, "n_sink_blocks": w.n_sink_blocks, "diag_halfwidth": w.diag_halfwidth,
            "values": w.values, "per_rank_bh": BH_rank, "parallelism": f"weak x{n} (independent heads per rank)",
            "l2": "inputs 3 x %.2f GB per step, larger than the 126 MB L2; no flush" %
                  (w.B * w.heads * w.S * w.D * 2 / 1e9)}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    n = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    qh, kh, vh = host_head(w, 0)
    BH = w.B * w.heads
    for _ in range(args.warmup):
        oracle_sample(w, qh, kh, vh, 2)
    tot_mask = tot_attn = 0.0
    tot_pairs = 0
    mean_cnt = 0.0
    t0 = time.perf_counter()
    for s in range(args.steps):
        m, a, p, mc = oracle_sample(w, qh, kh, vh, 4, seed=s)
        tot_mask += m
        tot_attn += a
        tot_pairs += p
        mean_cnt = mc
    wall = time.perf_counter() - t0
    value, est_s = cpu_estimate(w, BH, None, tot_mask / args.steps, tot_attn, tot_pairs, mean_cnt)
    cores = len(os.sched_getaffinity(0))
    sample = (f"head 0 of {BH}: tiling choice, permutation, summaries, scores and top-k in full; attention on "
              f"4 of {w.nb} query blocks per step; extrapolated by heads and by computed block pairs")
    # the step time is extrapolated from timed samples (see `sample`), not
    # timed whole: `estimated` says so
    line = {"impl": "reference", "metric": METRIC, "value": value * n, "unit": UNIT, "n_gpus": n,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": est_s * 1e3, "estimated": True,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, BH, n),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                             "wall_s": wall},
            "e2e": {"value": value * n, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def window_tile_pairs(S: int, window: int, sink: int, bn: int = 128) -> int:
    """128x128 (query tile, key tile) pairs the window kernel computes for one
    head: the local key range of each query tile plus the sink tiles
    (_key_ranges_for_block at tile granularity), or every pair when dense."""
    nt = (S + bn - 1) // bn
    if window >= S:
        return nt * nt
    half, sb = window // 2, (sink + bn - 1) // bn
    total = 0
    for t in range(nt):
        qs, qe = t * bn, min(S, t * bn + bn)
        lb0, lb1 = max(0, qs - half) // bn, (min(S, qe + half) + bn - 1) // bn
        if sb == 0:
            total += lb1 - lb0
        elif lb0 <= sb:
            total += max(lb1, sb)
        else:
            total += sb + lb1 - lb0
    return total


EXTRAS = ("window", "fixed", "padded", "structured", "explicit", "compensated", "topp", "profile")


def extra_workloads(steps: int, want=EXTRAS):
    """Secondary lines: window (S=30720), SPADE fixed tiling (S=30720), SPADE
    adaptive on a padded 16 x 45 x 80 grid (S=57600), structured masks on a
    CFG pair (S=122880), and dense SDPA context."""
    import block_sparse_self_b200 as vsa
    out = {}

    def timed(fn, n=steps, warm=2):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(n):
            fn()
        e.record()
        torch.cuda.synchronize()
        return s.elapsed_time(e) / n

    # window attention: computed 128x128 tiles counted by the kernel's enumeration
    if "window" in want:
        window_line(out, timed)
    if "fixed" in want:
        fixed_line(out, timed, steps)
    if "padded" in want:
        padded_line(out, timed, steps)
    if "structured" in want:
        structured_lines(out, timed, steps)
    return out


def window_line(out, timed):
    import block_sparse_self_b200 as vsa
    w = WORKLOADS["window_s30720"]
    q, k, v = make_qkv(w, device="cuda")
    ms = timed(lambda: vsa.window_attention(q, k, v, w.window, w.sink, chunk_size=w.chunk))
    pairs = window_tile_pairs(w.S, w.window, w.sink)
    flops = pairs * 4.0 * 128 * 128 * w.D * w.B * w.heads
    out[w.name] = {"ms_per_call": ms, "tflops": flops / ms / 1e9, "block_pairs_per_head": pairs}
    dense = timed(lambda: torch.nn.functional.scaled_dot_product_attention(q, k, v), n=3, warm=1)
    out[w.name]["dense_sdpa_ms_context"] = dense
    del q, k, v


def fixed_line(out, timed, steps):
    w = WORKLOADS["spade_fixed_s30720"]
    q, k, v = make_qkv(w, device="cuda")
    st = SpadeStep(w, q, k, v)
    ms = timed(lambda: st(True), n=steps)
    ph = st.phase_ms()
    fl = computed_flops(st.last["cnt"], st.block, w.D)
    out[w.name] = {"ms_per_step": ms, "tflops_step": fl / ms / 1e9, "attn_ms": ph["attention"],
                   "attn_tflops": fl / ph["attention"] / 1e9, "phase_ms": ph}
    del q, k, v, st


def padded_line(out, timed, steps):
    # SPADE with adaptive tiling on a grid the candidates do not divide
    # (16 x 45 x 80, zero-padded to 16 x 48 x 80 inside the kernels; every
    # 128-position query block of it holds real tokens, so the counted blocks
    # are the computed ones)
    import block_sparse_self_b200 as vsa
    w = WORKLOADS["spade_adaptive_pad_s57600"]
    q, k, v = make_qkv(w, device="cuda")
    st = SpadeStep(w, q, k, v)
    ms = timed(lambda: st(True), n=steps)
    ph = st.phase_ms()
    fl = computed_flops(st.last["cnt"], st.block, w.D)
    out[w.name] = {"ms_per_step": ms, "tflops_step": fl / ms / 1e9, "attn_ms": ph["attention"],
                   "attn_tflops": fl / ph["attention"] / 1e9, "phase_ms": ph,
                   "padded_grid": list(vsa.padded_grid(w.grid, w.tiles))}
    del q, k, v, st


def structured_lines(out, timed, steps):
    import block_sparse_self_b200 as vsa
    # structured masks on a CFG pair.  The attention kernel runs in the mode
    # structured_attention picks: T-major directly for whole-frame tiles
    # (spatial), through TMA boxes for sliding tiles, and for the temporal
    # tile through (T, 1, 128/T) boxes with a strided group mask.
    w = WORKLOADS["structured_s122880"]
    q, k, v = make_qkv(w, device="cuda")
    res = {}
    for kind in w.structured:
        stile = vsa.structured_tile(kind, w.grid, w.sliding_tile)
        idx, cnt, g = vsa.structured_block_list(kind, w.grid, 128, w.sliding_tile, w.sliding_radius,
                                                cap=1 if kind == "temporal" and 128 % w.grid[0] == 0 else None)
        if stile[1] == w.grid[1] and stile[2] == w.grid[2]:
            mode = "t-major"
            fn = lambda: vsa.block_sparse_attention(q, k, v, idx, cnt, 128, g)  # noqa: E731
        elif g == 0 and vsa.tiled_supported([stile]):
            mode = "tiled"
            fn = lambda: vsa.block_sparse_attention_tiled(q, k, v, w.grid, [stile], None, idx, cnt)  # noqa: E731
        elif kind == "temporal" and 128 % w.grid[0] == 0 and w.grid[2] % (128 // w.grid[0]) == 0:
            mode = "tiled, strided groups"
            sg = 128 // w.grid[0]
            fn = lambda: vsa.block_sparse_attention_tiled(q, k, v, w.grid, [(w.grid[0], 1, sg)], None, idx, cnt,  # noqa: E731
                                                          group_stride=sg if sg > 1 else 0)
        else:
            mode = "permuted copies"
            qp, kp, vp = (vsa.permute(x, w.grid, [stile]) for x in (q, k, v))
            fn = lambda: vsa.block_sparse_attention(qp, kp, vp, idx, cnt, 128, g)  # noqa: E731
        ms = timed(fn, n=max(2, steps // 2))
        call_ms = timed(lambda: vsa.structured_attention(q, k, v, kind, w.grid, 128, tile=w.sliding_tile,
                                                         radius=w.sliding_radius), n=max(2, steps // 2))
        fl = float(cnt.to(torch.int64).sum().item()) * 4.0 * 128 * 128 * w.D * w.B * w.heads
        res[kind] = {"attn_ms": ms, "tflops": fl / ms / 1e9, "group_size": g, "mode": mode,
                     "structured_attention_call_ms": call_ms}
        fn = None
        qp = kp = vp = None
    out[w.name] = res


def compensated_line(w, q, k, v, idx, cnt, n_rep: int):
    """Centroid-compensated attention against the plain block-sparse attention
    on the same inputs and lists, both in tiled mode (T-major q, k, v, each
    head's chosen tiling, no permuted copies).  Algorithmic FLOPs: 4 * 128 *
    128 * D per listed block pair plus 4 * 128 * D per (query block, skipped
    block) centroid."""
    import block_sparse_self_b200 as vsa
    tiles = list(w.tiles)
    choice = vsa.select_tiling(q, w.grid, tiles)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(n_rep):
            fn()
        e.record()
        torch.cuda.synchronize()
        return s.elapsed_time(e) / n_rep

    comp_ms = timed(lambda: vsa.centroid_compensated_attention_tiled(q, k, v, w.grid, tiles, choice, idx, cnt))
    plain_ms = timed(lambda: vsa.block_sparse_attention_tiled(q, k, v, w.grid, tiles, choice, idx, cnt))
    pairs = float(cnt.to(torch.int64).sum().item())
    BH, nb = w.B * w.heads, w.nb
    skipped = BH * nb * nb - pairs
    flops = pairs * 4.0 * 128 * 128 * w.D + skipped * 4.0 * 128 * w.D
    # tensor work the centroid pass runs: per query block, every 128-centroid
    # tile holding a skipped block, with the hi and lo halves of both products
    nct = (nb + 127) // 128
    rows = idx.view(-1, idx.shape[-1]).to(torch.int64)
    kept = torch.zeros(rows.shape[0], nct + 1, dtype=torch.int64, device=rows.device)
    kept.scatter_add_(1, torch.where(rows >= 0, rows // 128, nct), torch.ones_like(rows))
    size = torch.tensor([min(128, nb - 128 * c) for c in range(nct)], device=rows.device)
    tiles_run = float((kept[:, :nct] < size).sum().item())
    executed = pairs * 4.0 * 128 * 128 * w.D + tiles_run * 8.0 * 128 * 128 * w.D
    burst = load_peaks()[0].get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    return {"ms_per_call": comp_ms, "tflops": flops / comp_ms / 1e9, "frac_of_burst": flops / comp_ms / 1e9 / burst,
            "executed_tflops": executed / comp_ms / 1e9, "plain_attention_ms": plain_ms,
            "compensation_overhead": comp_ms / plain_ms - 1.0, "skipped_blocks_per_row": skipped / (BH * nb),
            "centroid_tiles_per_query_block": tiles_run / (BH * nb),
            "out_dtype": "bf16", "layout": "T-major, tiled (each head's chosen tiling, no permuted copies)"}


def run_ours(args, w):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    torch.cuda.set_device(local)
    if dist_on:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    import block_sparse_self_b200 as vsa
    vsa.lib()
    peaks, peak_src = load_peaks()

    # each rank: its own batch of heads (weak scaling, no data-path collective)
    wr = rank_workload(w, rank)
    q, k, v = make_qkv(wr, device="cuda")
    step = SpadeStep(wr, q, k, v)
    BH = w.B * w.heads

    clocks = ClockSampler(local)
    ms = time_steps(step, args.steps, args.warmup, dist_on)
    clk = clocks.stop()
    ph = step.phase_ms()
    flops = computed_flops(step.last["cnt"], step.block, w.D)
    vsa.device_status()

    ms_max = reduce_over_ranks(ms, "max", dist_on, "cuda")
    total_flops = reduce_over_ranks(flops, "sum", dist_on, "cuda")  # every rank's computed blocks
    value = total_flops / ms_max / 1e9  # TFLOP/s (ms -> 1e-3 s, 1e12)

    attn_ms = ph["attention"]
    achieved = flops / attn_ms / 1e9
    # the timed region lasts well under a second, so the burst figure is the
    # peak; the seconds-long sustained figure is reported beside it
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    mask_ms = ph["summaries"] + ph["scores"] + ph["topk"]
    mask_bytes = mask_pipeline_bytes(w, BH)
    mask_gbs = mask_bytes / mask_ms / 1e6
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    kname = ("attn_pp_kernel<128,false,true,false> (block-sparse, tiled)" if step.tiled
             else "attn_pp_kernel<128,false,false,false> (block-sparse)")
    mask = {"bound": "hbm", "kernels": "summaries (Q, K) + scores + top-k", "ms": mask_ms, "achieved": mask_gbs,
            "peak": hbm, "unit": "GB/s", "frac": mask_gbs / hbm, "bytes": mask_bytes,
            "peak_kind": f"hbm_gbs ({peak_src})"}
    roofline = {"bound": "tensor", "kernel": kname,
                "achieved": achieved, "peak": burst, "unit": "TFLOP/s", "frac": achieved / burst,
                "peak_kind": f"bf16_tflops, burst ({peak_src})",
                "frac_sustained": achieved / sustained, "peak_sustained": sustained,
                "traffic": profiled_traffic(w.name), "attn_ms_per_call": attn_ms,
                "flops_per_launch": flops, "mask_pipeline": mask,
                "phase_ms": {p: round(v, 4) for p, v in ph.items()}}

    e2e = None
    if not args.no_e2e:
        groups = args.e2e_groups if args.e2e_groups > 0 else w.B * w.heads
        e_ms, h2d, d2h = run_e2e(w, step, q, k, v, max(2, args.steps // 2), groups)
        e_max = reduce_over_ranks(e_ms, "max", dist_on, "cuda")
        e2e = {"value": total_flops / e_max / 1e9, "unit": UNIT, "ms_per_step": e_max,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "groups": groups}

    extra = None
    want = () if args.no_extra else tuple(args.extras.split(","))
    if rank == 0 and world == 1 and want:
        extra = extra_workloads(max(3, args.steps // 2), want)
        if step.tiled and "explicit" in want:  # the same step with explicit permuted copies, for comparison
            ex = SpadeStep(wr, q, k, v, tiled=False)
            ex_ms = time_steps(ex, max(3, args.steps // 2), 3, False)
            extra["explicit_permute_" + w.name] = {"ms_per_step": ex_ms, "phase_ms": ex.phase_ms(),
                                                   "same_output": bool(torch.equal(ex.last["o"], step.last["o"]))}
            del ex
        # centroid-compensated attention on the same lists: the kept blocks as
        # above plus every skipped block as its centroid (tiled mode, each
        # head's tiling; bf16 output)
        if "compensated" in want:
            extra["compensated_" + w.name] = compensated_line(w, q, k, v, step.last["idx"], step.last["cnt"],
                                                              max(3, args.steps // 2))
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        n_rep = 5
        if "topp" in want:
            # top-p (mass budget) lists on the same scores, in place of the top-k lists
            sc = step.last["scores"]
            p_mass, p_scale = 0.5, 1.0 / math.sqrt(w.D)
            tp = {}
            for _ in range(3):
                vsa.topp_block_mask(sc, p_mass, p_scale)
            ev[0].record()
            for _ in range(n_rep):
                ti, tc = vsa.topp_block_mask(sc, p_mass, p_scale)
            ev[1].record()
            torch.cuda.synchronize()
            tp["ms_per_call"] = ev[0].elapsed_time(ev[1]) / n_rep
            tp["p"], tp["scale"] = p_mass, p_scale
            tp["mean_blocks_per_row"] = float(tc.float().mean().item())
            tp["bytes"] = float(sc.numel() * 4 + ti.numel() * 4 + tc.numel() * 4)
            tp["gbs"] = tp["bytes"] / tp["ms_per_call"] / 1e6
            extra["topp_lists_" + w.name] = tp
            del ti, tc
        if "profile" in want:
            # head profile (spatial or temporal pattern per head) on 128 sampled query rows:
            # K is read once per head (the bound); Q contributes only the sampled rows
            rows = vsa.sample_query_rows(w.S, 128, seed=0, device=q.device)
            for _ in range(3):
                vsa.head_profile(q, k, w.grid, rows)
            ev[0].record()
            for _ in range(n_rep):
                hk, hm = vsa.head_profile(q, k, w.grid, rows)
            ev[1].record()
            torch.cuda.synchronize()
            hp_ms = ev[0].elapsed_time(ev[1]) / n_rep
            hk2, _ = vsa.head_profile(q, k, w.grid, rows, rule="mass_per_key")
            hp_bytes = float(k.numel() * 2 + BH * 128 * w.D * 2)
            extra["head_profile_" + w.name] = {
                "ms_per_call": hp_ms, "rows": 128, "bytes": hp_bytes, "gbs": hp_bytes / hp_ms / 1e6,
                "frac_hbm": hp_bytes / hp_ms / 1e6 / hbm,
                "tflops": 2.0 * 2 * 128 * w.S * w.D * BH / hp_ms / 1e9,
                "temporal_heads": int(hk.sum().item()), "temporal_heads_mass_per_key": int(hk2.sum().item()),
                "heads": BH}
            del hk, hm, hk2

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        qh, kh, vh = (x[0, 0].float().cpu().numpy() for x in (q, k, v))
        m, a, p, mc = oracle_sample(w, qh, kh, vh, 8)
        total_pairs = float(step.last["cnt"].to(torch.int64).sum().item())
        cval, _ = cpu_estimate(w, BH, total_pairs, m, a, p, mc)
        cpu = {"value": cval, "unit": UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
               "sample": f"head 0 of {BH}: tiling choice, permutation, summaries, scores and top-k in full "
                         f"({m:.1f} s); attention on 8 of {w.nb} query blocks ({a:.1f} s); extrapolated by "
                         f"heads and by computed block pairs"}

    if dist_on:
        torch.distributed.barrier()
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(w, BH, world),
                "roofline": roofline, "mask_pipeline": mask,
                "phase_ms": ph, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": step.launches() * args.steps, "clocks": clk, "per_workload": extra}
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-groups", type=int, default=0,
                    help="groups of (b, head) rows in the host-buffer run (0: one group per (b, head))")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--extras", default=",".join(EXTRAS),
                    help="comma-separated secondary lines to run (%s); --no-extra runs none" % ",".join(EXTRAS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--heads", type=int, default=None,
                    help="run the workload with this many heads (smaller cases for profilers; not a bench line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    unknown = set(args.extras.split(",")) - set(EXTRAS)
    if unknown:
        ap.error(f"unknown --extras {sorted(unknown)}; choose from {EXTRAS}")
    w = WORKLOADS[args.workload]
    if args.heads is not None:
        if args.heads < 1:
            ap.error("--heads must be >= 1")
        w = dataclasses.replace(w, heads=args.heads)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
