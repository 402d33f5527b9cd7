"""Seeded synthetic inputs for block-sparse video self-attention.

This module is shared by the tests, the benchmark and the oracle-based checks.
It holds no arithmetic of the attention method itself: it only draws tensors
of the shapes, value distributions and structure that the video-DiT workloads
have, and names those workloads.

Token order is T-major: token (t, h, w) of a (T, Hg, Wg) latent sits at
index (t * Hg + h) * Wg + w, as the "Sparse-attention roadmap for video DiTs"
page fixes in its shared conventions.

Two value distributions are provided:

* ``integer_grid`` -- i.i.d. values from {-4, ..., 4} / 4.  Every value is
  exact in bf16 and every product and short sum of them is exact in fp32, so
  block scores are exact and index outputs can be compared bit for bit.
* ``quantized_smooth_qkv`` -- the smooth fields below rounded onto that same
  {-4..4}/4 grid (per head, about two grid steps per standard deviation,
  clipped): exact scores like ``integer_grid``, but with the spatial or
  temporal cohesion of the smooth fields, so tiling choices have clear
  margins.
* ``smooth_qkv`` -- Q and K are smooth 3-D random fields over (t, h, w): per
  head 16 random low-frequency plane waves, mixed per channel with random
  amplitude and phase, plus N(0, 0.5^2) noise, then scaled per head so that
  the raw scaled scores have a standard deviation near 3.  V is N(0, 1).
  An "adaptive" variant draws, per head, either a spatially cohesive field
  (slow in h and w, fast in t) or a temporally cohesive one (slow in t, fast
  in h and w), so that different heads prefer different tilings.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence, Tuple

import torch

Dims3 = Tuple[int, int, int]


# --------------------------------------------------------------------------
# Workload catalogue (sizes of the video-DiT attention workloads)
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    grid: Dims3
    D: int
    dtype: torch.dtype
    values: str                       # "integer", "smooth" or "smooth_adaptive" ("integer_adaptive" on request)
    seed_base: int
    tiles: Tuple[Dims3, ...] = ()
    block: int = 128
    budget: Optional[float] = None    # fraction of key blocks kept by top-k
    topk: Optional[int] = None        # explicit k (overrides budget)
    n_sink_blocks: int = 1
    diag_halfwidth: int = 0
    window: Optional[int] = None
    sink: int = 0
    chunk: Optional[int] = None
    structured: Tuple[str, ...] = ()  # "spatial", "temporal", "sliding_tile", "sliding_tile_centered"
    sliding_tile: Dims3 = (4, 8, 8)
    sliding_radius: Dims3 = (1, 1, 1)

    @property
    def S(self) -> int:
        return self.grid[0] * self.grid[1] * self.grid[2]

    @property
    def nb(self) -> int:
        """Blocks of the grid itself (a grid the tiles do not divide has more
        blocks once padded; its workloads give topk explicitly)."""
        return self.S // self.block

    @property
    def k(self) -> int:
        """Top-k key blocks per query block: max(1, floor(budget * nb))."""
        if self.topk is not None:
            return self.topk
        return max(1, int(math.floor(self.budget * self.nb)))


WORKLOADS = {
    # Tiny correctness case: fp32, D=64, (4,8,8) grid, tile (2,4,4) -> 8 blocks
    # of 32, top-2 plus sink block 0 and the diagonal; and a window of 64 with
    # 16 sinks.
    "tiny_s256": Workload(
        name="tiny_s256", B=1, heads=2, grid=(4, 8, 8), D=64,
        dtype=torch.float32, values="integer", seed_base=0,
        tiles=((2, 4, 4),), block=32, topk=2, window=64, sink=16),
    # Symmetric sliding window with sinks, S = 30720.
    "window_s30720": Workload(
        name="window_s30720", B=1, heads=24, grid=(20, 32, 48), D=128,
        dtype=torch.bfloat16, values="smooth", seed_base=1000,
        window=4096, sink=256, chunk=128),
    # SPADE block-sparse attention, one fixed tiling, S = 30720, 17 % budget.
    "spade_fixed_s30720": Workload(
        name="spade_fixed_s30720", B=1, heads=40, grid=(20, 32, 48), D=128,
        dtype=torch.bfloat16, values="smooth", seed_base=2000,
        tiles=((1, 8, 16),), budget=0.17),
    # SPADE with per-head adaptive tiling, S = 122880, 10 % budget.
    "spade_adaptive_s122880": Workload(
        name="spade_adaptive_s122880", B=1, heads=24, grid=(32, 48, 80),
        D=128, dtype=torch.bfloat16, values="smooth_adaptive", seed_base=3000,
        tiles=((1, 8, 16), (2, 8, 8), (4, 4, 8)), budget=0.10),
    # SPADE with adaptive tiling on a grid the candidates do not divide: the
    # 16 x 45 x 80 latent the pages name for it (no candidate's height divides
    # 45).  S = 57600 real tokens; k = 48 is 10 % of the 480 blocks of the
    # zero-padded 16 x 48 x 80 grid the candidates tile.
    "spade_adaptive_pad_s57600": Workload(
        name="spade_adaptive_pad_s57600", B=1, heads=24, grid=(16, 45, 80),
        D=128, dtype=torch.bfloat16, values="smooth_adaptive", seed_base=5000,
        tiles=((1, 8, 16), (2, 8, 8), (4, 4, 8)), topk=48),
    # Structured static masks on a CFG pair, S = 122880.
    "structured_s122880": Workload(
        name="structured_s122880", B=2, heads=24, grid=(32, 48, 80), D=128,
        dtype=torch.bfloat16, values="smooth", seed_base=4000,
        structured=("spatial", "temporal", "sliding_tile", "sliding_tile_centered")),
}


# --------------------------------------------------------------------------
# Generators
# --------------------------------------------------------------------------

def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def integer_grid(shape: Sequence[int], seed: int, dtype=torch.bfloat16,
                 device="cpu") -> torch.Tensor:
    """I.i.d. values from {-4..4}/4 (exact in bf16 and fp32)."""
    g = _gen(seed, device)
    x = torch.randint(-4, 5, tuple(shape), generator=g, device=device,
                      dtype=torch.int32)
    return (x.to(torch.float32) / 4.0).to(dtype)


def _coords(grid: Dims3, device):
    T, Hg, Wg = grid
    t = torch.arange(T, device=device, dtype=torch.float32)
    h = torch.arange(Hg, device=device, dtype=torch.float32)
    w = torch.arange(Wg, device=device, dtype=torch.float32)
    tt = (t / T).repeat_interleave(Hg * Wg)
    hh = (h / Hg).repeat_interleave(Wg).repeat(T)
    ww = (w / Wg).repeat(T * Hg)
    return tt, hh, ww


# frequency ranges (max |f| along t, along h and w) per head kind
_KIND_FREQ = {
    "generic": (3, 3),
    "spatial": (8, 1),    # fast along t, slow along h, w: same-frame cohesion
    "temporal": (1, 6),   # slow along t, fast along h, w: same-(h,w) cohesion
}


def _wave_field(grid: Dims3, D: int, kind: str, g: torch.Generator, device,
                n_waves: int = 16, noise_sigma: float = 0.5) -> torch.Tensor:
    """One head's [S, D] smooth field: 16 plane waves mixed per channel."""
    ft_max, fs_max = _KIND_FREQ[kind]
    tt, hh, ww = _coords(grid, device)
    ft = torch.randint(-ft_max, ft_max + 1, (n_waves,), generator=g, device=device).float()
    fh = torch.randint(-fs_max, fs_max + 1, (n_waves,), generator=g, device=device).float()
    fw = torch.randint(-fs_max, fs_max + 1, (n_waves,), generator=g, device=device).float()
    phase = 2.0 * math.pi * (tt[:, None] * ft[None, :] + hh[:, None] * fh[None, :]
                             + ww[:, None] * fw[None, :])
    basis = torch.cat([torch.cos(phase), torch.sin(phase)], dim=1)      # [S, 2n]
    mix = torch.randn(2 * n_waves, D, generator=g, device=device) / 4.0  # amp+phase per channel
    noise = torch.randn(basis.shape[0], D, generator=g, device=device) * noise_sigma
    return basis @ mix + noise


def head_kinds(workload: Workload, device="cpu") -> list:
    """Per-(b, head) field kind; adaptive workloads draw a fair coin per head."""
    n = workload.B * workload.heads
    if workload.values != "smooth_adaptive":
        return ["generic"] * n
    g = _gen(workload.seed_base + 7, "cpu")
    coin = torch.randint(0, 2, (n,), generator=g)
    return ["spatial" if c == 0 else "temporal" for c in coin.tolist()]


def smooth_qkv(B: int, heads: int, grid: Dims3, D: int, seed: int,
               kinds: Optional[Sequence[str]] = None, dtype=torch.bfloat16,
               device="cpu", score_std: float = 3.0, n_pairs: int = 4096):
    """Smooth-field Q, K and N(0,1) V of shape [B, heads, S, D]."""
    S = grid[0] * grid[1] * grid[2]
    kinds = list(kinds) if kinds is not None else ["generic"] * (B * heads)
    q = torch.empty(B, heads, S, D, dtype=dtype, device=device)
    k = torch.empty_like(q)
    gq, gk, gv, gs = (_gen(seed + o, device) for o in (0, 1, 2, 3))
    scale = D ** -0.5
    for b in range(B):
        for h in range(heads):
            kind = kinds[b * heads + h]
            fq = _wave_field(grid, D, kind, gq, device)
            fk = _wave_field(grid, D, kind, gk, device)
            i = torch.randint(0, S, (n_pairs,), generator=gs, device=device)
            j = torch.randint(0, S, (n_pairs,), generator=gs, device=device)
            s = scale * (fq[i] * fk[j]).sum(-1)
            alpha = math.sqrt(score_std / max(float(s.std()), 1e-12))
            q[b, h] = (fq * alpha).to(dtype)
            k[b, h] = (fk * alpha).to(dtype)
    v = torch.randn(B, heads, S, D, generator=gv, device=device).to(dtype)
    return q, k, v


def quantized_smooth_qkv(B: int, heads: int, grid: Dims3, D: int, seed: int,
                         kinds: Optional[Sequence[str]] = None, dtype=torch.bfloat16,
                         device="cpu", steps_per_std: float = 2.0):
    """smooth_qkv's Q and K rounded onto the {-4..4}/4 grid (per (b, head):
    x / std(x) * steps_per_std, rounded, clipped to [-4, 4], divided by 4),
    and i.i.d. integer-grid V.  Every value is exact in bf16."""
    q, k, _ = smooth_qkv(B, heads, grid, D, seed, kinds=kinds, dtype=torch.float32, device=device)

    def grid_values(x):
        sd = x.flatten(2).std(dim=-1).clamp_min(1e-12)[..., None, None]
        # + 0.0 turns the -0.0 that rounding small negatives gives into +0.0
        return (torch.round(x / sd * steps_per_std).clamp(-4, 4) / 4.0 + 0.0).to(dtype)

    S = grid[0] * grid[1] * grid[2]
    v = integer_grid((B, heads, S, D), seed + 2, dtype, device)
    return grid_values(q), grid_values(k), v


def make_qkv(workload: Workload, device="cpu", values: Optional[str] = None,
             B: Optional[int] = None, heads: Optional[int] = None):
    """Q, K, V for a workload (optionally overriding value kind or sizes)."""
    values = values or workload.values
    B = workload.B if B is None else B
    heads = workload.heads if heads is None else heads
    shape = (B, heads, workload.S, workload.D)
    if values == "integer":
        s = workload.seed_base
        return tuple(integer_grid(shape, s + o, workload.dtype, device)
                     for o in (0, 1, 2))
    kinds = head_kinds(workload) if values in ("smooth_adaptive", "integer_adaptive") else None
    if kinds is not None:
        kinds = kinds[: B * heads] + ["generic"] * max(0, B * heads - len(kinds))
    if values == "integer_adaptive":
        return quantized_smooth_qkv(B, heads, workload.grid, workload.D, workload.seed_base,
                                    kinds=kinds, dtype=workload.dtype, device=device)
    return smooth_qkv(B, heads, workload.grid, workload.D, workload.seed_base,
                      kinds=kinds, dtype=workload.dtype, device=device)


def random_scores(shape: Sequence[int], seed: int, levels: int = 0,
                  device="cpu") -> torch.Tensor:
    """fp32 block-score rows for exercising top-k alone.

    ``levels > 0`` draws integers from [-levels, levels] (many exact ties);
    ``levels == 0`` draws N(0, 1) values.
    """
    g = _gen(seed, device)
    if levels > 0:
        x = torch.randint(-levels, levels + 1, tuple(shape), generator=g, device=device)
        return x.to(torch.float32)
    return torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
