"""fp64 CPU oracle for block-sparse video self-attention -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It shares no code with the CUDA library and
never calls it.  The arithmetic lives in ``vsa_oracle.c`` (plain C, double
precision); this module only moves numpy arrays in and out and loops over
(batch, head), in the order the "Adaptive tiling (SPADE)" Recipe composes the
steps: choose a tiling per head, permute, score, select, attend, permute back.

Inputs are taken as float32 numpy arrays (or torch tensors), which carry bf16
and fp32 values exactly.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.orc_tile_labels.argtypes = [i32] * 6 + [P]
        L.orc_tile_permutation.argtypes = [i32] * 6 + [P]
        L.orc_permute_rows.argtypes = [P, i64, i32, P, P]
        L.orc_unpermute_rows.argtypes = [P, i64, i32, P, P]
        L.orc_tile_sics.argtypes = [P] + [i32] * 7 + [P]
        L.orc_tile_counts.argtypes = [P] + [i32] * 7 + [P]
        L.orc_pad_grid.argtypes = [P] + [i32] * 7 + [P]
        L.orc_select_tiling.argtypes = [P, i32, i32, i32, i32, P, i32, P]
        L.orc_select_tiling.restype = i32
        L.orc_block_minmax.argtypes = [P, i64, i32, i32, P, P]
        L.orc_block_scores.argtypes = [P, P, P, P, i64, i32, P]
        L.orc_topk_block_list.argtypes = [P, i64, i32, i32, i32, i32, P, P]
        L.orc_topp_block_list.argtypes = [P, i64, dbl, dbl, i32, i32, i32, P, P]
        L.orc_topk_block_list.restype = i32
        L.orc_tile_neighbourhood_list.argtypes = [i32] * 11 + [P, P, P]
        L.orc_tile_neighbourhood_list.restype = i32
        L.orc_centered_tile_neighbourhood_list.argtypes = [i32] * 11 + [P, P, P]
        L.orc_centered_tile_neighbourhood_list.restype = i32
        L.orc_sampled_probs.argtypes = [P, P, i64, i32, P, i32, dbl, P]
        L.orc_pattern_masses.argtypes = [P, i32, i32, i32, P, i32, P]
        L.orc_centroid_compensated_attention.argtypes = [P, P, P, i64, i32, P, P, i32, i32, P, dbl, P, i64, P]
        L.orc_window_attention.argtypes = [P, P, P, i64, i32, i32, i32, dbl, i32, P, i64, P]
        L.orc_block_sparse_attention.argtypes = [P, P, P, i64, i32, i32, P, P, i32, i32, dbl, P, P, i64, P]
        L.orc_window_key_ranges.argtypes = [i64] * 5 + [P]
        L.orc_window_key_ranges.restype = i32
        _lib = L
    return _lib


def _f32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def default_scale(D: int, scale: Optional[float]) -> float:
    """_default_scale: the explicit scale, else D ** -0.5."""
    if scale is not None and scale > 0:
        return float(scale)
    if D <= 0:
        raise ValueError("head_dim must be positive")
    return float(D) ** -0.5


# --------------------------------------------------------------------------
# permutation
# --------------------------------------------------------------------------

def tile_labels(grid, tile) -> np.ndarray:
    T, H, W = grid
    out = np.empty(T * H * W, dtype=np.int64)
    lib().orc_tile_labels(T, H, W, *tile, _ptr(out))
    return out


def tile_permutation(grid, tile) -> np.ndarray:
    T, H, W = grid
    out = np.empty(T * H * W, dtype=np.int64)
    lib().orc_tile_permutation(T, H, W, *tile, _ptr(out))
    return out


def permute_rows(x, perm) -> np.ndarray:
    x = _f32(x)
    S, D = x.shape
    y = np.empty_like(x)
    lib().orc_permute_rows(_ptr(x), S, D, _ptr(np.ascontiguousarray(perm, np.int64)), _ptr(y))
    return y


def unpermute_rows(y, perm) -> np.ndarray:
    y = _f32(y)
    S, D = y.shape
    x = np.empty_like(y)
    lib().orc_unpermute_rows(_ptr(y), S, D, _ptr(np.ascontiguousarray(perm, np.int64)), _ptr(x))
    return x


# --------------------------------------------------------------------------
# grids the tiles do not divide ("Adaptive tiling (SPADE)", Deviations and
# notes: pad with zero tokens, excluded from the cohesion; mask padded keys)
# --------------------------------------------------------------------------

def padded_grid(grid, tiles):
    """Each axis rounded up to a multiple of every candidate's extent on it
    (their least common multiple), so that every candidate tiles it."""
    out = []
    for ax in range(3):
        l = 1
        for t in tiles:
            l = l * t[ax] // np.gcd(l, t[ax])
        out.append(-(-grid[ax] // l) * l)
    return tuple(int(x) for x in out)


def pad_grid(x, grid, padded) -> np.ndarray:
    """[T*H*W, D] T-major -> [Tp*Hp*Wp, D] with zero tokens outside (T, H, W)."""
    x = _f32(x)
    T, H, W = grid
    Tp, Hp, Wp = padded
    y = np.empty((Tp * Hp * Wp, x.shape[1]), np.float32)
    lib().orc_pad_grid(_ptr(x), T, H, W, x.shape[1], Tp, Hp, Wp, _ptr(y))
    return y


def real_tokens(grid, padded) -> np.ndarray:
    """Boolean mask over the padded grid's T-major tokens: inside (T, H, W)."""
    T, H, W = grid
    Tp, Hp, Wp = padded
    t, h, w = np.meshgrid(np.arange(Tp), np.arange(Hp), np.arange(Wp), indexing="ij")
    return ((t < T) & (h < H) & (w < W)).reshape(-1)


def tile_counts(q, grid, tile) -> np.ndarray:
    """Non-zero-norm queries per tile of one tiling."""
    q = _f32(q)
    T, H, W = grid
    n = (T * H * W) // (tile[0] * tile[1] * tile[2])
    out = np.empty(n, dtype=np.int64)
    lib().orc_tile_counts(_ptr(q), T, H, W, q.shape[1], *tile, _ptr(out))
    return out


# --------------------------------------------------------------------------
# tiling choice
# --------------------------------------------------------------------------

def tile_sics(q, grid, tile) -> np.ndarray:
    """SICS of every tile of one tiling, for one head's q [S, D]."""
    q = _f32(q)
    T, H, W = grid
    n = (T * H * W) // (tile[0] * tile[1] * tile[2])
    out = np.empty(n, dtype=np.float64)
    lib().orc_tile_sics(_ptr(q), T, H, W, q.shape[1], *tile, _ptr(out))
    return out


def select_tiling(q, grid, tiles):
    """(choice, cohesion[n_tiles]) for one head's q [S, D]."""
    q = _f32(q)
    T, H, W = grid
    t = np.ascontiguousarray(np.array(tiles, dtype=np.int32).reshape(-1))
    sc = np.empty(len(tiles), dtype=np.float64)
    c = lib().orc_select_tiling(_ptr(q), T, H, W, q.shape[1], _ptr(t), len(tiles), _ptr(sc))
    return int(c), sc


# --------------------------------------------------------------------------
# summaries, scores, top-k, structured lists
# --------------------------------------------------------------------------

def block_minmax(xp, block: int):
    xp = _f32(xp)
    S, D = xp.shape
    nb = S // block
    mx = np.empty((nb, D), np.float64)
    mn = np.empty((nb, D), np.float64)
    lib().orc_block_minmax(_ptr(xp), S, D, block, _ptr(mx), _ptr(mn))
    return mx, mn


def block_scores(qmax, qmin, kmax, kmin) -> np.ndarray:
    a = [np.ascontiguousarray(x, np.float64) for x in (qmax, qmin, kmax, kmin)]
    nb, D = a[0].shape
    s = np.empty((nb, nb), np.float64)
    lib().orc_block_scores(*(_ptr(x) for x in a), nb, D, _ptr(s))
    return s


def list_cap(nb: int, k: int, n_sink: int, diag_halfwidth: int) -> int:
    """Longest possible list: k top blocks, the sinks and the diagonal band
    (2 dw + 1 blocks; none when diag_halfwidth is -1)."""
    band = 2 * diag_halfwidth + 1 if diag_halfwidth >= 0 else 0
    return min(nb, k + n_sink + band)


def topk_block_list(score, k: int, n_sink: int = 1, diag_halfwidth: int = 0,
                    cap: Optional[int] = None):
    s = np.ascontiguousarray(score, np.float64)
    nb = s.shape[0]
    cap = cap if cap is not None else list_cap(nb, k, n_sink, diag_halfwidth)
    idx = np.empty((nb, cap), np.int32)
    cnt = np.empty(nb, np.int32)
    rc = lib().orc_topk_block_list(_ptr(s), nb, k, n_sink, diag_halfwidth, cap, _ptr(idx), _ptr(cnt))
    if rc != 0:
        raise ValueError("cap too small for the top-k list")
    return idx, cnt


def topp_block_list(score, p: float, scale: float, n_sink: int = 1, diag_halfwidth: int = 0,
                    cap: Optional[int] = None):
    """Top-p (mass budget) lists: per row, the shortest prefix in descending
    score order (ties: lower index) whose softmax(scale * score) mass reaches
    p, plus the sink and diagonal blocks (see orc_topp_block_list)."""
    s = np.ascontiguousarray(score, np.float64)
    nb = s.shape[0]
    cap = nb if cap is None else cap
    idx = np.empty((nb, cap), np.int32)
    cnt = np.empty(nb, np.int32)
    rc = lib().orc_topp_block_list(_ptr(s), nb, ctypes.c_double(p), ctypes.c_double(scale), n_sink,
                                   diag_halfwidth, cap, _ptr(idx), _ptr(cnt))
    if rc != 0:
        raise ValueError("cap too small for the top-p list")
    return idx, cnt


STRUCTURED_KINDS = ("spatial", "temporal", "sliding_tile", "sliding_tile_centered")


def structured_tile(kind: str, grid, tile=(4, 8, 8), radius=(1, 1, 1)):
    """(tile, radius) of a structured mask: spatial_only = same frame,
    temporal_only = same (h, w), sliding_tile = tile neighbourhood clipped at
    the border, sliding_tile_centered = a window of 2r+1 tiles shifted to fit."""
    T, H, W = grid
    if kind == "spatial":
        return (1, H, W), (0, 0, 0)
    if kind == "temporal":
        return (T, 1, 1), (0, 0, 0)
    if kind in ("sliding_tile", "sliding_tile_centered"):
        return tuple(tile), tuple(radius)
    raise ValueError(kind)


def tile_neighbourhood_list(grid, tile, radius, block: int, cap: Optional[int] = None, centered: bool = False):
    """Block list of a tile-neighbourhood mask in the tile-contiguous order of
    `tile`: clipped at the grid border, or with `centered` a window of
    min(2r+1, n) tiles per axis moved inside the grid."""
    T, H, W = grid
    S = T * H * W
    nb = S // block
    trim = cap is None
    if trim:
        cap = nb
    idx = np.empty((nb, cap), np.int32)
    cnt = np.empty(nb, np.int32)
    g = ctypes.c_int(0)
    fn = lib().orc_centered_tile_neighbourhood_list if centered else lib().orc_tile_neighbourhood_list
    rc = fn(T, H, W, *tile, *radius, block, cap, _ptr(idx), _ptr(cnt), ctypes.byref(g))
    if rc != 0:
        raise ValueError(f"unsupported tile/radius/block combination (rc={rc})")
    if trim:
        idx = idx[:, :int(cnt.max())].copy()
    return idx, cnt, int(g.value)


# --------------------------------------------------------------------------
# head profile: spatial or temporal pattern per head
# --------------------------------------------------------------------------

PATTERN_KINDS = ("spatial", "temporal")


def sampled_probs(q, k, rows, scale=None):
    """Attention probabilities [R, S] of the sampled query rows of one head."""
    q, k = _f32(q), _f32(k)
    S, D = q.shape
    r = np.ascontiguousarray(rows, np.int32)
    probs = np.empty((len(r), S), np.float64)
    lib().orc_sampled_probs(_ptr(q), _ptr(k), S, D, _ptr(r), len(r), default_scale(D, scale), _ptr(probs))
    return probs


def pattern_masses(probs, grid, rows):
    """[R, 2]: each sampled row's probability mass on its own frame (spatial)
    and on its own (h, w) position (temporal)."""
    T, H, W = grid
    probs = np.ascontiguousarray(probs, np.float64)
    r = np.ascontiguousarray(rows, np.int32)
    mass = np.empty((len(r), 2), np.float64)
    lib().orc_pattern_masses(_ptr(probs), T, H, W, _ptr(r), len(r), _ptr(mass))
    return mass


PROFILE_RULES = ("mass", "mass_per_key")


def classify_head(q, k, grid, rows, scale=None, rule="mass"):
    """(kind, mean masses [2]) of one head, 0 = spatial, 1 = temporal, ties to
    spatial.  rule "mass": the pattern holding the larger mean mass over the
    sampled rows.  rule "mass_per_key": the larger mean mass per key of the
    pattern, spatial mass / (H W) against temporal mass / T (the attention a
    query pays each key of its frame, or each key at its (h, w))."""
    if rule not in PROFILE_RULES:
        raise ValueError(f"rule must be one of {PROFILE_RULES}")
    mass = pattern_masses(sampled_probs(q, k, rows, scale), grid, rows).mean(axis=0)
    T, H, W = grid
    sp, tp = (mass[0], mass[1]) if rule == "mass" else (mass[0] / (H * W), mass[1] / T)
    return (0 if sp >= tp else 1), mass


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def _rows(rows, S):
    if rows is None:
        return np.arange(S, dtype=np.int64)
    return np.ascontiguousarray(rows, np.int64)


def window_attention(q, k, v, window: int, sink: int = 0, scale=None, rows=None):
    """windowed_attention for one head [S, D]; returns rows x D doubles."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    S, D = q.shape
    r = _rows(rows, S)
    out = np.empty((len(r), D), np.float64)
    lib().orc_window_attention(_ptr(q), _ptr(k), _ptr(v), S, D, window, sink,
                               default_scale(D, scale), 0, _ptr(r), len(r), _ptr(out))
    return out


def centroid_compensated_attention(q, k, v, q_labels, k_labels, block_mask, scale=None, rows=None):
    """centroid_compensated_attention for one head [S, D]: kept key blocks
    exactly, each skipped key block as its mean key and mean value weighted by
    its size.  q_labels / k_labels give each token's block, block_mask
    [n_q_blocks, n_k_blocks] (bool) the kept pairs.  Returns rows x D doubles."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    S, D = q.shape
    ql = np.ascontiguousarray(q_labels, np.int32)
    kl = np.ascontiguousarray(k_labels, np.int32)
    m = np.ascontiguousarray(block_mask, np.uint8)
    n_qb, n_kb = m.shape
    if len(ql) != S or len(kl) != S or ql.min() < 0 or ql.max() >= n_qb or kl.min() < 0 or kl.max() >= n_kb:
        raise ValueError("labels must give every token a block of block_mask")
    r = _rows(rows, S)
    out = np.empty((len(r), D), np.float64)
    lib().orc_centroid_compensated_attention(_ptr(q), _ptr(k), _ptr(v), S, D, _ptr(ql), _ptr(kl), n_qb, n_kb,
                                             _ptr(m), default_scale(D, scale), _ptr(r), len(r), _ptr(out))
    return out


def dense_attention(q, k, v, scale=None, rows=None):
    """full_attention for one head [S, D]."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    S, D = q.shape
    r = _rows(rows, S)
    out = np.empty((len(r), D), np.float64)
    lib().orc_window_attention(_ptr(q), _ptr(k), _ptr(v), S, D, 1, 0,
                               default_scale(D, scale), 1, _ptr(r), len(r), _ptr(out))
    return out


def block_sparse_attention(qp, kp, vp, idx, cnt, block: int, group_size: int = 0,
                           scale=None, rows=None, key_ok=None):
    """Block-list attention for one head in the permuted order; key_ok[p] == 0
    masks key p (padding)."""
    qp, kp, vp = _f32(qp), _f32(kp), _f32(vp)
    S, D = qp.shape
    idx = np.ascontiguousarray(idx, np.int32)
    cnt = np.ascontiguousarray(cnt, np.int32)
    r = _rows(rows, S)
    ok = None if key_ok is None else np.ascontiguousarray(key_ok, np.uint8)
    out = np.empty((len(r), D), np.float64)
    lib().orc_block_sparse_attention(_ptr(qp), _ptr(kp), _ptr(vp), S, D, block,
                                     _ptr(idx), _ptr(cnt), idx.shape[1], group_size,
                                     default_scale(D, scale), None if ok is None else _ptr(ok),
                                     _ptr(r), len(r), _ptr(out))
    return out


def window_key_ranges(qs: int, qe: int, S: int, half: int, sink: int):
    out = np.zeros(4, np.int64)
    n = lib().orc_window_key_ranges(qs, qe, S, half, sink, _ptr(out))
    return [(int(out[2 * i]), int(out[2 * i + 1])) for i in range(n)]


# --------------------------------------------------------------------------
# the SPADE composition for one head
# --------------------------------------------------------------------------

def spade_head(q, k, v, grid, tiles, k_blocks: int, n_sink: int = 1,
               diag_halfwidth: int = 0, scale=None, query_blocks=None):
    """Adaptive tiling -> permutation -> min/max scores -> top-k + sink +
    diagonal -> block-sparse attention -> inverse permutation, for one head.

    A grid the candidates do not divide is first zero-padded to padded_grid()
    (the pages' recipe); the zero tokens drop out of the cohesion by having
    zero norm, take part in the summaries, and are masked as keys.  ``out``
    then holds the real tokens only; ``perm`` and the blocks refer to the
    padded grid.

    Returns a dict with every intermediate.  With ``query_blocks`` only those
    query blocks (in the permuted order) are attended; ``out_perm`` then holds
    just their rows and ``out`` is None.
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    real_grid = tuple(grid)
    grid = padded_grid(real_grid, tiles)
    padded = grid != real_grid
    if padded:  # zero tokens up to a grid every candidate tiles; padded keys masked below
        q, k, v = (pad_grid(x, real_grid, grid) for x in (q, k, v))
    choice, cohesion = select_tiling(q, grid, tiles) if len(tiles) > 1 else (0, None)
    tile = tiles[choice]
    block = tile[0] * tile[1] * tile[2]
    perm = tile_permutation(grid, tile)
    qp, kp, vp = (permute_rows(x, perm) for x in (q, k, v))
    key_ok = real_tokens(real_grid, grid)[perm].astype(np.uint8) if padded else None
    qmax, qmin = block_minmax(qp, block)
    kmax, kmin = block_minmax(kp, block)
    score = block_scores(qmax, qmin, kmax, kmin)
    idx, cnt = topk_block_list(score, k_blocks, n_sink, diag_halfwidth)
    res = dict(choice=choice, cohesion=cohesion, perm=perm, block=block,
               qmax=qmax, qmin=qmin, kmax=kmax, kmin=kmin, score=score,
               idx=idx, cnt=cnt, padded_grid=grid, key_ok=key_ok)
    if query_blocks is None:
        op = block_sparse_attention(qp, kp, vp, idx, cnt, block, 0, scale, key_ok=key_ok)
        res["out_perm"] = op
        out = _unpermute64(op, perm)
        res["out"] = out[real_tokens(real_grid, grid)] if padded else out
    else:
        rows = np.concatenate([np.arange(b * block, (b + 1) * block) for b in query_blocks])
        res["out_perm"] = block_sparse_attention(qp, kp, vp, idx, cnt, block, 0, scale, rows, key_ok=key_ok)
        res["rows"] = rows
        res["out"] = None
    return res


def _unpermute64(y: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """x[perm[p]] = y[p] for double rows (the inverse permutation)."""
    x = np.empty_like(y)
    x[perm] = y
    return x
