"""block_sparse_self_b200 -- Python binding of libvsa (B200 / sm_100a).

Structured and input-adaptive block-sparse self-attention over a video DiT's
T-major token sequence.  Every function here only checks and marshals
arguments (torch CUDA tensors -> device pointers, the current CUDA stream)
and calls the C ABI declared in include/vsa.h; all arithmetic runs in the
library's CUDA kernels.  There is no CPU fallback: if libvsa.so is missing or
a tensor is not on a CUDA device, the call raises.

Errors follow the pages' convention ("ADR-0001", Conventions: Validation):
invalid arguments raise ValueError, violated device-side invariants raise
RuntimeError, unsupported-but-valid requests raise NotImplementedError.
"""

from __future__ import annotations

import ctypes
import math
import os
import re
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvsa.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "vsa.h")

OK, ERR_INVALID_ARGUMENT, ERR_RUNTIME, ERR_CUDA, ERR_UNSUPPORTED, ERR_TIMEOUT = range(6)
BF16, F32 = 0, 1
MASK_SPATIAL, MASK_TEMPORAL, MASK_SLIDING_TILE, MASK_SLIDING_TILE_CENTERED = 0, 1, 2, 3


class Dims3(ctypes.Structure):
    _fields_ = [("t", ctypes.c_int32), ("h", ctypes.c_int32), ("w", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libvsa.so (built in-tree by ``python -m block_sparse_self_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m block_sparse_self_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    D3 = Dims3
    sig = {
        "vsa_last_error": ([], ctypes.c_char_p),
        "vsa_device_status": ([P], I),
        "vsa_padded_grid": ([D3, P, I, P], I),
        "vsa_select_tiling_workspace_size": ([I, I, D3, P, I], SZ),
        "vsa_select_tiling": ([P, I, I, I, I, I, D3, P, I, P, P, P, SZ, P], I),
        "vsa_select_tiling_noalloc": ([P, I, I, I, I, I, D3, P, I, P, P, P], I),
        "vsa_permute": ([P, P, I, I, I, I, I, D3, P, I, P, P], I),
        "vsa_unpermute": ([P, P, I, I, I, I, I, D3, P, I, P, P], I),
        "vsa_block_summaries": ([P, I, I, I, I, I, I, P, P, P], I),
        "vsa_block_summaries_tiled": ([P, I, I, I, I, I, D3, P, I, P, I, P, P, P], I),
        "vsa_block_scores": ([P, P, P, P, I, I, I, I, I, P, P], I),
        "vsa_topk_block_mask": ([P, I, I, I, I, I, I, P, P, I, P], I),
        "vsa_block_scores_topk": ([P, P, P, P, I, I, I, I, I, I, I, I, P, P, I, P], I),
        "vsa_topp_block_mask": ([P, I, I, I, F, F, I, I, P, P, I, P], I),
        "vsa_structured_block_list": ([I, D3, D3, D3, I, P, P, I, P, P], I),
        "vsa_block_sparse_attention": ([P, P, P, P, I, I, I, I, I, I, P, P, I, I, I, F, P], I),
        "vsa_block_sparse_attention_tiled": ([P, P, P, P, I, I, I, I, I, D3, P, I, P, P, P, I, I, I, F, P], I),
        "vsa_window_attention": ([P, P, P, P, I, I, I, I, I, I, I, F, I, P], I),
        "vsa_head_profile_workspace_size": ([I, I, I, I], SZ),
        "vsa_head_profile": ([P, P, I, I, I, I, D3, P, I, F, I, P, P, P, SZ, P], I),
        "vsa_centroid_compensated_attention_workspace_size": ([I, I, I, I, I], SZ),
        "vsa_centroid_compensated_attention": ([P, P, P, P, I, I, I, I, I, I, P, P, I, I, F, P, SZ, P], I),
        "vsa_centroid_compensated_attention_tiled": ([P, P, P, P, I, I, I, I, I, D3, P, I, P, P, P, I, I, F, P, SZ, P],
                                                     I),
        "vsa_spade_attention_host_workspace_size": ([I, I, I, I, D3, P, I, I, I, I, I, I], SZ),
        "vsa_spade_attention_host": ([P, P, P, P, I, I, I, I, I, D3, P, I, I, I, I, F, I, P, SZ, P], I),
        "vsa_cast_f32_to_bf16": ([P, P, I64, P], I),
        "vsa_debug_wait_timeout": ([I64, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def declared_functions() -> list:
    """Names of the functions include/vsa.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vsa_[a-z0-9_]+)\s*\(", text)))


def last_error() -> str:
    return lib().vsa_last_error().decode()


def _check(status: int) -> None:
    if status == OK:
        return
    msg = last_error()
    if status == ERR_INVALID_ARGUMENT:
        raise ValueError(msg)
    if status == ERR_UNSUPPORTED:
        raise NotImplementedError(msg)
    if status == ERR_TIMEOUT:
        raise RuntimeError("timeout: " + msg)
    raise RuntimeError(msg)


def _stream(device=None) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _cuda(t: torch.Tensor, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _dtype_code(t: torch.Tensor, name: str) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise ValueError(f"{name} must be bfloat16 or float32, got {t.dtype}")


def _bhsd(t: torch.Tensor, name: str) -> Tuple[int, int, int, int]:
    if t.dim() != 4:
        raise ValueError(f"{name} must be rank-4 (B, H, S, D); got shape {tuple(t.shape)}")
    return tuple(t.shape)


def _tiles_arg(tiles: Sequence[Sequence[int]]):
    tiles = [tuple(int(v) for v in t) for t in tiles]
    arr = (Dims3 * len(tiles))(*[Dims3(*t) for t in tiles])
    return arr, len(tiles)


def padded_grid(grid, tiles) -> Tuple[int, int, int]:
    """The grid every candidate tiles: each axis rounded up to a multiple of the
    candidates' lcm on it (equal to grid when they all divide it).  Positions,
    tilings and block indices of the calls below refer to this grid."""
    arr, n = _tiles_arg(tiles)
    out = Dims3()
    _check(lib().vsa_padded_grid(Dims3(*grid), arr, n, ctypes.byref(out)))
    return (out.t, out.h, out.w)


def _grid_tokens(grid) -> int:
    return int(grid[0]) * int(grid[1]) * int(grid[2])


def device_status(stream=None) -> None:
    """Synchronise the stream; raise if a kernel recorded a device-side failure."""
    _check(lib().vsa_device_status(_stream() if stream is None else stream))


# --------------------------------------------------------------------------
# the steps of the path
# --------------------------------------------------------------------------

def select_tiling(q: torch.Tensor, grid, tiles, return_sics: bool = False):
    """Per-(b, head) index of the most cohesive candidate tiling (int32 [B*H])."""
    _cuda(q, "q")
    B, H, S, D = _bhsd(q, "q")
    arr, n = _tiles_arg(tiles)
    g = Dims3(*grid)
    choice = torch.empty(B * H, dtype=torch.int32, device=q.device)
    sics = torch.empty(B * H, n, dtype=torch.float32, device=q.device) if return_sics else None
    ws_bytes = lib().vsa_select_tiling_workspace_size(B, H, g, arr, n)
    ws = torch.empty(max(ws_bytes, 256) // 4, dtype=torch.float32, device=q.device)
    _check(lib().vsa_select_tiling(_ptr(q), _dtype_code(q, "q"), B, H, S, D, g, arr, n, _ptr(choice),
                                   _ptr(sics), _ptr(ws), ws.numel() * 4, _stream(q.device)))
    return (choice, sics) if return_sics else choice


def select_tiling_noalloc(q: torch.Tensor, grid, tiles, return_sics: bool = False):
    """select_tiling for callers that cannot allocate device scratch: the
    library's own fixed scratch array is used (see vsa_select_tiling_noalloc
    in include/vsa.h for its size limit, and note that overlapping calls on
    one GPU race on it).  Only the outputs are allocated here."""
    _cuda(q, "q")
    B, H, S, D = _bhsd(q, "q")
    arr, n = _tiles_arg(tiles)
    choice = torch.empty(B * H, dtype=torch.int32, device=q.device)
    sics = torch.empty(B * H, n, dtype=torch.float32, device=q.device) if return_sics else None
    _check(lib().vsa_select_tiling_noalloc(_ptr(q), _dtype_code(q, "q"), B, H, S, D, Dims3(*grid), arr, n,
                                           _ptr(choice), _ptr(sics), _stream(q.device)))
    return (choice, sics) if return_sics else choice


def _permute(x, grid, tiles, choice, inverse):
    _cuda(x, "x")
    B, H, rows, D = _bhsd(x, "x")
    if choice is not None:
        _cuda(choice, "choice")
        if choice.dtype != torch.int32 or choice.numel() != B * H:
            raise ValueError("choice must be int32 with B*H entries")
    arr, n = _tiles_arg(tiles)
    S, Sp = _grid_tokens(grid), _grid_tokens(padded_grid(grid, tiles))
    if rows != (Sp if inverse else S):
        raise ValueError(f"x has {rows} rows per head; expected {Sp if inverse else S} "
                         f"({'padded' if inverse else 'real'} tokens of grid {tuple(grid)})")
    y = torch.empty(B, H, S if inverse else Sp, D, dtype=x.dtype, device=x.device)
    fn = lib().vsa_unpermute if inverse else lib().vsa_permute
    _check(fn(_ptr(x), _ptr(y), _dtype_code(x, "x"), B, H, S, D, Dims3(*grid), arr, n, _ptr(choice),
              _stream(x.device)))
    return y


def permute(x: torch.Tensor, grid, tiles, choice: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Tile-contiguous order: y[b, h, p] = x[b, h, perm_c(p)] (c = choice[b*H+h] or 0).
    On a grid the tiles do not divide, y covers padded_grid(grid, tiles), with
    zero rows at padding positions."""
    return _permute(x, grid, tiles, choice, False)


def unpermute(y: torch.Tensor, grid, tiles, choice: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Inverse of permute: back to T-major order (padding rows dropped)."""
    return _permute(y, grid, tiles, choice, True)


def block_summaries(x_perm: torch.Tensor, block: int):
    """(x_max, x_min), each [B, H, S/block, D]: per-block element-wise max / min."""
    _cuda(x_perm, "x_perm")
    B, H, S, D = _bhsd(x_perm, "x_perm")
    if block <= 0 or S % block:
        raise ValueError(f"block ({block}) must divide S ({S})")
    xmax = torch.empty(B, H, S // block, D, dtype=x_perm.dtype, device=x_perm.device)
    xmin = torch.empty_like(xmax)
    _check(lib().vsa_block_summaries(_ptr(x_perm), _dtype_code(x_perm, "x_perm"), B, H, S, D, block,
                                     _ptr(xmax), _ptr(xmin), _stream(x_perm.device)))
    return xmax, xmin


def _choice_arg(choice, BH):
    if choice is not None:
        _cuda(choice, "choice")
        if choice.dtype != torch.int32 or choice.numel() != BH:
            raise ValueError("choice must be int32 with B*H entries")
    return _ptr(choice)


def block_summaries_tiled(x: torch.Tensor, grid, tiles, choice: Optional[torch.Tensor], block: int):
    """block_summaries(permute(x, grid, tiles, choice), block) read straight from T-major x
    (blocks of padded_grid(grid, tiles); padding positions count as zero rows)."""
    _cuda(x, "x")
    B, H, S, D = _bhsd(x, "x")
    Sp = _grid_tokens(padded_grid(grid, tiles))
    if block <= 0 or Sp % block:
        raise ValueError(f"block ({block}) must divide the padded token count ({Sp})")
    arr, n = _tiles_arg(tiles)
    xmax = torch.empty(B, H, Sp // block, D, dtype=x.dtype, device=x.device)
    xmin = torch.empty_like(xmax)
    _check(lib().vsa_block_summaries_tiled(_ptr(x), _dtype_code(x, "x"), B, H, S, D, Dims3(*grid), arr, n,
                                           _choice_arg(choice, B * H), int(block), _ptr(xmax), _ptr(xmin),
                                           _stream(x.device)))
    return xmax, xmin


def block_scores(q_max, q_min, k_max, k_min) -> torch.Tensor:
    """fp32 [B, H, nb, nb]: max((q_max+q_min).k_max, (q_max+q_min).k_min)."""
    for t, nm in ((q_max, "q_max"), (q_min, "q_min"), (k_max, "k_max"), (k_min, "k_min")):
        _cuda(t, nm)
        if t.shape != q_max.shape or t.dtype != q_max.dtype:
            raise ValueError("summaries must share shape and dtype")
    B, H, nb, D = _bhsd(q_max, "q_max")
    out = torch.empty(B, H, nb, nb, dtype=torch.float32, device=q_max.device)
    _check(lib().vsa_block_scores(_ptr(q_max), _ptr(q_min), _ptr(k_max), _ptr(k_min), _dtype_code(q_max, "q_max"),
                                  B, H, nb, D, _ptr(out), _stream(q_max.device)))
    return out


def list_cap(nb: int, k: int, n_sink_blocks: int, diag_halfwidth: int) -> int:
    extra = 2 * diag_halfwidth + 1 if diag_halfwidth >= 0 else 0
    return min(nb, k + n_sink_blocks + extra)


def topk_block_mask(scores: torch.Tensor, k: int, n_sink_blocks: int = 1, diag_halfwidth: int = 0,
                    cap: Optional[int] = None):
    """(idx [B,H,nb,cap] int32, cnt [B,H,nb] int32): top-k + sink + diagonal, ascending, -1 padded."""
    _cuda(scores, "scores")
    if scores.dtype != torch.float32 or scores.dim() != 4 or scores.shape[-1] != scores.shape[-2]:
        raise ValueError("scores must be fp32 [B, H, nb, nb]")
    B, H, nb, _ = scores.shape
    cap = list_cap(nb, k, n_sink_blocks, diag_halfwidth) if cap is None else int(cap)
    idx = torch.empty(B, H, nb, max(cap, 1), dtype=torch.int32, device=scores.device)
    cnt = torch.empty(B, H, nb, dtype=torch.int32, device=scores.device)
    _check(lib().vsa_topk_block_mask(_ptr(scores), B, H, nb, int(k), int(n_sink_blocks), int(diag_halfwidth),
                                     _ptr(idx), _ptr(cnt), cap, _stream(scores.device)))
    return idx, cnt


def block_scores_topk(q_max, q_min, k_max, k_min, k: int, n_sink_blocks: int = 1, diag_halfwidth: int = 0,
                      cap: Optional[int] = None):
    """topk_block_mask(block_scores(q_max, q_min, k_max, k_min), k, ...) in one
    kernel, without the score matrix: (idx [B,H,nb,cap] int32, cnt [B,H,nb] int32)."""
    for t, nm in ((q_max, "q_max"), (q_min, "q_min"), (k_max, "k_max"), (k_min, "k_min")):
        _cuda(t, nm)
        if t.shape != q_max.shape or t.dtype != q_max.dtype:
            raise ValueError("summaries must share shape and dtype")
    B, H, nb, D = _bhsd(q_max, "q_max")
    cap = list_cap(nb, k, n_sink_blocks, diag_halfwidth) if cap is None else int(cap)
    idx = torch.empty(B, H, nb, max(cap, 1), dtype=torch.int32, device=q_max.device)
    cnt = torch.empty(B, H, nb, dtype=torch.int32, device=q_max.device)
    _check(lib().vsa_block_scores_topk(_ptr(q_max), _ptr(q_min), _ptr(k_max), _ptr(k_min),
                                       _dtype_code(q_max, "q_max"), B, H, nb, D, int(k), int(n_sink_blocks),
                                       int(diag_halfwidth), _ptr(idx), _ptr(cnt), cap, _stream(q_max.device)))
    return idx, cnt


def topp_block_mask(scores: torch.Tensor, p: float, scale: float, n_sink_blocks: int = 1, diag_halfwidth: int = 0,
                    cap: Optional[int] = None):
    """(idx [B,H,nb,cap] int32, cnt [B,H,nb] int32): per row the shortest
    descending-score prefix whose softmax(scale * scores) mass reaches p, plus
    sink and diagonal blocks, ascending, -1 padded (see include/vsa.h)."""
    _cuda(scores, "scores")
    if scores.dtype != torch.float32 or scores.dim() != 4 or scores.shape[-1] != scores.shape[-2]:
        raise ValueError("scores must be fp32 [B, H, nb, nb]")
    B, H, nb, _ = scores.shape
    cap = nb if cap is None else int(cap)
    idx = torch.empty(B, H, nb, max(cap, 1), dtype=torch.int32, device=scores.device)
    cnt = torch.empty(B, H, nb, dtype=torch.int32, device=scores.device)
    _check(lib().vsa_topp_block_mask(_ptr(scores), B, H, nb, float(p), float(scale), int(n_sink_blocks),
                                     int(diag_halfwidth), _ptr(idx), _ptr(cnt), cap, _stream(scores.device)))
    return idx, cnt


_KINDS = {"spatial": MASK_SPATIAL, "temporal": MASK_TEMPORAL, "sliding_tile": MASK_SLIDING_TILE,
          "sliding_tile_centered": MASK_SLIDING_TILE_CENTERED}


def structured_tile(kind: str, grid, tile=(4, 8, 8)):
    """The tile whose tile-contiguous order a structured list is expressed in."""
    T, Hg, Wg = grid
    return {"spatial": (1, Hg, Wg), "temporal": (T, 1, 1), "sliding_tile": tuple(tile),
            "sliding_tile_centered": tuple(tile)}[kind]


def structured_block_list(kind: str, grid, block: int = 128, tile=(4, 8, 8), radius=(1, 1, 1),
                          device="cuda", cap: Optional[int] = None):
    """(idx [nb,cap], cnt [nb], group_size) of a structured mask in its tile-contiguous order."""
    if kind not in _KINDS:
        raise ValueError(f"kind must be one of {sorted(_KINDS)}")
    T, Hg, Wg = grid
    S = T * Hg * Wg
    if block <= 0 or S % block:
        raise ValueError(f"block ({block}) must divide S ({S})")
    nb = S // block
    cap = nb if cap is None else int(cap)
    idx = torch.empty(nb, max(cap, 1), dtype=torch.int32, device=device)
    cnt = torch.empty(nb, dtype=torch.int32, device=device)
    g = ctypes.c_int(0)
    _check(lib().vsa_structured_block_list(_KINDS[kind], Dims3(*grid), Dims3(*tile), Dims3(*radius), block,
                                           _ptr(idx), _ptr(cnt), cap, ctypes.byref(g), _stream(idx.device)))
    return idx, cnt, int(g.value)


PATTERN_KINDS = ("spatial", "temporal")
PROFILE_RULES = {"mass": 0, "mass_per_key": 1}


def sample_query_rows(S: int, n_rows: int = 128, seed: int = 0, device="cuda") -> torch.Tensor:
    """A seeded draw of distinct query positions for the head profile (int32 [n_rows])."""
    if not 1 <= n_rows <= min(128, S):
        raise ValueError(f"n_rows must be in [1, min(128, S)], got {n_rows}")
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    rows = torch.randperm(S, generator=g)[:n_rows].sort().values
    return rows.to(device=device, dtype=torch.int32)


def head_profile(q, k, grid, rows=None, scale: Optional[float] = None, n_rows: int = 128, seed: int = 0,
                 rule: str = "mass"):
    """Per-(b, head) attention mass on the spatial (same frame) and temporal
    (same (h, w)) patterns over sampled query rows, and the head's kind
    (0 = spatial, 1 = temporal): (kind int32 [B, H], masses fp32 [B, H, 2]).
    `rows` (int32 [R], R <= 128) defaults to sample_query_rows(S, n_rows, seed).
    rule "mass" picks the pattern with the larger mean mass, "mass_per_key"
    the larger mean mass per key of the pattern (see include/vsa.h)."""
    if rule not in PROFILE_RULES:
        raise ValueError(f"rule must be one of {sorted(PROFILE_RULES)}")
    B, H, S, D = _bhsd(q, "q")
    if tuple(k.shape) != (B, H, S, D):
        raise ValueError(f"q/k shapes must match exactly; got q={tuple(q.shape)}, k={tuple(k.shape)}")
    qb, kb = _bf16(q, "q"), _bf16(k, "k")
    if rows is None:
        rows = sample_query_rows(S, min(n_rows, S), seed, q.device)
    _cuda(rows, "rows")
    if rows.dtype != torch.int32 or rows.dim() != 1:
        raise ValueError("rows must be a 1-D int32 tensor")
    rows = rows.contiguous()
    masses = torch.empty(B, H, 2, dtype=torch.float32, device=q.device)
    kind = torch.empty(B, H, dtype=torch.int32, device=q.device)
    ws_bytes = lib().vsa_head_profile_workspace_size(B, H, S, D)
    ws = torch.empty(max(ws_bytes, 256) // 4 + 1, dtype=torch.float32, device=q.device)
    _check(lib().vsa_head_profile(_ptr(qb), _ptr(kb), B, H, S, D, Dims3(*grid), _ptr(rows), rows.numel(),
                                  0.0 if scale is None else float(scale), PROFILE_RULES[rule], _ptr(masses),
                                  _ptr(kind), _ptr(ws),
                                  ws.numel() * 4, _stream(q.device)))
    return kind, masses


def _bf16(t: torch.Tensor, name: str) -> torch.Tensor:
    _cuda(t, name)
    if t.dtype == torch.bfloat16:
        return t
    if t.dtype != torch.float32:
        raise ValueError(f"{name} must be bfloat16 or float32")
    y = torch.empty(t.shape, dtype=torch.bfloat16, device=t.device)
    _check(lib().vsa_cast_f32_to_bf16(_ptr(t), _ptr(y), t.numel(), _stream(t.device)))
    return y


def _out_dtype(out_dtype, ref):
    dt = ref.dtype if out_dtype is None else out_dtype
    if dt not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bfloat16 or float32")
    return dt


def block_sparse_attention(q, k, v, idx, cnt, block: int, group_size: int = 0, scale: Optional[float] = None,
                           out_dtype=None) -> torch.Tensor:
    """Softmax attention of each query block over the key blocks its list names (tile-contiguous order)."""
    B, H, S, D = _bhsd(q, "q")
    if tuple(k.shape) != (B, H, S, D) or tuple(v.shape) != (B, H, S, D):
        raise ValueError(f"q/k/v shapes must match exactly; got q={tuple(q.shape)}, k={tuple(k.shape)}, "
                         f"v={tuple(v.shape)}")
    odt = _out_dtype(out_dtype, q)
    qb, kb, vb = _bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v")
    _cuda(idx, "idx")
    _cuda(cnt, "cnt")
    if idx.dtype != torch.int32 or cnt.dtype != torch.int32:
        raise ValueError("idx and cnt must be int32")
    per_head = idx.dim() == 4
    cap = idx.shape[-1]
    o = torch.empty(B, H, S, D, dtype=odt, device=q.device)
    _check(lib().vsa_block_sparse_attention(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(o), BF16 if odt == torch.bfloat16
                                            else F32, B, H, S, D, int(block), _ptr(idx), _ptr(cnt), int(cap),
                                            1 if per_head else 0, int(group_size),
                                            0.0 if scale is None else float(scale), _stream(q.device)))
    return o


def centroid_compensated_attention(q, k, v, idx, cnt, block: int = 128, scale: Optional[float] = None,
                                   out_dtype=None) -> torch.Tensor:
    """Block-sparse attention (tile-contiguous order, 128-token blocks) in which
    every key block a query block's list skips still takes part, as one key:
    the block's mean key, with its mean value, weighted by its key count (see
    include/vsa.h for the reading of the pages' call)."""
    B, H, S, D = _bhsd(q, "q")
    if tuple(k.shape) != (B, H, S, D) or tuple(v.shape) != (B, H, S, D):
        raise ValueError(f"q/k/v shapes must match exactly; got q={tuple(q.shape)}, k={tuple(k.shape)}, "
                         f"v={tuple(v.shape)}")
    odt = _out_dtype(out_dtype, q)
    qb, kb, vb = _bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v")
    _cuda(idx, "idx")
    _cuda(cnt, "cnt")
    if idx.dtype != torch.int32 or cnt.dtype != torch.int32:
        raise ValueError("idx and cnt must be int32")
    oc = BF16 if odt == torch.bfloat16 else F32
    need = lib().vsa_centroid_compensated_attention_workspace_size(B, H, S, D, oc)
    if need == 0:
        raise ValueError(f"no workspace size for B={B}, H={H}, S={S}, D={D} (S must be a multiple of 128, D 64 or 128)")
    ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    o = torch.empty(B, H, S, D, dtype=odt, device=q.device)
    _check(lib().vsa_centroid_compensated_attention(
        _ptr(qb), _ptr(kb), _ptr(vb), _ptr(o), oc, B, H, S, D, int(block), _ptr(idx), _ptr(cnt), int(idx.shape[-1]),
        1 if idx.dim() == 4 else 0, 0.0 if scale is None else float(scale), _ptr(ws), need, _stream(q.device)))
    return o


def centroid_compensated_attention_tiled(q, k, v, grid, tiles, choice, idx, cnt, scale: Optional[float] = None,
                                         out_dtype=None) -> torch.Tensor:
    """unpermute(centroid_compensated_attention(permute(q), permute(k), permute(v), idx, cnt)) with no
    permuted copies: q, k, v and the result in T-major order, each head's 128-token blocks those of
    tiles[choice[b, h]] (tiling 0 without a choice); the tiles must divide the grid."""
    B, H, S, D = _bhsd(q, "q")
    if tuple(k.shape) != (B, H, S, D) or tuple(v.shape) != (B, H, S, D):
        raise ValueError(f"q/k/v shapes must match exactly; got q={tuple(q.shape)}, k={tuple(k.shape)}, "
                         f"v={tuple(v.shape)}")
    odt = _out_dtype(out_dtype, q)
    qb, kb, vb = _bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v")
    _cuda(idx, "idx")
    _cuda(cnt, "cnt")
    if idx.dtype != torch.int32 or cnt.dtype != torch.int32:
        raise ValueError("idx and cnt must be int32")
    oc = BF16 if odt == torch.bfloat16 else F32
    need = lib().vsa_centroid_compensated_attention_workspace_size(B, H, S, D, oc)
    if need == 0:
        raise ValueError(f"no workspace size for B={B}, H={H}, S={S}, D={D} (S must be a multiple of 128, D 64 or 128)")
    arr, n = _tiles_arg(tiles)
    ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    o = torch.empty(B, H, S, D, dtype=odt, device=q.device)
    _check(lib().vsa_centroid_compensated_attention_tiled(
        _ptr(qb), _ptr(kb), _ptr(vb), _ptr(o), oc, B, H, S, D, Dims3(*grid), arr, n, _choice_arg(choice, B * H),
        _ptr(idx), _ptr(cnt), int(idx.shape[-1]), 1 if idx.dim() == 4 else 0, 0.0 if scale is None else float(scale),
        _ptr(ws), need, _stream(q.device)))
    return o


def block_sparse_attention_tiled(q, k, v, grid, tiles, choice, idx, cnt, scale: Optional[float] = None,
                                 out_dtype=None, group_stride: int = 0) -> torch.Tensor:
    """unpermute(block_sparse_attention(permute(q), permute(k), permute(v), idx, cnt, block)) in one
    kernel: q, k, v and the result stay in T-major order; lists number the blocks of each
    head's tile-contiguous order (block = the tile volume if 32 or 64, else 128 tokens).
    group_stride s > 0 (128-token blocks) restricts each query to keys whose position
    differs from its own by a multiple of s (see include/vsa.h)."""
    B, H, S, D = _bhsd(q, "q")
    if tuple(k.shape) != (B, H, S, D) or tuple(v.shape) != (B, H, S, D):
        raise ValueError(f"q/k/v shapes must match exactly; got q={tuple(q.shape)}, k={tuple(k.shape)}, "
                         f"v={tuple(v.shape)}")
    odt = _out_dtype(out_dtype, q)
    qb, kb, vb = _bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v")
    _cuda(idx, "idx")
    _cuda(cnt, "cnt")
    if idx.dtype != torch.int32 or cnt.dtype != torch.int32:
        raise ValueError("idx and cnt must be int32")
    arr, n = _tiles_arg(tiles)
    o = torch.empty(B, H, S, D, dtype=odt, device=q.device)
    _check(lib().vsa_block_sparse_attention_tiled(
        _ptr(qb), _ptr(kb), _ptr(vb), _ptr(o), BF16 if odt == torch.bfloat16 else F32, B, H, S, D, Dims3(*grid),
        arr, n, _choice_arg(choice, B * H), _ptr(idx), _ptr(cnt), int(idx.shape[-1]), 1 if idx.dim() == 4 else 0,
        int(group_stride), 0.0 if scale is None else float(scale), _stream(q.device)))
    return o


def tiled_supported(tiles) -> bool:
    """Whether every candidate tiling can run through the T-major (tiled) attention:
    one common volume V, either 32 or 64 (a block is the tile) or a multiple of 128
    (a block is 128 tokens: each tile.t divisible by V/128)."""
    tiles = [tuple(t) for t in tiles]
    vols = {t[0] * t[1] * t[2] for t in tiles}
    if len(vols) != 1:
        return False
    vol = vols.pop()
    if vol in (32, 64):
        return True
    return vol % 128 == 0 and all(t[0] % (vol // 128) == 0 for t in tiles)


def window_attention(q, k, v, window: int, sink: int = 0, scale: Optional[float] = None,
                     chunk_size: Optional[int] = None, out_dtype=None) -> torch.Tensor:
    """Symmetric sliding-window attention with `sink` global keys (dense when window >= S)."""
    B, H, S, D = _bhsd(q, "q")
    if tuple(k.shape) != (B, H, S, D) or tuple(v.shape) != (B, H, S, D):
        raise ValueError(f"q/k/v shapes must match exactly; got q={tuple(q.shape)}, k={tuple(k.shape)}, "
                         f"v={tuple(v.shape)}")
    if chunk_size is not None and int(chunk_size) < 1:
        raise ValueError(f"chunk_size must be >= 1, got {chunk_size}")
    odt = _out_dtype(out_dtype, q)
    qb, kb, vb = _bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v")
    o = torch.empty(B, H, S, D, dtype=odt, device=q.device)
    _check(lib().vsa_window_attention(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(o), BF16 if odt == torch.bfloat16 else F32,
                                      B, H, S, D, int(window), int(sink), 0.0 if scale is None else float(scale),
                                      0 if chunk_size is None else int(chunk_size), _stream(q.device)))
    return o


def cast_f32_to_bf16(x: torch.Tensor) -> torch.Tensor:
    _cuda(x, "x")
    if x.dtype != torch.float32:
        raise ValueError("x must be float32")
    return _bf16(x, "x")


def debug_wait_timeout(timeout_ns: int, stream=None) -> None:
    _check(lib().vsa_debug_wait_timeout(int(timeout_ns), _stream() if stream is None else stream))


# --------------------------------------------------------------------------
# compositions
# --------------------------------------------------------------------------

def topk_budget(nb: int, budget: float) -> int:
    """k = max(1, floor(budget * n_blocks)) ("Adaptive tiling (SPADE)", Recipe)."""
    return max(1, int(math.floor(budget * nb)))


def _select_blocks(scores, kk, n_sink_blocks, diag_halfwidth, top_p, top_p_scale, D):
    if top_p is None:
        return topk_block_mask(scores, kk, n_sink_blocks, diag_halfwidth)
    sc = (1.0 / math.sqrt(D)) if top_p_scale is None else float(top_p_scale)
    return topp_block_mask(scores, top_p, sc, n_sink_blocks, diag_halfwidth)


def spade_attention(q, k, v, grid, tiles, budget: Optional[float] = None, topk: Optional[int] = None,
                    n_sink_blocks: int = 1, diag_halfwidth: int = 0, scale: Optional[float] = None,
                    out_dtype=None, return_intermediates: bool = False, tiled: Optional[bool] = None,
                    top_p: Optional[float] = None, top_p_scale: Optional[float] = None,
                    compensate: bool = False):
    """Adaptive tiling -> permutation -> min/max block scores -> top-k + sink +
    diagonal -> block-sparse attention -> inverse permutation, all on the GPU.

    compensate=True takes the Recipe's attention call: every key block a
    query block skips still takes part as its centroid
    (centroid_compensated_attention, or its tiled form); it needs 128-token
    blocks and grids the tiles divide.

    Every candidate tile must have the same volume (the block size).  With a
    single candidate the tiling choice is skipped (choice 0 for every head).
    A grid the candidates do not divide is zero-padded (padded_grid): the
    padding holds no query of the cohesion, takes part in the summaries as
    zero tokens and is masked as keys; the result holds the real tokens only.
    Padded grids run in tiled mode, which masks the padding keys.

    top_p selects key blocks by mass instead of count (topp_block_mask), with
    probabilities softmax(top_p_scale * scores), top_p_scale defaulting to
    1/sqrt(D); budget and topk are then unused.

    tiled=True runs the permutation inside the summaries and attention kernels
    (no permuted copies; blocks of 32, 64 or 128 tokens, see tiled_supported); tiled=False
    runs the explicit permute / unpermute steps; None picks tiled when it is
    supported.  Both give identical results.  In tiled mode the permuted
    tensors in the intermediates are computed afterwards, for inspection only.
    """
    tiles = [tuple(t) for t in tiles]
    vols = {t[0] * t[1] * t[2] for t in tiles}
    if len(vols) != 1:
        raise ValueError("candidate tiles must share one volume (the block size)")
    block = vols.pop()
    B, H, S, D = _bhsd(q, "q")
    pgrid = padded_grid(grid, tiles)
    nb = _grid_tokens(pgrid) // block
    kk = topk if topk is not None else topk_budget(nb, budget if budget is not None else 0.17)
    can_tile = block in (32, 64, 128) and tiled_supported(tiles)
    if compensate:
        if block != 128:
            raise NotImplementedError("compensated attention takes 128-token blocks")
        if tuple(pgrid) != tuple(grid):
            raise NotImplementedError(f"compensated attention needs a grid the tiles divide; {tuple(grid)} "
                                      f"is padded to {pgrid}")
    if tiled is None:
        tiled = can_tile
    elif tiled and not can_tile:
        raise ValueError("tiled mode needs blocks of 32, 64 or 128 tokens whose tiles satisfy tiled_supported()")
    if not tiled and tuple(pgrid) != tuple(grid):
        raise NotImplementedError(f"grid {tuple(grid)} is padded to {pgrid}: its padding keys are masked in "
                                  "tiled mode only (see tiled_supported)")
    choice = select_tiling(q, grid, tiles) if len(tiles) > 1 else None
    if tiled:
        qb, kb, vb = _bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v")
        qmax, qmin = block_summaries_tiled(q, grid, tiles, choice, block)
        kmax, kmin = block_summaries_tiled(k, grid, tiles, choice, block)
        scores = block_scores(qmax, qmin, kmax, kmin)
        idx, cnt = _select_blocks(scores, kk, n_sink_blocks, diag_halfwidth, top_p, top_p_scale, D)
        if compensate:
            o = centroid_compensated_attention_tiled(qb, kb, vb, grid, tiles, choice, idx, cnt, scale, out_dtype)
        else:
            o = block_sparse_attention_tiled(qb, kb, vb, grid, tiles, choice, idx, cnt, scale, out_dtype)
        if return_intermediates:
            qp, kp, vp, op = (permute(x, grid, tiles, choice) for x in (q, k, v, o))
    else:
        qp, kp, vp = (permute(x, grid, tiles, choice) for x in (q, k, v))
        qmax, qmin = block_summaries(qp, block)
        kmax, kmin = block_summaries(kp, block)
        scores = block_scores(qmax, qmin, kmax, kmin)
        idx, cnt = _select_blocks(scores, kk, n_sink_blocks, diag_halfwidth, top_p, top_p_scale, D)
        if compensate:
            op = centroid_compensated_attention(qp, kp, vp, idx, cnt, block, scale, out_dtype)
        else:
            op = block_sparse_attention(qp, kp, vp, idx, cnt, block, 0, scale, out_dtype)
        o = unpermute(op, grid, tiles, choice)
    if return_intermediates:
        return o, dict(choice=choice, qp=qp, kp=kp, vp=vp, qmax=qmax, qmin=qmin, kmax=kmax, kmin=kmin,
                       scores=scores, idx=idx, cnt=cnt, out_perm=op, block=block, k=kk, padded_grid=pgrid)
    return o


def spade_attention_host(q, k, v, grid, tiles, out: Optional[torch.Tensor] = None, chunks: Optional[int] = None,
                         device=None, budget: Optional[float] = None, topk: Optional[int] = None,
                         n_sink_blocks: int = 1, diag_halfwidth: int = 0, scale: Optional[float] = None,
                         out_dtype=None) -> torch.Tensor:
    """spade_attention for bf16 inputs and an output in (pinned) host memory,
    through vsa_spade_attention_host: the B*H (batch, head) rows are taken in
    `chunks` groups (default: one per (batch, head)) whose copies to the
    device and back overlap the kernels of other groups (see include/vsa.h).
    Allocates the device workspace and `out` (pinned) when not given, and
    returns `out` once the call's stream has finished with it."""
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{nm} must be a contiguous host tensor")
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{nm} must be bfloat16")
    B, H, S, D = _bhsd(q, "q")
    if tuple(k.shape) != (B, H, S, D) or tuple(v.shape) != (B, H, S, D):
        raise ValueError("q/k/v shapes must match exactly")
    chunks = B * H if chunks is None else int(chunks)
    odt = _out_dtype(out_dtype, q)
    if out is None:
        out = torch.empty(q.shape, dtype=odt, pin_memory=True)
    elif out.shape != q.shape or out.dtype != odt or out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous host tensor of q's shape and the output dtype")
    tiles = [tuple(t) for t in tiles]
    block = min(128, tiles[0][0] * tiles[0][1] * tiles[0][2])
    nb = _grid_tokens(padded_grid(grid, tiles)) // block
    kk = topk if topk is not None else topk_budget(nb, budget if budget is not None else 0.17)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    arr, n = _tiles_arg(tiles)
    g = Dims3(*grid)
    oc = BF16 if odt == torch.bfloat16 else F32
    need = lib().vsa_spade_attention_host_workspace_size(B, H, S, D, g, arr, n, int(kk), int(n_sink_blocks),
                                                         int(diag_halfwidth), oc, int(chunks))
    if need == 0:
        raise ValueError(f"no valid workspace size for these arguments ({last_error() or 'check the shapes'})")
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = torch.cuda.current_stream(dev)
        _check(lib().vsa_spade_attention_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), oc, B, H, S, D, g, arr, n,
                                              int(kk), int(n_sink_blocks), int(diag_halfwidth),
                                              0.0 if scale is None else float(scale), int(chunks), _ptr(ws), need,
                                              ctypes.c_void_p(st.cuda_stream)))
        st.synchronize()
    return out


def structured_attention(q, k, v, kind: str, grid, block: int = 128, tile=(4, 8, 8), radius=(1, 1, 1),
                         scale: Optional[float] = None, out_dtype=None):
    """A structured static mask as block-sparse attention, in and out in T-major order."""
    st = structured_tile(kind, grid, tile)
    # when T divides the block, temporal-only lists hold the diagonal block
    # alone: a one-slot list lets the attention use its one-key-block kernel
    one = kind == "temporal" and block % grid[0] == 0
    idx, cnt, g = structured_block_list(kind, grid, block, tile, radius, device=q.device, cap=1 if one else None)
    if st[1] == grid[1] and st[2] == grid[2]:  # whole frames: the tile-contiguous order is T-major itself
        return block_sparse_attention(q, k, v, idx, cnt, block, g, scale, out_dtype)
    T = grid[0]
    if kind == "temporal" and block == 128 and T <= 128 and 128 % T == 0 and grid[2] % (128 // T) == 0:
        # tile (T, 1, 128/T): a block is all frames of 128/T neighbouring columns, position
        # t * s + w with s = 128/T, and the temporal mask is "same w", i.e. equal mod s;
        # the diagonal list is the same as for tile (T, 1, 1)
        s = 128 // T
        return block_sparse_attention_tiled(q, k, v, grid, [(T, 1, s)], None, idx, cnt, scale, out_dtype,
                                            group_stride=s if s > 1 else 0)
    if g == 0 and block == 128 and tiled_supported([st]):
        return block_sparse_attention_tiled(q, k, v, grid, [st], None, idx, cnt, scale, out_dtype)
    qp, kp, vp = (permute(x, grid, [st]) for x in (q, k, v))
    op = block_sparse_attention(qp, kp, vp, idx, cnt, block, g, scale, out_dtype)
    return unpermute(op, grid, [st])
