"""Parity of the CUDA path (through the C ABI) against the fp64 oracle.

Integer and index outputs (permutations, summaries, block lists, tiling
choices with a clear margin) must match bit for bit.  Attention outputs, with
bf16 inputs and fp32 accumulation, must be within max-abs 1e-2 and relative-L2
2e-3 of the fp64 oracle; that bar is applied to the kernel's fp32-output mode.
A bf16 output is that fp32 result rounded once to nearest-even (checked bit
for bit): bf16's unit roundoff 2^-8 alone puts about 1.6e-3 of relative-L2
error on any bf16 output.  Inputs come from the seeded generators in
`workloads`.
"""

import numpy as np
import pytest
import torch

import block_sparse_self_b200 as vsa
import oracle
from workloads import WORKLOADS, integer_grid, make_qkv, random_scores, smooth_qkv

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 1e-2, 2e-3
DEV = "cuda"


@pytest.fixture(autouse=True)
def _no_device_errors():
    yield
    vsa.device_status()  # raises if any kernel of the test recorded a failure


def _np(t):
    return t.detach().float().cpu().numpy()


def assert_attn_close(got, want, what=""):
    g = np.asarray(got, np.float64)
    w = np.asarray(want, np.float64)
    err = np.abs(g - w).max()
    rl2 = np.linalg.norm(g - w) / max(np.linalg.norm(w), 1e-30)
    assert np.isfinite(g).all(), what
    assert err <= MAX_ABS and rl2 <= REL_L2, f"{what}: max-abs {err:.3e}, rel-L2 {rl2:.3e}"


# --------------------------------------------------------------------------
# permutation
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,D", [(torch.float32, 64), (torch.bfloat16, 128), (torch.bfloat16, 64),
                                     (torch.float32, 128)])
def test_permute_matches_oracle_permutation(dtype, D):
    grid, tiles = (4, 8, 16), [(1, 8, 16), (2, 8, 8), (4, 4, 8)]
    x = integer_grid((2, 3, 512, D), 11, dtype, DEV)
    choice = torch.tensor([2, 0, 1, 1, 2, 0], dtype=torch.int32, device=DEV)
    y = vsa.permute(x, grid, tiles, choice)
    xb = x.cpu()
    for bh, c in enumerate(choice.tolist()):
        perm = torch.as_tensor(oracle.tile_permutation(grid, tiles[c]))
        assert torch.equal(y.cpu().view(6, 512, D)[bh], xb.view(6, 512, D)[bh][perm])
    assert torch.equal(vsa.unpermute(y, grid, tiles, choice), x)


def test_permute_without_choice_and_ragged_rows():
    grid, tile = (3, 4, 6), (1, 2, 3)   # S = 72: fewer rows than one work item
    x = integer_grid((1, 2, 72, 64), 12, torch.bfloat16, DEV)
    y = vsa.permute(x, grid, [tile])
    perm = torch.as_tensor(oracle.tile_permutation(grid, tile))
    assert torch.equal(y.cpu(), x.cpu()[:, :, perm])
    assert torch.equal(vsa.unpermute(y, grid, [tile]), x)


def test_permute_bad_choice_sets_runtime_status():
    grid, tiles = (2, 8, 8), [(1, 8, 8), (2, 4, 4)]
    x = integer_grid((1, 2, 128, 64), 13, torch.bfloat16, DEV)
    choice = torch.tensor([0, 5], dtype=torch.int32, device=DEV)
    vsa.permute(x, grid, tiles, choice)
    with pytest.raises(RuntimeError):
        vsa.device_status()


# --------------------------------------------------------------------------
# summaries, scores, top-k
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,D,block", [(torch.bfloat16, 128, 128), (torch.bfloat16, 64, 16),
                                           (torch.float32, 64, 32), (torch.float32, 128, 256)])
def test_block_summaries_bit_exact(dtype, D, block):
    S = 1024
    x = torch.randn(2, 2, S, D, generator=torch.Generator(DEV).manual_seed(3), device=DEV).to(dtype)
    mx, mn = vsa.block_summaries(x, block)
    for bh in range(4):
        omx, omn = oracle.block_minmax(_np(x.view(4, S, D)[bh]), block)
        assert np.array_equal(_np(mx.view(4, -1, D)[bh]), omx)
        assert np.array_equal(_np(mn.view(4, -1, D)[bh]), omn)


@pytest.mark.parametrize("dtype,D,block", [(torch.bfloat16, 128, 128), (torch.float32, 64, 32),
                                           (torch.bfloat16, 64, 256), (torch.float32, 128, 16)])
def test_block_summaries_tiled_matches_oracle_and_permuted_path(dtype, D, block):
    """Summaries read from T-major x through each head's tiling equal those of
    the permuted copy, bit for bit, and the oracle's."""
    grid, tiles = (4, 8, 16), [(1, 8, 16), (2, 8, 8), (4, 4, 8)]
    S = 512
    x = torch.randn(2, 3, S, D, generator=torch.Generator(DEV).manual_seed(71), device=DEV).to(dtype)
    choice = torch.tensor([2, 0, 1, 1, 2, 0], dtype=torch.int32, device=DEV)
    mx, mn = vsa.block_summaries_tiled(x, grid, tiles, choice, block)
    wmx, wmn = vsa.block_summaries(vsa.permute(x, grid, tiles, choice), block)
    assert torch.equal(mx, wmx) and torch.equal(mn, wmn)
    for bh, c in enumerate(choice.tolist()):
        xp = oracle.permute_rows(_np(x.view(6, S, D)[bh]), oracle.tile_permutation(grid, tiles[c]))
        omx, omn = oracle.block_minmax(xp, block)
        assert np.array_equal(_np(mx.view(6, -1, D)[bh]), omx)
        assert np.array_equal(_np(mn.view(6, -1, D)[bh]), omn)
    # no choice: tile 0 for every head
    mx0, _ = vsa.block_summaries_tiled(x, grid, tiles, None, block)
    assert torch.equal(mx0, vsa.block_summaries(vsa.permute(x, grid, tiles[:1]), block)[0])


@pytest.mark.parametrize("grid,tiles,block", [((2, 8, 8), [(1, 8, 8), (2, 4, 4)], 64),
                                              ((2, 8, 16), [(1, 8, 16), (2, 8, 8)], 128)])
def test_block_summaries_tiled_bad_choice_sets_runtime_status(grid, tiles, block):
    """A choice out of range leaves that head unwritten and sets the status, in
    the row-gather kernel (64-token blocks) and the TMA one (128-token boxes);
    the other head is still summarised."""
    S = grid[0] * grid[1] * grid[2]
    x = integer_grid((1, 2, S, 64), 72, torch.bfloat16, DEV)
    mx, mn = vsa.block_summaries_tiled(x, grid, tiles, torch.tensor([1, -1], dtype=torch.int32, device=DEV), block)
    with pytest.raises(RuntimeError):
        vsa.device_status()
    want = vsa.block_summaries(vsa.permute(x[:, :1], grid, tiles[1:]), block)
    assert torch.equal(mx[:, :1], want[0]) and torch.equal(mn[:, :1], want[1])


@pytest.mark.parametrize("dtype,D,nb", [(torch.bfloat16, 128, 40), (torch.float32, 64, 70), (torch.bfloat16, 64, 1),
                                        (torch.bfloat16, 128, 300), (torch.bfloat16, 64, 129)])
def test_block_scores_exact_on_integer_grid(dtype, D, nb):
    summ = [integer_grid((1, 2, nb, D), 20 + i, dtype, DEV) for i in range(4)]
    s = vsa.block_scores(*summ)
    for h in range(2):
        want = oracle.block_scores(*(_np(t[0, h]) for t in summ))
        assert np.array_equal(_np(s[0, h]).astype(np.float64), want)


def test_block_scores_smooth_within_fp32_bound():
    q, k, _ = smooth_qkv(1, 2, (4, 16, 32), 128, seed=5, device=DEV)
    qp, kp = (vsa.permute(t, (4, 16, 32), [(1, 8, 16)]) for t in (q, k))
    qmax, qmin = vsa.block_summaries(qp, 128)
    kmax, kmin = vsa.block_summaries(kp, 128)
    s = vsa.block_scores(qmax, qmin, kmax, kmin)
    for h in range(2):
        a = [_np(t[0, h]).astype(np.float64) for t in (qmax, qmin, kmax, kmin)]
        want = oracle.block_scores(*a)
        # fp32 accumulation of q_max.k + q_min.k over 2D exact products
        bound = 4 * np.finfo(np.float32).eps * ((np.abs(a[0]) + np.abs(a[1])) @ np.maximum(np.abs(a[2]), np.abs(a[3])).T)
        assert (np.abs(_np(s[0, h]) - want) <= bound + 1e-30).all()


@pytest.mark.parametrize("nb,levels", [(1, 3), (5, 2), (33, 3), (240, 4), (240, 0), (960, 6)])
def test_topk_lists_bit_exact(nb, levels):
    sc = random_scores((2, 2, nb, nb), seed=nb + levels, levels=levels, device=DEV)
    if levels == 0:
        sc[0, 0, :, 3] = -0.0   # -0 and +0 must rank as equal
        sc[0, 0, :, 4] = 0.0
    settings = [(max(1, nb // 6), 1, 0), (1, 0, -1), (nb, 1, 0), (max(1, nb // 10), min(3, nb), 2)]
    for k, n_sink, dw in settings:
        idx, cnt = vsa.topk_block_mask(sc, k, n_sink, dw)
        for bh in range(4):
            oi, oc = oracle.topk_block_list(_np(sc.view(4, nb, nb)[bh]).astype(np.float64), k, n_sink, dw,
                                            cap=idx.shape[-1])
            assert np.array_equal(idx.view(4, nb, -1)[bh].cpu().numpy(), oi), (nb, k, n_sink, dw, bh)
            assert np.array_equal(cnt.view(4, nb)[bh].cpu().numpy(), oc)


@pytest.mark.parametrize("nb", [200, 960, 1000])
@pytest.mark.parametrize("kind", ["negative", "narrow", "wide_ties", "spread", "infinite", "clustered"])
def test_topk_threshold_search_paths(nb, kind):
    """Score rows that drive the threshold search down each of its paths: all
    negative (padded slots share the threshold's prefix), values within a few
    ulps of each other (many keys share every prefix), exact ties wider than
    the candidate buffer, magnitudes spread over many octaves (most of a
    row's histogram in its end bins), infinite scores (no finite value range
    to bin) and two far-apart clusters (the threshold's bin crowded)."""
    g = torch.Generator(DEV).manual_seed(nb + len(kind))
    x = torch.randn(2, 1, nb, nb, generator=g, device=DEV)
    if kind == "negative":
        sc = -x.abs() - 100.0
    elif kind == "narrow":
        sc = 1.0 + x * 1e-6
    elif kind == "wide_ties":
        sc = torch.where(x > -0.5, torch.full_like(x, 2.5), x)  # ~70% of each row ties at the top
    elif kind == "infinite":
        sc = x.clone()
        sc[..., 5] = float("inf")
        sc[..., 9] = float("-inf")
        sc[..., 11] = float("inf")
    elif kind == "clustered":
        sc = torch.where(x > 0.3, 1e6 + x, x)
    else:
        sc = torch.sign(x) * torch.exp2(x * 20.0)
    sc = sc.contiguous()
    for k, n_sink, dw in [(max(1, nb // 10), 1, 0), (max(1, nb // 3), 0, -1)]:
        idx, cnt = vsa.topk_block_mask(sc, k, n_sink, dw)
        for bh in range(2):
            oi, oc = oracle.topk_block_list(_np(sc.view(2, nb, nb)[bh]).astype(np.float64), k, n_sink, dw,
                                            cap=idx.shape[-1])
            assert np.array_equal(idx.view(2, nb, -1)[bh].cpu().numpy(), oi), (kind, nb, k, bh)
            assert np.array_equal(cnt.view(2, nb)[bh].cpu().numpy(), oc)


@pytest.mark.parametrize("nb,D", [(1, 64), (33, 128), (240, 128), (300, 64), (960, 128), (1024, 64)])
def test_fused_scores_topk_bit_exact(nb, D):
    """The fused scores-and-lists kernel on integer-grid summaries (exact
    scores): lists equal the oracle's and the separate scores -> top-k path's
    bit for bit, for several budgets, sink counts and diagonal widths."""
    summ = [integer_grid((2, 2, nb, D), 40 + i, torch.bfloat16, DEV) for i in range(4)]
    settings = [(max(1, nb // 10), 1, 0), (1, 0, -1), (nb, 1, 0), (max(1, nb // 6), min(3, nb), 2)]
    for k, n_sink, dw in settings:
        fi, fc = vsa.block_scores_topk(*summ, k, n_sink, dw)
        si, sc_ = vsa.topk_block_mask(vsa.block_scores(*summ), k, n_sink, dw)
        assert torch.equal(fi, si) and torch.equal(fc, sc_), (nb, D, k, n_sink, dw)
        for bh in range(4):
            s = oracle.block_scores(*(_np(x.view(4, nb, D)[bh]) for x in summ))
            oi, oc = oracle.topk_block_list(s, k, n_sink, dw, cap=fi.shape[-1])
            assert np.array_equal(fi.view(4, nb, -1)[bh].cpu().numpy(), oi), (nb, k, n_sink, dw, bh)
            assert np.array_equal(fc.view(4, nb)[bh].cpu().numpy(), oc)


def test_fused_scores_topk_adaptive_full_size():
    """The S = 122880 adaptive step's summaries (smooth fields, 24 heads, k =
    96): the fused kernel's lists against the separate path's and, where they
    differ, as valid top-k sets under the oracle's scores within the fp32
    allowance."""
    w = WORKLOADS["spade_adaptive_s122880"]
    q, k, v = make_qkv(w, device=DEV)
    choice = vsa.select_tiling(q, w.grid, list(w.tiles))
    summ = [*vsa.block_summaries_tiled(q, w.grid, list(w.tiles), choice, 128),
            *vsa.block_summaries_tiled(k, w.grid, list(w.tiles), choice, 128)]
    fi, fc = vsa.block_scores_topk(*summ, w.k)
    si, sc_ = vsa.topk_block_mask(vsa.block_scores(*summ), w.k)
    same = (fi == si).all(-1)
    print(f"rows whose fused list differs from the separate path's: {int((~same).sum())} of {same.numel()}")
    for h in torch.nonzero(~same.all(-1).view(-1)).flatten().tolist()[:3]:
        res = {"qmax": _np(summ[0][0, h]).astype(np.float64), "qmin": _np(summ[1][0, h]).astype(np.float64),
               "kmax": _np(summ[2][0, h]).astype(np.float64), "kmin": _np(summ[3][0, h]).astype(np.float64)}
        s = oracle.block_scores(res["qmax"], res["qmin"], res["kmax"], res["kmin"])
        bound = SCORE_EPS * _abs_terms(res)
        gi, gc = fi[0, h].cpu().numpy(), fc[0, h].cpu().numpy()
        for i in range(w.nb):
            sel = set(gi[i, :gc[i]].tolist())
            forced = {0, i}
            assert forced <= sel and w.k <= len(sel) <= w.k + len(forced)
            order = np.lexsort((np.arange(w.nb), -s[i]))
            kth = order[w.k - 1]
            tol = bound[i] + bound[i, kth]
            assert all(s[i, j] >= s[i, kth] - tol[j] for j in sel - forced), (h, i)
            assert all(s[i, j] <= s[i, kth] + tol[j] for j in set(range(w.nb)) - sel), (h, i)


# --------------------------------------------------------------------------
# structured lists
# --------------------------------------------------------------------------

@pytest.mark.parametrize("grid,block,tile", [((32, 48, 80), 128, (4, 8, 8)), ((8, 4, 8), 32, (2, 2, 8)),
                                             ((6, 12, 16), 64, (2, 4, 8))])
def test_structured_lists_match_oracle(grid, block, tile):
    for kind in ("spatial", "temporal", "sliding_tile", "sliding_tile_centered"):
        try:
            idx, cnt, g = vsa.structured_block_list(kind, grid, block, tile=tile, radius=(1, 1, 1))
        except NotImplementedError:   # e.g. temporal groups of 6 tokens in blocks of 64
            t, r = oracle.structured_tile(kind, grid, tile, (1, 1, 1))
            with pytest.raises(ValueError):
                oracle.tile_neighbourhood_list(grid, t, r, block)
            continue
        t, r = oracle.structured_tile(kind, grid, tile, (1, 1, 1))
        oi, oc, og = oracle.tile_neighbourhood_list(grid, t, r, block, cap=idx.shape[1],
                                                    centered=kind == "sliding_tile_centered")
        assert g == og
        assert np.array_equal(cnt.cpu().numpy(), oc)
        assert np.array_equal(idx.cpu().numpy(), oi)


# --------------------------------------------------------------------------
# adaptive tiling choice
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_select_tiling_matches_oracle(dtype, D):
    grid, tiles = (8, 16, 32), [(1, 8, 16), (2, 8, 8), (4, 4, 8)]
    kinds = ["spatial", "temporal", "generic", "spatial", "temporal", "generic"]
    q, _, _ = smooth_qkv(1, 6, grid, D, seed=9, kinds=kinds, dtype=dtype, device=DEV)
    choice, sics = vsa.select_tiling(q, grid, tiles, return_sics=True)
    flips = 0
    for h in range(6):
        oc, osc = oracle.select_tiling(_np(q[0, h]), grid, tiles)
        np.testing.assert_allclose(_np(sics[h]), osc, atol=2e-5, rtol=0)
        margin = np.sort(osc)[-1] - np.sort(osc)[-2]
        if margin > 1e-4:
            assert int(choice[h]) == oc, (h, osc)
        else:
            flips += 1
    assert flips <= 1


# Region geometries of the tiling choice: the candidates' per-axis lcm region
# and gcd cells in several shapes (one frame per 128-token box of the region,
# several frames, a cell spanning several frames, a padded grid).
SICS_TILE_SETS = [
    ((8, 16, 32), [(1, 8, 16), (2, 8, 8), (4, 4, 8)]),   # 16 cells of 1 x 4 x 8
    ((8, 16, 32), [(2, 4, 8), (4, 4, 4)]),               # cells two frames deep
    ((16, 16, 32), [(4, 8, 16), (8, 8, 16)]),            # two cells of 512 tokens
    ((8, 16, 16), [(4, 4, 8), (2, 8, 8)]),
    ((8, 16, 32), [(1, 16, 8), (2, 8, 8)]),
    ((6, 21, 36), [(1, 8, 16), (2, 8, 8), (4, 4, 8)]),   # padded grid: regions cross its edge
]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("case", range(len(SICS_TILE_SETS)))
def test_select_tiling_region_geometries(case, D):
    """Each head's cohesion per candidate against the oracle's on several
    region geometries, bf16 and fp32 inputs of the same values agreeing."""
    grid, tiles = SICS_TILE_SETS[case]
    kinds = ["spatial", "temporal", "generic", "spatial"]
    q, _, _ = smooth_qkv(1, 4, grid, D, seed=300 + case, kinds=kinds, device=DEV)
    choice, sics = vsa.select_tiling(q, grid, tiles, return_sics=True)
    choice32, sics32 = vsa.select_tiling(q.float(), grid, tiles, return_sics=True)
    np.testing.assert_allclose(_np(sics), _np(sics32), atol=2e-6, rtol=0)
    pg = oracle.padded_grid(grid, tiles)
    for h in range(4):
        qh = _np(q[0, h])
        if tuple(pg) != tuple(grid):
            qh = oracle.pad_grid(qh, grid, pg)
        oc, osc = oracle.select_tiling(qh, pg, tiles)
        np.testing.assert_allclose(_np(sics[h]), osc, atol=2e-5, rtol=0)
        if np.sort(osc)[-1] - np.sort(osc)[-2] > 1e-4:
            assert int(choice[h]) == oc and int(choice32[h]) == oc, (h, osc)
    assert torch.equal(choice, vsa.select_tiling_noalloc(q, grid, tiles))


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def _random_lists(nb, cap, bh, seed, full_row=True):
    rng = np.random.default_rng(seed)
    idx = np.full((bh, nb, cap), -1, np.int32)
    cnt = np.zeros((bh, nb), np.int32)
    for b in range(bh):
        for i in range(nb):
            n = int(rng.integers(1, cap + 1))
            if full_row and i == nb - 1:
                n = cap
            sel = np.sort(rng.choice(nb, n, replace=False))
            idx[b, i, :n] = sel
            cnt[b, i] = n
    return idx, cnt


@pytest.mark.parametrize("D,block,values", [(64, 32, "integer"), (128, 64, "smooth"), (128, 128, "smooth"),
                                            (64, 128, "integer"), (128, 32, "smooth"), (64, 64, "smooth")])
def test_block_sparse_attention_random_lists(D, block, values):
    B, H, S = 1, 2, 768
    nb = S // block
    if values == "integer":
        q, k, v = (integer_grid((B, H, S, D), 40 + i, torch.bfloat16, DEV) for i in range(3))
    else:
        q, k, v = smooth_qkv(B, H, (3, 16, 16), D, seed=41, device=DEV)
    idx, cnt = _random_lists(nb, min(nb, 5), B * H, seed=block + D)
    ti = torch.as_tensor(idx, device=DEV).view(B, H, nb, -1)
    tc = torch.as_tensor(cnt, device=DEV).view(B, H, nb)
    o = vsa.block_sparse_attention(q, k, v, ti, tc, block, out_dtype=torch.float32)
    ob = vsa.block_sparse_attention(q, k, v, ti, tc, block, out_dtype=torch.bfloat16)
    assert torch.equal(ob, o.to(torch.bfloat16))
    for h in range(H):
        want = oracle.block_sparse_attention(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), idx[h], cnt[h], block)
        assert_attn_close(_np(o[0, h]), want, f"head {h}")


@pytest.mark.parametrize("D,grid,tiles,values", [
    (128, (4, 8, 16), [(1, 8, 16), (2, 8, 8), (4, 4, 8)], "smooth"),   # volume 128: one block per tile
    (64, (4, 8, 16), [(2, 8, 16), (4, 8, 8)], "integer"),               # volume 256: two blocks per tile
    (128, (8, 8, 8), [(4, 8, 8), (8, 4, 8)], "smooth"),                 # volume 256, every tile.t even
])
def test_block_sparse_attention_tiled_matches_oracle_and_permuted_path(D, grid, tiles, values):
    """T-major attention through each head's tiling (TMA boxes in, token rows
    out) equals permute -> attention -> unpermute bit for bit, and the oracle."""
    B, H = 2, 2
    S = grid[0] * grid[1] * grid[2]
    nb = S // 128
    if values == "integer":
        q, k, v = (integer_grid((B, H, S, D), 73 + i, torch.bfloat16, DEV) for i in range(3))
    else:
        q, k, v = smooth_qkv(B, H, grid, D, seed=74, device=DEV)
    choice = torch.tensor([(i * 5 + 1) % len(tiles) for i in range(B * H)], dtype=torch.int32, device=DEV)
    idx, cnt = _random_lists(nb, min(nb, 3), B * H, seed=D + nb)
    ti = torch.as_tensor(idx, device=DEV).view(B, H, nb, -1)
    tc = torch.as_tensor(cnt, device=DEV).view(B, H, nb)
    o = vsa.block_sparse_attention_tiled(q, k, v, grid, tiles, choice, ti, tc, out_dtype=torch.float32)
    ob = vsa.block_sparse_attention_tiled(q, k, v, grid, tiles, choice, ti, tc, out_dtype=torch.bfloat16)
    assert torch.equal(ob, o.to(torch.bfloat16))
    qp, kp, vp = (vsa.permute(x, grid, tiles, choice) for x in (q, k, v))
    op = vsa.block_sparse_attention(qp, kp, vp, ti, tc, 128, out_dtype=torch.float32)
    assert torch.equal(o, vsa.unpermute(op, grid, tiles, choice))
    for bh, c in enumerate(choice.tolist()):
        b, h = divmod(bh, H)
        perm = oracle.tile_permutation(grid, tiles[c])
        qo, ko, vo = (oracle.permute_rows(_np(x[b, h]), perm) for x in (q, k, v))
        want = oracle.block_sparse_attention(qo, ko, vo, idx[bh], cnt[bh], 128)
        assert_attn_close(_np(o[b, h])[perm], want, f"b{b} h{h}")


def test_block_sparse_attention_tiled_bad_choice_and_lists():
    grid, tiles = (2, 8, 16), [(1, 8, 16), (2, 8, 8)]
    q, k, v = (integer_grid((1, 2, 256, 64), 75 + i, torch.bfloat16, DEV) for i in range(3))
    idx = torch.tensor([[0, 1], [0, 1], [1, 0], [0, 1]], dtype=torch.int32, device=DEV).view(1, 2, 2, 2)
    cnt = torch.full((1, 2, 2), 2, dtype=torch.int32, device=DEV)
    o = vsa.block_sparse_attention_tiled(q, k, v, grid, tiles, torch.tensor([0, 1], dtype=torch.int32, device=DEV),
                                         idx, cnt, out_dtype=torch.float32)
    with pytest.raises(RuntimeError):   # head 1's first list is descending
        vsa.device_status()
    perm1 = torch.as_tensor(oracle.tile_permutation(grid, tiles[1]), device=DEV)
    assert (o[0, 1][perm1[:128]] == 0).all()
    o2 = vsa.block_sparse_attention_tiled(q, k, v, grid, tiles, torch.tensor([0, 2], dtype=torch.int32, device=DEV),
                                          idx[:, :1].expand(1, 2, 2, 2).contiguous(), cnt, out_dtype=torch.float32)
    with pytest.raises(RuntimeError):   # choice 2 is out of range
        vsa.device_status()
    assert torch.isfinite(o2[0, 0]).all()
    with pytest.raises(ValueError):     # mixed volumes
        vsa.block_sparse_attention_tiled(q, k, v, grid, [(1, 8, 16), (1, 8, 8)], None, idx, cnt)
    with pytest.raises(ValueError):     # volume 256 with tile.t = 1: a block is not whole planes
        vsa.block_sparse_attention_tiled(q, k, v, (1, 16, 16), [(1, 16, 16)], None, idx, cnt)


@pytest.mark.parametrize("D,grid", [(64, (16, 4, 16)), (128, (32, 2, 8))])
def test_temporal_attention_through_strided_groups(D, grid):
    """temporal_only via tile (T, 1, 128/T) and a strided group mask, with no
    permuted copies, against the oracle's same-(h, w) attention."""
    q, k, v = smooth_qkv(1, 2, grid, D, seed=76, device=DEV)
    o = vsa.structured_attention(q, k, v, "temporal", grid, 128, out_dtype=torch.float32)
    t, r = oracle.structured_tile("temporal", grid)
    idx, cnt, g = oracle.tile_neighbourhood_list(grid, t, r, 128)
    perm = oracle.tile_permutation(grid, t)
    for h in range(2):
        qp, kp, vp = (oracle.permute_rows(_np(x[0, h]), perm) for x in (q, k, v))
        op = oracle.block_sparse_attention(qp, kp, vp, idx, cnt, 128, g)
        want = np.empty_like(op)
        want[perm] = op
        assert_attn_close(_np(o[0, h]), want, f"h{h}")
    qb, kb, vb = (x.to(torch.bfloat16) for x in (q, k, v))
    ti = torch.as_tensor(idx, device=DEV)
    tc = torch.as_tensor(cnt, device=DEV)
    with pytest.raises(ValueError):   # a stride must be a power of two
        vsa.block_sparse_attention_tiled(qb, kb, vb, grid, [(grid[0], 1, 128 // grid[0])], None, ti, tc,
                                         group_stride=3)


def test_block_sparse_attention_group_mask_and_shared_list():
    """temporal_only: tile (T,1,1) with T=8 inside blocks of 32 -> group mask."""
    grid, block = (8, 8, 8), 32
    q, k, v = smooth_qkv(2, 2, grid, 64, seed=44, device=DEV)
    o = vsa.structured_attention(q, k, v, "temporal", grid, block, out_dtype=torch.float32)
    t, r = oracle.structured_tile("temporal", grid)
    idx, cnt, g = oracle.tile_neighbourhood_list(grid, t, r, block)
    assert g == 8
    perm = oracle.tile_permutation(grid, t)
    for b in range(2):
        for h in range(2):
            qp, kp, vp = (oracle.permute_rows(_np(x[b, h]), perm) for x in (q, k, v))
            op = oracle.block_sparse_attention(qp, kp, vp, idx, cnt, block, g)
            want = np.empty_like(op)
            want[perm] = op
            assert_attn_close(_np(o[b, h]), want, f"b{b} h{h}")


def test_block_sparse_attention_invalid_lists_write_zeros_and_set_status():
    B, H, S, D, block = 1, 1, 512, 64, 128
    q, k, v = (integer_grid((B, H, S, D), 50 + i, torch.bfloat16, DEV) for i in range(3))
    idx = torch.tensor([[[0, 1], [1, 0], [2, 9], [3, -1]]], dtype=torch.int32, device=DEV).view(1, 1, 4, 2)
    cnt = torch.tensor([2, 2, 2, 0], dtype=torch.int32, device=DEV).view(1, 1, 4)
    o = vsa.block_sparse_attention(q, k, v, idx, cnt, block, out_dtype=torch.float32)
    with pytest.raises(RuntimeError):
        vsa.device_status()
    oo = o.cpu()
    assert (oo[0, 0, 128:] == 0).all()          # descending, out of range, empty
    want = oracle.block_sparse_attention(_np(q[0, 0]), _np(k[0, 0]), _np(v[0, 0]), np.array([[0, 1]], np.int32),
                                         np.array([2], np.int32), block, rows=np.arange(128))
    assert_attn_close(_np(oo[0, 0, :128]), want)


@pytest.mark.parametrize("S,D,window,sink", [(256, 64, 64, 16), (300, 128, 100, 7), (1000, 64, 2000, 0),
                                             (384, 128, 1, 0), (640, 64, 257, 300), (1280, 128, 300, 128),
                                             (129, 64, 128, 1)])
def test_window_attention_matches_oracle(S, D, window, sink):
    q, k, v = (integer_grid((1, 2, S, D), 60 + i, torch.bfloat16, DEV) for i in range(3))
    o = vsa.window_attention(q, k, v, window, sink, out_dtype=torch.float32)
    assert torch.equal(vsa.window_attention(q, k, v, window, sink), o.to(torch.bfloat16))
    for h in range(2):
        want = oracle.window_attention(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), window, sink)
        assert_attn_close(_np(o[0, h]), want, f"head {h}")
    # the page's query chunk size groups the work but never changes the result
    o2 = vsa.window_attention(q, k, v, window, sink, chunk_size=7, out_dtype=torch.float32)
    assert torch.equal(o, o2)


def test_wait_timeout_is_reported():
    vsa.debug_wait_timeout(2_000_000)  # 2 ms
    with pytest.raises(RuntimeError, match="timeout"):
        vsa.device_status()


# --------------------------------------------------------------------------
# end to end on the tiny workload, then sampled checks at full size
# --------------------------------------------------------------------------

def test_tiny_workload_end_to_end():
    w = WORKLOADS["tiny_s256"]
    q, k, v = make_qkv(w, device=DEV)                  # fp32 values on the {-4..4}/4 grid
    o, mid = vsa.spade_attention(q, k, v, w.grid, list(w.tiles), topk=w.k, n_sink_blocks=1, diag_halfwidth=0,
                                 out_dtype=torch.float32, return_intermediates=True)
    ow = vsa.window_attention(q, k, v, w.window, w.sink, out_dtype=torch.float32)
    for h in range(w.heads):
        res = oracle.spade_head(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), w.grid, list(w.tiles), w.k)
        assert np.array_equal(mid["idx"][0, h].cpu().numpy(), res["idx"])
        assert np.array_equal(mid["cnt"][0, h].cpu().numpy(), res["cnt"])
        assert np.array_equal(_np(mid["scores"][0, h]).astype(np.float64), res["score"])
        assert_attn_close(_np(o[0, h]), res["out"], f"spade head {h}")
        want = oracle.window_attention(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), w.window, w.sink)
        assert_attn_close(_np(ow[0, h]), want, f"window head {h}")


@pytest.mark.parametrize("chunks", [1, 3, 8])
def test_spade_attention_host_buffers_match_device(chunks):
    """The host-buffer entry point (copies of one group of heads overlapping
    the kernels of another) returns exactly the device result."""
    grid, tiles = (4, 8, 16), [(1, 8, 16), (2, 8, 8), (4, 4, 8)]
    q, k, v = smooth_qkv(2, 3, grid, 128, seed=77, device=DEV)
    want = vsa.spade_attention(q, k, v, grid, tiles, topk=2, out_dtype=torch.float32)
    qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
    got = vsa.spade_attention_host(qh, kh, vh, grid, tiles, chunks=chunks, topk=2, out_dtype=torch.float32)
    assert not got.is_cuda and torch.equal(got, want.cpu())


@pytest.mark.parametrize("grid,tiles,chunks,out", [
    ((4, 9, 16), [(1, 8, 16), (2, 8, 8), (4, 4, 8)], 4, torch.float32),   # padded to (4, 16, 16)
    ((4, 8, 16), [(2, 8, 8)], 2, torch.bfloat16),                        # one candidate: no tiling choice
    ((4, 8, 16), [(1, 4, 16), (1, 8, 8)], 64, torch.float32),           # 64-token tiles; more groups than heads
])
def test_spade_attention_host_more_shapes(grid, tiles, chunks, out):
    """The host-buffer entry point on a padded grid, with a single candidate,
    with 64-token candidate tiles and with more groups than (b, head) rows:
    the device composition's result bit for bit."""
    q, k, v = smooth_qkv(1, 3, grid, 64, seed=78, device=DEV)
    want = vsa.spade_attention(q, k, v, grid, tiles, topk=2, out_dtype=out)
    qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
    got = vsa.spade_attention_host(qh, kh, vh, grid, tiles, chunks=chunks, topk=2, out_dtype=out)
    assert got.dtype == out and torch.equal(got, want.cpu())


def _sample_blocks(nb, seed, n=16):
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, nb - 1), n - 2, replace=False)
    return sorted({0, nb - 1, *mid.tolist()})


def test_spade_fixed_full_size_sampled():
    """40 heads, S = 30720, tile (1,8,16), k = 40: integer-grid values make
    the block scores exact, so whole lists must match bit for bit."""
    w = WORKLOADS["spade_fixed_s30720"]
    q, k, v = make_qkv(w, device=DEV, values="integer")
    o, mid = vsa.spade_attention(q, k, v, w.grid, list(w.tiles), topk=w.k, out_dtype=torch.float32,
                                 return_intermediates=True)
    for h in (0, 23, 39):
        blocks = _sample_blocks(w.nb, h)
        res = oracle.spade_head(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), w.grid, list(w.tiles), w.k,
                                query_blocks=blocks)
        assert np.array_equal(mid["idx"][0, h].cpu().numpy(), res["idx"])
        assert np.array_equal(mid["cnt"][0, h].cpu().numpy(), res["cnt"])
        got = _np(mid["out_perm"][0, h])[res["rows"]]
        assert_attn_close(got, res["out_perm"], f"head {h}")
    # the unpermuted output is the permuted one scattered back
    perm = torch.as_tensor(oracle.tile_permutation(w.grid, w.tiles[0]), device=DEV)
    assert torch.equal(o[0, 5][perm], mid["out_perm"][0, 5])
    # tiled (in-kernel permutation) and explicit permute paths agree bit for bit
    assert torch.equal(o, vsa.spade_attention(q, k, v, w.grid, list(w.tiles), topk=w.k, out_dtype=torch.float32,
                                              tiled=False))


# Scores are fp32 sums of exact bf16 products; a GPU score may differ from the
# exact one by at most SCORE_EPS * sum|terms| (4 machine epsilons of fp32),
# the allowance for comparing lists on smooth fields.  Tiling choices are
# compared where the oracle's margin between the best two candidates exceeds
# CHOICE_MARGIN (the fp32 cohesion may rank closer candidates either way).
SCORE_EPS = 4 * float(np.finfo(np.float32).eps)
CHOICE_MARGIN = 1e-5


def _abs_terms(res):
    """sum_d |q_max d * k_d| + |q_min d * k_d| for each (i, j), taken for the
    summary (k_max or k_min) whose sum is the larger: the scale of the fp32
    rounding error of each score."""
    aq, bq = np.abs(res["qmax"]), np.abs(res["qmin"])
    a_max = aq @ np.abs(res["kmax"]).T + bq @ np.abs(res["kmax"]).T
    a_min = aq @ np.abs(res["kmin"]).T + bq @ np.abs(res["kmin"]).T
    return np.maximum(a_max, a_min)


def _check_choice(h, gpu_choice, cohesion):
    best = np.sort(cohesion)
    if best[-1] - best[-2] > CHOICE_MARGIN:
        assert gpu_choice == int(np.argmax(cohesion)), (h, cohesion)
        return True
    assert cohesion[gpu_choice] >= best[-1] - CHOICE_MARGIN, (h, cohesion)
    return False


def _near_tied(cohesion):
    """Candidate tilings the oracle cannot separate from its own choice (within
    CHOICE_MARGIN of the best), its argmax first: the set of correct choices,
    decided by the oracle alone."""
    best = int(np.argmax(cohesion))
    return [best] + [c for c in range(len(cohesion)) if c != best and cohesion[c] >= cohesion[best] - CHOICE_MARGIN]


def _in_some_tiling(h, cohesion, check):
    """check(c) raises AssertionError unless the GPU's results for head h are
    the oracle's in candidate tiling c.  Passes if they are for one of the
    near-tied tilings (scores alone may not tell them apart: on i.i.d. grid
    values every block summary saturates and every score is 0)."""
    failures = []
    for c in _near_tied(cohesion):
        try:
            return check(c)
        except AssertionError as e:
            failures.append(f"tiling {c}: {e}")
    raise AssertionError(f"head {h}: " + "; ".join(failures))


@pytest.mark.parametrize("values", ["integer", "integer_adaptive"])
def test_spade_adaptive_full_size_integer_lists(values):
    """24 heads, S = 122880, three candidate tilings, k = 96, on {-4..4}/4 grid
    values: i.i.d. ("integer") and smooth fields rounded onto the grid
    ("integer_adaptive", whose heads have clear tiling preferences).  Scores
    are exact, so every head's whole score matrix and its whole lists must
    equal the oracle's bit for bit; the tiling choice must equal the oracle's
    wherever its margin is clear (where it is not, the GPU's results must be
    the oracle's in one of the near-tied tilings); sampled query blocks of
    every head are within the attention tolerance."""
    w = WORKLOADS["spade_adaptive_s122880"]
    q, k, v = make_qkv(w, device=DEV, values=values)
    o, mid = vsa.spade_attention(q, k, v, w.grid, list(w.tiles), topk=w.k, out_dtype=torch.float32,
                                 return_intermediates=True)
    choice = mid["choice"].cpu().numpy()
    clear = 0
    for h in range(w.heads):
        qh, kh, vh = (_np(x[0, h]) for x in (q, k, v))
        _, cohesion = oracle.select_tiling(qh, w.grid, list(w.tiles))
        clear += _check_choice(h, int(choice[h]), cohesion)
        blocks = _sample_blocks(w.nb, 300 + h, n=16 if h in (0, 13) else 4)
        got_scores = _np(mid["scores"][0, h]).astype(np.float64)
        got_idx, got_cnt = mid["idx"][0, h].cpu().numpy(), mid["cnt"][0, h].cpu().numpy()
        got_out = _np(mid["out_perm"][0, h])

        def check(c):
            res = oracle.spade_head(qh, kh, vh, w.grid, [w.tiles[c]], w.k, query_blocks=blocks)
            assert np.array_equal(got_scores, res["score"]), "scores"
            assert np.array_equal(got_idx, res["idx"]), "idx"
            assert np.array_equal(got_cnt, res["cnt"]), "cnt"
            assert_attn_close(got_out[res["rows"]], res["out_perm"], "attention")

        _in_some_tiling(h, cohesion, check)
    if values == "integer_adaptive":
        assert clear == w.heads and len(set(choice.tolist())) >= 2


def test_spade_adaptive_full_size_sampled():
    """24 heads, S = 122880, three candidate tilings, k = 96, smooth fields.
    Every head: the tiling choice equals the oracle's wherever its margin is
    clear.  Three heads: every GPU score is within SCORE_EPS * sum|terms| of
    the exact one; every list is a valid top-k set under the oracle's scores
    (a block may differ from the oracle's list only where its score and the
    k-th score lie within that allowance of each other); sampled query blocks
    whose list equals the oracle's are compared with the oracle's attention
    over its own lists (a block whose list flipped at a near-tie was checked
    valid above; at most one per head may be left out)."""
    w = WORKLOADS["spade_adaptive_s122880"]
    q, k, v = make_qkv(w, device=DEV)
    o, mid = vsa.spade_attention(q, k, v, w.grid, list(w.tiles), topk=w.k, out_dtype=torch.float32,
                                 return_intermediates=True)
    choice = mid["choice"].cpu().numpy()
    for h in range(w.heads):
        _, cohesion = oracle.select_tiling(_np(q[0, h]), w.grid, list(w.tiles))
        _check_choice(h, int(choice[h]), cohesion)
    assert len(set(choice.tolist())) >= 2   # the heads do not all pick one tiling
    # tiled (in-kernel permutation) and explicit permute paths agree bit for bit
    assert torch.equal(o, vsa.spade_attention(q, k, v, w.grid, list(w.tiles), topk=w.k, out_dtype=torch.float32,
                                              tiled=False))
    differing_rows = 0
    for h in (0, 13, 22):
        qh, kh, vh = (_np(x[0, h]) for x in (q, k, v))
        _, cohesion = oracle.select_tiling(qh, w.grid, list(w.tiles))
        blocks = _sample_blocks(w.nb, 100 + h)
        got_scores = _np(mid["scores"][0, h]).astype(np.float64)
        gi, gc = mid["idx"][0, h].cpu().numpy(), mid["cnt"][0, h].cpu().numpy()
        got_out = _np(mid["out_perm"][0, h])

        def check(c):
            tile = w.tiles[c]
            res = oracle.spade_head(qh, kh, vh, w.grid, [tile], w.k, query_blocks=blocks[:1])
            s, terms = res["score"], _abs_terms(res)
            bound = SCORE_EPS * terms
            err = np.abs(got_scores - s)
            assert (err <= bound).all(), f"score error {np.max(err / np.maximum(terms, 1e-30)):.3e} x sum|terms|"
            differing = 0
            for i in range(w.nb):
                sel = set(gi[i, :gc[i]].tolist())
                forced = {0, i}
                assert forced <= sel and w.k <= len(sel) <= w.k + len(forced), i
                order = np.lexsort((np.arange(w.nb), -s[i]))      # descending score, ties: lower index
                kth = order[w.k - 1]
                tol = bound[i] + bound[i, kth]
                assert all(s[i, j] >= s[i, kth] - tol[j] for j in sel - forced), i
                assert all(s[i, j] <= s[i, kth] + tol[j] for j in set(range(w.nb)) - sel), i
                differing += int(not np.array_equal(gi[i], res["idx"][i]))
            perm = oracle.tile_permutation(w.grid, tile)
            qp, kp, vp = (oracle.permute_rows(x, perm) for x in (qh, kh, vh))
            rows = np.concatenate([np.arange(b * 128, (b + 1) * 128) for b in blocks])
            want = oracle.block_sparse_attention(qp, kp, vp, res["idx"], res["cnt"], 128, 0, None, rows)
            got = got_out[rows]
            compared = 0
            for bi, b in enumerate(blocks):
                if np.array_equal(gi[b], res["idx"][b]):
                    assert_attn_close(got[bi * 128:(bi + 1) * 128], want[bi * 128:(bi + 1) * 128], f"block {b}")
                    compared += 1
            assert compared >= len(blocks) - 1, (compared, len(blocks))
            return differing

        differing_rows += _in_some_tiling(h, cohesion, check)
    print(f"rows whose list differs from the oracle's by near-ties: {differing_rows} of {3 * w.nb}")


def test_window_full_size_sampled():
    w = WORKLOADS["window_s30720"]
    q, k, v = make_qkv(w, device=DEV)
    o = vsa.window_attention(q, k, v, w.window, w.sink, chunk_size=w.chunk, out_dtype=torch.float32)
    for h in (0, 17):
        rows = np.concatenate([np.arange(b * 128, (b + 1) * 128) for b in _sample_blocks(w.S // 128, h)])
        want = oracle.window_attention(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), w.window, w.sink, rows=rows)
        assert_attn_close(_np(o[0, h])[rows], want, f"head {h}")


@pytest.mark.parametrize("grid,block,tile,radius", [
    ((8, 16, 32), 128, (2, 8, 8), (1, 1, 1)),    # 4 x 2 x 4 tiles of one 128-token block, through TMA boxes
    ((6, 16, 40), 64, (1, 8, 8), (2, 0, 1)),     # 64-token tiles through permuted copies, unequal radii
])
def test_sliding_tile_centered_attention_every_row(grid, block, tile, radius):
    """All rows of the centred sliding-tile mask against the oracle, for shapes
    where most query tiles sit at a border and the window is shifted."""
    q, k, v = smooth_qkv(1, 2, grid, 64, seed=77, device=DEV)
    for kind in ("sliding_tile_centered", "sliding_tile"):
        o = vsa.structured_attention(q, k, v, kind, grid, block, tile=tile, radius=radius, out_dtype=torch.float32)
        idx, cnt, g = oracle.tile_neighbourhood_list(grid, tile, radius, block,
                                                     centered=kind == "sliding_tile_centered")
        perm = oracle.tile_permutation(grid, tile)
        for h in range(2):
            qp, kp, vp = (oracle.permute_rows(_np(x[0, h]), perm) for x in (q, k, v))
            want = oracle.block_sparse_attention(qp, kp, vp, idx, cnt, block, g)
            assert_attn_close(_np(o[0, h])[perm], want, f"{kind} head {h}")


@pytest.mark.parametrize("kind", ["spatial", "temporal", "sliding_tile", "sliding_tile_centered"])
def test_structured_full_size_sampled(kind):
    """The CFG pair at S = 122880: sampled query blocks of a head of each batch
    entry (the conditional and the unconditional half) against the oracle."""
    w = WORKLOADS["structured_s122880"]
    q, k, v = make_qkv(w, device=DEV, B=2, heads=2)
    o = vsa.structured_attention(q, k, v, kind, w.grid, 128, tile=w.sliding_tile, radius=w.sliding_radius,
                                 out_dtype=torch.float32)
    t, r = oracle.structured_tile(kind, w.grid, w.sliding_tile, w.sliding_radius)
    idx, cnt, g = oracle.tile_neighbourhood_list(w.grid, t, r, 128, centered=kind == "sliding_tile_centered")
    perm = oracle.tile_permutation(w.grid, t)
    for b, h in ((0, 0), (1, 1)):
        qp, kp, vp = (oracle.permute_rows(_np(x[b, h]), perm) for x in (q, k, v))
        blocks = _sample_blocks(w.nb, 7 + b)
        rows = np.concatenate([np.arange(bb * 128, (bb + 1) * 128) for bb in blocks])
        want = oracle.block_sparse_attention(qp, kp, vp, idx, cnt, 128, g, rows=rows)
        got = _np(o[b, h])[perm[rows]]
        assert_attn_close(got, want, f"{kind} batch {b} head {h}")


# --------------------------------------------------------------------------
# tiled mode with 32- and 64-token tiles (a block is the tile itself)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("D,grid,tiles,values", [
    (128, (4, 16, 32), [(1, 4, 16), (1, 8, 8)], "smooth"),    # 64-token candidates, as in SPADE's own configs
    (64, (4, 16, 32), [(1, 4, 16), (1, 8, 8)], "integer"),
    (64, (4, 8, 16), [(2, 4, 4), (1, 4, 8)], "integer"),      # 32-token candidates
])
def test_small_block_tiled_attention_matches_permuted_path_and_oracle(D, grid, tiles, values):
    """Blocks of 32 and 64 tokens read as TMA boxes from T-major tensors equal
    permute -> attention -> unpermute bit for bit, and the oracle."""
    B, H = 1, 3
    S = grid[0] * grid[1] * grid[2]
    block = tiles[0][0] * tiles[0][1] * tiles[0][2]
    nb = S // block
    if values == "integer":
        q, k, v = (integer_grid((B, H, S, D), 91 + i, torch.bfloat16, DEV) for i in range(3))
    else:
        q, k, v = smooth_qkv(B, H, grid, D, seed=92, device=DEV)
    choice = torch.tensor([1, 0, 1], dtype=torch.int32, device=DEV)
    idx, cnt = _random_lists(nb, min(nb, 5), B * H, seed=D + nb + block)
    ti = torch.as_tensor(idx, device=DEV).view(B, H, nb, -1)
    tc = torch.as_tensor(cnt, device=DEV).view(B, H, nb)
    o = vsa.block_sparse_attention_tiled(q, k, v, grid, tiles, choice, ti, tc, out_dtype=torch.float32)
    qp, kp, vp = (vsa.permute(x, grid, tiles, choice) for x in (q, k, v))
    op = vsa.block_sparse_attention(qp, kp, vp, ti, tc, block, out_dtype=torch.float32)
    assert torch.equal(o, vsa.unpermute(op, grid, tiles, choice))
    for h, c in enumerate(choice.tolist()):
        perm = oracle.tile_permutation(grid, tiles[c])
        qo, ko, vo = (oracle.permute_rows(_np(x[0, h]), perm) for x in (q, k, v))
        want = oracle.block_sparse_attention(qo, ko, vo, idx[h], cnt[h], block)
        assert_attn_close(_np(o[0, h])[perm], want, f"head {h}")


def test_spade_64_token_candidates_tiled_equals_explicit():
    """The whole composition with SPADE's 64-token candidates: tiled mode (boxes)
    and the explicit permute path give the same bits, and the lists match the
    oracle's on integer-grid values."""
    grid, tiles = (4, 16, 32), [(1, 4, 16)]
    S = grid[0] * grid[1] * grid[2]
    q, k, v = (integer_grid((1, 2, S, 128), 93 + i, torch.bfloat16, DEV) for i in range(3))
    o, mid = vsa.spade_attention(q, k, v, grid, tiles, topk=4, out_dtype=torch.float32, return_intermediates=True)
    oe = vsa.spade_attention(q, k, v, grid, tiles, topk=4, out_dtype=torch.float32, tiled=False)
    assert torch.equal(o, oe)
    for h in range(2):
        res = oracle.spade_head(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), grid, tiles, 4)
        assert np.array_equal(mid["idx"][0, h].cpu().numpy(), res["idx"])
        assert_attn_close(_np(o[0, h]), res["out"], f"head {h}")


# --------------------------------------------------------------------------
# top-p (mass budget) lists
# --------------------------------------------------------------------------

def _check_topp_row(kept, row, p, scale, what):
    """kept must be an upper set of the row (ties by lower index) whose mass
    reaches p while it would not without its last block, within fp32 error."""
    nb = row.shape[0]
    e = np.exp(scale * (row - row.max()))
    pr = e / e.sum()
    order = sorted(range(nb), key=lambda j: (-row[j], j))
    n = len(kept)
    assert kept == set(order[:n]), what
    tol = 1e-5
    assert pr[order[:n]].sum() >= p - tol, what
    assert n == 1 or pr[order[:n - 1]].sum() < p + tol, what


@pytest.mark.parametrize("nb", [1, 5, 33, 240, 960])
@pytest.mark.parametrize("p,scale", [(0.1, 0.3), (0.5, 0.05), (0.9, 0.3), (0.99, 1.0)])
def test_topp_lists_against_oracle(nb, p, scale):
    scores = random_scores((1, 2, nb, nb), seed=nb + int(p * 100), device=DEV) * 4.0
    idx, cnt = vsa.topp_block_mask(scores, p, scale, n_sink_blocks=0, diag_halfwidth=-1)
    s = _np(scores).astype(np.float64)
    same = 0
    for h in range(2):
        oi, oc = oracle.topp_block_list(s[0, h], p, scale, 0, -1)
        gi, gc = idx[0, h].cpu().numpy(), cnt[0, h].cpu().numpy()
        for i in range(nb):
            kept = set(gi[i, :gc[i]].tolist())
            assert (gi[i, :gc[i]] == np.sort(gi[i, :gc[i]])).all() and (gi[i, gc[i]:] == -1).all()
            _check_topp_row(kept, s[0, h, i], p, scale, (h, i))
            same += int(gc[i] == oc[i] and (gi[i, :gc[i]] == oi[i, :oc[i]]).all())
    assert same >= 0.98 * 2 * nb   # a block whose mass straddles p within fp32 error may differ


def test_topp_static_blocks_and_uniform_case():
    nb = 96
    scores = random_scores((1, 1, nb, nb), seed=7, device=DEV) * 4.0
    s = _np(scores).astype(np.float64)[0, 0]
    idx, cnt = vsa.topp_block_mask(scores, 0.3, 0.2, n_sink_blocks=2, diag_halfwidth=1)
    oi, oc = oracle.topp_block_list(s, 0.3, 0.2, 2, 1)
    gi, gc = idx[0, 0].cpu().numpy(), cnt[0, 0].cpu().numpy()
    for i in range(nb):
        assert {0, 1} | {j for j in range(max(0, i - 1), min(nb, i + 2))} <= set(gi[i, :gc[i]].tolist())
    assert (np.array([np.array_equal(gi[i, :gc[i]], oi[i, :oc[i]]) for i in range(nb)])).mean() >= 0.98
    # scale 0: every block equally likely, so the list is the top-k list, k = ceil(p nb)
    p = 0.37   # p * nb = 35.52
    ui, uc = vsa.topp_block_mask(scores, p, 0.0, n_sink_blocks=0, diag_halfwidth=-1)
    ki, kc = vsa.topk_block_mask(scores, 36, n_sink_blocks=0, diag_halfwidth=-1, cap=nb)
    assert torch.equal(uc, kc) and torch.equal(ui, ki)


def test_spade_top_p_end_to_end():
    w = WORKLOADS["tiny_s256"]
    q, k, v = make_qkv(w, device=DEV)
    o, mid = vsa.spade_attention(q, k, v, w.grid, list(w.tiles), top_p=0.6, top_p_scale=0.25,
                                 out_dtype=torch.float32, return_intermediates=True)
    for h in range(w.heads):
        perm = oracle.tile_permutation(w.grid, w.tiles[0])
        qo, ko, vo = (oracle.permute_rows(_np(x[0, h]), perm) for x in (q, k, v))
        s = oracle.block_scores(*oracle.block_minmax(qo, w.block), *oracle.block_minmax(ko, w.block))
        oi, oc = oracle.topp_block_list(s, 0.6, 0.25, 1, 0)
        gi, gc = mid["idx"][0, h].cpu().numpy(), mid["cnt"][0, h].cpu().numpy()
        assert np.array_equal(gc, oc) and all(np.array_equal(gi[i, :gc[i]], oi[i, :oc[i]]) for i in range(len(gc)))
        want = oracle.block_sparse_attention(qo, ko, vo, oi, oc, w.block)
        assert_attn_close(_np(o[0, h])[perm], want, f"head {h}")


# --------------------------------------------------------------------------
# lists of one key block: the one-block kernel (two CTAs per SM)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("mode,grid", [("permuted", (4, 8, 16)), ("tiled", (4, 8, 16)), ("padded", (5, 12, 20)),
                                       ("padded", (5, 44, 76))])   # 720 tiles: several per persistent CTA
def test_one_block_lists_match_two_tile_kernel_and_oracle(mode, grid):
    """One-slot lists run through the one-key-block kernel; the same lists in
    two slots (cnt 1, second slot -1) run through the two-tile kernel.  Both
    must give the same bits, and the oracle's result."""
    tiles = [(1, 8, 16), (2, 8, 8), (4, 4, 8)]
    B, H, D = 1, 3, 128
    S = grid[0] * grid[1] * grid[2]
    pg = vsa.padded_grid(grid, tiles)
    nb = pg[0] * pg[1] * pg[2] // 128
    q, k, v = smooth_qkv(B, H, grid, D, seed=95, device=DEV)
    rng = np.random.default_rng(96)
    # padded grid: the diagonal block (it holds the query itself, so every real
    # query has a real key); otherwise random blocks for heads 1 and 2
    idx1 = np.stack([np.arange(nb) if h == 0 or mode == "padded" else rng.integers(0, nb, nb)
                     for h in range(H)]).astype(np.int32)
    cnt = np.ones((H, nb), np.int32)
    ti1 = torch.as_tensor(idx1, device=DEV).view(B, H, nb, 1)
    ti2 = torch.as_tensor(np.concatenate([idx1[..., None], np.full((H, nb, 1), -1, np.int32)], -1),
                          device=DEV).view(B, H, nb, 2)
    tc = torch.as_tensor(cnt, device=DEV).view(B, H, nb)
    opg = tuple(oracle.padded_grid(grid, tiles))   # the oracle's own padded grid
    assert tuple(pg) == opg
    if mode == "permuted":
        qp, kp, vp = (vsa.permute(x, grid, tiles[:1]) for x in (q, k, v))
        o1 = vsa.block_sparse_attention(qp, kp, vp, ti1, tc, 128, out_dtype=torch.float32)
        o2 = vsa.block_sparse_attention(qp, kp, vp, ti2, tc, 128, out_dtype=torch.float32)
        assert torch.equal(o1, o2)
        perm = oracle.tile_permutation(grid, tiles[0])
        for h in range(H):
            qo, ko, vo = (oracle.permute_rows(_np(x[0, h]), perm) for x in (q, k, v))
            want = oracle.block_sparse_attention(qo, ko, vo, idx1[h][:, None], cnt[h], 128)
            assert_attn_close(_np(o1[0, h]), want, f"head {h}")
        return
    choice = torch.tensor([0, 1, 2], dtype=torch.int32, device=DEV)
    o1 = vsa.block_sparse_attention_tiled(q, k, v, grid, tiles, choice, ti1, tc, out_dtype=torch.float32)
    o2 = vsa.block_sparse_attention_tiled(q, k, v, grid, tiles, choice, ti2, tc, out_dtype=torch.float32)
    assert torch.equal(o1, o2)
    ob = vsa.block_sparse_attention_tiled(q, k, v, grid, tiles, choice, ti1, tc, out_dtype=torch.bfloat16)
    assert torch.equal(ob, o1.to(torch.bfloat16))
    for h, c in enumerate(choice.tolist()):
        perm = oracle.tile_permutation(opg, tiles[c])
        real = oracle.real_tokens(grid, opg)
        qo, ko, vo = (oracle.permute_rows(oracle.pad_grid(_np(x[0, h]), grid, opg), perm) for x in (q, k, v))
        want_p = oracle.block_sparse_attention(qo, ko, vo, idx1[h][:, None], cnt[h], 128,
                                               key_ok=real[perm].astype(np.uint8) if mode == "padded" else None)
        want = np.zeros((opg[0] * opg[1] * opg[2], D))
        want[perm] = want_p
        assert_attn_close(_np(o1[0, h]), want[real], f"head {h}")


def test_one_block_kernel_many_tiles_per_cta_with_invalid_lists():
    """1024 query tiles of four heads in three tilings, with tiles whose list
    is invalid (zeros and an error status) among them: the one-block kernel
    gives the two-tile kernel's bits on the same lists, and the oracle's
    result on sampled blocks."""
    grid, tiles = (16, 32, 64), [(1, 8, 16), (2, 8, 8), (4, 4, 8)]
    B, H, D = 1, 4, 128
    nb = grid[0] * grid[1] * grid[2] // 128
    q, k, v = smooth_qkv(B, H, grid, D, seed=97, device=DEV)
    rng = np.random.default_rng(98)
    idx1 = rng.integers(0, nb, (H, nb)).astype(np.int32)
    cnt = np.ones((H, nb), np.int32)
    choice = torch.tensor([0, 1, 2, 1], dtype=torch.int32, device=DEV)

    def run(idx):
        ti1 = torch.as_tensor(idx, device=DEV).view(B, H, nb, 1)
        ti2 = torch.as_tensor(np.concatenate([idx[..., None], np.full((H, nb, 1), -1, np.int32)], -1),
                              device=DEV).view(B, H, nb, 2)
        tc = torch.as_tensor(cnt, device=DEV).view(B, H, nb)
        o1 = vsa.block_sparse_attention_tiled(q, k, v, grid, tiles, choice, ti1, tc, out_dtype=torch.float32)
        o2 = vsa.block_sparse_attention_tiled(q, k, v, grid, tiles, choice, ti2, tc, out_dtype=torch.float32)
        return o1, o2

    o1, o2 = run(idx1)
    vsa.device_status()
    assert torch.equal(o1, o2)
    for h, c in enumerate(choice.tolist()):
        perm = oracle.tile_permutation(grid, tiles[c])
        qo, ko, vo = (oracle.permute_rows(_np(x[0, h]), perm) for x in (q, k, v))
        blocks = [0, 1, 100, 201, nb - 1]
        rows = np.concatenate([np.arange(b * 128, (b + 1) * 128) for b in blocks])
        want = oracle.block_sparse_attention(qo, ko, vo, idx1[h][:, None], cnt[h], 128, rows=rows)
        assert_attn_close(_np(o1[0, h])[perm[rows]], want, f"head {h}")
    bad = idx1.copy()
    bad[1, ::5] = nb          # out of range
    bad[3, 3::7] = -1
    o1b, o2b = run(bad)
    with pytest.raises(RuntimeError):
        vsa.device_status()
    assert torch.equal(o1b, o2b)
    for h, sel in ((1, slice(0, None, 5)), (3, slice(3, None, 7))):
        perm = oracle.tile_permutation(grid, tiles[int(choice[h])])
        dead = np.zeros(nb, bool)
        dead[sel] = True
        rows = perm[np.repeat(dead, 128)]
        assert torch.count_nonzero(o1b[0, h, torch.as_tensor(rows, device=DEV)]) == 0
        live = perm[np.repeat(~dead, 128)]
        assert torch.equal(o1b[0, h, torch.as_tensor(live, device=DEV)], o1[0, h, torch.as_tensor(live, device=DEV)])


def test_temporal_mask_with_more_frames_than_a_block():
    """T = 256 frames: a temporal tile is two blocks, so the lists hold two
    blocks and the composition must not ask for one-slot lists."""
    grid = (256, 1, 2)
    q, k, v = smooth_qkv(1, 1, grid, 64, seed=99, device=DEV)
    o = vsa.structured_attention(q, k, v, "temporal", grid, 128, out_dtype=torch.float32)
    t, r = oracle.structured_tile("temporal", grid)
    idx, cnt, g = oracle.tile_neighbourhood_list(grid, t, r, 128)
    perm = oracle.tile_permutation(grid, t)
    qp, kp, vp = (oracle.permute_rows(_np(x[0, 0]), perm) for x in (q, k, v))
    op = oracle.block_sparse_attention(qp, kp, vp, idx, cnt, 128, g)
    want = np.empty_like(op)
    want[perm] = op
    assert_attn_close(_np(o[0, 0]), want, "T = 256")
