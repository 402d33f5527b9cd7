"""Grids the candidate tiles do not divide, through the C ABI, against the
fp64 oracle ("Adaptive tiling (SPADE)", Deviations and notes: pad with zero
tokens, leave them out of the cohesion, mask the padded keys).

The oracle pads explicitly (oracle.pad_grid) and masks keys with key_ok; the
library works on the real T-major tensors and treats padding positions by
their coordinates.  Index outputs (permutations, summaries, lists) must match
bit for bit; attention within the bounds of test_gpu_parity.
"""

import numpy as np
import pytest
import torch

import block_sparse_self_b200 as vsa
import oracle
from workloads import WORKLOADS, integer_grid, make_qkv, smooth_qkv

from test_gpu_parity import _np, _sample_blocks, assert_attn_close

pytestmark = pytest.mark.gpu

DEV = "cuda"
TILES3 = [(1, 8, 16), (2, 8, 8), (4, 4, 8)]


@pytest.fixture(autouse=True)
def _no_device_errors():
    yield
    vsa.device_status()


def _padded(grid, tiles, tile):
    pg = oracle.padded_grid(grid, tiles)
    return pg, oracle.tile_permutation(pg, tile), oracle.real_tokens(grid, pg)


def _oracle_perm_padded(x, grid, tiles, tile):
    """The oracle's permuted copy of one head on the padded grid."""
    pg, perm, _ = _padded(grid, tiles, tile)
    return oracle.permute_rows(oracle.pad_grid(x, grid, pg), perm)


# --------------------------------------------------------------------------
# permutation and summaries
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,D,grid", [(torch.float32, 64, (3, 5, 13)), (torch.bfloat16, 128, (5, 12, 20)),
                                          (torch.bfloat16, 64, (7, 9, 17))])
def test_permute_on_padded_grid(dtype, D, grid):
    S = grid[0] * grid[1] * grid[2]
    pg = vsa.padded_grid(grid, TILES3)
    assert pg == oracle.padded_grid(grid, TILES3) and pg != grid
    Sp = pg[0] * pg[1] * pg[2]
    x = integer_grid((2, 3, S, D), 81, dtype, DEV)
    choice = torch.tensor([2, 0, 1, 1, 2, 0], dtype=torch.int32, device=DEV)
    y = vsa.permute(x, grid, TILES3, choice)
    assert tuple(y.shape) == (2, 3, Sp, D)
    for bh, c in enumerate(choice.tolist()):
        want = _oracle_perm_padded(_np(x.view(6, S, D)[bh]), grid, TILES3, TILES3[c])
        assert np.array_equal(_np(y.view(6, Sp, D)[bh]), want)
    assert torch.equal(vsa.unpermute(y, grid, TILES3, choice), x)
    with pytest.raises(ValueError):   # the inverse takes the padded rows
        vsa.unpermute(x, grid, TILES3, choice)


@pytest.mark.parametrize("dtype,D,block", [(torch.bfloat16, 128, 128), (torch.float32, 64, 64),
                                           (torch.bfloat16, 64, 256), (torch.float32, 128, 32)])
def test_block_summaries_tiled_on_padded_grid(dtype, D, block):
    """Padding positions take part as zero rows: a block holding padding has a
    max >= 0 and a min <= 0 in every channel, exactly as the oracle's."""
    grid = (5, 12, 20)
    S = grid[0] * grid[1] * grid[2]
    x = torch.randn(2, 3, S, D, generator=torch.Generator(DEV).manual_seed(82), device=DEV).to(dtype)
    choice = torch.tensor([1, 2, 0, 0, 1, 2], dtype=torch.int32, device=DEV)
    mx, mn = vsa.block_summaries_tiled(x, grid, TILES3, choice, block)
    wmx, wmn = vsa.block_summaries(vsa.permute(x, grid, TILES3, choice), block)
    assert torch.equal(mx, wmx) and torch.equal(mn, wmn)
    for bh, c in enumerate(choice.tolist()):
        xp = _oracle_perm_padded(_np(x.view(6, S, D)[bh]), grid, TILES3, TILES3[c])
        omx, omn = oracle.block_minmax(xp, block)
        assert np.array_equal(_np(mx.view(6, -1, D)[bh]), omx)
        assert np.array_equal(_np(mn.view(6, -1, D)[bh]), omn)


# --------------------------------------------------------------------------
# tiling choice
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,D,grid", [(torch.bfloat16, 128, (6, 21, 36)), (torch.float32, 64, (5, 12, 20))])
def test_select_tiling_on_padded_grid(dtype, D, grid):
    """The cohesion is the mean over the tiles of the padded grid that hold a
    query; tiles made only of padding (T = 6 padded to 8 leaves whole frames
    of padding) are not counted."""
    kinds = ["spatial", "temporal", "generic", "spatial", "temporal", "generic"]
    q, _, _ = smooth_qkv(1, 6, grid, D, seed=83, kinds=kinds, dtype=dtype, device=DEV)
    choice, sics = vsa.select_tiling(q, grid, TILES3, return_sics=True)
    pg = oracle.padded_grid(grid, TILES3)
    flips = 0
    for h in range(6):
        oc, osc = oracle.select_tiling(oracle.pad_grid(_np(q[0, h]), grid, pg), pg, TILES3)
        np.testing.assert_allclose(_np(sics[h]), osc, atol=2e-5, rtol=0)
        margin = np.sort(osc)[-1] - np.sort(osc)[-2]
        if margin > 1e-4:
            assert int(choice[h]) == oc, (h, osc)
        else:
            flips += 1
    assert flips <= 1
    assert torch.equal(choice, vsa.select_tiling_noalloc(q, grid, TILES3))


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def _lists_with_diagonal(nb, cap, bh, seed):
    """Random ascending lists that always hold the query block itself (a real
    query then always has a real key)."""
    rng = np.random.default_rng(seed)
    idx = np.full((bh, nb, cap), -1, np.int32)
    cnt = np.zeros((bh, nb), np.int32)
    for b in range(bh):
        for i in range(nb):
            n = int(rng.integers(1, cap + 1))
            others = rng.choice(np.setdiff1d(np.arange(nb), [i]), n - 1, replace=False)
            sel = np.sort(np.concatenate([[i], others]))
            idx[b, i, :n] = sel
            cnt[b, i] = n
    return idx, cnt


@pytest.mark.parametrize("D,grid,values", [(128, (5, 12, 20), "smooth"), (64, (7, 9, 17), "integer"),
                                           (128, (4, 13, 31), "integer")])
def test_tiled_attention_masks_padding_keys(D, grid, values):
    """Keys at padding positions are masked, rows at padding positions are not
    written, and the real rows equal the oracle with key_ok."""
    B, H = 1, 3
    S = grid[0] * grid[1] * grid[2]
    pg = vsa.padded_grid(grid, TILES3)
    Sp = pg[0] * pg[1] * pg[2]
    nb = Sp // 128
    if values == "integer":
        q, k, v = (integer_grid((B, H, S, D), 84 + i, torch.bfloat16, DEV) for i in range(3))
    else:
        q, k, v = smooth_qkv(B, H, grid, D, seed=85, device=DEV)
    choice = torch.tensor([0, 1, 2], dtype=torch.int32, device=DEV)
    idx, cnt = _lists_with_diagonal(nb, min(nb, 4), B * H, seed=D + nb)
    ti = torch.as_tensor(idx, device=DEV).view(B, H, nb, -1)
    tc = torch.as_tensor(cnt, device=DEV).view(B, H, nb)
    o = vsa.block_sparse_attention_tiled(q, k, v, grid, TILES3, choice, ti, tc, out_dtype=torch.float32)
    ob = vsa.block_sparse_attention_tiled(q, k, v, grid, TILES3, choice, ti, tc, out_dtype=torch.bfloat16)
    assert torch.equal(ob, o.to(torch.bfloat16))
    for h, c in enumerate(choice.tolist()):
        _, perm, real = _padded(grid, TILES3, TILES3[c])
        qo, ko, vo = (_oracle_perm_padded(_np(x[0, h]), grid, TILES3, TILES3[c]) for x in (q, k, v))
        want_p = oracle.block_sparse_attention(qo, ko, vo, idx[h], cnt[h], 128, key_ok=real[perm].astype(np.uint8))
        want = np.zeros((Sp, D))
        want[perm] = want_p
        assert_attn_close(_np(o[0, h]), want[real], f"head {h}")


def test_tiled_attention_padding_limits():
    grid = (3, 5, 13)   # (4, 4, 8) boxes are taller than T = 3
    q, k, v = (integer_grid((1, 1, 195, 64), 86 + i, torch.bfloat16, DEV) for i in range(3))
    idx = torch.zeros(1, 1, 4, 1, dtype=torch.int32, device=DEV)
    cnt = torch.ones(1, 1, 4, dtype=torch.int32, device=DEV)
    with pytest.raises(NotImplementedError):
        vsa.block_sparse_attention_tiled(q, k, v, grid, TILES3, None, idx, cnt)
    # the permuted path has no key mask: padded grids need tiled mode
    with pytest.raises(NotImplementedError):
        vsa.spade_attention(q, k, v, (5, 3, 13), [(1, 8, 16)], topk=1, tiled=False)


# --------------------------------------------------------------------------
# the whole path
# --------------------------------------------------------------------------

def test_spade_on_padded_grid_integer_lists_exact():
    """One candidate, integer-grid values: scores are exact, so the lists must
    equal the oracle's bit for bit; the output within the attention bounds."""
    grid, tiles = (5, 12, 20), [(2, 8, 8)]
    S = grid[0] * grid[1] * grid[2]
    q, k, v = (integer_grid((1, 2, S, 128), 87 + i, torch.bfloat16, DEV) for i in range(3))
    o, mid = vsa.spade_attention(q, k, v, grid, tiles, topk=3, out_dtype=torch.float32, return_intermediates=True)
    assert mid["padded_grid"] == oracle.padded_grid(grid, tiles)
    for h in range(2):
        res = oracle.spade_head(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), grid, tiles, 3)
        assert np.array_equal(mid["idx"][0, h].cpu().numpy(), res["idx"])
        assert np.array_equal(mid["cnt"][0, h].cpu().numpy(), res["cnt"])
        assert np.array_equal(_np(mid["scores"][0, h]).astype(np.float64), res["score"])
        assert_attn_close(_np(o[0, h]), res["out"], f"head {h}")


def test_spade_on_padded_grid_adaptive():
    """Three candidates on a padded grid, smooth fields: heads whose choice is
    clear must agree with the oracle's whole composition."""
    grid = (6, 21, 36)
    kinds = ["spatial", "temporal", "spatial", "temporal"]
    q, k, v = smooth_qkv(1, 4, grid, 128, seed=88, kinds=kinds, device=DEV)
    o, mid = vsa.spade_attention(q, k, v, grid, TILES3, topk=6, out_dtype=torch.float32, return_intermediates=True)
    checked = 0
    for h in range(4):
        res = oracle.spade_head(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), grid, TILES3, 6)
        margin = np.sort(res["cohesion"])[-1] - np.sort(res["cohesion"])[-2]
        if margin <= 1e-4:
            continue
        assert int(mid["choice"][h]) == res["choice"]
        gi, gc = mid["idx"][0, h].cpu().numpy(), mid["cnt"][0, h].cpu().numpy()
        same = [i for i in range(gi.shape[0]) if np.array_equal(gi[i], res["idx"][i])]
        assert len(same) >= 0.9 * gi.shape[0]
        if len(same) == gi.shape[0]:
            assert_attn_close(_np(o[0, h]), res["out"], f"head {h}")
        checked += 1
    assert checked >= 2


def test_spade_padded_full_size_sampled():
    """The 16 x 45 x 80 grid (padded to 16 x 48 x 80), 24 heads, three
    candidates, k = 48: choices where the oracle's margin is clear, lists
    valid top-k sets under the oracle's scores, sampled real rows compared."""
    w = WORKLOADS["spade_adaptive_pad_s57600"]
    q, k, v = make_qkv(w, device=DEV)
    o, mid = vsa.spade_attention(q, k, v, w.grid, list(w.tiles), topk=w.k, out_dtype=torch.float32,
                                 return_intermediates=True)
    pg = oracle.padded_grid(w.grid, list(w.tiles))
    nb = pg[0] * pg[1] * pg[2] // 128
    assert mid["padded_grid"] == pg and mid["idx"].shape[2] == nb
    choice = mid["choice"].cpu().numpy()
    clear = []
    for h in range(w.heads):
        oc, osc = oracle.select_tiling(oracle.pad_grid(_np(q[0, h]), w.grid, pg), pg, list(w.tiles))
        margin = np.sort(osc)[-1] - np.sort(osc)[-2]
        if margin > 1e-4:
            assert choice[h] == oc, (h, osc)
            clear.append(h)
    assert len(clear) >= w.heads - 2
    for h in clear[:2]:
        blocks = _sample_blocks(nb, 200 + h)
        res = oracle.spade_head(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), w.grid, list(w.tiles), w.k,
                                query_blocks=blocks)
        gi, gc = mid["idx"][0, h].cpu().numpy(), mid["cnt"][0, h].cpu().numpy()
        s = res["score"]
        same = 0
        for i in range(nb):
            sel = set(gi[i, :gc[i]].tolist())
            forced = {0, i}
            assert forced <= sel and w.k <= len(sel) <= w.k + len(forced)
            kth = np.sort(s[i])[::-1][w.k - 1]
            tol = 1e-5 * max(1.0, float(np.abs(s[i]).max()))
            assert all(s[i, j] >= kth - tol for j in sel - forced), (h, i)
            assert all(s[i, j] <= kth + tol for j in set(range(nb)) - sel), (h, i)
            same += int(np.array_equal(gi[i], res["idx"][i]))
        assert same >= 0.9 * nb
        real_p = oracle.real_tokens(w.grid, pg)[res["perm"]]
        got = _np(mid["out_perm"][0, h])
        for bi, b in enumerate(blocks):
            if not np.array_equal(gi[b], res["idx"][b]):
                continue
            rows = np.arange(b * 128, (b + 1) * 128)
            keep = real_p[rows]
            if keep.any():
                assert_attn_close(got[rows][keep], res["out_perm"][bi * 128:(bi + 1) * 128][keep],
                                  f"head {h} block {b}")


# --------------------------------------------------------------------------
# SPADE's own 64-token candidates on grids they do not divide
# --------------------------------------------------------------------------

SPADE64 = [(1, 4, 16), (1, 8, 8)]


@pytest.mark.parametrize("D,grid", [(64, (3, 13, 20)), (128, (5, 10, 18))])
def test_tiled_attention_64_token_boxes_mask_padding_keys(D, grid):
    B, H = 1, 2
    S = grid[0] * grid[1] * grid[2]
    pg = vsa.padded_grid(grid, SPADE64)
    Sp = pg[0] * pg[1] * pg[2]
    nb = Sp // 64
    q, k, v = (integer_grid((B, H, S, D), 94 + i, torch.bfloat16, DEV) for i in range(3))
    choice = torch.tensor([0, 1], dtype=torch.int32, device=DEV)
    idx, cnt = _lists_with_diagonal(nb, min(nb, 5), B * H, seed=D + nb)
    ti = torch.as_tensor(idx, device=DEV).view(B, H, nb, -1)
    tc = torch.as_tensor(cnt, device=DEV).view(B, H, nb)
    o = vsa.block_sparse_attention_tiled(q, k, v, grid, SPADE64, choice, ti, tc, out_dtype=torch.float32)
    for h, c in enumerate(choice.tolist()):
        _, perm, real = _padded(grid, SPADE64, SPADE64[c])
        qo, ko, vo = (_oracle_perm_padded(_np(x[0, h]), grid, SPADE64, SPADE64[c]) for x in (q, k, v))
        want_p = oracle.block_sparse_attention(qo, ko, vo, idx[h], cnt[h], 64, key_ok=real[perm].astype(np.uint8))
        want = np.zeros((Sp, D))
        want[perm] = want_p
        assert_attn_close(_np(o[0, h]), want[real], f"head {h}")


def test_spade_64_token_candidates_on_padded_grid():
    """The pages' case in small: a height no 64-token candidate divides.  One
    candidate, integer-grid values: lists bit-exact with the oracle's."""
    grid, tiles = (3, 13, 20), [(1, 8, 8)]
    S = grid[0] * grid[1] * grid[2]
    q, k, v = (integer_grid((1, 2, S, 64), 97 + i, torch.bfloat16, DEV) for i in range(3))
    o, mid = vsa.spade_attention(q, k, v, grid, tiles, topk=3, out_dtype=torch.float32, return_intermediates=True)
    for h in range(2):
        res = oracle.spade_head(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), grid, tiles, 3)
        assert np.array_equal(mid["idx"][0, h].cpu().numpy(), res["idx"])
        assert np.array_equal(mid["cnt"][0, h].cpu().numpy(), res["cnt"])
        assert_attn_close(_np(o[0, h]), res["out"], f"head {h}")


def test_spade_64_token_candidates_wan_grid_sampled():
    """16 x 45 x 80 with SPADE's (1, 4, 16) and (1, 8, 8) candidates (padded to
    16 x 48 x 80, 960 blocks of 64), 4 heads, k = 96: choices where clear, lists
    valid top-k sets under the oracle's scores, sampled real rows compared."""
    grid = (16, 45, 80)
    kinds = ["spatial", "temporal", "spatial", "temporal"]
    q, k, v = smooth_qkv(1, 4, grid, 128, seed=98, kinds=kinds, device=DEV)
    kk = 96
    o, mid = vsa.spade_attention(q, k, v, grid, SPADE64, topk=kk, out_dtype=torch.float32, return_intermediates=True)
    pg = oracle.padded_grid(grid, SPADE64)
    nb = pg[0] * pg[1] * pg[2] // 64
    assert mid["idx"].shape[2] == nb
    checked = 0
    for h in range(4):
        res = oracle.spade_head(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), grid, SPADE64, kk,
                                query_blocks=_sample_blocks(nb, 300 + h))
        margin = np.sort(res["cohesion"])[-1] - np.sort(res["cohesion"])[-2]
        if margin <= 1e-4:
            continue
        assert int(mid["choice"][h]) == res["choice"]
        gi, gc = mid["idx"][0, h].cpu().numpy(), mid["cnt"][0, h].cpu().numpy()
        s = res["score"]
        same = 0
        for i in range(nb):
            sel = set(gi[i, :gc[i]].tolist())
            forced = {0, i}
            assert forced <= sel and kk <= len(sel) <= kk + len(forced)
            kth = np.sort(s[i])[::-1][kk - 1]
            tol = 1e-5 * max(1.0, float(np.abs(s[i]).max()))
            assert all(s[i, j] >= kth - tol for j in sel - forced), (h, i)
            same += int(np.array_equal(gi[i], res["idx"][i]))
        assert same >= 0.9 * nb
        real_p = oracle.real_tokens(grid, pg)[res["perm"]]
        got = _np(mid["out_perm"][0, h])
        blocks = _sample_blocks(nb, 300 + h)
        for bi, b in enumerate(blocks):
            if not np.array_equal(gi[b], res["idx"][b]):
                continue
            rows = np.arange(b * 64, (b + 1) * 64)
            keep = real_p[rows]
            if keep.any():
                assert_attn_close(got[rows][keep], res["out_perm"][bi * 64:(bi + 1) * 64][keep], f"head {h} block {b}")
        checked += 1
    assert checked >= 2
