"""Pins of the fp64 oracle to what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: worked
examples done by hand (tests/golden), coordinate properties that determine a
result uniquely, brute force over tiny inputs, or special cases that reduce to
a library routine (torch scaled_dot_product_attention in fp64, numpy).
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import integer_grid, smooth_qkv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _coords(grid):
    T, H, W = grid
    i = np.arange(T * H * W)
    return i // (H * W), (i // W) % H, i % W


def _sdpa64(q, k, v, scale, mask=None):
    """torch SDPA in fp64 on the CPU; mask is a bool [S, S] (True = visible)."""
    q, k, v = (torch.as_tensor(np.asarray(x, np.float64))[None, None] for x in (q, k, v))
    m = None if mask is None else torch.as_tensor(mask)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale)
    return o[0, 0].numpy()


# --------------------------------------------------------------------------
# permutation (ADR step 6; SPADE Recipe: argsort of tile labels)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("grid,tile", [((4, 8, 8), (2, 4, 4)), ((3, 4, 6), (1, 2, 3)),
                                       ((4, 6, 10), (4, 1, 1)), ((2, 4, 4), (1, 4, 4)),
                                       ((6, 6, 8), (3, 2, 4))])
def test_permutation_determined_by_coordinates(grid, tile):
    """Runs of tile-volume positions hold exactly one tile each, tiles in
    row-major tile order, tokens inside a tile in ascending T-major order,
    and every token appears once."""
    perm = oracle.tile_permutation(grid, tile)
    S = grid[0] * grid[1] * grid[2]
    vol = tile[0] * tile[1] * tile[2]
    assert sorted(perm.tolist()) == list(range(S))
    t, h, w = _coords(grid)
    ntile = (grid[1] // tile[1], grid[2] // tile[2])
    for r in range(S // vol):
        run = perm[r * vol:(r + 1) * vol]
        ct, ch, cw = t[run] // tile[0], h[run] // tile[1], w[run] // tile[2]
        assert len(set(zip(ct, ch, cw))) == 1
        assert (ct[0] * ntile[0] + ch[0]) * ntile[1] + cw[0] == r
        assert np.all(np.diff(run) > 0)


def test_unpermute_inverts_permute():
    grid, tile = (4, 8, 8), (2, 4, 4)
    x = integer_grid((256, 64), seed=5, dtype=torch.float32).numpy()
    perm = oracle.tile_permutation(grid, tile)
    y = oracle.permute_rows(x, perm)
    assert np.array_equal(oracle.unpermute_rows(y, perm), x)
    assert np.array_equal(y, x[perm])
    assert not np.array_equal(y, x)


def test_identity_permutation_for_whole_frames():
    """A (1, H, W) tile is a whole frame: T-major order is already tile order."""
    perm = oracle.tile_permutation((5, 4, 6), (1, 4, 6))
    assert np.array_equal(perm, np.arange(120))


# --------------------------------------------------------------------------
# SICS and the tiling choice (SPADE step 1; block_self_similarity; select_tiling)
# --------------------------------------------------------------------------

def test_sics_golden():
    g = json.load(open(os.path.join(GOLDEN, "sics_tiny.json")))
    got = oracle.tile_sics(np.array(g["q"], np.float32), tuple(g["grid"]), tuple(g["tile"]))
    np.testing.assert_allclose(got, g["tile_sics"], rtol=0, atol=1e-15)


def _pairwise_mean_cos(x):
    """Brute force: mean cosine over distinct ordered pairs of non-zero rows."""
    x = np.asarray(x, np.float64)
    x = x[np.linalg.norm(x, axis=1) > 0]
    m = len(x)
    if m < 2:
        return 0.0
    tot = 0.0
    for i in range(m):
        for j in range(m):
            if i != j:
                tot += x[i] @ x[j] / (np.linalg.norm(x[i]) * np.linalg.norm(x[j]))
    return tot / (m * (m - 1))


@pytest.mark.parametrize("grid,tile", [((2, 4, 4), (1, 2, 2)), ((4, 4, 4), (2, 2, 1)),
                                       ((2, 2, 8), (2, 2, 4))])
def test_sics_brute_force(grid, tile):
    S = grid[0] * grid[1] * grid[2]
    q = np.random.default_rng(3).normal(size=(S, 8)).astype(np.float32)
    q[5] = 0.0  # one zero-norm query, excluded
    got = oracle.tile_sics(q, grid, tile)
    t, h, w = _coords(grid)
    nth, ntw = grid[1] // tile[1], grid[2] // tile[2]
    lab = ((t // tile[0]) * nth + h // tile[1]) * ntw + w // tile[2]
    want = [_pairwise_mean_cos(q[lab == c]) for c in range(len(got))]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_sics_special_cases():
    # constant direction: 1; m = 2: the plain cosine
    grid, tile = (1, 1, 4), (1, 1, 2)
    q = np.array([[1, 2, 3], [2, 4, 6], [1, 0, 1], [0, 1, 1]], np.float32)
    got = oracle.tile_sics(q, grid, tile)
    assert got[0] == pytest.approx(1.0, abs=1e-15)
    assert got[1] == pytest.approx(0.5, abs=1e-15)  # cos((1,0,1),(0,1,1)) = 1/2


def test_select_tiling_picks_the_cohesive_tiling_and_breaks_ties_low():
    grid = (4, 4, 4)
    t, h, w = _coords(grid)
    rng = np.random.default_rng(0)
    # every frame is one direction, frames differ: whole-frame tiles are cohesive
    dirs = rng.normal(size=(4, 16))
    q = dirs[t].astype(np.float32)
    tiles = [(4, 1, 1), (1, 4, 4), (2, 2, 2)]
    choice, sc = oracle.select_tiling(q, grid, tiles)
    assert choice == 1 and sc[1] == pytest.approx(1.0)
    # identical candidates tie exactly: the lower index wins
    choice, sc = oracle.select_tiling(q, grid, [(2, 2, 2), (2, 2, 2), (1, 4, 4)])
    assert choice == 2
    choice, sc = oracle.select_tiling(q, grid, [(2, 2, 2), (2, 2, 2)])
    assert choice == 0 and sc[0] == sc[1]


def test_self_pair_reading_gives_the_same_choice():
    """Counting self-pairs maps SICS to (m-1)/m * SICS + 1/m: monotone for a
    common tile volume, so the choice does not depend on that reading."""
    grid = (4, 8, 8)
    q, _, _ = smooth_qkv(1, 2, grid, 32, seed=11, kinds=["spatial", "temporal"],
                         dtype=torch.float32)
    tiles = [(1, 4, 8), (2, 4, 4), (4, 2, 4)]
    for hd in range(2):
        c, sc = oracle.select_tiling(q[0, hd], grid, tiles)
        m = 32
        alt = (m - 1) / m * sc + 1 / m
        assert int(np.argmax(alt)) == c


# --------------------------------------------------------------------------
# summaries and scores (SPADE step 3; minmax_block_scores)
# --------------------------------------------------------------------------

def test_block_scores_golden():
    g = json.load(open(os.path.join(GOLDEN, "block_scores_tiny.json")))
    qmax, qmin = oracle.block_minmax(np.array(g["q"], np.float32), g["block"])
    kmax, kmin = oracle.block_minmax(np.array(g["k"], np.float32), g["block"])
    assert np.array_equal(qmax, g["q_max"]) and np.array_equal(qmin, g["q_min"])
    assert np.array_equal(kmax, g["k_max"]) and np.array_equal(kmin, g["k_min"])
    s = oracle.block_scores(qmax, qmin, kmax, kmin)
    assert np.array_equal(s, g["scores"])
    idx, cnt = oracle.topk_block_list(s, 1, n_sink=0, diag_halfwidth=-1, cap=1)
    assert idx.tolist() == g["top1_plain"]
    idx, cnt = oracle.topk_block_list(s, 1, n_sink=1, diag_halfwidth=0, cap=2)
    assert idx.tolist() == g["top1_sink_diag"] and cnt.tolist() == [2, 2]


def test_block_minmax_against_numpy():
    x = integer_grid((512, 64), seed=9, dtype=torch.float32).numpy()
    mx, mn = oracle.block_minmax(x, 32)
    r = x.reshape(16, 32, 64).astype(np.float64)
    assert np.array_equal(mx, r.max(1)) and np.array_equal(mn, r.min(1))


def test_singleton_blocks_reduce_to_twice_the_dot_product():
    """With one token per block, q_max = q_min = q and k_max = k_min = k, so
    the score is 2 q . k."""
    x = integer_grid((2, 40, 16), seed=4, dtype=torch.float32).numpy()
    qmax, qmin = oracle.block_minmax(x[0], 1)
    kmax, kmin = oracle.block_minmax(x[1], 1)
    s = oracle.block_scores(qmax, qmin, kmax, kmin)
    want = 2.0 * x[0].astype(np.float64) @ x[1].astype(np.float64).T
    assert np.array_equal(s, want)


def test_scores_symmetric_in_the_key_summaries_and_positively_homogeneous():
    rng = np.random.default_rng(1)
    a, b, c, d = (rng.normal(size=(6, 8)) for _ in range(4))
    s = oracle.block_scores(a, b, c, d)
    assert np.array_equal(s, oracle.block_scores(a, b, d, c))
    np.testing.assert_allclose(oracle.block_scores(2 * a, 2 * b, c, d), 2 * s, rtol=1e-14)
    assert not np.allclose(s, oracle.block_scores(a, b, -c, -d))


# --------------------------------------------------------------------------
# top-k + sink + diagonal (SPADE step 4; top_k_block_mask; recipe note)
# --------------------------------------------------------------------------

def _brute_topk(row, k):
    """The unique k-subset whose every member outranks every non-member,
    ranking by larger score, then lower index."""
    nb = len(row)
    key = lambda j: (-row[j], j)
    found = []
    for sub in itertools.combinations(range(nb), k):
        rest = [j for j in range(nb) if j not in sub]
        if not rest or max(key(j) for j in sub) < min(key(j) for j in rest):
            found.append(set(sub))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_with_ties(seed):
    nb = 7
    rng = np.random.default_rng(seed)
    s = rng.integers(-2, 3, size=(nb, nb)).astype(np.float64)  # many ties
    for k, n_sink, dhw in [(1, 0, -1), (2, 1, 0), (3, 2, 1), (nb, 1, 0)]:
        idx, cnt = oracle.topk_block_list(s, k, n_sink, dhw, cap=nb)
        for i in range(nb):
            want = _brute_topk(s[i], k)
            want |= {j for j in range(nb) if j < n_sink or abs(j - i) <= dhw}
            got = idx[i, :cnt[i]].tolist()
            assert got == sorted(want)
            assert (idx[i, cnt[i]:] == -1).all()


def test_sink_and_diagonal_always_present():
    nb = 40
    s = np.random.default_rng(2).normal(size=(nb, nb))
    s[:, 0] = -1e9                      # the sink block never wins on score
    np.fill_diagonal(s, -1e9)           # nor does the diagonal
    idx, cnt = oracle.topk_block_list(s, 5, n_sink=1, diag_halfwidth=0)
    for i in range(nb):
        row = idx[i, :cnt[i]].tolist()
        assert 0 in row and i in row
        assert cnt[i] == (6 if i == 0 else 7)


# --------------------------------------------------------------------------
# structured masks (ADR step 1)
# --------------------------------------------------------------------------

def _expand_list_to_tmajor(idx, cnt, g, block, perm):
    """Element mask in T-major order from a block list in the permuted order."""
    S = len(perm)
    m = np.zeros((S, S), bool)
    for i in range(S // block):
        for c in range(cnt[i]):
            j = idx[i, c]
            m[i * block:(i + 1) * block, j * block:(j + 1) * block] = True
    if g > 0:
        p = np.arange(S)
        m &= (p[:, None] // g) == (p[None, :] // g)
    out = np.zeros_like(m)
    out[np.ix_(perm, perm)] = m
    return out


@pytest.mark.parametrize("grid,block", [((4, 4, 8), 32), ((2, 4, 8), 16), ((8, 4, 4), 16)])
def test_spatial_and_temporal_lists_are_exactly_frame_and_pixel_masks(grid, block):
    t, h, w = _coords(grid)
    for kind, want in [("spatial", t[:, None] == t[None, :]),
                       ("temporal", (h[:, None] == h[None, :]) & (w[:, None] == w[None, :]))]:
        tile, rad = oracle.structured_tile(kind, grid)
        idx, cnt, g = oracle.tile_neighbourhood_list(grid, tile, rad, block)
        perm = oracle.tile_permutation(grid, tile)
        got = _expand_list_to_tmajor(idx, cnt, g, block, perm)
        assert np.array_equal(got, want), kind


def test_sliding_tile_list_is_the_clipped_tile_neighbourhood():
    grid, tile, block = (6, 12, 12), (2, 4, 4), 16
    idx, cnt, g = oracle.tile_neighbourhood_list(grid, tile, (1, 1, 1), block)
    perm = oracle.tile_permutation(grid, tile)
    got = _expand_list_to_tmajor(idx, cnt, g, block, perm)
    t, h, w = _coords(grid)
    ct, ch, cw = t // 2, h // 4, w // 4
    want = ((np.abs(ct[:, None] - ct[None, :]) <= 1) & (np.abs(ch[:, None] - ch[None, :]) <= 1)
            & (np.abs(cw[:, None] - cw[None, :]) <= 1))
    assert g == 0 and np.array_equal(got, want)
    # a corner tile has 2*2*2 neighbours, an interior one 3*3*3; 2 blocks per tile
    assert cnt.min() == 2 * 8 and cnt.max() == 2 * 27
    for i in range(len(cnt)):
        assert np.all(np.diff(idx[i, :cnt[i]]) > 0)


def _nearest_start(c, r, n):
    """Brute force: of the in-grid windows of min(2r+1, n) tiles, the one whose
    start is nearest the centred start c - r."""
    w = min(2 * r + 1, n)
    starts = range(0, n - w + 1)
    s = min(starts, key=lambda s0: abs(s0 - (c - r)))
    return s, s + w - 1


_CENTERED_CASES = [((6, 12, 12), (2, 4, 4), (1, 1, 1), 16),   # 3 x 3 x 3 tiles: every window is the grid
                   ((8, 20, 12), (2, 4, 4), (1, 1, 1), 32),   # 4 x 5 x 3 tiles
                   ((8, 24, 8), (1, 4, 4), (2, 1, 0), 16),    # 8 x 6 x 2 tiles, unequal radii
                   ((4, 8, 16), (1, 2, 2), (1, 2, 3), 4)]     # 4 x 4 x 8 tiles, a radius beyond the grid


@pytest.mark.parametrize("grid,tile,radius,block", _CENTERED_CASES)
def test_centered_sliding_tile_is_the_nearest_in_grid_window(grid, tile, radius, block):
    idx, cnt, g = oracle.tile_neighbourhood_list(grid, tile, radius, block, centered=True)
    perm = oracle.tile_permutation(grid, tile)
    got = _expand_list_to_tmajor(idx, cnt, g, block, perm)
    t, h, w = _coords(grid)
    cs = [t // tile[0], h // tile[1], w // tile[2]]
    ns = [grid[a] // tile[a] for a in range(3)]
    want = np.ones_like(got)
    for a in range(3):
        lohi = np.array([_nearest_start(c, radius[a], ns[a]) for c in range(ns[a])])
        lo, hi = lohi[cs[a], 0], lohi[cs[a], 1]
        want &= (cs[a][None, :] >= lo[:, None]) & (cs[a][None, :] <= hi[:, None])
    assert g == 0 and np.array_equal(got, want)
    # every query sees the same number of key tiles, itself among them
    per_tile = np.prod([min(2 * radius[a] + 1, ns[a]) for a in range(3)])
    assert np.all(cnt == per_tile * (np.prod(tile) // block))
    assert np.all(np.diag(got))
    for i in range(len(cnt)):
        assert np.all(np.diff(idx[i, :cnt[i]]) > 0)


@pytest.mark.parametrize("grid,tile,radius,block", _CENTERED_CASES)
def test_centered_sliding_tile_agrees_with_clipped_inside_and_is_mirror_symmetric(grid, tile, radius, block):
    ci, cc, _ = oracle.tile_neighbourhood_list(grid, tile, radius, block, centered=True)
    pi, pc, _ = oracle.tile_neighbourhood_list(grid, tile, radius, block)
    ns = [grid[a] // tile[a] for a in range(3)]
    bpt = np.prod(tile) // block
    for i in range(len(cc)):
        tl = i // bpt
        c = (tl // (ns[1] * ns[2]), (tl // ns[2]) % ns[1], tl % ns[2])
        inside = all(radius[a] <= c[a] <= ns[a] - 1 - radius[a] for a in range(3))
        if inside:
            assert cc[i] == pc[i] and np.array_equal(ci[i, :cc[i]], pi[i, :pc[i]])
        else:
            # the clipped window is the centred one cut at the border
            assert set(pi[i, :pc[i]]) <= set(ci[i, :cc[i]])
    perm = oracle.tile_permutation(grid, tile)
    m = _expand_list_to_tmajor(ci, cc, 0, block, perm)
    t, h, w = _coords(grid)
    T, H, W = grid
    for refl in ((T - 1 - t) * H * W + h * W + w, t * H * W + (H - 1 - h) * W + w, t * H * W + h * W + (W - 1 - w)):
        assert np.array_equal(m[np.ix_(refl, refl)], m)


def test_centered_sliding_tile_is_not_symmetric_at_the_border():
    # 4 tiles along w, radius 1: tile 0 sees tiles 0..2, tile 2 sees 1..3
    grid, tile, block = (1, 4, 16), (1, 4, 4), 16
    ci, cc, _ = oracle.tile_neighbourhood_list(grid, tile, (0, 0, 1), block, centered=True)
    assert [list(ci[i, :cc[i]]) for i in range(4)] == [[0, 1, 2], [0, 1, 2], [1, 2, 3], [1, 2, 3]]
    pi, pc, _ = oracle.tile_neighbourhood_list(grid, tile, (0, 0, 1), block)
    assert [list(pi[i, :pc[i]]) for i in range(4)] == [[0, 1], [0, 1, 2], [1, 2, 3], [2, 3]]


# --------------------------------------------------------------------------
# head profile (ADR step 2; SVG: spatial or temporal pattern per head)
# --------------------------------------------------------------------------

def test_head_profile_uniform_attention_masses_are_the_pattern_sizes():
    # q = 0: every key has the same logit, so a pattern's mass is its size / S
    grid = (5, 3, 4)
    S, HW = 60, 12
    k = np.random.default_rng(3).standard_normal((S, 16)).astype(np.float32)
    q = np.zeros((S, 16), np.float32)
    rows = [0, 7, 59, 31]
    mass = oracle.pattern_masses(oracle.sampled_probs(q, k, rows), grid, rows)
    assert np.allclose(mass[:, 0], HW / S, rtol=0, atol=1e-15)
    assert np.allclose(mass[:, 1], 5 / S, rtol=0, atol=1e-15)


@pytest.mark.parametrize("alpha", [0.5, 2.0, 6.0])
def test_head_profile_closed_forms_of_one_hot_fields(alpha):
    grid = (4, 4, 4)
    T, HW, S = 4, 16, 64
    t, h, w = _coords(grid)
    hw = h * 4 + w
    rows = [0, 21, 42, 63]
    e = math.exp(alpha)
    # frame-coded field: logit alpha inside the query's frame, 0 elsewhere
    q = np.zeros((S, 16), np.float32)
    k = np.zeros((S, 16), np.float32)
    q[np.arange(S), t] = alpha
    k[np.arange(S), t] = 1.0
    kind, mass = oracle.classify_head(q, k, grid, rows, scale=1.0)
    z = HW * e + (S - HW)
    assert kind == 0
    assert mass[0] == pytest.approx(HW * e / z, rel=1e-13)
    assert mass[1] == pytest.approx((e + T - 1) / z, rel=1e-13)
    # position-coded field: logit alpha at the query's (h, w), 0 elsewhere
    q[:] = 0.0
    k[:] = 0.0
    q[np.arange(S), hw] = alpha
    k[np.arange(S), hw] = 1.0
    kind, mass = oracle.classify_head(q, k, grid, rows, scale=1.0)
    z = T * e + (S - T)
    sp, tp = (e + HW - 1) / z, T * e / z
    assert mass[1] == pytest.approx(tp, rel=1e-13)
    assert mass[0] == pytest.approx(sp, rel=1e-13)
    # a weak position code still leaves more mass on the 16-token frame than on
    # the 4 keys at the query's position
    assert kind == (0 if sp >= tp else 1) and kind == (1 if alpha >= 2 else 0)


@pytest.mark.parametrize("alpha", [0.05, 0.5, 2.0, 6.0])
def test_head_profile_mass_per_key_rule_closed_forms(alpha):
    """The per-key rule compares spatial mass / (H W) with temporal mass / T.
    With a frame code every key of the frame holds e^alpha / z and the keys at
    the query's (h, w) hold (e^alpha + T - 1) / (T z) on average, so the head is
    spatial for every alpha > 0; with a position code it is temporal for every
    alpha > 0 (the mass rule calls weak position codes spatial, see above)."""
    grid = (4, 4, 4)
    T, HW, S = 4, 16, 64
    t, h, w = _coords(grid)
    hw = h * 4 + w
    rows = [0, 21, 42, 63]
    q = np.zeros((S, 16), np.float32)
    k = np.zeros((S, 16), np.float32)
    q[np.arange(S), t] = alpha
    k[np.arange(S), t] = 1.0
    kind, mass = oracle.classify_head(q, k, grid, rows, scale=1.0, rule="mass_per_key")
    assert kind == 0 and mass[0] / HW > mass[1] / T
    q[:] = 0.0
    k[:] = 0.0
    q[np.arange(S), hw] = alpha
    k[np.arange(S), hw] = 1.0
    kind, mass = oracle.classify_head(q, k, grid, rows, scale=1.0, rule="mass_per_key")
    assert kind == 1 and mass[1] / T > mass[0] / HW
    assert kind == oracle.classify_head(q, k, grid, rows, scale=1.0, rule="mass")[0] or alpha < 2


def test_head_profile_mass_per_key_uniform_tie_and_equal_sizes():
    # q = 0: every key carries 1/S, so both patterns hold 1/S per key exactly
    # (1/64 and its multiples are exact): a tie, which goes to spatial
    grid = (4, 4, 4)
    k = np.random.default_rng(7).standard_normal((64, 8)).astype(np.float32)
    q = np.zeros((64, 8), np.float32)
    kind, mass = oracle.classify_head(q, k, grid, [0, 9, 33, 63], rule="mass_per_key")
    assert mass[0] / 16 == mass[1] / 4 and kind == 0
    # T = H W: the two rules are one
    grid = (4, 2, 2)
    rng = np.random.default_rng(8)
    for _ in range(5):
        q = rng.standard_normal((16, 8)).astype(np.float32)
        k = rng.standard_normal((16, 8)).astype(np.float32)
        assert (oracle.classify_head(q, k, grid, [0, 3, 9], rule="mass_per_key")[0]
                == oracle.classify_head(q, k, grid, [0, 3, 9], rule="mass")[0])
    with pytest.raises(ValueError):
        oracle.classify_head(q, k, grid, [0], rule="density")


def test_head_profile_matches_torch_softmax_and_coordinate_masks():
    grid = (6, 4, 5)
    S = 120
    rng = np.random.default_rng(11)
    q = (rng.standard_normal((S, 32)) * 0.7).astype(np.float32)
    k = (rng.standard_normal((S, 32)) * 0.7).astype(np.float32)
    rows = np.array([0, 1, 19, 20, 64, 119], np.int32)
    scale = 0.3
    logits = torch.as_tensor(q, dtype=torch.float64)[rows] @ torch.as_tensor(k, dtype=torch.float64).T * scale
    want_p = torch.softmax(logits, dim=-1).numpy()
    got_p = oracle.sampled_probs(q, k, rows, scale)
    assert np.allclose(got_p, want_p, rtol=1e-12, atol=1e-15)
    t, h, w = _coords(grid)
    same_t = t[rows][:, None] == t[None, :]
    same_hw = (h[rows][:, None] == h[None, :]) & (w[rows][:, None] == w[None, :])
    mass = oracle.pattern_masses(got_p, grid, rows)
    assert np.allclose(mass[:, 0], (want_p * same_t).sum(1), rtol=1e-12)
    assert np.allclose(mass[:, 1], (want_p * same_hw).sum(1), rtol=1e-12)
    # the patterns meet only at the query itself
    self_p = want_p[np.arange(len(rows)), rows]
    assert np.all(mass >= 0) and np.all(mass <= 1 + 1e-12)
    assert np.all(mass[:, 0] + mass[:, 1] - self_p <= 1 + 1e-12)


def test_head_profile_tie_goes_to_spatial():
    # T = H*W and uniform attention: both patterns hold 4/16 of every row
    grid = (4, 2, 2)
    q = np.zeros((16, 8), np.float32)
    k = np.random.default_rng(5).standard_normal((16, 8)).astype(np.float32)
    kind, mass = oracle.classify_head(q, k, grid, [0, 5, 10, 15])
    assert mass[0] == mass[1] and kind == 0


# --------------------------------------------------------------------------
# attention (windowed_attention / full_attention; recipe note: dropped blocks)
# --------------------------------------------------------------------------

def _qkv(S, D, seed):
    q, k, v = (integer_grid((S, D), seed + o, torch.float32).numpy() for o in range(3))
    return q, k, v


@pytest.mark.parametrize("window", [64, 200, 257])
def test_window_at_least_S_is_dense_sdpa(window):
    q, k, v = _qkv(64, 16, 20)
    scale = 16 ** -0.5
    got = oracle.window_attention(q, k, v, window=window, sink=3)
    want = _sdpa64(q, k, v, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle.dense_attention(q, k, v), want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("S,window,sink", [(64, 1, 0), (64, 9, 0), (64, 10, 5), (50, 31, 7),
                                           (64, 63, 64), (37, 2, 37)])
def test_window_matches_sdpa_with_the_docstring_mask(S, window, sink):
    """Mask built from the module docstring's statement: sinks j in [0, sink)
    and local j in [max(0, i - half), min(S, i + half + 1))."""
    q, k, v = _qkv(S, 16, 30)
    half = window // 2
    m = np.zeros((S, S), bool)
    for i in range(S):
        m[i, :sink] = True
        m[i, max(0, i - half):min(S, i + half + 1)] = True
    got = oracle.window_attention(q, k, v, window=window, sink=sink, scale=0.3)
    np.testing.assert_allclose(got, _sdpa64(q, k, v, 0.3, m), rtol=0, atol=1e-12)


def test_window_formula_covers_everything_from_2S_minus_1():
    """|i - j| <= floor(window/2) reaches every key once window >= 2S - 1."""
    S = 40
    q, k, v = _qkv(S, 8, 40)
    half = (2 * S - 1) // 2
    assert all(abs(i - j) <= half for i in range(S) for j in range(S))
    got = oracle.window_attention(q, k, v, window=2 * S - 1, sink=0)
    np.testing.assert_allclose(got, _sdpa64(q, k, v, 8 ** -0.5), atol=1e-12, rtol=0)


def test_default_scale_is_inverse_sqrt_head_dim():
    q, k, v = _qkv(32, 16, 50)
    np.testing.assert_array_equal(oracle.dense_attention(q, k, v),
                                  oracle.dense_attention(q, k, v, scale=0.25))
    assert oracle.default_scale(64, None) == 0.125


@pytest.mark.parametrize("S,chunk,half,sink", [(300, 128, 32, 16), (300, 64, 100, 0),
                                               (513, 512, 7, 300), (90, 7, 3, 10)])
def test_key_ranges_cover_exactly_the_chunk_union(S, chunk, half, sink):
    """_key_ranges_for_block returns exactly the union, over the chunk's rows,
    of the per-element visible keys, without overlap."""
    for qs in range(0, S, chunk):
        qe = min(S, qs + chunk)
        ranges = oracle.window_key_ranges(qs, qe, S, half, sink)
        got = [j for a, b in ranges for j in range(a, b)]
        assert len(got) == len(set(got))
        want = {j for i in range(qs, qe) for j in range(S) if j < sink or abs(i - j) <= half}
        assert set(got) == want


def test_block_list_attention_equals_sdpa_with_the_expanded_mask():
    S, D, block = 96, 16, 16
    q, k, v = _qkv(S, D, 60)
    nb = S // block
    rng = np.random.default_rng(7)
    idx = np.full((nb, 4), -1, np.int32)
    cnt = np.zeros(nb, np.int32)
    m = np.zeros((S, S), bool)
    for i in range(nb):
        sel = sorted(set(rng.choice(nb, 3, replace=False).tolist()) | {i})
        cnt[i] = len(sel)
        idx[i, :len(sel)] = sel
        for j in sel:
            m[i * block:(i + 1) * block, j * block:(j + 1) * block] = True
    got = oracle.block_sparse_attention(q, k, v, idx, cnt, block, 0, 0.2)
    np.testing.assert_allclose(got, _sdpa64(q, k, v, 0.2, m), atol=1e-12, rtol=0)
    # group mask: only keys of the query's own group of 4 tokens
    g = 4
    p = np.arange(S)
    got = oracle.block_sparse_attention(q, k, v, idx, cnt, block, g, 0.2)
    want = _sdpa64(q, k, v, 0.2, m & ((p[:, None] // g) == (p[None, :] // g)))
    np.testing.assert_allclose(got, want, atol=1e-12, rtol=0)


def test_all_blocks_budget_equals_dense_attention():
    """k = number of blocks keeps every block: the SPADE composition must then
    be dense attention in the original T-major order."""
    grid = (4, 8, 8)
    q, k, v = (integer_grid((256, 64), 70 + o, torch.float32).numpy() for o in range(3))
    tiles = [(2, 4, 4), (1, 8, 4), (4, 2, 4)]
    res = oracle.spade_head(q, k, v, grid, tiles, k_blocks=8)
    assert (res["cnt"] == 8).all()
    np.testing.assert_allclose(res["out"], _sdpa64(q, k, v, 64 ** -0.5), atol=1e-12, rtol=0)


def test_sampled_rows_match_full_rows():
    grid = (4, 8, 8)
    q, k, v = (integer_grid((256, 64), 80 + o, torch.float32).numpy() for o in range(3))
    full = oracle.spade_head(q, k, v, grid, [(2, 4, 4)], k_blocks=2)
    part = oracle.spade_head(q, k, v, grid, [(2, 4, 4)], k_blocks=2, query_blocks=[0, 5, 7])
    np.testing.assert_array_equal(part["out_perm"], full["out_perm"][part["rows"]])


# --------------------------------------------------------------------------
# grids the tiles do not divide ("Adaptive tiling (SPADE)", Deviations and
# notes: pad to a multiple of the tiles with zero tokens, excluded from the
# cohesion, and mask the padded keys)
# --------------------------------------------------------------------------

def test_padded_grid_is_the_per_axis_lcm_multiple():
    tiles = [(1, 8, 16), (2, 8, 8), (4, 4, 8)]
    assert oracle.padded_grid((16, 45, 80), tiles) == (16, 48, 80)   # Wan's 16 x 45 x 80
    assert oracle.padded_grid((13, 45, 81), tiles) == (16, 48, 96)
    assert oracle.padded_grid((32, 48, 80), tiles) == (32, 48, 80)   # divisible: unchanged
    assert oracle.padded_grid((3, 5, 6), [(1, 2, 4), (2, 2, 2)]) == (4, 6, 8)


def test_pad_grid_keeps_coordinates_and_zero_fills():
    grid, padded = (3, 5, 6), (4, 6, 8)
    x = np.arange(3 * 5 * 6 * 2, dtype=np.float32).reshape(-1, 2) + 1
    y = oracle.pad_grid(x, grid, padded)
    real = oracle.real_tokens(grid, padded)
    assert real.sum() == 90 and np.array_equal(y[real], x)
    assert (y[~real] == 0).all()
    # token (t, h, w) of the real grid sits at (t, h, w) of the padded one
    t, h, w = 2, 4, 5
    assert np.array_equal(y[(t * 6 + h) * 8 + w], x[(t * 5 + h) * 6 + w])


def test_padded_all_blocks_budget_equals_dense_attention_over_the_real_tokens():
    """pad = mask: with every block kept, the padded composition must be dense
    attention over the real tokens alone (the padding takes no part)."""
    grid = (3, 5, 6)
    tiles = [(1, 2, 4), (2, 2, 2)]
    q, k, v = (integer_grid((90, 16), 90 + o, torch.float32).numpy() for o in range(3))
    nb = 4 * 6 * 8 // 8
    res = oracle.spade_head(q, k, v, grid, tiles, k_blocks=nb, n_sink=0, diag_halfwidth=-1)
    assert res["padded_grid"] == (4, 6, 8) and (res["cnt"] == nb).all()
    np.testing.assert_allclose(res["out"], _sdpa64(q, k, v, 16 ** -0.5), atol=1e-12, rtol=0)


def test_padded_cohesion_by_brute_force():
    """Cohesion on a padded grid: per tile the mean cosine over distinct pairs
    of its non-zero queries, averaged over the tiles that hold any query; the
    zero padding adds neither queries nor tiles."""
    grid, tiles = (3, 5, 6), [(1, 2, 4), (2, 2, 2), (1, 2, 2)]
    padded = oracle.padded_grid(grid, tiles)
    q = integer_grid((90, 8), 95, torch.float32).numpy()
    q[7] = 0.0                                   # one real zero-norm query too
    qp = oracle.pad_grid(q, grid, padded)
    _, got = oracle.select_tiling(qp, padded, tiles)
    tp, hp, wp = _coords(padded)
    for c, (tt, th, tw) in enumerate(tiles):
        label = ((tp // tt) * (padded[1] // th) + hp // th) * (padded[2] // tw) + wp // tw
        vals = []
        for lab in np.unique(label):
            rows = qp[label == lab]
            rows = rows[np.linalg.norm(rows, axis=1) > 0].astype(np.float64)
            if len(rows) == 0:
                continue
            n = rows / np.linalg.norm(rows, axis=1, keepdims=True)
            if len(n) < 2:
                vals.append(0.0)
                continue
            pairs = [n[i] @ n[j] for i in range(len(n)) for j in range(len(n)) if i != j]
            vals.append(float(np.mean(pairs)))
        assert abs(got[c] - np.mean(vals)) < 1e-12, (c, got[c], np.mean(vals))


# --------------------------------------------------------------------------
# top-p (mass budget) lists: the pages name top_p_block_mask only; the
# reading (softmax(scale * score) mass, shortest descending prefix reaching
# p, ties to the lower index, static blocks ORed in) is pinned by properties
# that do not restate the algorithm
# --------------------------------------------------------------------------

def _topp_sets(score, p, scale, n_sink=0, dw=-1):
    idx, cnt = oracle.topp_block_list(score, p, scale, n_sink, dw)
    return [set(idx[i, :cnt[i]].tolist()) for i in range(score.shape[0])]


def _probs(row, scale):
    e = np.exp(scale * (row - row.max()))
    return e / e.sum()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_topp_is_the_smallest_upper_set_reaching_p(seed):
    rng = np.random.default_rng(seed)
    nb = 23
    score = rng.normal(size=(nb, nb)) * 4
    for p in (0.05, 0.3, 0.6, 0.9, 0.999):
        for i, kept in enumerate(_topp_sets(score, p, 0.7)):
            pr = _probs(score[i], 0.7)
            rest = set(range(nb)) - kept
            # an upper set: no dropped block scores above a kept one
            assert not rest or min(score[i, list(kept)]) >= max(score[i, list(rest)])
            # it reaches p, and without its lowest block it would not
            assert pr[list(kept)].sum() >= p - 1e-12
            low = min(kept, key=lambda j: (score[i, j], -j))
            assert pr[list(kept - {low})].sum() < p + 1e-12


def test_topp_closed_forms():
    rng = np.random.default_rng(5)
    nb = 17
    score = rng.normal(size=(nb, nb))
    # p = 1 keeps every block; a vanishing p keeps the row's maximum alone
    assert all(k == set(range(nb)) for k in _topp_sets(score, 1.0, 1.0))
    assert all(k == {int(np.argmax(score[i]))} for i, k in enumerate(_topp_sets(score, 1e-12, 1.0)))
    # scale 0: uniform probabilities, so the mass budget is a count budget: the
    # ceil(p nb) highest scores, i.e. the top-k list with k = ceil(p nb)
    for p in (0.1, 0.5, 0.77):
        k = int(np.ceil(p * nb - 1e-9))
        ti, tc = oracle.topk_block_list(score, k, 0, -1)
        assert _topp_sets(score, p, 0.0) == [set(ti[i, :tc[i]].tolist()) for i in range(nb)]
    # equal scores rank the lower index first
    tie = np.zeros((4, 4))
    assert _topp_sets(tie, 0.5, 1.0)[0] == {0, 1}


def test_topp_invariances_and_static_blocks():
    rng = np.random.default_rng(6)
    nb = 19
    score = rng.normal(size=(nb, nb)) * 2
    base = _topp_sets(score, 0.6, 1.3)
    assert _topp_sets(score + 7.5, 0.6, 1.3) == base           # softmax is shift invariant
    assert _topp_sets(score * 2.0, 0.6, 0.65) == base          # only scale * score matters
    prev = None
    for p in (0.2, 0.4, 0.6, 0.8):                             # monotone in p
        cur = _topp_sets(score, p, 1.3)
        if prev is not None:
            assert all(a <= b for a, b in zip(prev, cur))
        prev = cur
    with_static = _topp_sets(score, 0.6, 1.3, n_sink=2, dw=1)
    for i, (k, ks) in enumerate(zip(base, with_static)):
        assert ks == k | {0, 1} | {j for j in range(nb) if abs(j - i) <= 1}


# --------------------------------------------------------------------------
# centroid-compensated attention (SPADE Recipe: skipped blocks compensated)
# --------------------------------------------------------------------------

def _labels_irregular(S, seed):
    """Block labels with blocks of unequal sizes (1 to 12 tokens), in order."""
    rng = np.random.default_rng(seed)
    sizes = []
    while sum(sizes) < S:
        sizes.append(int(rng.integers(1, 13)))
    sizes[-1] -= sum(sizes) - S
    return np.repeat(np.arange(len(sizes)), sizes).astype(np.int32), len(sizes)


def test_compensated_attention_with_every_block_kept_is_dense():
    q, k, v = _qkv(96, 16, 40)
    lab = (np.arange(96) // 16).astype(np.int32)
    got = oracle.centroid_compensated_attention(q, k, v, lab, lab, np.ones((6, 6), bool), scale=0.25)
    assert np.allclose(got, _sdpa64(q, k, v, 0.25), rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_compensated_attention_is_exact_when_block_keys_are_equal(seed):
    # every key of a block is the same vector (values differ): a skipped block's
    # centroid then stands for its keys exactly, whatever the mask
    S, D = 120, 16
    rng = np.random.default_rng(100 + seed)
    kl, nkb = _labels_irregular(S, seed)
    ql = (np.arange(S) // 10).astype(np.int32)
    q = rng.standard_normal((S, D)).astype(np.float32)
    kb = rng.standard_normal((nkb, D)).astype(np.float32)
    k = kb[kl]
    v = rng.standard_normal((S, D)).astype(np.float32)
    mask = rng.random((12, nkb)) < 0.3
    mask[0] = False       # query block 0 keeps nothing: centroids only
    mask[1] = True        # query block 1 keeps everything
    got = oracle.centroid_compensated_attention(q, k, v, ql, kl, mask, scale=0.5)
    assert np.allclose(got, _sdpa64(q, k, v, 0.5), rtol=0, atol=1e-12)


def test_compensated_attention_with_nothing_kept_is_attention_over_weighted_centroids():
    S, D = 90, 8
    q, k, v = _qkv(S, D, 50)
    kl, nkb = _labels_irregular(S, 7)
    ql = np.zeros(S, np.int32)
    got = oracle.centroid_compensated_attention(q, k, v, ql, kl, np.zeros((1, nkb), bool), scale=0.7)
    n = np.bincount(kl, minlength=nkb).astype(np.float64)
    kbar = np.stack([k[kl == b].astype(np.float64).mean(0) for b in range(nkb)])
    vbar = np.stack([v[kl == b].astype(np.float64).mean(0) for b in range(nkb)])
    # a weight n_b on a key is an additive log(n_b) on its logit
    bias = torch.as_tensor(np.log(n))[None, None, None, :].expand(1, 1, S, nkb)
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.as_tensor(q, dtype=torch.float64)[None, None], torch.as_tensor(kbar)[None, None],
        torch.as_tensor(vbar)[None, None], attn_mask=bias, scale=0.7)[0, 0].numpy()
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_compensated_attention_reduces_to_dropped_blocks_when_skipped_weights_vanish():
    # queries positive, skipped blocks' keys strongly negative: their centroid
    # weights underflow next to the kept keys, leaving the recipe note's
    # dropped-block attention
    S, D, block = 64, 8, 16
    rng = np.random.default_rng(9)
    q = rng.uniform(0.5, 1.0, (S, D)).astype(np.float32)
    k = rng.uniform(-0.5, 0.5, (S, D)).astype(np.float32)
    v = rng.standard_normal((S, D)).astype(np.float32)
    lab = (np.arange(S) // block).astype(np.int32)
    mask = np.eye(4, dtype=bool)
    mask[:, 0] = True
    for b in (1, 2, 3):
        k[lab == b] -= 40.0
    got = oracle.centroid_compensated_attention(q, k, v, lab, lab, mask, scale=1.0)
    idx = np.full((4, 2), -1, np.int32)
    cnt = np.zeros(4, np.int32)
    for a in range(4):
        js = np.flatnonzero(mask[a])
        idx[a, :len(js)] = js
        cnt[a] = len(js)
    want = oracle.block_sparse_attention(q, k, v, idx, cnt, block, 0, scale=1.0)
    assert np.allclose(got, want, rtol=0, atol=1e-12)
