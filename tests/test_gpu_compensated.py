"""Centroid-compensated block-sparse attention (through the C ABI) against the
fp64 oracle.

"Adaptive tiling (SPADE)", Recipe: centroid_compensated_attention(q, k, v,
q_labels, k_labels, block_mask).  Blocks are the 128-position blocks of the
tile-contiguous order, so the oracle gets labels = position // 128 and the
block mask the lists expand to.  Outputs are held to the attention tolerance
(max-abs 1e-2, relative-L2 2e-3 in the fp32-output mode); a bf16 output must
be the fp32 result rounded once, and a list that keeps every block must give
the plain block-sparse attention bit for bit.
"""

import numpy as np
import pytest
import torch

import block_sparse_self_b200 as vsa
import oracle
from workloads import WORKLOADS, integer_grid, make_qkv, smooth_qkv

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 1e-2, 2e-3
DEV = "cuda"
BLOCK = 128


@pytest.fixture(autouse=True)
def _no_device_errors():
    yield
    vsa.device_status()


def _np(t):
    return t.detach().float().cpu().numpy()


def assert_close(got, want, what=""):
    g = np.asarray(got, np.float64)
    w = np.asarray(want, np.float64)
    assert np.isfinite(g).all(), what
    err = np.abs(g - w).max()
    rl2 = np.linalg.norm(g - w) / max(np.linalg.norm(w), 1e-30)
    assert err <= MAX_ABS and rl2 <= REL_L2, f"{what}: max-abs {err:.3e}, rel-L2 {rl2:.3e}"


def _block_mask(idx, cnt, nb):
    m = np.zeros((nb, nb), np.uint8)
    for i in range(nb):
        m[i, idx[i, :cnt[i]]] = 1
    return m


def _oracle_rows(q, k, v, idx, cnt, rows=None):
    """Oracle over one head's permuted rows with labels = position // 128."""
    S = q.shape[0]
    nb = S // BLOCK
    labels = np.arange(S, dtype=np.int32) // BLOCK
    return oracle.centroid_compensated_attention(q, k, v, labels, labels, _block_mask(idx, cnt, nb), rows=rows)


def _lists(nb, cap, bh, seed, keep_forced_only=()):
    """Random ascending lists that always hold block 0 and the diagonal;
    query blocks in keep_forced_only keep nothing else."""
    rng = np.random.default_rng(seed)
    idx = np.full((bh, nb, cap), -1, np.int32)
    cnt = np.zeros((bh, nb), np.int32)
    for h in range(bh):
        for i in range(nb):
            forced = {0, i}
            if i in keep_forced_only:
                chosen = sorted(forced)
            else:
                extra = rng.choice(nb, size=min(nb, rng.integers(1, cap - 1)), replace=False).tolist()
                chosen = sorted((forced | set(extra)))[:cap]
                if i not in chosen:
                    chosen = sorted(set(chosen[:cap - 1]) | {i})
            idx[h, i, :len(chosen)] = chosen
            cnt[h, i] = len(chosen)
    return idx, cnt


@pytest.mark.parametrize("S,D,cap", [(1024, 64, 4), (2560, 128, 6), (25600, 128, 20), (38400, 64, 31)])
def test_compensated_matches_oracle(S, D, cap):
    """Several heads, per-head lists, nb from 8 to 300 (centroid tiles cut by
    the end of the block range), fp32 and bf16 outputs."""
    grid = {1024: (4, 16, 16), 2560: (10, 16, 16), 25600: (25, 32, 32), 38400: (24, 40, 40)}[S]
    H, nb = 3, S // BLOCK
    q, k, v = smooth_qkv(1, H, grid, D, seed=S + D, device=DEV)
    idx, cnt = _lists(nb, cap, H, seed=S, keep_forced_only={nb // 2})
    ti, tc = torch.tensor(idx, device=DEV).view(1, H, nb, cap), torch.tensor(cnt, device=DEV).view(1, H, nb)
    o32 = vsa.centroid_compensated_attention(q, k, v, ti, tc, out_dtype=torch.float32)
    o16 = vsa.centroid_compensated_attention(q, k, v, ti, tc, out_dtype=torch.bfloat16)
    assert torch.equal(o16, o32.to(torch.bfloat16))
    for h in range(H):
        blocks = sorted({0, nb // 2, nb - 1, *range(1, nb, max(1, nb // 6))})
        rows = np.concatenate([np.arange(b * BLOCK, (b + 1) * BLOCK) for b in blocks])
        want = _oracle_rows(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), idx[h], cnt[h], rows)
        assert_close(_np(o32[0, h])[rows], want, f"S={S} head {h}")


def test_compensated_shared_list_and_every_block_kept():
    """A list shared by every head; a list of every block compensates nothing
    and equals the plain block-sparse attention bit for bit."""
    grid, D = (8, 16, 16), 128
    S, nb = 2048, 16
    q, k, v = smooth_qkv(2, 2, grid, D, seed=5, device=DEV)
    idx, cnt = _lists(nb, 5, 1, seed=9)
    ti, tc = torch.tensor(idx[0], device=DEV), torch.tensor(cnt[0], device=DEV)
    o = vsa.centroid_compensated_attention(q, k, v, ti, tc, out_dtype=torch.float32)
    for b in range(2):
        for h in range(2):
            want = _oracle_rows(_np(q[b, h]), _np(k[b, h]), _np(v[b, h]), idx[0], cnt[0])
            assert_close(_np(o[b, h]), want, f"shared list b={b} h={h}")
    full = torch.arange(nb, dtype=torch.int32, device=DEV).repeat(nb, 1).contiguous()
    fcnt = torch.full((nb,), nb, dtype=torch.int32, device=DEV)
    oc = vsa.centroid_compensated_attention(q, k, v, full, fcnt, out_dtype=torch.float32)
    assert torch.equal(oc, vsa.block_sparse_attention(q, k, v, full, fcnt, BLOCK, out_dtype=torch.float32))


def test_compensated_one_block_lists():
    """Lists of one block (the diagonal): the kept block runs through the
    one-key-block kernel with its per-row softmax state, every other block
    through the centroid pass."""
    grid, D = (8, 16, 16), 128
    S, nb, H = 2048, 16, 2
    q, k, v = smooth_qkv(1, H, grid, D, seed=21, device=DEV)
    idx = np.tile(np.arange(nb, dtype=np.int32)[None, :, None], (H, 1, 1))
    cnt = np.ones((H, nb), np.int32)
    o = vsa.centroid_compensated_attention(q, k, v, torch.tensor(idx, device=DEV).view(1, H, nb, 1),
                                           torch.tensor(cnt, device=DEV).view(1, H, nb), out_dtype=torch.float32)
    for h in range(H):
        want = _oracle_rows(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), idx[h], cnt[h])
        assert_close(_np(o[0, h]), want, f"head {h}")


def test_compensated_equal_keys_within_blocks_is_dense_attention():
    """Keys (and values) equal within each block: every skipped block's
    centroid stands for it exactly, so the result is dense attention whatever
    the lists keep (the oracle's own pin, on the GPU path)."""
    grid, D = (4, 16, 32), 64
    S, nb, H = 2048, 16, 2
    q = integer_grid((1, H, S, D), 31, torch.bfloat16, DEV)
    kb = integer_grid((1, H, nb, 1, D), 32, torch.bfloat16, DEV)
    vb = integer_grid((1, H, nb, 1, D), 33, torch.bfloat16, DEV)
    k = kb.expand(1, H, nb, BLOCK, D).reshape(1, H, S, D).contiguous()
    v = vb.expand(1, H, nb, BLOCK, D).reshape(1, H, S, D).contiguous()
    idx, cnt = _lists(nb, 4, H, seed=3, keep_forced_only={3, 7})
    o = vsa.centroid_compensated_attention(q, k, v, torch.tensor(idx, device=DEV).view(1, H, nb, 4),
                                           torch.tensor(cnt, device=DEV).view(1, H, nb), out_dtype=torch.float32)
    for h in range(H):
        assert_close(_np(o[0, h]), oracle.dense_attention(_np(q[0, h]), _np(k[0, h]), _np(v[0, h])), f"head {h}")


def test_compensated_invalid_list_writes_zeros_and_sets_status():
    grid, D = (4, 16, 16), 64
    S, nb = 1024, 8
    q, k, v = smooth_qkv(1, 1, grid, D, seed=2, device=DEV)
    idx = torch.tensor([[0, 1], [1, 0]] + [[0, i] for i in range(2, nb)], dtype=torch.int32, device=DEV)
    idx[0, 1] = 0                       # row 0: 0, 0 is not strictly ascending
    cnt = torch.full((nb,), 2, dtype=torch.int32, device=DEV)
    o = vsa.centroid_compensated_attention(q, k, v, idx, cnt, out_dtype=torch.float32)
    with pytest.raises(RuntimeError):
        vsa.device_status()
    assert torch.count_nonzero(o[0, 0, :BLOCK]) == 0     # rows of the invalid list
    assert torch.count_nonzero(o[0, 0, BLOCK:2 * BLOCK]) == 0   # row 1: 1, 0 descends
    assert torch.isfinite(o).all()


def test_compensated_adaptive_full_size_sampled():
    """The S = 122880 adaptive workload in each head's tiling (explicit
    permuted copies) with its top-k lists, k = 96, both taken from the oracle
    and given to the GPU as inputs: sampled query blocks of two heads, one of
    them keeping only its sink and diagonal blocks."""
    w = WORKLOADS["spade_adaptive_s122880"]
    H = 4
    q, k, v = make_qkv(w, device=DEV, heads=H)
    choices, perms, idx_o, cnt_o = [], [], [], []
    for h in range(H):
        qh, kh = _np(q[0, h]), _np(k[0, h])
        c, _ = oracle.select_tiling(qh, w.grid, list(w.tiles))
        perm = oracle.tile_permutation(w.grid, w.tiles[c])
        qmax, qmin = oracle.block_minmax(oracle.permute_rows(qh, perm), BLOCK)
        kmax, kmin = oracle.block_minmax(oracle.permute_rows(kh, perm), BLOCK)
        i_, c_ = oracle.topk_block_list(oracle.block_scores(qmax, qmin, kmax, kmin), w.k)
        choices.append(c)
        perms.append(perm)
        idx_o.append(i_)
        cnt_o.append(c_)
    idx_np, cnt_np = np.stack(idx_o), np.stack(cnt_o)
    # head 3: query block 500 keeps only its forced blocks (0 and 500)
    idx_np[3, 500] = -1
    idx_np[3, 500, :2] = (0, 500)
    cnt_np[3, 500] = 2
    choice = torch.tensor(choices, dtype=torch.int32, device=DEV)
    qp, kp, vp = (vsa.permute(x, w.grid, list(w.tiles), choice) for x in (q, k, v))
    idx = torch.as_tensor(idx_np, device=DEV).view(1, H, w.nb, -1)
    cnt = torch.as_tensor(cnt_np, device=DEV).view(1, H, w.nb)
    o = vsa.centroid_compensated_attention(qp, kp, vp, idx, cnt, out_dtype=torch.float32)
    for h in (1, 3):
        blocks = [0, 17, 500, 958, w.nb - 1]
        rows = np.concatenate([np.arange(b * BLOCK, (b + 1) * BLOCK) for b in blocks])
        qo, ko, vo = (oracle.permute_rows(_np(x[0, h]), perms[h]) for x in (q, k, v))
        want = _oracle_rows(qo, ko, vo, idx_np[h], cnt_np[h], rows)
        got = _np(o[0, h])[rows]
        for bi, b in enumerate(blocks):
            assert_close(got[bi * BLOCK:(bi + 1) * BLOCK], want[bi * BLOCK:(bi + 1) * BLOCK], f"head {h} block {b}")


def test_spade_attention_compensated_composition():
    """spade_attention(compensate=True): tiling choice, permutation, scores,
    top-k lists and the compensated attention, back in T-major order, against
    the oracle's steps on every head (integer-grid values: exact lists), in
    the oracle's tiling or in one within 1e-5 of its best cohesion (the
    tiling choice's fp32 resolution), a set the oracle alone decides."""
    grid, tiles = (8, 16, 16), [(1, 8, 16), (2, 8, 8), (4, 4, 8)]
    q = integer_grid((1, 3, 2048, 64), 51, torch.bfloat16, DEV)
    k = integer_grid((1, 3, 2048, 64), 52, torch.bfloat16, DEV)
    v = integer_grid((1, 3, 2048, 64), 53, torch.bfloat16, DEV)
    o, mid = vsa.spade_attention(q, k, v, grid, tiles, topk=3, out_dtype=torch.float32, compensate=True,
                                 return_intermediates=True)
    for h in range(3):
        qh, kh, vh = (_np(x[0, h]) for x in (q, k, v))
        _, cohesion = oracle.select_tiling(qh, grid, tiles)
        best = int(np.argmax(cohesion))
        near = [best] + [c for c in range(len(tiles)) if c != best and cohesion[c] >= cohesion[best] - 1e-5]
        failures = []
        for c in near:
            res = oracle.spade_head(qh, kh, vh, grid, [tiles[c]], 3, query_blocks=[0])
            perm = res["perm"]
            qp, kp, vp = (oracle.permute_rows(x, perm) for x in (qh, kh, vh))
            want_p = _oracle_rows(qp, kp, vp, res["idx"], res["cnt"])
            want = np.empty_like(want_p)
            want[perm] = want_p
            try:
                assert np.array_equal(mid["idx"][0, h].cpu().numpy(), res["idx"]), "lists"
                assert_close(_np(o[0, h]), want, "attention")
                break
            except AssertionError as e:
                failures.append(f"tiling {c}: {e}")
        else:
            raise AssertionError(f"head {h}: " + "; ".join(failures))
    # tiled mode: no permuted copies, the same bits
    ot = vsa.spade_attention(q, k, v, grid, tiles, topk=3, out_dtype=torch.float32, compensate=True, tiled=True)
    oe = vsa.spade_attention(q, k, v, grid, tiles, topk=3, out_dtype=torch.float32, compensate=True, tiled=False)
    assert torch.equal(ot, oe) and torch.equal(ot, o)


@pytest.mark.parametrize("D,grid,cap", [(128, (8, 16, 32), 5), (64, (16, 16, 16), 1), (128, (8, 24, 32), 1)])
def test_compensated_tiled_equals_permuted_path(D, grid, cap):
    """T-major q, k, v through each head's tiling give unpermute of the
    permuted path's result bit for bit, in both output dtypes, with lists of
    several blocks (two-tile kernel) or of one (one-key-block kernel)."""
    tiles = [(1, 8, 16), (2, 8, 8), (4, 4, 8)]
    B, H = 2, 2
    S = grid[0] * grid[1] * grid[2]
    nb = S // BLOCK
    q, k, v = smooth_qkv(B, H, grid, D, seed=S + cap, device=DEV)
    choice = torch.tensor([2, 0, 1, 2], dtype=torch.int32, device=DEV)
    if cap == 1:
        idx = np.tile(np.arange(nb, dtype=np.int32)[None, None, :, None], (B, H, 1, 1))
        cnt = np.ones((B, H, nb), np.int32)
    else:
        idx_h, cnt_h = _lists(nb, cap, B * H, seed=S, keep_forced_only={nb // 3})
        idx, cnt = idx_h.reshape(B, H, nb, cap), cnt_h.reshape(B, H, nb)
    ti, tc = torch.tensor(idx, device=DEV), torch.tensor(cnt, device=DEV)
    for odt in (torch.float32, torch.bfloat16):
        ot = vsa.centroid_compensated_attention_tiled(q, k, v, grid, tiles, choice, ti, tc, out_dtype=odt)
        qp, kp, vp = (vsa.permute(x, grid, tiles, choice) for x in (q, k, v))
        op = vsa.centroid_compensated_attention(qp, kp, vp, ti, tc, out_dtype=odt)
        vsa.device_status()
        assert torch.equal(ot, vsa.unpermute(op, grid, tiles, choice)), odt


def test_compensated_tiled_bad_choice_sets_runtime_status():
    grid, tiles, D = (8, 16, 16), [(1, 8, 16), (2, 8, 8)], 64
    S, nb = 2048, 16
    q, k, v = smooth_qkv(1, 2, grid, D, seed=8, device=DEV)
    idx = torch.arange(nb, dtype=torch.int32, device=DEV).view(nb, 1).contiguous()
    cnt = torch.ones(nb, dtype=torch.int32, device=DEV)
    o = vsa.centroid_compensated_attention_tiled(q, k, v, grid, tiles, torch.tensor([1, 5], dtype=torch.int32,
                                                                                    device=DEV), idx, cnt,
                                                 out_dtype=torch.float32)
    with pytest.raises(RuntimeError):
        vsa.device_status()
    good = vsa.centroid_compensated_attention_tiled(q[:, :1], k[:, :1], v[:, :1], grid, tiles,
                                                    torch.tensor([1], dtype=torch.int32, device=DEV), idx, cnt,
                                                    out_dtype=torch.float32)
    assert torch.equal(o[:, :1], good)
