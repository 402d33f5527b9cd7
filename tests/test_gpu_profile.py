"""Head profile on the GPU against the fp64 oracle: per-(b, head) attention
mass on the spatial (same frame) and temporal (same (h, w)) patterns over
sampled query rows, and the kind that follows from them."""

import numpy as np
import pytest
import torch

import block_sparse_self_b200 as vsa
import oracle
from workloads import WORKLOADS, make_qkv, smooth_qkv

pytestmark = pytest.mark.gpu

DEV = "cuda"
# fp32 softmax sums over bf16 x bf16 products (exact) accumulated in fp32
MASS_TOL = 1e-4


@pytest.fixture(autouse=True)
def _no_device_errors():
    yield
    vsa.device_status()


def _np(t):
    return t.detach().float().cpu().numpy()


def _check_against_oracle(q, k, grid, rows, kind, masses, heads=None, scale=None, rule="mass"):
    """Masses within MASS_TOL of the oracle's; the kind equal to the oracle's
    wherever the two compared quantities (masses, or masses per key) differ
    by more than the masses' tolerance allows, else consistent with the GPU's
    own masses."""
    B, H = q.shape[:2]
    r = rows.cpu().numpy()
    T, Hg, Wg = grid
    w = (1.0, 1.0) if rule == "mass" else (1.0 / (Hg * Wg), 1.0 / T)
    for b in range(B):
        for h in (range(H) if heads is None else heads):
            ok, om = oracle.classify_head(_np(q[b, h]), _np(k[b, h]), grid, r, scale, rule=rule)
            got = masses[b, h].cpu().numpy().astype(np.float64)
            assert np.abs(got - om).max() <= MASS_TOL, (b, h, got, om)
            if abs(om[0] * w[0] - om[1] * w[1]) > 2 * MASS_TOL * max(w):
                assert int(kind[b, h]) == ok, (b, h, got, om, rule)
            else:
                assert int(kind[b, h]) in (0, 1)


@pytest.mark.parametrize("grid,D,R", [
    ((4, 8, 16), 64, 128),     # S = 512: four key tiles, frames of 128 keys
    ((3, 5, 7), 128, 50),      # S = 105: one ragged key tile, R < S
    ((5, 9, 13), 64, 100),     # frames of 117 keys: frame edges inside key tiles
    ((40, 4, 5), 128, 128),    # frames of 20 keys: several temporal keys per 32-key chunk
    ((7, 24, 40), 128, 77),    # S = 6720 over several CTAs per head
])
def test_head_profile_matches_oracle_smooth(grid, D, R):
    kinds = ["spatial", "temporal", "temporal", "spatial"]
    q, k, _ = smooth_qkv(2, 2, grid, D, seed=321, kinds=kinds, device=DEV)
    S = q.shape[2]
    rows = vsa.sample_query_rows(S, R, seed=9, device=DEV)
    for rule in ("mass", "mass_per_key"):
        kind, masses = vsa.head_profile(q, k, grid, rows, rule=rule)
        _check_against_oracle(q, k, grid, rows, kind, masses, rule=rule)


def test_head_profile_one_hot_fields_pick_their_pattern():
    grid = (8, 4, 4)
    T, HW, S, D = 8, 16, 128, 64
    t = torch.arange(S) // HW
    hw = torch.arange(S) % HW
    q = torch.zeros(1, 2, S, D)
    k = torch.zeros(1, 2, S, D)
    q[0, 0, torch.arange(S), t] = 3.0    # head 0: logit 3 within the frame, 0 elsewhere
    k[0, 0, torch.arange(S), t] = 1.0
    q[0, 1, torch.arange(S), 16 + hw] = 3.0  # head 1: logit 3 at the same (h, w), 0 elsewhere
    k[0, 1, torch.arange(S), 16 + hw] = 1.0
    q, k = q.to(DEV, torch.bfloat16), k.to(DEV, torch.bfloat16)
    rows = vsa.sample_query_rows(S, 64, seed=1, device=DEV)
    kind, masses = vsa.head_profile(q, k, grid, rows, scale=1.0)
    assert kind[0].tolist() == [0, 1]
    _check_against_oracle(q, k, grid, rows, kind, masses, scale=1.0)
    # closed forms: weight e = exp(3) inside the pattern, 1 outside
    e = float(np.exp(3.0))
    sp0 = HW * e / (HW * e + S - HW)
    tp1 = T * e / (T * e + S - T)
    assert abs(float(masses[0, 0, 0]) - sp0) < MASS_TOL and abs(float(masses[0, 1, 1]) - tp1) < MASS_TOL
    # per key as well: a frame code is spatial and a position code temporal
    kind2, masses2 = vsa.head_profile(q, k, grid, rows, scale=1.0, rule="mass_per_key")
    assert kind2[0].tolist() == [0, 1] and torch.equal(masses2, masses)
    # a weak position code: spatial by mass (16 keys in a frame against 8
    # frames), temporal per key
    q[0, 1] *= 1.0 / 12.0
    kind, _ = vsa.head_profile(q, k, grid, rows, scale=1.0)
    kind2, masses2 = vsa.head_profile(q, k, grid, rows, scale=1.0, rule="mass_per_key")
    assert int(kind[0, 1]) == 0 and int(kind2[0, 1]) == 1
    _check_against_oracle(q, k, grid, rows, kind2, masses2, scale=1.0, rule="mass_per_key")


def test_head_profile_uniform_attention_gives_pattern_sizes():
    grid = (6, 10, 16)
    S = 960
    q = torch.zeros(1, 3, S, 128, dtype=torch.bfloat16, device=DEV)
    k = torch.randn(1, 3, S, 128, device=DEV).to(torch.bfloat16)
    kind, masses = vsa.head_profile(q, k, grid, n_rows=128, seed=4)
    assert torch.allclose(masses[0, :, 0].cpu(), torch.full((3,), 160 / S), atol=1e-6)
    assert torch.allclose(masses[0, :, 1].cpu(), torch.full((3,), 6 / S), atol=1e-6)
    assert kind.cpu().tolist() == [[0, 0, 0]]


def test_head_profile_fp32_inputs_are_rounded_to_bf16():
    grid = (4, 8, 8)
    q, k, _ = smooth_qkv(1, 2, grid, 64, seed=17, dtype=torch.float32, device=DEV)
    rows = vsa.sample_query_rows(256, 40, seed=2, device=DEV)
    kind, masses = vsa.head_profile(q, k, grid, rows)
    k2, m2 = vsa.head_profile(q.to(torch.bfloat16), k.to(torch.bfloat16), grid, rows)
    assert torch.equal(masses, m2) and torch.equal(kind, k2)


def test_head_profile_full_size_sampled():
    """The adaptive S = 122880 workload (24 heads of spatial- or temporal-
    leaning fields): 4 heads against the oracle on 32 sampled rows."""
    w = WORKLOADS["spade_adaptive_s122880"]
    q, k, _ = make_qkv(w, device=DEV)
    rows = vsa.sample_query_rows(w.S, 32, seed=123, device=DEV)
    kind, masses = vsa.head_profile(q, k, w.grid, rows)
    assert torch.isfinite(masses).all()
    _check_against_oracle(q, k, w.grid, rows, kind, masses, heads=[0, 5, 11, 23])
    kind2, masses2 = vsa.head_profile(q, k, w.grid, rows, rule="mass_per_key")
    assert torch.equal(masses2, masses)
    _check_against_oracle(q, k, w.grid, rows, kind2, masses2, heads=[0, 5, 11, 23], rule="mass_per_key")
    print(f"temporal heads: {int(kind.sum())} by mass, {int(kind2.sum())} per key, of {w.heads}")


def test_head_profile_bad_row_sets_runtime_status():
    grid = (2, 8, 8)
    q = torch.randn(1, 1, 128, 64, device=DEV).to(torch.bfloat16)
    rows = torch.tensor([0, 5, 128], dtype=torch.int32, device=DEV)  # 128 is past S
    vsa.head_profile(q, q, grid, rows)
    with pytest.raises(RuntimeError):
        vsa.device_status()


def test_head_profile_argument_errors():
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):
        vsa.head_profile(q, q, (2, 8, 9))          # grid does not hold S tokens
    with pytest.raises(ValueError):
        vsa.head_profile(q, q, (2, 8, 8), rows=torch.zeros(129, dtype=torch.int32, device=DEV))
    with pytest.raises(ValueError):
        vsa.head_profile(q, q[..., :32].contiguous(), (2, 8, 8))
