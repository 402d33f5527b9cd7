"""The allocation-free tiling choice, checked against the workspace variant.

Some callers cannot allocate device memory where they choose tilings: code
running inside an allocator or a memory pool, a process whose device memory is
already reserved by another framework, or a plugin that is handed inputs and
outputs but no allocator and no workspace.  vsa_select_tiling_noalloc serves
them with a fixed scratch array inside the library.  Called twice in a row on
different inputs (the second call reuses the array the first one left behind),
it must give the same choices as vsa_select_tiling with a caller workspace and
the same cohesion values within the tolerance the other tiling tests use.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""

import ctypes

import pytest
import torch

import block_sparse_self_b200 as vsa
from block_sparse_self_b200 import Dims3
from workloads import smooth_qkv

pytestmark = pytest.mark.gpu

TILES = [(1, 8, 16), (2, 8, 8), (4, 4, 8)]


def _noalloc(q, grid, tiles):
    """Call the C ABI directly; only the outputs are allocated, by the test."""
    B, H, S, D = q.shape
    arr = (Dims3 * len(tiles))(*[Dims3(*t) for t in tiles])
    choice = torch.full((B * H,), -7, dtype=torch.int32, device=q.device)
    sics = torch.full((B * H, len(tiles)), float("nan"), dtype=torch.float32, device=q.device)
    code = vsa.BF16 if q.dtype == torch.bfloat16 else vsa.F32
    st = vsa.lib().vsa_select_tiling_noalloc(
        ctypes.c_void_p(q.data_ptr()), code, B, H, S, D, Dims3(*grid), arr, len(tiles),
        ctypes.c_void_p(choice.data_ptr()), ctypes.c_void_p(sics.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == vsa.OK, vsa.last_error()
    return choice, sics


def test_noalloc_matches_the_workspace_variant_on_two_calls_in_a_row():
    cases = [((8, 16, 32), 1, 6, 128, torch.bfloat16, 17),
             ((4, 16, 16), 2, 3, 64, torch.float32, 18)]
    for grid, B, H, D, dtype, seed in cases:
        kinds = ["spatial", "temporal", "generic"] * (B * H // 3 + 1)
        q, _, _ = smooth_qkv(B, H, grid, D, seed=seed, kinds=kinds[:B * H], dtype=dtype, device="cuda")
        want_c, want_s = vsa.select_tiling(q, grid, TILES, return_sics=True)
        got_c, got_s = _noalloc(q, grid, TILES)
        torch.cuda.synchronize()
        assert torch.equal(got_c, want_c)
        torch.testing.assert_close(got_s, want_s, atol=2e-5, rtol=0)
    vsa.device_status()


def test_noalloc_rejects_requests_larger_than_its_scratch():
    """256 heads x 240 regions x 3 candidates x 8 bytes (a SICS sum and a tile
    count each) is 1.47 MB, above the 1 MiB array: the call must refuse before
    launching anything (the fake pointers are never read).  The shape is valid
    for every other check, and the workspace variant would accept it."""
    arr = (Dims3 * 3)(*[Dims3(*t) for t in TILES])
    grid = Dims3(32, 48, 80)
    need = vsa.lib().vsa_select_tiling_workspace_size(1, 256, grid, arr, 3)
    assert need > 1 << 20
    fake = ctypes.c_void_p(1 << 20)
    st = vsa.lib().vsa_select_tiling_noalloc(fake, vsa.BF16, 1, 256, 122880, 64, grid, arr, 3, fake, None, None)
    assert st == vsa.ERR_INVALID_ARGUMENT
    assert "at most" in vsa.last_error()
