"""The C ABI without a GPU: libvsa.so loads, exports every function that
include/vsa.h declares, and rejects invalid arguments on the host before any
launch (the pages raise ValueError for these: "ADR-0001", Conventions;
windowed_attention's and _validate_qkv's checks)."""

import ctypes

import pytest

import block_sparse_self_b200 as vsa
from block_sparse_self_b200 import Dims3

FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced
NULL = ctypes.c_void_p(0)
MIS = ctypes.c_void_p(0x10004)       # misaligned


@pytest.fixture(scope="module")
def L():
    return vsa.lib()


def test_every_declared_symbol_is_exported(L):
    names = vsa.declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n


def _tiles(*ts):
    arr = (Dims3 * len(ts))(*[Dims3(*t) for t in ts])
    return arr, len(ts)


def test_window_attention_argument_errors(L):
    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=ctypes.c_void_p(0x20000), o=ctypes.c_void_p(0x40000), out=vsa.BF16, B=1, H=2,
                 S=256, D=64, window=64, sink=16, scale=0.0, chunk=0)
        a.update(kw)
        return L.vsa_window_attention(a["q"], a["k"], a["v"], a["o"], a["out"], a["B"], a["H"], a["S"], a["D"],
                                      a["window"], a["sink"], a["scale"], a["chunk"], NULL)
    assert call(window=0) == vsa.ERR_INVALID_ARGUMENT
    assert "window must be >= 1" in vsa.last_error()
    assert call(sink=-1) == vsa.ERR_INVALID_ARGUMENT
    assert call(sink=257) == vsa.ERR_INVALID_ARGUMENT
    assert "cannot exceed sequence length" in vsa.last_error()
    assert call(chunk=-3) == vsa.ERR_INVALID_ARGUMENT
    assert call(S=0) == vsa.ERR_INVALID_ARGUMENT
    assert call(D=0) == vsa.ERR_INVALID_ARGUMENT
    assert call(D=96) == vsa.ERR_UNSUPPORTED
    assert call(q=NULL) == vsa.ERR_INVALID_ARGUMENT
    assert call(k=MIS) == vsa.ERR_INVALID_ARGUMENT
    assert call(out=7) == vsa.ERR_INVALID_ARGUMENT
    assert call(o=FAKE) == vsa.ERR_INVALID_ARGUMENT  # output aliases q
    assert call(scale=float("nan")) == vsa.ERR_INVALID_ARGUMENT


def test_block_sparse_attention_argument_errors(L):
    def call(**kw):
        a = dict(B=1, H=2, S=256, D=64, block=32, cap=4, group=0)
        a.update(kw)
        return L.vsa_block_sparse_attention(FAKE, ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000),
                                            ctypes.c_void_p(0x40000), vsa.F32, a["B"], a["H"], a["S"], a["D"],
                                            a["block"], FAKE, FAKE, a["cap"], 1, a["group"], 0.0, NULL)
    assert call(block=48) == vsa.ERR_INVALID_ARGUMENT
    assert call(S=250) == vsa.ERR_INVALID_ARGUMENT
    assert call(cap=0) == vsa.ERR_INVALID_ARGUMENT
    assert call(group=-1) == vsa.ERR_INVALID_ARGUMENT
    assert call(B=0) == vsa.ERR_INVALID_ARGUMENT


def test_topk_argument_errors(L):
    def call(nb=8, k=2, sink=1, dw=0, cap=4):
        return L.vsa_topk_block_mask(FAKE, 1, 2, nb, k, sink, dw, ctypes.c_void_p(0x20000),
                                     ctypes.c_void_p(0x30000), cap, NULL)
    assert call(k=0) == vsa.ERR_INVALID_ARGUMENT
    assert call(k=9) == vsa.ERR_INVALID_ARGUMENT
    assert call(sink=-1) == vsa.ERR_INVALID_ARGUMENT
    assert call(dw=-2) == vsa.ERR_INVALID_ARGUMENT
    assert call(cap=3) == vsa.ERR_INVALID_ARGUMENT       # needs k + sink + 1 = 4
    assert "cap" in vsa.last_error()
    assert call(nb=0) == vsa.ERR_INVALID_ARGUMENT


def test_permute_and_select_tiling_argument_errors(L):
    arr, n = _tiles((2, 4, 4))
    g = Dims3(4, 8, 8)
    y = ctypes.c_void_p(0x100000)
    assert L.vsa_permute(FAKE, y, vsa.F32, 1, 2, 256, 64, Dims3(4, 8, 4), arr, n, NULL, NULL) == \
        vsa.ERR_INVALID_ARGUMENT  # grid product != S
    bad, nb_ = _tiles((0, 4, 4))
    assert L.vsa_permute(FAKE, y, vsa.F32, 1, 2, 256, 64, g, bad, nb_, NULL, NULL) == vsa.ERR_INVALID_ARGUMENT
    assert "must be positive" in vsa.last_error()
    assert L.vsa_permute(FAKE, FAKE, vsa.F32, 1, 2, 256, 64, g, arr, n, NULL, NULL) == vsa.ERR_INVALID_ARGUMENT
    assert L.vsa_permute(FAKE, y, vsa.F32, 1, 2, 256, 64, g, arr, 0, NULL, NULL) == vsa.ERR_INVALID_ARGUMENT
    # select_tiling: workspace size, then a too-small workspace
    t3, n3 = _tiles((1, 8, 16), (2, 8, 8), (4, 4, 8))
    ws = L.vsa_select_tiling_workspace_size(1, 24, Dims3(32, 48, 80), t3, n3)
    assert ws == 24 * 240 * 2 * 3 * 4   # per region and candidate: a SICS sum and a tile count
    assert L.vsa_select_tiling(FAKE, vsa.BF16, 1, 24, 122880, 128, Dims3(32, 48, 80), t3, n3, FAKE, NULL,
                               y, ws - 256, NULL) == vsa.ERR_INVALID_ARGUMENT
    # an lcm region of too many gcd cells is reported as unsupported
    big, nbig = _tiles((1, 1, 7), (1, 1, 9), (1, 5, 1), (3, 1, 1))
    assert L.vsa_select_tiling(FAKE, vsa.BF16, 1, 1, 3 * 5 * 63, 128, Dims3(3, 5, 63), big, nbig, FAKE, NULL,
                               y, 1 << 20, NULL) == vsa.ERR_UNSUPPORTED


@pytest.mark.parametrize("grid,tiles", [
    ((16, 45, 80), [(1, 8, 16), (2, 8, 8), (4, 4, 8)]),   # the height no candidate divides
    ((21, 45, 80), [(1, 8, 16), (2, 8, 8), (4, 4, 8)]),
    ((32, 48, 80), [(1, 8, 16), (2, 8, 8), (4, 4, 8)]),   # divisible: unchanged
    ((3, 5, 13), [(2, 3, 4), (3, 2, 6)]),
    ((1, 1, 1), [(4, 4, 8)]),
])
def test_padded_grid_matches_oracle(L, grid, tiles):
    import oracle
    assert vsa.padded_grid(grid, tiles) == oracle.padded_grid(grid, tiles)


def test_padded_grid_argument_errors(L):
    out = Dims3()
    arr, n = _tiles((2, 4, 4))
    assert L.vsa_padded_grid(Dims3(0, 8, 8), arr, n, ctypes.byref(out)) == vsa.ERR_INVALID_ARGUMENT
    assert L.vsa_padded_grid(Dims3(4, 8, 8), arr, n, None) == vsa.ERR_INVALID_ARGUMENT
    assert L.vsa_padded_grid(Dims3(4, 8, 8), arr, 9, ctypes.byref(out)) == vsa.ERR_INVALID_ARGUMENT
    big, nbig = _tiles((1, 1, 1 << 15), (1, 1, (1 << 15) - 1))   # lcm above 2^20
    assert L.vsa_padded_grid(Dims3(4, 8, 8), big, nbig, ctypes.byref(out)) == vsa.ERR_INVALID_ARGUMENT
    huge, nh = _tiles((1, 1, 1))
    assert L.vsa_padded_grid(Dims3(2048, 2048, 1024), huge, nh, ctypes.byref(out)) == vsa.ERR_INVALID_ARGUMENT


def test_topp_argument_errors(L):
    idx, cnt = FAKE, ctypes.c_void_p(0x20000)
    ok = dict(B=1, H=1, nb=8, p=0.5, scale=1.0, sink=1, dw=0, cap=8)
    def call(**kw):
        a = dict(ok, **kw)
        return L.vsa_topp_block_mask(FAKE, a["B"], a["H"], a["nb"], a["p"], a["scale"], a["sink"], a["dw"],
                                     idx, cnt, a["cap"], NULL)
    assert call(p=0.0) == vsa.ERR_INVALID_ARGUMENT
    assert call(p=1.5) == vsa.ERR_INVALID_ARGUMENT
    assert call(scale=-1.0) == vsa.ERR_INVALID_ARGUMENT
    assert call(cap=7) == vsa.ERR_INVALID_ARGUMENT     # a list can hold every block
    assert call(sink=9) == vsa.ERR_INVALID_ARGUMENT
    assert call(dw=-2) == vsa.ERR_INVALID_ARGUMENT
    assert call(nb=2000, cap=2000) == vsa.ERR_UNSUPPORTED


def test_structured_list_argument_errors(L):
    g = ctypes.c_int(0)
    grid = Dims3(32, 48, 80)
    idx, cnt = FAKE, ctypes.c_void_p(0x20000)
    # sliding tile whose volume is neither a multiple nor a divisor of the block
    assert L.vsa_structured_block_list(vsa.MASK_SLIDING_TILE, grid, Dims3(2, 3, 4), Dims3(1, 1, 1), 128, idx, cnt,
                                       960, ctypes.byref(g), NULL) == vsa.ERR_UNSUPPORTED
    assert L.vsa_structured_block_list(vsa.MASK_SLIDING_TILE, grid, Dims3(4, 8, 8), Dims3(1, 1, 1), 128, idx, cnt,
                                       50, ctypes.byref(g), NULL) == vsa.ERR_INVALID_ARGUMENT  # longest list is 54
    assert L.vsa_structured_block_list(7, grid, Dims3(4, 8, 8), Dims3(1, 1, 1), 128, idx, cnt, 960,
                                       ctypes.byref(g), NULL) == vsa.ERR_INVALID_ARGUMENT
    # the centred window holds the same 54 blocks for every query
    assert L.vsa_structured_block_list(vsa.MASK_SLIDING_TILE_CENTERED, grid, Dims3(4, 8, 8), Dims3(1, 1, 1), 128,
                                       idx, cnt, 53, ctypes.byref(g), NULL) == vsa.ERR_INVALID_ARGUMENT
    assert L.vsa_structured_block_list(vsa.MASK_SLIDING_TILE_CENTERED, grid, Dims3(2, 3, 4), Dims3(1, 1, 1), 128,
                                       idx, cnt, 960, ctypes.byref(g), NULL) == vsa.ERR_UNSUPPORTED
    assert L.vsa_structured_block_list(vsa.MASK_SLIDING_TILE_CENTERED, grid, Dims3(4, 8, 8), Dims3(-1, 1, 1), 128,
                                       idx, cnt, 960, ctypes.byref(g), NULL) == vsa.ERR_INVALID_ARGUMENT


def test_head_profile_argument_errors(L):
    ws = ctypes.c_void_p(0x20000)
    need = L.vsa_head_profile_workspace_size(1, 2, 512, 64)
    assert need > 0 and L.vsa_head_profile_workspace_size(1, 2, 512, 96) == 0

    def call(S=512, D=64, grid=Dims3(4, 8, 16), R=128, wsb=need, scale=0.0, rule=0):
        return L.vsa_head_profile(FAKE, FAKE, 1, 2, S, D, grid, FAKE, R, scale, rule, FAKE, FAKE, ws, wsb, NULL)

    assert call(R=0) == vsa.ERR_INVALID_ARGUMENT
    assert call(R=129) == vsa.ERR_INVALID_ARGUMENT
    assert call(D=96) == vsa.ERR_UNSUPPORTED
    assert call(grid=Dims3(4, 8, 8)) == vsa.ERR_INVALID_ARGUMENT
    assert call(wsb=need - 1) == vsa.ERR_INVALID_ARGUMENT
    assert call(scale=float("nan")) == vsa.ERR_INVALID_ARGUMENT
    assert call(rule=2) == vsa.ERR_INVALID_ARGUMENT
    assert call(S=1 << 30, grid=Dims3(1 << 10, 1 << 10, 1 << 10)) == vsa.ERR_INVALID_ARGUMENT


def test_python_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 128, 64)
    with pytest.raises(ValueError):
        vsa.window_attention(q, q, q, window=8)
    with pytest.raises(ValueError):
        vsa.permute(q, (2, 8, 8), [(1, 8, 8)])


def test_missing_library_fails_loudly():
    """No CPU fallback: without libvsa.so every call raises (run in a child
    process so this process keeps its loaded library)."""
    import os
    import subprocess
    import sys
    code = ("import block_sparse_self_b200 as v, torch\n"
            "v.LIB_PATH = '/nonexistent/libvsa.so'\n"
            "v._lib = None\n"
            "try:\n"
            "    v.lib()\n"
            "except RuntimeError as e:\n"
            "    print('raised:', e)\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert "raised:" in r.stdout and "missing" in r.stdout


def test_sample_query_rows_is_a_seeded_sorted_distinct_draw():
    import torch
    r = vsa.sample_query_rows(1000, 128, seed=3, device="cpu")
    assert r.dtype == torch.int32 and r.shape == (128,)
    assert torch.all(r[1:] > r[:-1]) and int(r.min()) >= 0 and int(r.max()) < 1000
    assert torch.equal(r, vsa.sample_query_rows(1000, 128, seed=3, device="cpu"))
    assert not torch.equal(r, vsa.sample_query_rows(1000, 128, seed=4, device="cpu"))
    assert vsa.sample_query_rows(50, 50, device="cpu").tolist() == list(range(50))
    with pytest.raises(ValueError):
        vsa.sample_query_rows(1000, 129, device="cpu")
    with pytest.raises(ValueError):
        vsa.sample_query_rows(10, 11, device="cpu")


def test_head_profile_and_centred_kind_reject_bad_host_arguments():
    import torch
    q = torch.zeros(1, 1, 128, 64)
    with pytest.raises(ValueError):   # CPU tensors never reach the library
        vsa.head_profile(q, q, (2, 8, 8))
    with pytest.raises(ValueError):
        vsa.structured_block_list("sliding_tile_centred", (8, 16, 16), 128)   # the kind is spelt "centered"
    assert vsa.structured_tile("sliding_tile_centered", (8, 16, 16), (2, 8, 8)) == (2, 8, 8)


def test_spade_attention_host_argument_errors(L):
    """The host-buffer path refuses bad arguments before creating a stream or
    issuing a copy (the host pointers here are never read)."""
    arr, n = _tiles((1, 8, 16), (2, 8, 8), (4, 4, 8))
    g = Dims3(8, 16, 32)

    def size(**kw):
        a = dict(B=1, H=3, S=4096, D=128, k=4, sink=1, dw=0, out=vsa.BF16, groups=2)
        a.update(kw)
        return L.vsa_spade_attention_host_workspace_size(a["B"], a["H"], a["S"], a["D"], g, arr, n, a["k"],
                                                         a["sink"], a["dw"], a["out"], a["groups"])

    need = size()
    assert need > 3 * 2 * 2 * 4096 * 128 * 2   # two slots of q, k, v and the output slots
    assert size(groups=0) == 0 and size(k=33) == 0 and size(k=0) == 0

    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, out=vsa.BF16, B=1, H=3, S=4096, D=128, topk=4, sink=1, dw=0,
                 scale=0.0, groups=2, ws=ctypes.c_void_p(1 << 20), wsb=need)
        a.update(kw)
        return L.vsa_spade_attention_host(a["q"], a["k"], a["v"], a["o"], a["out"], a["B"], a["H"], a["S"], a["D"],
                                          g, arr, n, a["topk"], a["sink"], a["dw"], a["scale"], a["groups"], a["ws"],
                                          a["wsb"], NULL)
    assert call(q=NULL) == vsa.ERR_INVALID_ARGUMENT
    assert call(out=5) == vsa.ERR_INVALID_ARGUMENT
    assert call(topk=33) == vsa.ERR_INVALID_ARGUMENT
    assert "k must be in [1, nb]" in vsa.last_error()
    assert call(groups=0) == vsa.ERR_INVALID_ARGUMENT
    assert call(wsb=need - 1) == vsa.ERR_INVALID_ARGUMENT
    assert "needed" in vsa.last_error()
    assert call(ws=ctypes.c_void_p((1 << 20) + 16)) == vsa.ERR_INVALID_ARGUMENT
    assert call(S=4095) == vsa.ERR_INVALID_ARGUMENT
    assert call(sink=-1) == vsa.ERR_INVALID_ARGUMENT
    assert call(dw=-2) == vsa.ERR_INVALID_ARGUMENT
    assert call(scale=float("inf")) == vsa.ERR_INVALID_ARGUMENT
    assert call(D=96, wsb=1 << 40) == vsa.ERR_UNSUPPORTED


def test_compensated_attention_argument_errors(L):
    def call(**kw):
        a = dict(q=FAKE, k=ctypes.c_void_p(0x100000), v=ctypes.c_void_p(0x200000), o=ctypes.c_void_p(0x400000),
                 out=vsa.F32, B=1, H=2, S=512, D=64, block=128, cap=2, per_head=1, scale=0.0,
                 ws=ctypes.c_void_p(1 << 24), wsb=None)
        a.update(kw)
        wsb = a["wsb"] if a["wsb"] is not None else L.vsa_centroid_compensated_attention_workspace_size(
            a["B"], a["H"], max(a["S"], 128), a["D"] if a["D"] in (64, 128) else 64, a["out"] if a["out"] in (0, 1) else 1)
        return L.vsa_centroid_compensated_attention(a["q"], a["k"], a["v"], a["o"], a["out"], a["B"], a["H"], a["S"],
                                                    a["D"], a["block"], FAKE, FAKE, a["cap"], a["per_head"],
                                                    a["scale"], a["ws"], wsb, NULL)
    f32 = L.vsa_centroid_compensated_attention_workspace_size(1, 2, 512, 64, vsa.F32)
    bf = L.vsa_centroid_compensated_attention_workspace_size(1, 2, 512, 64, vsa.BF16)
    assert bf >= f32 + 2 * 512 * 64 * 4          # a bf16 output also holds the kept keys' fp32 output
    assert L.vsa_centroid_compensated_attention_workspace_size(1, 2, 500, 64, vsa.F32) == 0
    assert call(block=64) == vsa.ERR_UNSUPPORTED
    assert call(S=500) == vsa.ERR_INVALID_ARGUMENT
    assert call(cap=0) == vsa.ERR_INVALID_ARGUMENT
    assert call(D=96) == vsa.ERR_UNSUPPORTED
    assert call(wsb=f32 - 1) == vsa.ERR_INVALID_ARGUMENT
    assert "needed" in vsa.last_error()
    assert call(ws=ctypes.c_void_p((1 << 24) + 16)) == vsa.ERR_INVALID_ARGUMENT
    assert call(ws=ctypes.c_void_p(0x400000)) == vsa.ERR_INVALID_ARGUMENT  # workspace over o
    assert call(ws=ctypes.c_void_p(0x100000)) == vsa.ERR_INVALID_ARGUMENT  # workspace over k
    assert call(o=FAKE) == vsa.ERR_INVALID_ARGUMENT                        # o over q


def test_compensated_tiled_argument_errors(L):
    q, k, v, o = (ctypes.c_void_p(0x100000 * (i + 1)) for i in range(4))
    idx, cnt = ctypes.c_void_p(0x800000), ctypes.c_void_p(0x900000)
    ws = ctypes.c_void_p(0x10000000)
    big = 1 << 34

    def call(grid=Dims3(8, 16, 16), tiles=((1, 8, 16), (2, 8, 8)), S=2048, D=64, cap=2, wsz=big, w=ws):
        arr, n = _tiles(*tiles)
        return L.vsa_centroid_compensated_attention_tiled(q, k, v, o, vsa.F32, 1, 1, S, D, grid, arr, n, None,
                                                          idx, cnt, cap, 0, 0.0, w, wsz, None)

    assert call(grid=Dims3(5, 12, 20), S=1200) == vsa.ERR_UNSUPPORTED            # padded grid
    assert call(tiles=((1, 4, 16), (2, 4, 8))) == vsa.ERR_UNSUPPORTED            # 64-token tiles
    assert call(tiles=((1, 8, 16), (1, 8, 8))) == vsa.ERR_INVALID_ARGUMENT       # volumes differ
    assert call(S=2000) == vsa.ERR_INVALID_ARGUMENT                              # grid product != S
    assert call(cap=0) == vsa.ERR_INVALID_ARGUMENT
    assert call(wsz=16) == vsa.ERR_INVALID_ARGUMENT                              # workspace too small
    assert call(w=ctypes.c_void_p(0x100000 * 2)) == vsa.ERR_INVALID_ARGUMENT     # workspace over k


def test_fused_scores_topk_argument_errors(L):
    def call(**kw):
        a = dict(dt=vsa.BF16, B=1, H=2, nb=240, D=128, k=24, sink=1, dw=0, cap=26)
        a.update(kw)
        return L.vsa_block_scores_topk(FAKE, FAKE, FAKE, FAKE, a["dt"], a["B"], a["H"], a["nb"], a["D"], a["k"],
                                       a["sink"], a["dw"], FAKE, FAKE, a["cap"], NULL)
    assert call(k=0) == vsa.ERR_INVALID_ARGUMENT
    assert call(k=241) == vsa.ERR_INVALID_ARGUMENT
    assert call(cap=25) == vsa.ERR_INVALID_ARGUMENT
    assert call(sink=-1) == vsa.ERR_INVALID_ARGUMENT
    assert call(dw=-2) == vsa.ERR_INVALID_ARGUMENT
    assert call(dt=vsa.F32) == vsa.ERR_UNSUPPORTED
    assert call(nb=1025, k=100, cap=102) == vsa.ERR_UNSUPPORTED
    assert "at most 1024" in vsa.last_error()
    assert call(D=96) == vsa.ERR_UNSUPPORTED


def test_header_is_plain_c(tmp_path):
    """include/vsa.h is a C header: it compiles as C99 and as C++17 on its own,
    with no CUDA or torch types in the signatures."""
    import os
    import shutil
    import subprocess
    header = os.path.abspath(vsa.HEADER_PATH)
    src = tmp_path / "use.c"
    src.write_text('#include "%s"\nint main(void) { return vsa_last_error() == 0; }\n' % header)
    for compiler, std in (("gcc", "-std=c99"), ("g++", "-std=c++17")):
        if shutil.which(compiler) is None:
            pytest.skip(f"{compiler} not found")
        lang = ["-x", "c++"] if compiler == "g++" else []
        r = subprocess.run([compiler, std, "-Wall", "-Werror", "-fsyntax-only", *lang, str(src)],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
