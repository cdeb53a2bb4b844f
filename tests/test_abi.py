"""The C ABI library builds for sm_100a, loads, exports every function the public
header declares, and rejects invalid arguments on the host before touching the
GPU (these checks run without a GPU: they fail before any CUDA call)."""
import ctypes

import pytest

import moe_expert_gemm_mxfp4_b200 as mx
from moe_expert_gemm_mxfp4_b200 import _lib
from moe_expert_gemm_mxfp4_b200 import build as mxbuild


@pytest.fixture(scope="module")
def lib():
    mxbuild.build()
    return _lib.load()


def test_header_declares_the_api():
    names = _lib.header_symbols()
    for n in ("mxfp4_quantize", "mxfp4_dequantize", "mxfp4_gemm", "moe_mxfp4_mlp",
              "moe_mxfp4_route", "mxfp4_get_device_status"):
        assert n in names


def test_library_exports_every_header_symbol(lib):
    for name in _lib.header_symbols():
        assert hasattr(lib, name), f"{name} declared in include/mxfp4.h but not exported"
        assert name in _lib._SIGS, f"{name} has no ctypes signature in the binding"


def test_status_strings(lib):
    for code in range(8):
        assert lib.mxfp4_status_string(code).startswith(b"MXFP4_")


A = ctypes.c_void_p(0x10000)      # aligned fake device pointer (never dereferenced)
U = ctypes.c_void_p(0x10001)      # misaligned fake pointer
N = ctypes.c_void_p(0)


def test_quantize_argument_checks(lib):
    q = lib.mxfp4_quantize
    assert q(N, 0, 4, 64, A, A, 0, N) == _lib.ERR_INVALID_ARG
    assert q(A, 0, 0, 64, A, A, 0, N) == _lib.ERR_INVALID_ARG
    assert q(A, 0, 4, -32, A, A, 0, N) == _lib.ERR_INVALID_ARG
    assert q(A, 7, 4, 64, A, A, 0, N) == _lib.ERR_INVALID_ARG
    assert q(A, 0, 4, 64, A, A, 9, N) == _lib.ERR_INVALID_ARG
    assert q(A, 0, 4, 48, A, A, 0, N) == _lib.ERR_UNSUPPORTED_SHAPE
    assert q(U, 0, 4, 64, A, A, 0, N) == _lib.ERR_MISALIGNED
    assert lib.mxfp4_dequantize(A, N, 4, 64, A, N) == _lib.ERR_INVALID_ARG
    assert lib.mxfp4_dequantize(A, A, 4, 40, A, N) == _lib.ERR_UNSUPPORTED_SHAPE
    assert lib.mxfp4_dequantize(A, A, 4, 64, U, N) == _lib.ERR_MISALIGNED


def test_gemm_argument_checks(lib):
    g = lib.mxfp4_gemm
    assert g(A, 8, 256, A, A, 512, N, 0, N, 0, N) == _lib.ERR_INVALID_ARG
    assert g(A, 0, 256, A, A, 512, A, 0, N, 0, N) == _lib.ERR_INVALID_ARG
    assert g(A, 8, 256, A, A, 512, A, 5, N, 0, N) == _lib.ERR_INVALID_ARG
    assert g(A, 8, 96, A, A, 512, A, 0, N, 0, N) == _lib.ERR_UNSUPPORTED_SHAPE
    # the largest K is 7680 (the tile's block scales are staged whole in shared memory)
    assert g(A, 8, 7680 + 64, A, A, 512, A, 0, N, 0, N) == _lib.ERR_UNSUPPORTED_SHAPE
    assert g(A, 8, 256, U, A, 512, A, 0, N, 0, N) == _lib.ERR_MISALIGNED
    assert g(A, 8, 256, A, A, 512, A, 1, N, 0, N) == _lib.ERR_WORKSPACE   # W4A4 needs ws
    assert lib.mxfp4_gemm_workspace_size(8, 256, 512, 0) == 0
    # W4A4: x as MXFP4 codes + block scales (+16 readable bytes past the scales)
    assert lib.mxfp4_gemm_workspace_size(8, 256, 512, 1) >= 8 * 256 // 2 + 8 * 256 // 32 + 16


# Switch points of the W4A16 token-tiling rule: least tile cost x tiles (costs 1.0, 1.0,
# 1.04, 1.14, 1.43 for 16- to 192-row tiles) for a group one standard deviation (the
# square root of the mean) above the mean rows per group.
W4A16_TILES = [(1, 16), (12, 16), (13, 32), (26, 32), (27, 64), (56, 64), (57, 128),
               (117, 128), (118, 192), (178, 192), (179, 128), (240, 128), (241, 192),
               (552, 192), (553, 128), (615, 128), (616, 192), (1024, 192)]


@pytest.mark.parametrize("avg,nt", W4A16_TILES)
def test_w4a16_token_tiles(lib, avg, nt):
    assert lib.mxfp4_token_tile_rows(avg, 1, 0) == nt
    # the mean is rows / groups, rounded up
    assert lib.mxfp4_token_tile_rows(avg * 32 - 31, 32, 0) == nt
    assert mx.mxfp4_token_tile_rows(avg * 32, 32) == nt


def test_token_tile_rule_between_switch_points(lib):
    """Between two listed switch points the choice does not change, and a brute-force
    restatement of the rule agrees at every mean up to 2048."""
    import math
    cost = {16: 1.0, 32: 1.0, 64: 1.04, 128: 1.14, 192: 1.43}
    for avg in range(1, 2049):
        hi = avg + math.sqrt(avg)
        want = min(cost, key=lambda n: (cost[n] * math.ceil(hi / n), n))
        assert lib.mxfp4_token_tile_rows(avg, 1, 0) == want, avg


def test_w4a4_token_tiles_and_invalid_queries(lib):
    for avg, nt in [(1, 16), (16, 16), (17, 32), (32, 32), (33, 64), (64, 64), (65, 128), (4096, 128)]:
        assert lib.mxfp4_token_tile_rows(avg, 1, 1) == nt
    assert lib.mxfp4_token_tile_rows(0, 1, 0) == 0
    assert lib.mxfp4_token_tile_rows(8, 0, 0) == 0
    assert lib.mxfp4_token_tile_rows(8, 1, 7) == 0
    assert lib.mxfp4_token_tile_rows(1 << 62, 1, 0) == 0          # no overflow in the mean
    assert lib.mxfp4_token_tile_rows((1 << 62) - 1, 1 << 40, 0) == 192


def test_route_and_moe_argument_checks(lib):
    r = lib.moe_mxfp4_route
    assert r(A, 64, 32, 0, A, A, A, A, A, A, A, 1 << 20, N) == _lib.ERR_INVALID_ARG
    assert r(A, 64, 32, 9, A, A, A, A, A, A, A, 1 << 20, N) == _lib.ERR_UNSUPPORTED_SHAPE
    assert r(A, 64, 300, 4, A, A, A, A, A, A, A, 1 << 20, N) == _lib.ERR_UNSUPPORTED_SHAPE
    assert r(A, 64, 3, 4, A, A, A, A, A, A, A, 1 << 20, N) == _lib.ERR_UNSUPPORTED_SHAPE
    assert r(A, 64, 32, 4, A, A, A, A, A, A, N, 0, N) == _lib.ERR_WORKSPACE
    m = lib.moe_mxfp4_mlp
    big = 1 << 40
    assert m(A, 64, 2880, A, 32, 4, A, A, 2880, A, A, A, 0, N, 0, N) == _lib.ERR_WORKSPACE
    assert m(A, 64, 2880 + 32, A, 32, 4, A, A, 2880, A, A, A, 0, A, big, N) == _lib.ERR_UNSUPPORTED_SHAPE
    assert m(A, 64, 2880, A, 32, 4, A, A, 2880 + 32, A, A, A, 0, A, big, N) == _lib.ERR_UNSUPPORTED_SHAPE
    assert m(A, 64, 2880, A, 32, 4, U, A, 2880, A, A, A, 0, A, big, N) == _lib.ERR_MISALIGNED
    assert m(A, 64, 2880, A, 32, 4, A, A, 2880, A, A, A, 3, A, big, N) == _lib.ERR_INVALID_ARG
    ws = lib.moe_mxfp4_workspace_size(64, 2880, 2880, 32, 4, 0)
    assert ws >= 64 * 4 * (2880 * 2 * 2 + 2880 * 2)


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(_lib, "_LIB", None)
    with pytest.raises(_lib.Mxfp4LibraryMissing):
        _lib.load(str(tmp_path / "nope.so"))


def test_workspace_layout_mirror_matches_the_library():
    # the tests' copy of the workspace carving (used to read h for the W4A4 staged
    # check) must describe the library's workspace exactly
    from helpers import moe_ws_layout
    lib = _lib.load()
    for T, H, I, E, k in ((1, 64, 64, 1, 1), (37, 192, 128, 8, 2), (256, 2880, 2880, 32, 4),
                          (4096, 2880, 2880, 128, 4), (513, 64, 128, 3, 1)):
        for mode in (0, 1):
            assert moe_ws_layout(T, H, I, E, k, mode == 1)["total"] == \
                lib.moe_mxfp4_workspace_size(T, H, I, E, k, mode), (T, H, I, E, k, mode)
