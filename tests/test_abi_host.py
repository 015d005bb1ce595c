"""Host-side checks of the C ABI: the library loads, exports every entry point
include/nvfp4.h declares, and rejects bad arguments before touching a GPU.
No call here reaches a kernel launch (all fail validation first)."""
import ctypes

import pytest

import gemm_decode_nvfp4_b200 as nv

OK, INVALID, SHAPE, ALIGN = 0, 1, 2, 3
A = 1 << 20  # a fake, 16-byte aligned "device address": never dereferenced here


def test_exports_every_declared_symbol():
    names = nv.declared_symbols()
    assert set(names) >= {"nvfp4_amax", "nvfp4_quantize", "nvfp4_gemv", "nvfp4_gemm",
                          "nvfp4_gemm_workspace_size", "nvfp4_last_error", "nvfp4_version",
                          "nvfp4_status_string"}
    raw = ctypes.CDLL(nv.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n


def test_version_and_status_strings():
    assert nv.version() >= 100
    assert nv.lib.nvfp4_status_string(0) == b"NVFP4_OK"
    assert nv.lib.nvfp4_status_string(3) == b"NVFP4_ERR_ALIGNMENT"
    assert nv.lib.nvfp4_status_string(99) == b"NVFP4_ERR_UNKNOWN"


@pytest.mark.parametrize("K", [0, -16, 8, 24, 100])
def test_bad_k_rejected(K):
    assert nv.lib.nvfp4_gemv(A, A, A, A, A + 4096, 16, K, None) == SHAPE
    assert nv.lib.nvfp4_quantize(A, 16, K, 64, A, A, A, A + 64, None) == SHAPE
    assert nv.lib.nvfp4_gemm(A, 64, A, A, A, A, 64, 4, 16, K, None, 0, None) == SHAPE
    assert b"multiple of 16" in nv.lib.nvfp4_last_error()


def test_gemv_validation():
    assert nv.lib.nvfp4_gemv(A, A, A, A, A, -1, 64, None) == SHAPE
    assert nv.lib.nvfp4_gemv(A, A, A, A, A, 0, 64, None) == OK          # no-op, no device needed
    assert nv.lib.nvfp4_gemv(None, A, A, A, A, 4, 64, None) == INVALID
    assert nv.lib.nvfp4_gemv(A + 8, A, A, A, A + 4096, 4, 64, None) == ALIGN
    assert nv.lib.nvfp4_gemv(A, A, A, A + 2, A + 4096, 4, 64, None) == ALIGN
    assert nv.lib.nvfp4_gemv(A, A, A, A, A + 4097, 4, 64, None) == ALIGN
    assert nv.lib.nvfp4_gemv(A, A, A, A, A + 4096, 4, 49152 + 16, None) == SHAPE
    # y overlapping x
    assert nv.lib.nvfp4_gemv(A, A + 8192, A + 16384, A + 32768, A + 16, 4, 64, None) == INVALID


def test_quantize_validation():
    assert nv.lib.nvfp4_quantize(A, 4, 64, 64, None, A + 4096, A + 8192, None, None) == INVALID
    assert nv.lib.nvfp4_quantize(A, 4, 64, 64, A, A + 4096, A + 8192, A, None) == INVALID   # alias
    assert nv.lib.nvfp4_quantize(A, 4, 64, 32, A + 100, A + 4096, A + 8192, None, None) == INVALID  # ldw < K
    assert nv.lib.nvfp4_quantize(A, 4, 64, 68, A + 100, A + 4096, A + 8192, None, None) == ALIGN
    assert nv.lib.nvfp4_quantize(A, -1, 64, 64, A + 100, A + 4096, A + 8192, None, None) == SHAPE
    # q overlapping w
    assert nv.lib.nvfp4_quantize(A, 4, 64, 64, A + 100000, A + 16, A + 8192, None, None) == INVALID


def test_amax_validation():
    assert nv.lib.nvfp4_amax(A, 4, 12, 16, A + 4096, None) == SHAPE
    assert nv.lib.nvfp4_amax(A, 0, 16, 16, None, None) == OK
    assert nv.lib.nvfp4_amax(None, 4, 16, 16, A, None) == INVALID
    assert nv.lib.nvfp4_amax(A + 2, 4, 16, 16, A + 4096, None) == ALIGN


def test_gemm_validation():
    assert nv.lib.nvfp4_gemm(A, 64, A, A, A, A, 64, 0, 64, 64, None, 0, None) == OK
    assert nv.lib.nvfp4_gemm(A, 32, A, A, A, A, 64, 4, 64, 64, None, 0, None) == INVALID  # ldx < K
    assert nv.lib.nvfp4_gemm(A, 68, A, A, A, A + 4096, 64, 4, 64, 64, None, 0, None) == ALIGN   # ldx % 8
    assert nv.lib.nvfp4_gemm(A, 64, A, A, A, A + 4097, 64, 4, 64, 64, None, 0, None) == ALIGN   # odd Y
    assert nv.lib.nvfp4_gemm(A, 64, A, A, A, None, 64, 4, 64, 64, None, 0, None) == INVALID


def test_unknown_flags_rejected():
    assert nv.lib.nvfp4_gemv_ex(A, A, A, A, A + 4096, 4, 64, 0x80, None) == INVALID
    assert nv.lib.nvfp4_gemm_ex(A, 64, A, A, A, A + 4096, 64, 4, 64, 64, None, 0, 0x2, None) == INVALID
    assert nv.lib.nvfp4_gemv_ex(A, A, A, A, A + 4096, 0, 64, 1, None) == OK   # N == 0: no-op


def test_quantize_mse_validation():
    """The micro-scale search entry point checks its window, then the same
    arguments as nvfp4_quantize, before any device work."""
    assert "nvfp4_quantize_mse" in nv.declared_symbols()
    for window in (-1, 126, 1000):
        assert nv.lib.nvfp4_quantize_mse(A, 4, 64, 64, A + 100, window, A + 4096, A + 8192, None, None) == INVALID
    assert nv.lib.nvfp4_quantize_mse(A, 4, 40, 64, A + 100, 8, A + 4096, A + 8192, None, None) == SHAPE
    assert nv.lib.nvfp4_quantize_mse(A, 4, 64, 32, A + 100, 8, A + 4096, A + 8192, None, None) == INVALID
    assert nv.lib.nvfp4_quantize_mse(A, 4, 64, 68, A + 100, 8, A + 4096, A + 8192, None, None) == ALIGN
    assert nv.lib.nvfp4_quantize_mse(A, 4, 64, 64, None, 8, A + 4096, A + 8192, None, None) == INVALID


def test_ksplit_flag_values():
    """NVFP4_FLAG_KSPLIT(c) takes c in {1, 2, 4, 8} on the GEMV entry points
    only; anything else is rejected before any device work."""
    for c in (3, 5, 6, 7, 9, 15):
        assert nv.lib.nvfp4_gemv_ex(A, A, A, A, A + 4096, 4, 1024, c << 8, None) == INVALID
        assert nv.lib.mxfp4_gemv_ex(A, A, A, A + 4096, 4, 1024, c << 8, None) == INVALID
        assert b"KSPLIT" in nv.lib.nvfp4_last_error()
    for c in (0, 1, 2, 4, 8):
        assert nv.lib.nvfp4_gemv_ex(A, A, A, A, A + 4096, 0, 1024, c << 8, None) == OK   # N == 0: no-op
    # the GEMM does not take the GEMV's split flag
    assert nv.lib.nvfp4_gemm_ex(A, 64, A, A, A, A + 4096, 64, 4, 64, 64, None, 0, 2 << 8, None) == INVALID
    with pytest.raises(ValueError):
        nv._ksplit_flag(3)


def test_mxfp4_exports_and_validation():
    names = set(nv.declared_symbols())
    assert {"mxfp4_quantize", "mxfp4_gemv", "mxfp4_gemv_ex"} <= names
    for K in (0, 16, 48, -32):
        assert nv.lib.mxfp4_quantize(A, 4, K, 64, A + 4096, A + 8192, None) == SHAPE
        assert nv.lib.mxfp4_gemv(A, A, A, A + 4096, 4, K, None) == SHAPE
    assert b"multiple of 32" in nv.lib.nvfp4_last_error()
    assert nv.lib.mxfp4_quantize(A, 0, 64, 64, A, A, None) == OK              # no-op
    assert nv.lib.mxfp4_quantize(A, 4, 64, 32, A + 4096, A + 8192, None) == INVALID   # ldw < K
    assert nv.lib.mxfp4_quantize(A, 4, 64, 64, A + 16, A + 8192, None) == INVALID     # q inside w
    assert nv.lib.mxfp4_quantize(A, 4, 64, 64, A + 4096, A + 8200, None) == ALIGN
    assert nv.lib.mxfp4_gemv(A, A, A, A, 0, 64, None) == OK
    assert nv.lib.mxfp4_gemv(None, A, A, A, 4, 64, None) == INVALID
    assert nv.lib.mxfp4_gemv(A + 8, A, A, A + 4096, 4, 64, None) == ALIGN
    assert nv.lib.mxfp4_gemv(A, A + 8192, A + 16384, A + 16, 4, 64, None) == INVALID  # y overlaps x
    assert nv.lib.mxfp4_gemv_ex(A, A, A, A + 4096, 4, 64, 2, None) == INVALID         # unknown flag


def test_grouped_validation():
    assert "nvfp4_gemv_grouped" in nv.declared_symbols()
    f = nv.lib.nvfp4_gemv_grouped
    # X, ldx, q, s, g, experts, tokens, Y, ldy, P, E, T, N, K, flags, stream
    assert f(A, 64, A, A, A, A, A, A, 16, 0, 4, 1, 16, 64, 0, None) == OK           # P == 0: no-op
    assert f(A, 64, A, A, A, A, A, A, 16, -1, 4, 1, 16, 64, 0, None) == SHAPE
    assert f(A, 64, A, A, A, A, A, A, 16, 4, 0, 1, 16, 64, 0, None) == SHAPE        # E == 0
    assert f(A, 64, A, A, A, A, A, A, 16, 70000, 4, 1, 16, 64, 0, None) == SHAPE    # too many problems
    assert f(A, 64, A, A, A, A, A, A, 16, 4, 4, 1, 16, 24, 0, None) == SHAPE        # K % 16
    assert f(A, 64, A, A, A, None, A, A + 8192, 16, 4, 4, 1, 16, 64, 0, None) == INVALID
    assert f(A, 60, A, A, A, A, A, A + 8192, 16, 4, 4, 1, 16, 64, 0, None) == INVALID  # ldx < K
    assert f(A, 68, A, A, A, A, A, A + 8192, 16, 4, 4, 1, 16, 64, 0, None) == ALIGN    # ldx % 8
    assert f(A, 64, A, A, A, A + 2, A, A + 8192, 16, 4, 4, 1, 16, 64, 0, None) == ALIGN
    assert f(A, 64, A + 8192, A + 16384, A + 24576, A + 32768, A + 32800, A, 16, 4, 4, 1, 16, 64, 0, None) == INVALID  # Y over X
    assert f(A, 64, A, A, A, A, A, A + 8192, 16, 4, 4, 1, 16, 64, 4, None) == INVALID  # unknown flag


def test_w4a4_sizes_and_validation():
    L = nv.lib
    assert L.nvfp4_w4a4_weight_scales_bytes(300, 512) == 384 * 32
    assert L.nvfp4_w4a4_x_scales_bytes(300, 512) == 512 * 32
    assert L.nvfp4_w4a4_x_scales_bytes(300, 500) == 0
    assert L.nvfp4_w4a4_workspace_size(300, 512) == 300 * 256 + 512 * 32 + 260 * 4
    assert L.nvfp4_w4a4_weight_scales_bytes(1, 256) == 128 * 16
    # K must be a multiple of 256
    assert L.nvfp4_w4a4_prepare_weights(A, 16, 128, A + 65536, None) == SHAPE
    assert L.nvfp4_w4a4_quantize_x(A, 128, 4, 128, A + 8192, A + 16384, A + 32768, 0, None) == SHAPE
    assert L.nvfp4_w4a4_gemm(A, A, A, A, A, A, A, 16, 4, 16, 128, 0, None) == SHAPE
    # no-ops need no device
    assert L.nvfp4_w4a4_prepare_weights(A, 0, 256, A + 65536, None) == OK
    assert L.nvfp4_w4a4_quantize_x(A, 256, 0, 256, A, A, A, 0, None) == OK
    assert L.nvfp4_w4a4_gemm(A, A, A, A, A, A, A, 16, 0, 16, 256, 0, None) == OK
    # null, alignment, overlap, flags
    assert L.nvfp4_w4a4_prepare_weights(None, 16, 256, A, None) == INVALID
    assert L.nvfp4_w4a4_prepare_weights(A, 16, 256, A + 8, None) == ALIGN
    assert L.nvfp4_w4a4_prepare_weights(A, 16, 256, A + 64, None) == INVALID          # s_mma overlaps s
    assert L.nvfp4_w4a4_quantize_x(A, 256, 4, 256, A + 8192, A + 16384, A + 32768, 4, None) == INVALID
    assert L.nvfp4_w4a4_quantize_x(A, 128, 4, 256, A + 8192, A + 16384, A + 32768, 0, None) == INVALID  # ldx < K
    assert L.nvfp4_w4a4_quantize_x(A, 260, 4, 256, A + 8192, A + 16384, A + 32768, 0, None) == ALIGN
    assert L.nvfp4_w4a4_quantize_x(A, 256, 4, 256, A + 16, A + 16384, A + 32768, 0, None) == INVALID   # qx in X
    assert L.nvfp4_w4a4_quantize_x(A, 256, 4, 256, A + 8192, A + 16384, A + 32770, 0, None) == ALIGN
    assert L.nvfp4_w4a4_gemm(A, A + 4096, A + 8192, A + 16384, A + 32768, A + 65536, A + 131072, 8, 4, 16, 256,
                             0, None) == INVALID                                       # ldy < N
    assert L.nvfp4_w4a4_gemm(A, A + 4096, A + 8192, A + 16384, A + 32768, A + 65536, A + 16, 16, 4, 16, 256,
                             0, None) == INVALID                                       # Y over qx
    assert L.nvfp4_w4a4_gemm(A, A + 4096, A + 8192, A + 16384, A + 32768, A + 65536, A + 131072, 16, 4, 16, 256,
                             8, None) == INVALID                                       # unknown flag
    assert L.nvfp4_w4a4_linear(A, 256, None, A + 16384, A + 32768, A + 65536, A + 131072, 16, 4, 16, 256,
                               None, 0, 0, None) == 6                                  # workspace missing
    assert L.nvfp4_w4a4_linear(A, 256, None, A + 16384, A + 32768, A + 65536, A + 131072, 16, 4, 16, 256,
                               A + 8, 1 << 20, 0, None) == ALIGN


def test_w4a4_binding_constants_match_header():
    import re
    with open(nv.W4A4_HEADER_PATH) as f:
        text = f.read()
    assert int(re.search(r"#define NVFP4_W4A4_AMAX_FLOATS (\d+)", text).group(1)) == nv.AMAX_FLOATS
    assert int(re.search(r"#define NVFP4_W4A4_GIVEN_AMAX (\d+)u", text).group(1)) == nv.GIVEN_AMAX


def test_w4a4_tile_count_bound():
    """2^24 tokens x 2^31 - 128 weight rows is within the per-dimension limits
    but has more 128 x 256 tiles than a 32-bit tile index holds."""
    L = nv.lib
    big_n = (1 << 31) - 128
    assert L.nvfp4_w4a4_gemm(A, A, A, A, A, A, A, big_n, 1 << 24, big_n, 256, 0, None) == SHAPE
    assert b"tiles" in L.nvfp4_last_error()


def test_mxfp4_to_nvfp4_scales_validation():
    L = nv.lib
    assert "mxfp4_to_nvfp4_scales" in nv.declared_symbols()
    for K in (0, 48, -32):
        assert L.mxfp4_to_nvfp4_scales(A, A + 4096, 4, K, A + 8192, A + 12288, None) == SHAPE
    assert L.mxfp4_to_nvfp4_scales(A, A + 4096, 0, 64, A + 8192, A + 12288, None) == OK      # no-op
    assert L.mxfp4_to_nvfp4_scales(None, A + 4096, 4, 64, A + 8192, A + 12288, None) == INVALID
    assert L.mxfp4_to_nvfp4_scales(A, A + 4096, 4, 64, A + 8200, A + 12288, None) == ALIGN   # s_nv
    assert L.mxfp4_to_nvfp4_scales(A, A + 4096, 4, 64, A + 8192, A + 12290, None) == ALIGN   # g_out
    assert L.mxfp4_to_nvfp4_scales(A, A + 4096, 4, 64, A + 64, A + 12288, None) == INVALID   # s_nv in q
    assert L.mxfp4_to_nvfp4_scales(A, A + 4096, 4, 64, A + 8192, A + 4100, None) == INVALID  # g_out in s_mx


def test_w4a4_pair_flag():
    """NVFP4_FLAG_W4A4_PAIR (bit 12) is taken by the W4A4 entry points only;
    the flags are checked before any device work (M == 0 is a no-op)."""
    pair = nv.FLAG_W4A4_PAIR
    assert pair == 1 << 12
    assert nv.lib.nvfp4_w4a4_gemm(A, A, A, A, A, A, A + 4096, 64, 0, 64, 256, pair | 1, None) == OK
    assert nv.lib.nvfp4_w4a4_gemm(A, A, A, A, A, A, A + 4096, 64, 0, 64, 256, 1 << 13, None) == INVALID
    assert nv.lib.nvfp4_w4a4_linear(A, 256, None, A, A, A, A + 4096, 64, 0, 64, 256, A + 8192, 0, pair, None) == OK
    assert nv.lib.nvfp4_gemm_ex(A, 64, A, A, A, A + 4096, 64, 4, 64, 64, None, 0, pair, None) == INVALID
    assert nv.lib.nvfp4_gemv_ex(A, A, A, A, A + 4096, 4, 1024, pair, None) == INVALID
