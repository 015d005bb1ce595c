"""Pins of the MXFP4 -> NVFP4 scale conversion of the oracle: the NVFP4
dequantization of the converted scales equals the MXFP4 dequantization
exactly (both pinned to library decodes), E4M3 codes of powers of two match
the library cast, and out-of-window blocks are counted."""
import ml_dtypes
import numpy as np

import oracle

F8 = ml_dtypes.float8_e4m3fn


def test_pow2_codes_match_library():
    for j in range(-9, 9):
        byte = oracle._e4m3_byte_of_pow2(j)
        assert np.array([byte], np.uint8).view(F8).astype(np.float64)[0] == 2.0 ** j


def _mx(N, K, seed, lo, hi):
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    s = rng.integers(lo, hi + 1, (N, K // 32), dtype=np.uint8)
    return q, s


def test_conversion_is_exact_within_window():
    q, s = _mx(12, 256, 1, 110, 127)               # exponents span 17 binades
    q[0, :16] = 0x88                               # an all-(-0) block: its scale is free
    s[0, 0] = 3
    s_nv, g, bad = oracle.mx_to_nvfp4(q, s)
    assert bad == 0
    np.testing.assert_array_equal(oracle.dequantize(q, s_nv, g), oracle.mx_dequantize(q, s))
    assert s_nv[0, 0] == 0 and s_nv[0, 1] == 0


def test_out_of_window_blocks_are_counted():
    q, s = _mx(6, 128, 2, 120, 130)
    q[3, 16:32] = 0x11                             # make block (3, 1) non-zero
    s[3, 1] = 100                                  # 30 binades below the top
    s_nv, g, bad = oracle.mx_to_nvfp4(q, s)
    assert bad == 1 and s_nv[3, 2] == 0 and s_nv[3, 3] == 0
    assert g == np.float32(2.0 ** (int(s.max()) - 127 - 8))


def test_all_zero_tensor():
    q = np.zeros((3, 64), np.uint8)
    s = np.full((3, 4), 200, np.uint8)
    s_nv, g, bad = oracle.mx_to_nvfp4(q, s)
    assert bad == 0 and g == 1.0 and not s_nv.any()


def test_nan_scale_blocks_are_counted_and_ignored():
    """Scale byte 255 is NaN in UE8M0 (library decode): such blocks, zero codes
    or not, are counted and leave G to the finite blocks."""
    q, s = _mx(4, 128, 3, 118, 124)
    assert np.isnan(np.array([255], np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)[0])
    s[1, 2] = 255
    q[2, 0:16] = 0
    s[2, 0] = 255
    s_nv, g, bad = oracle.mx_to_nvfp4(q, s)
    assert bad == 2 and not s_nv[1, 4:6].any() and not s_nv[2, 0:2].any()
    assert g == np.float32(2.0 ** (int(s[s != 255].max()) - 127 - 8))
