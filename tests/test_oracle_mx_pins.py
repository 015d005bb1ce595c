"""Pins of the MXFP4 part of the CPU oracle against facts outside it.

MXFP4 on the pages (imp docs/quantization.md, MXFP4 paragraph): the NVFP4
nibble layout, one UE8M0 micro-scale per 32 elements, no tensor scale,
round-to-nearest quantization.  The checks use library casts (ml_dtypes
UE8M0 and E2M1), closed forms of the scale rule, exact round trips and a
numpy fp64 matrix product; none compares the oracle with itself.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import workloads

F4 = ml_dtypes.float4_e2m1fn
E8 = ml_dtypes.float8_e8m0fnu


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)


def _codes(q: np.ndarray) -> np.ndarray:
    """[N, K/2] packed bytes -> [N, K] codes, element k in the low nibble for even k."""
    out = np.empty((q.shape[0], q.shape[1] * 2), np.uint8)
    out[:, 0::2] = q & 15
    out[:, 1::2] = q >> 4
    return out


def test_e8m0_decode_all_bytes_matches_library():
    lib = np.arange(256, dtype=np.uint8).view(E8).astype(np.float64)
    for b in range(256):
        got = oracle.e8m0_decode(b)
        if b == 255:
            assert math.isnan(got) and math.isnan(lib[b])
        else:
            assert got == lib[b] == 2.0 ** (b - 127)


def _blocks(seed: int, rows: int, K: int) -> np.ndarray:
    """Rows of 32-blocks at magnitudes from BF16 subnormals to 2^100, with
    zeros, negative zeros and exact ties sprinkled in."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((rows, K)).astype(np.float32)
    mags = 2.0 ** rng.integers(-130, 100, size=(rows, K // 32, 1))
    w = (w.reshape(rows, K // 32, 32) * mags).reshape(rows, K)
    w[0, :32] = 0.0                                        # all-zero block
    w[0, 32:64] = -0.0                                     # all negative zeros
    w[1, :32] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 4.0] * 4, np.float32)  # ties at X = 1
    w[1, 5] = -w[1, 5]
    return w


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_mx_codes_are_library_rne_of_w_over_scale(seed):
    """Every code is the ml_dtypes E2M1 cast (round to nearest even,
    saturating, sign kept) of w / 2^(b - 127) with the block's scale byte b."""
    K = 256
    wb = _bf16(_blocks(seed, 24, K))
    q, s = oracle.mx_quantize(wb)
    w = wb.float().numpy().astype(np.float64)
    scale = np.repeat(2.0 ** (s.astype(np.float64) - 127), 32, axis=1)
    lib_codes = (w / scale).astype(np.float32).astype(F4).view(np.uint8) & 15
    assert np.array_equal(_codes(q), lib_codes)


@pytest.mark.parametrize("seed", [3, 4])
def test_mx_scale_closed_form(seed):
    """The block scale X = 2^(b-127) puts the block max in [4, 8): 4X <= amax < 8X,
    unless amax < 2^-125 (byte clamped to 0) or the block is zero (byte 0)."""
    K = 512
    wb = _bf16(_blocks(seed, 16, K))
    _, s = oracle.mx_quantize(wb)
    amax = np.abs(wb.float().numpy().astype(np.float64)).reshape(16, K // 32, 32).max(axis=2)
    X = 2.0 ** (s.astype(np.float64) - 127)
    small = amax < 2.0 ** -125
    assert np.all(s[small] == 0)
    big = ~small
    assert np.all(4 * X[big] <= amax[big]) and np.all(amax[big] < 8 * X[big])
    assert s[0, 0] == 0 and s[0, 1] == 0


def test_mx_zero_blocks_keep_sign():
    wb = _bf16(_blocks(5, 4, 64))
    q, _ = oracle.mx_quantize(wb)
    c = _codes(q)
    assert np.all(c[0, :32] == 0) and np.all(c[0, 32:64] == 8)


def test_mx_round_trip_exact():
    """Blocks built from E2M1 values times a power of two whose largest
    magnitude is 4 or 6 times it come back exactly."""
    rng = np.random.default_rng(7)
    vals = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    N, K = 8, 128
    w = np.empty((N, K))
    for n in range(N):
        for b in range(K // 32):
            e = int(rng.integers(-20, 20))
            blk = rng.choice(vals, 32) * rng.choice([-1.0, 1.0], 32)
            blk[int(rng.integers(0, 32))] = rng.choice([4.0, 6.0])
            w[n, 32 * b:32 * b + 32] = blk * 2.0 ** e
    wb = _bf16(w)
    q, s = oracle.mx_quantize(wb)
    assert np.array_equal(oracle.mx_dequantize(q, s), w)


def test_mx_dequantize_matches_library_decode():
    rng = np.random.default_rng(9)
    q = rng.integers(0, 256, (5, 64), dtype=np.uint8)
    s = rng.integers(100, 150, (5, 4), dtype=np.uint8)
    ref = _codes(q).view(F4).astype(np.float64) * np.repeat(s.view(E8).astype(np.float64), 32, axis=1)
    assert np.array_equal(oracle.mx_dequantize(q, s), ref)


@pytest.mark.parametrize("M,N,K", [(1, 7, 64), (3, 5, 256)])
def test_mx_linear_is_matmul_of_dequantized(M, N, K):
    """y = x . W_deq^T and bound = |x| . |W_deq|^T, against numpy fp64 products
    (exact here: every partial sum is a short sum of exact products)."""
    rng = np.random.default_rng(M * 100 + N)
    q = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    s = rng.integers(120, 134, (N, K // 32), dtype=np.uint8)
    x = workloads.random_bf16((M, K), 11)
    xf = x.float().numpy().astype(np.float64)
    wd = oracle.mx_dequantize(q, s)
    y, bound = oracle.mx_linear(x, q, s)
    np.testing.assert_allclose(y, xf @ wd.T, rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(bound, np.abs(xf) @ np.abs(wd).T, rtol=1e-12, atol=1e-300)
    ys, bs = oracle.mx_linear(x, q, s, rows=[M - 1, 0], cols=[0, N - 1])
    assert ys[0] == y[M - 1, 0] and ys[1] == y[0, N - 1] and bs[1] == bound[0, N - 1]


def test_mx_quantization_error_bound():
    """Unsaturated elements are within half an E2M1 step of w / X (at most X
    in absolute terms: the step is 2 between 4 and 6); saturated ones (w / X
    in (6, 8)) are off by less than 2X."""
    wb = _bf16(_blocks(12, 16, 256))
    q, s = oracle.mx_quantize(wb)
    w = wb.float().numpy().astype(np.float64)
    X = np.repeat(2.0 ** (s.astype(np.float64) - 127), 32, axis=1)
    err = np.abs(w - oracle.mx_dequantize(q, s))
    sat = np.abs(w) / X > 6
    assert np.all(err[~sat] <= X[~sat]) and np.all(err[sat] < 2 * X[sat])
