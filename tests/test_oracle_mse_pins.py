"""Pins of the micro-scale search (MSE) quantizer of the oracle
(imp docs/quantization.md, micro-scale search paragraph: each E4M3 micro-scale
chosen by the least reconstruction error over FP8 candidates around the
absmax scale; window, error precision and tie rule are readings).

The checks tie it to facts outside its own code: window 0 reduces it to the
separately pinned round-to-nearest quantizer, a block worked out by hand,
a brute force over the window with library casts (ml_dtypes E4M3 and E2M1)
and plain Python sums, and the defining property (never worse than
round-to-nearest) measured through the pinned dequantizer."""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import workloads

F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)


@pytest.mark.parametrize("seed", [0, 1])
def test_window_zero_is_round_to_nearest(seed):
    w = workloads.random_bf16((12, 512), seed, 0.02)
    q0, s0, g0 = oracle.quantize(w)
    q1, s1, g1 = oracle.quantize_mse(w, window=0)
    assert g0 == g1 and np.array_equal(q0, q1) and np.array_equal(s0, s1)


def test_worked_block():
    """Sixteen values 2.5, g = 1.  Round-to-nearest: 2.5 / 6 = 0.4167 rounds to
    the E4M3 value 0.40625 (0x2D), and 2.5 / 0.40625 = 6.15 rounds to the code
    of 6 (0x7): error 16 * 0.0625^2.  The E4M3 value 0.625 (0x32) is 5 codes
    above 0x2D, inside the window of 8, and 2.5 / 0.625 = 4 exactly (code 0x6):
    error 0, and no other candidate in the window reaches 0 (2.5 / v for the
    other E2M1 values v is not an E4M3 value in range), so it is chosen."""
    w = _bf16(np.full((1, 16), 2.5))
    q, s, _ = oracle.quantize(w, np.float32(1.0))
    assert s[0, 0] == 0x2D and np.all(q == 0x77)
    q, s, _ = oracle.quantize_mse(w, np.float32(1.0))
    assert s[0, 0] == 0x32 and np.all(q == 0x66)
    assert np.array_equal(oracle.dequantize(q, s, np.float32(1.0)), np.full((1, 16), 2.5))


def _library_choice(block, g, window):
    """Brute force with library casts and Python fp64 sums, same readings."""
    f = block.astype(np.float32)
    amax_b = np.float32(np.max(np.abs(f)))
    c0 = int(np.array([(amax_b / np.float32(6.0)) / g], np.float32).astype(F8).view(np.uint8)[0])
    if c0 == 0:
        return 0, np.zeros(16, np.uint8)
    best = None
    for c in range(max(1, c0 - window), min(126, c0 + window) + 1):
        d = np.float32(np.array([c], np.uint8).view(F8).astype(np.float32)[0] * g)
        r = np.float32(np.float32(1.0) / d)
        codes = (f * r).astype(np.float32).astype(F4)
        vals = codes.astype(np.float64)
        err = 0.0
        for i in range(16):
            e = float(f[i]) - float(vals[i]) * float(d)
            err += e * e
        key = (err, abs(c - c0), c)
        if best is None or key < best[0]:
            best = (key, c, codes.view(np.uint8) & 15)
    return best[1], best[2]


@pytest.mark.parametrize("seed", [2, 3, 4])
def test_brute_force_with_library_casts(seed):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((6, 64)).astype(np.float32) * np.float32(0.02)
    w[0, :16] = 0.0
    w[1, 16:32] *= 1e3
    wb = _bf16(w)
    q, s, g = oracle.quantize_mse(wb)
    wf = wb.float().numpy()
    codes = np.empty((6, 64), np.uint8)
    codes[:, 0::2] = q & 15
    codes[:, 1::2] = q >> 4
    for n in range(6):
        for b in range(4):
            blk = wf[n, 16 * b:16 * b + 16]
            c, cc = _library_choice(blk, np.float32(g), 8)
            assert s[n, b] == c, (n, b)
            got = codes[n, 16 * b:16 * b + 16]
            nz = blk != 0
            assert np.array_equal(got[nz], cc[nz]), (n, b)
            if c != 0:  # zeros keep their sign bit
                assert np.array_equal(got[~nz], np.where(np.signbit(blk[~nz]), 8, 0)), (n, b)


def test_never_worse_than_round_to_nearest():
    w = workloads.random_bf16((32, 1024), 5, 0.02)
    q0, s0, g = oracle.quantize(w)
    q1, s1, _ = oracle.quantize_mse(w, g)
    wf = w.float().numpy().astype(np.float64)
    e0 = ((wf - oracle.dequantize(q0, s0, g)) ** 2).reshape(32, -1, 16).sum(axis=2)
    e1 = ((wf - oracle.dequantize(q1, s1, g)) ** 2).reshape(32, -1, 16).sum(axis=2)
    assert np.all(e1 <= e0 * (1 + 1e-12))
    assert e1.sum() < e0.sum()          # and it does change something on a weight-like tensor
