"""Pins of the W4A4 part of the CPU oracle (X quantized to NVFP4 by the weights'
round-to-nearest rule, then the product of the two dequantized operands).

The checks tie it to facts outside its own formula: inputs that NVFP4 holds
exactly reduce it to the (separately pinned) W4A16 oracle, a worked example is
computed by hand, powers of two pass through the tensor scale exactly, and a
too-small calibrated amax saturates at the format's largest value."""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import workloads

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)


def _representable_x(M, K, seed, E=-2):
    """X whose NVFP4 quantization is lossless: the tensor max is 2688 * 2^E, so
    g_x = 2^E exactly; each 16-block is E2M1 values times s_b * 2^E with an E4M3
    value s_b <= 448 and one element at +-6 * s_b * 2^E, so the block scale
    (amax_b / 6) / g_x is exactly s_b and every element is a code times the
    step s_b * g_x.  (Every value has at most 6 significant bits: exact in BF16.)"""
    rng = np.random.default_rng(seed)
    e4m3_normal = np.arange(0x08, 0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    x = np.empty((M, K))
    for m in range(M):
        for b in range(K // 16):
            sb = float(rng.choice(e4m3_normal))
            blk = rng.choice(E2M1, 16) * rng.choice([-1.0, 1.0], 16)
            blk[int(rng.integers(0, 16))] = 6.0 * rng.choice([-1.0, 1.0])
            x[m, 16 * b:16 * b + 16] = blk * sb * 2.0 ** E
    x[0, :16] = 0.0
    x[0, 0] = 6.0 * 448.0 * 2.0 ** E
    return x


@pytest.mark.parametrize("M,N,K", [(3, 5, 64), (8, 12, 256)])
def test_lossless_x_reduces_to_w4a16(M, N, K):
    x = _representable_x(M, K, M * N)
    xb = _bf16(x)
    w = workloads.random_bf16((N, K), N + K)
    q, s, g = oracle.quantize(w)
    y4, b4, (qx, sx, g_x) = oracle.w4a4_linear(xb, q, s, g)
    assert g_x == np.float32(0.25)
    np.testing.assert_array_equal(oracle.dequantize(qx, sx, g_x), x)
    y16, b16 = oracle.linear(xb, q, s, g)
    np.testing.assert_allclose(y4, y16, rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(b4, b16, rtol=1e-12, atol=1e-300)


def test_worked_example_by_hand():
    """One 16-block.  x = (5.25, 1.75, 0.4375, -3.5, 0 ...): amax 5.25 = 2688 / 512,
    so g_x = 2^-9; block scale (5.25 / 6) / 2^-9 = 448 (an E4M3 value), step
    448 * 2^-9 = 0.875, and x / 0.875 = (6, 2, 0.5, -4) are E2M1 values, so
    X_deq = x.  W: code 1.0 (0x2) times scale 1 (E4M3 0x38) times g = 2 in every
    element, so y = 2 * 3.9375 = 7.875 and the bound is 2 * 10.9375 = 21.875."""
    x = np.zeros((1, 16))
    x[0, :4] = [5.25, 1.75, 0.4375, -3.5]
    q = np.full((1, 8), 0x22, np.uint8)
    s = np.full((1, 1), 0x38, np.uint8)
    y, bound, (qx, sx, g_x) = oracle.w4a4_linear(_bf16(x), q, s, np.float32(2.0))
    assert g_x == np.float32(2.0 ** -9) and sx[0, 0] == 0x7E
    assert list(qx[0, :2]) == [0x47, 0xE1]   # codes 6 (0x7) | 2 (0x4) << 4, 0.5 (0x1) | -4 (0xE) << 4
    assert y[0, 0] == 7.875 and bound[0, 0] == 21.875


def test_power_of_two_scaling_is_exact():
    """X * 2^j changes only g_x (by exactly 2^j): codes and block scales stay,
    so y scales by 2^j exactly."""
    x = workloads.random_bf16((4, 128), 3)
    w = workloads.random_bf16((6, 128), 4)
    q, s, g = oracle.quantize(w)
    y, bound, (qx, sx, g_x) = oracle.w4a4_linear(x, q, s, g)
    for j in (-7, 5):
        xj = (x.float() * 2.0 ** j).to(torch.bfloat16)
        yj, bj, (qj, sj, gj) = oracle.w4a4_linear(xj, q, s, g)
        assert gj == np.float32(g_x * np.float32(2.0 ** j))
        assert np.array_equal(qj, qx) and np.array_equal(sj, sx)
        np.testing.assert_array_equal(yj, y * 2.0 ** j)
        np.testing.assert_array_equal(bj, bound * 2.0 ** j)


def test_small_calibrated_amax_saturates():
    """With x_amax below max |X| the largest elements clip to 6 * 448 * g_x,
    the format's largest value, and nothing exceeds it."""
    x = workloads.random_bf16((4, 64), 5)
    true_max = float(oracle.amax(x))
    w = workloads.random_bf16((3, 64), 6)
    q, s, g = oracle.quantize(w)
    _, _, (qx, sx, g_x) = oracle.w4a4_linear(x, q, s, g, x_amax=true_max / 4)
    xd = oracle.dequantize(qx, sx, g_x)
    top = 6.0 * 448.0 * float(g_x)
    assert np.max(np.abs(xd)) == top
    assert np.all(np.abs(xd) <= top)


def test_sampled_outputs_match_full():
    x = workloads.random_bf16((5, 96), 7)
    w = workloads.random_bf16((9, 96), 8)
    q, s, g = oracle.quantize(w)
    y, bound, _ = oracle.w4a4_linear(x, q, s, g)
    rows, cols = np.array([4, 0, 2]), np.array([8, 3, 0])
    ys, bs, _ = oracle.w4a4_linear(x, q, s, g, rows=rows, cols=cols)
    np.testing.assert_allclose(ys, y[rows, cols], rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(bs, bound[rows, cols], rtol=1e-13, atol=1e-300)
