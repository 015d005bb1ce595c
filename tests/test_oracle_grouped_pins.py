"""Pins of the grouped (MoE) GEMV of the oracle: it reduces to the pinned
single-layer linear for one expert, equals a numpy fp64 product of each
expert's dequantized matrix, and permuting the problems permutes the rows."""
import numpy as np

import oracle
import workloads


def _experts(E, N, K, seed):
    q = np.stack([workloads.random_codes(N, K, seed + e)[0].numpy() for e in range(E)])
    s = np.stack([workloads.random_codes(N, K, seed + e)[1].numpy() for e in range(E)])
    g = np.array([0.01 * (e + 1) for e in range(E)], np.float32)
    return q, s, g


def test_one_expert_reduces_to_linear():
    q, s, g = _experts(1, 9, 64, 3)
    x = workloads.random_bf16((2, 64), 4)
    y, b = oracle.linear_grouped(x, q, s, g, [0, 0], [1, 0])
    y1, b1 = oracle.linear(x, q[0], s[0], g[0])
    assert np.array_equal(y[0], y1[1]) and np.array_equal(y[1], y1[0])
    assert np.array_equal(b[0], b1[1])


def test_grouped_equals_dequantized_products():
    E, N, K = 4, 7, 96
    q, s, g = _experts(E, N, K, 11)
    x = workloads.random_bf16((3, K), 12)
    xf = x.float().numpy().astype(np.float64)
    experts, tokens = [2, 0, 3, 2, 1], [0, 2, 1, 1, 0]
    y, b = oracle.linear_grouped(x, q, s, g, experts, tokens)
    for p, (e, t) in enumerate(zip(experts, tokens)):
        wd = oracle.dequantize(q[e], s[e], g[e])
        np.testing.assert_allclose(y[p], wd @ xf[t], rtol=1e-12, atol=1e-300)
        np.testing.assert_allclose(b[p], np.abs(wd) @ np.abs(xf[t]), rtol=1e-12, atol=1e-300)


def test_problem_order_permutes_rows():
    q, s, g = _experts(3, 5, 32, 21)
    x = workloads.random_bf16((2, 32), 22)
    e, t = np.array([0, 1, 2, 1]), np.array([1, 0, 1, 1])
    perm = np.array([3, 1, 0, 2])
    y, _ = oracle.linear_grouped(x, q, s, g, e, t)
    yp, _ = oracle.linear_grouped(x, q, s, g, e[perm], t[perm])
    assert np.array_equal(yp, y[perm])
