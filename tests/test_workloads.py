"""The seeded input recipe shared by the oracle and the GPU tests: the same
seed gives the same tensors, and the generators have the distributions the
design notes state (per-row scale spread and outliers of the layer weights,
the 3.7x amax spread of the merged members, the shapes of the workloads)."""
import numpy as np
import torch

import workloads


def test_deterministic_and_seed_dependent():
    a = workloads.layer_weight_f32(64, 256, 7)
    b = workloads.layer_weight_f32(64, 256, 7)
    c = workloads.layer_weight_f32(64, 256, 8)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    assert torch.equal(workloads.activations(4, 128, 3), workloads.activations(4, 128, 3))
    assert torch.equal(workloads.random_bf16((5, 32), 1), workloads.random_bf16((5, 32), 1))


def test_layer_weight_row_scales_and_outliers():
    """N(0, 0.02) times a per-row factor in [0.5, 2], and about one element in
    a thousand multiplied by 20."""
    w = workloads.layer_weight_f32(512, 4096, 1)
    # robust row scale (the outliers inflate a plain std): median |N(0, s)| = 0.6745 s
    row_factor = np.median(np.abs(w), axis=1) / (0.6745 * 0.02)
    assert row_factor.min() > 0.5 * 0.95 and row_factor.max() < 2.0 * 1.05
    assert row_factor.min() < 0.55 and row_factor.max() > 1.9   # the whole [0.5, 2] range is used
    z = np.abs(w) / (row_factor[:, None] * 0.02)
    # beyond 8 sigma: only the x20 outliers, 1e-3 * P(|N(0, 1)| > 0.4) = 6.9e-4 of all elements
    frac = float(np.mean(z > 8.0))
    assert 5.5e-4 < frac < 8.5e-4


def test_merged_members_amax_spread():
    members = workloads.merged_members(0, K=256, rows=(64, 64, 64, 96, 96))
    amax = [float(m.float().abs().max()) for m in members]
    rel = np.array(amax) / amax[0]
    np.testing.assert_allclose(rel, workloads.MERGED_MEMBER_AMAX, rtol=1e-2)
    assert max(amax) / min(amax) > 3.6


def test_workload_shapes():
    c = workloads.CONFIGS
    assert (c["decode"].N, c["decode"].K) == (17408, 5120)
    assert (c["batch32"].M, c["prefill"].M) == (32, 512)
    assert c["merged"].N == 3 * 5120 + 2 * 17408
    x = workloads.activations(3, 64, 0)
    assert x.dtype == torch.bfloat16 and tuple(x.shape) == (3, 64)
