"""GPU quantizer (nvfp4_amax / nvfp4_quantize) against the oracle: bit-exact
codes, scales and tensor scale."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import guarded_empty

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import gemm_decode_nvfp4_b200 as m
    assert torch.cuda.is_available()
    return m


def _gpu_quantize(nv, w_cpu, amax=None):
    w = w_cpu.cuda()
    N, K = w.shape
    q, cq = guarded_empty((N, K // 2), torch.uint8)
    s, cs = guarded_empty((N, K // 16), torch.uint8)
    g, cg = guarded_empty((1,), torch.float32)
    nv.quantize(w, q, s, g, amax=amax)
    torch.cuda.synchronize()
    cq(); cs(); cg()
    return q.cpu().numpy(), s.cpu().numpy(), np.float32(g.cpu().item())


def _planted(shape, seed, std):
    w = workloads.random_bf16(shape, seed, std).float()
    N, K = shape
    w[0, min(5, K - 1)] *= 40                    # outlier
    if N > 1 and K >= 32:
        w[1, 16:32] = 0.0                        # zero block
    if N > 2:
        w[2, 0:16] = -0.0                        # negative zeros
    if N > 3 and K >= 48:
        w[3, 32:48] *= 1e-6                      # tiny block
    if N > 4:
        w[4, :16] = torch.tensor([-1e-30] * 16)  # underflows to signed zero codes
    return w.to(torch.bfloat16)


@pytest.mark.parametrize("N,K,seed,std", [(1, 16, 0, 1.0), (3, 48, 1, 0.02), (37, 160, 2, 3.0),
                                          (128, 1024, 3, 0.02), (257, 5120, 4, 0.02), (64, 96, 5, 1e-20)])
def test_quantize_bit_exact(nv, N, K, seed, std):
    w = _planted((N, K), seed, std)
    q_ref, s_ref, g_ref = oracle.quantize(w)
    q, s, g = _gpu_quantize(nv, w)
    assert g == g_ref
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_array_equal(q, q_ref)


def test_quantize_given_amax_and_strided_rows(nv):
    N, K, ld = 40, 256, 384
    full = workloads.random_bf16((N, ld), 7, 0.1)
    w = full[:, :K]
    amax = torch.tensor([0.37], dtype=torch.float32, device="cuda")  # any amax >= the tensor's own
    g_ref = oracle.tensor_scale(np.float32(0.37))
    q_ref, s_ref, _ = oracle.quantize(w.contiguous(), g_ref)
    wd = full.cuda()[:, :K]
    assert wd.stride(0) == ld
    q = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    s = torch.empty((N, K // 16), dtype=torch.uint8, device="cuda")
    g = torch.empty((1,), dtype=torch.float32, device="cuda")
    nv.quantize(wd, q, s, g, amax=amax)
    torch.cuda.synchronize()
    assert np.float32(g.item()) == g_ref
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)


def test_quantize_rounding_ties_and_grid(nv):
    """Blocks whose d is a power of two, so w * r hits every E2M1 midpoint and
    every BF16 value in [2^-60, 6] exactly; plus saturation above 6."""
    g = np.float32(2.0 ** -10)
    d = np.float32(2.0 ** -3) * g           # scale 2^-3 (E4M3 exact), power-of-two d
    vals = np.arange(0, 1 << 15, dtype=np.uint32)
    bf = (vals << 16).view(np.float32)
    grid = bf[((bf >= 2.0 ** -60) & (bf <= 6.0)) | (bf == 0)]  # every BF16 in [2^-60, 6], and 0
    t = np.concatenate([grid, -grid, [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]])
    n_el = ((len(t) + 14) // 15) * 15
    t = np.resize(t, n_el).reshape(-1, 15)
    blocks = np.concatenate([t, np.full((t.shape[0], 1), 6.0)], axis=1)  # amax_b = 6 -> scale 2^-3
    over = bf[(bf > 6.0) & (bf < 8.0)]       # blocks whose scale rounds down: w * r above 6
    over = np.resize(over, ((len(over) + 15) // 16) * 16).reshape(-1, 16)
    w = np.concatenate([blocks, over], axis=0) * float(d)
    first = np.zeros((1, 16), np.float64)    # fixes the tensor amax at 2688 g
    first[0, 0] = 2688.0 * float(g)
    w = np.concatenate([first, w], axis=0)
    pad = (-w.shape[0]) % 4
    w = np.concatenate([w, np.zeros((pad, 16))], axis=0).astype(np.float32).reshape(-1, 64)
    wt = torch.from_numpy(w).to(torch.bfloat16)
    assert np.array_equal(wt.float().numpy(), w)   # all exactly BF16
    q_ref, s_ref, g_ref = oracle.quantize(wt)
    assert g_ref == g
    q, s, gg = _gpu_quantize(nv, wt)
    assert gg == g_ref
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_array_equal(q, q_ref)


def test_quantize_all_zero_tensor(nv):
    w = torch.zeros((8, 64), dtype=torch.bfloat16)
    q, s, g = _gpu_quantize(nv, w)
    assert g == 0.0
    assert not q.any() and not s.any()


def test_quantize_merged_shared_scale(nv):
    """nvfp4_amax over the five members into one accumulator, then each member
    quantized with the shared amax, equals the oracle with the shared g."""
    K = 256
    members = workloads.merged_members(21, K=K, rows=(32, 32, 32, 96, 96))
    acc = torch.zeros((1,), dtype=torch.float32, device="cuda")
    dev = [m.cuda() for m in members]
    for m in dev:
        nv.amax(m, acc)
    torch.cuda.synchronize()
    amax_ref = max(oracle.amax(m) for m in members)
    assert np.float32(acc.item()) == amax_ref
    g_ref = oracle.tensor_scale(amax_ref)
    for m_cpu, m in zip(members, dev):
        q = torch.empty((m.shape[0], K // 2), dtype=torch.uint8, device="cuda")
        s = torch.empty((m.shape[0], K // 16), dtype=torch.uint8, device="cuda")
        g = torch.empty((1,), dtype=torch.float32, device="cuda")
        nv.quantize(m, q, s, g, amax=acc)
        torch.cuda.synchronize()
        q_ref, s_ref, _ = oracle.quantize(m_cpu, g_ref)
        assert np.float32(g.item()) == g_ref
        np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
        np.testing.assert_array_equal(s.cpu().numpy(), s_ref)


def test_quantize_full_size_prefill_tensor(nv):
    """The 512-token prefill workload's quantizer input, BF16 [17408, 5120]
    N(0, 0.02): every byte against the oracle."""
    w = workloads.to_bf16(workloads.plain_weight_f32(workloads.MLP, workloads.HIDDEN, 4))
    q_ref, s_ref, g_ref = oracle.quantize(w)
    q, s, g = _gpu_quantize(nv, w)
    assert g == g_ref
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_array_equal(q, q_ref)
