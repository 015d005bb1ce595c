"""Micro-scale search (MSE) quantizer on the GPU (nvfp4_quantize_mse,
imp docs/quantization.md, micro-scale search paragraph) against the oracle,
byte for byte: every scale byte and every code byte must equal the oracle's,
which takes the same readings (candidates within `window` E4M3 codes of the
round-to-nearest scale, fp64 squared error summed in index order, ties to
the code nearest it, then the smaller code)."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import gemm_decode_nvfp4_b200 as m
    assert torch.cuda.is_available()
    return m


def _gpu_mse(nv, w_cpu, window=8, g=None, ldw_pad=0):
    N, K = w_cpu.shape
    if ldw_pad:
        big = torch.zeros((N, K + ldw_pad), dtype=torch.bfloat16)
        big[:, :K] = w_cpu
        wd = big.cuda()[:, :K]
    else:
        wd = w_cpu.cuda()
    q = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    s = torch.empty((N, K // 16), dtype=torch.uint8, device="cuda")
    gout = torch.empty((1,), dtype=torch.float32, device="cuda")
    if g is None:
        nv.quantize_mse(wd, q, s, gout, window=window)
    else:
        a = torch.tensor([float(np.float32(g) * np.float32(2688.0))], dtype=torch.float32, device="cuda")
        nv.quantize_mse(wd, q, s, gout, amax=a, window=window)
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy(), np.float32(gout.item())


def _assert_same(nv, w, window=8, what=""):
    q, s, g = _gpu_mse(nv, w, window)
    q_ref, s_ref, g_ref = oracle.quantize_mse(w, window=window)
    assert g == g_ref, what
    assert np.array_equal(s, s_ref), f"{what}: {int((s != s_ref).sum())} scale bytes differ"
    assert np.array_equal(q, q_ref), f"{what}: {int((q != q_ref).sum())} code bytes differ"


def test_worked_block(nv):
    """Sixteen 2.5s with g = 1: scale 0x32 (0.625) and codes 0x6 (4.0) reproduce
    the block exactly, where round-to-nearest gives 0x2D and 0x7."""
    w = torch.full((1, 16), 2.5, dtype=torch.bfloat16)
    q, s, g = _gpu_mse(nv, w, g=np.float32(1.0))
    assert g == np.float32(1.0)
    assert s[0, 0] == 0x32 and np.all(q == 0x66)


@pytest.mark.parametrize("window", [0, 1, 3, 8, 16])
def test_windows_match_oracle(nv, window):
    w = workloads.random_bf16((96, 1024), 10 + window, 0.02)
    _assert_same(nv, w, window, f"window {window}")


def test_window_zero_equals_round_to_nearest_kernel(nv):
    w = workloads.random_bf16((64, 2048), 21, 0.02).cuda()
    q0, s0, g0 = nv.quantize_new(w)
    q1 = torch.empty_like(q0)
    s1 = torch.empty_like(s0)
    g1 = torch.empty_like(g0)
    nv.quantize_mse(w, q1, s1, g1, window=0)
    torch.cuda.synchronize()
    assert torch.equal(q0, q1) and torch.equal(s0, s1) and torch.equal(g0, g1)


def test_special_blocks(nv):
    """Zero blocks, signed zeros inside blocks, a block 1000x larger than the
    rest (scales near 448), tiny blocks (scales near the E4M3 subnormals), and
    ties between equally good candidates (constant blocks)."""
    rng = np.random.default_rng(31)
    w = rng.standard_normal((8, 256)).astype(np.float32) * np.float32(0.02)
    w[0, :16] = 0.0
    w[0, 16:32] = -0.0
    w[1, 3] = -0.0
    w[1, 40] = 0.0
    w[2, 16:32] *= 1e3
    w[3, :64] *= 1e-4
    w[4, :16] = 1.0
    w[4, 16:32] = -3.0
    w[5, :] = 0.125
    _assert_same(nv, workloads.to_bf16(w), 8, "special blocks")


def test_decode_workload_full(nv):
    """The 27B layer weight [17408, 5120] (jittered rows, 0.1% outliers),
    every byte."""
    _assert_same(nv, workloads.weight_bf16(workloads.CONFIGS["decode"]), 8, "decode layer")


def test_prefill_quantizer_input_full(nv):
    """The plain N(0, 0.02) [17408, 5120] tensor of the prefill configuration's
    quantizer, every byte."""
    w = workloads.to_bf16(workloads.plain_weight_f32(workloads.MLP, workloads.HIDDEN, 4))
    _assert_same(nv, w, 8, "prefill quantizer input")


def test_given_amax_and_row_stride(nv):
    """A merged layer's shared amax passed in, and rows with a leading dimension
    larger than K."""
    w = workloads.random_bf16((40, 512), 41, 0.02)
    g = np.float32(0.0001)
    q, s, g_out = _gpu_mse(nv, w, 8, g=g, ldw_pad=64)
    g_ref = np.float32(np.float32(g * np.float32(2688.0)) / np.float32(2688.0))
    q_ref, s_ref, _ = oracle.quantize_mse(w, g_ref, window=8)
    assert g_out == g_ref
    assert np.array_equal(s, s_ref) and np.array_equal(q, q_ref)


def test_bad_window_rejected(nv):
    w = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((4, 32), dtype=torch.uint8, device="cuda")
    s = torch.empty((4, 4), dtype=torch.uint8, device="cuda")
    g = torch.empty((1,), dtype=torch.float32, device="cuda")
    for window in (-1, 126):
        with pytest.raises(nv.Nvfp4Error, match="INVALID_ARG"):
            nv.quantize_mse(w, q, s, g, window=window)
