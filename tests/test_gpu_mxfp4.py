"""GPU MXFP4 quantizer (bit-exact) and decode GEMV (within the stated
tolerance 1e-3 * sum|w x| + 1e-2 * |y_ref|) against the oracle.

MXFP4 on the pages (imp docs/quantization.md, MXFP4 paragraph): E2M1 nibbles
as NVFP4, one UE8M0 micro-scale per 32 elements, no tensor scale."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import assert_within_tolerance, guarded_empty

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import gemm_decode_nvfp4_b200 as m
    assert torch.cuda.is_available()
    return m


def _extreme_weights(N, K, seed):
    """Blocks at magnitudes from BF16 subnormals to 2^60, exact ties, zeros."""
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((N, K)).astype(np.float32)
    mags = 2.0 ** rng.integers(-135, 60, size=(N, K // 32, 1))
    w = (w.reshape(N, K // 32, 32) * mags).reshape(N, K)
    w[0, :32] = 0.0
    w[0, 32:64] = -0.0
    w[1, :32] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 4.0] * 4, np.float32)
    return torch.from_numpy(w).to(torch.bfloat16)


@pytest.mark.parametrize("which", ["tiny", "decode", "extreme"])
def test_mx_quantize_bit_exact(nv, which):
    if which == "extreme":
        w = _extreme_weights(96, 1024, 3)
    else:
        w = workloads.weight_bf16(workloads.CONFIGS[which])
    q_ref, s_ref = oracle.mx_quantize(w)
    q, s = nv.mx_quantize_new(w.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_mx_quantize_strided_rows(nv):
    """Rows of a wider tensor (ldw > K) quantize as if contiguous."""
    wide = _extreme_weights(40, 1024, 5)
    w = wide[:, 256:256 + 512]
    q_ref, s_ref = oracle.mx_quantize(w.contiguous())
    wd = wide.cuda()[:, 256:256 + 512]
    q = torch.empty((40, 256), dtype=torch.uint8, device="cuda")
    s = torch.empty((40, 16), dtype=torch.uint8, device="cuda")
    nv.mx_quantize(wd, q, s)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref) and np.array_equal(s.cpu().numpy(), s_ref)


def _mx_codes(N, K, seed):
    """Random codes and UE8M0 scales around 2^-8 .. 2^4 (trained-weight range)."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    s = rng.integers(119, 132, (N, K // 32), dtype=np.uint8)
    return q, s


def _run(nv, x, q, s, static=False):
    N = q.shape[0]
    y, check = guarded_empty((N,), torch.bfloat16)
    nv.mx_gemv(x.reshape(-1).cuda(), torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), y,
               static_weights=static)
    check()
    return y


@pytest.mark.parametrize("N,K", [(17408, 5120),     # ring kernel, one row block per CTA
                                 (148 * 120 + 9, 1024),  # ring, two row blocks
                                 (333, 1536),       # ring, half-empty last column of 256 bytes
                                 (77, 1056),        # K % 512 != 0: register kernel
                                 (64, 12288),       # K above the ring's limit: register kernel
                                 (1, 32), (5, 96)])
@pytest.mark.parametrize("static", [False, True])
def test_mx_gemv_shapes(nv, N, K, static):
    q, s = _mx_codes(N, K, N + K)
    x = workloads.random_bf16((1, K), 7 * N + K)
    y_ref, bound = oracle.mx_linear(x, q, s)
    y = _run(nv, x, q, s, static)
    assert_within_tolerance(y, y_ref[0], bound[0], f"mx N={N} K={K} static={static}")
    nv.check_device_errors()


@pytest.mark.parametrize("N,K", [(600, 5120), (90, 1056)])
@pytest.mark.parametrize("kind", ["wide", "zero"])
def test_mx_gemv_x_range_paths(nv, N, K, kind):
    """x spanning more than 2^32 takes the exact fp32 path; all-zero x gives 0."""
    q, s = _mx_codes(N, K, 21)
    x = workloads.random_bf16((1, K), 22).float()
    if kind == "wide":
        x[0, 0] = 2.0 ** 90
        x[0, 3] = -(2.0 ** -70)
    else:
        x = x * 0.0
    x = x.to(torch.bfloat16)
    y_ref, bound = oracle.mx_linear(x, q, s)
    y = _run(nv, x, q, s)
    assert_within_tolerance(y, y_ref[0], bound[0], f"mx {kind} N={N} K={K}")


def test_mx_quantize_then_gemv(nv):
    """The 27B decode layer quantized to MXFP4 on the GPU, then the GEMV on the
    same stream, against the oracle on the oracle's own quantization."""
    cfg = workloads.CONFIGS["decode"]
    w = workloads.weight_bf16(cfg)
    x = workloads.activations(1, cfg.K, cfg.seed)
    q_ref, s_ref = oracle.mx_quantize(w)
    q, s = nv.mx_quantize_new(w.cuda())
    y = torch.empty((cfg.N,), dtype=torch.bfloat16, device="cuda")
    nv.mx_gemv(x.reshape(-1).cuda(), q, s, y)
    torch.cuda.synchronize()
    rows = np.arange(0, cfg.N, 97)
    y_ref, bound = oracle.mx_linear(x, q_ref, s_ref, rows=np.zeros_like(rows), cols=rows)
    assert_within_tolerance(y.cpu()[rows], y_ref, bound, "mx decode layer")
