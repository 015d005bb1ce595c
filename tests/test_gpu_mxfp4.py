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


# MXFP4 weights on the NVFP4 kernels: the scales restated once (include/mxfp4.h,
# mxfp4_to_nvfp4_scales) and the GEMMs run unchanged on them.

def _convert(nv, q, s):
    s_nv, g = nv.mx_to_nvfp4(torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    return s_nv.cpu().numpy(), g.cpu().numpy()[0]


@pytest.mark.parametrize("N,K", [(17408, 5120), (333, 1536), (1, 32), (7, 96)])
def test_mx_to_nvfp4_bit_exact(nv, N, K):
    q, s = _mx_codes(N, K, 3 * N + K)
    q[0, :16] = 0x88                     # an all-(-0) block: scale 0
    s_ref, g_ref, bad = oracle.mx_to_nvfp4(q, s)
    assert bad == 0
    s_nv, g = _convert(nv, q, s)
    assert np.array_equal(s_nv, s_ref) and g == g_ref
    nv.check_device_errors()


def test_mx_to_nvfp4_edge_scales(nv):
    """All-zero tensor (g = 1), a tensor scale below the normal range (G < -126),
    NaN scale bytes and blocks far below the largest (counted, scale 0)."""
    q = np.zeros((3, 64), np.uint8)
    s = np.full((3, 4), 200, np.uint8)
    s_nv, g = _convert(nv, q, s)
    assert g == 1.0 and not s_nv.any()
    nv.check_device_errors()

    q, s = _mx_codes(16, 256, 4)
    s[:] = np.random.default_rng(5).integers(0, 6, s.shape, dtype=np.uint8)   # 2^-127 .. 2^-122
    s_ref, g_ref, bad = oracle.mx_to_nvfp4(q, s)
    assert bad == 0 and g_ref < np.float32(2.0 ** -126) and g_ref > 0
    s_nv, g = _convert(nv, q, s)
    assert np.array_equal(s_nv, s_ref) and g == g_ref
    nv.check_device_errors()

    q, s = _mx_codes(16, 256, 6)
    s[2, 1] = 255
    s[5, 3] = 100
    s_ref, g_ref, bad = oracle.mx_to_nvfp4(q, s)
    assert bad == 2
    s_nv, g = _convert(nv, q, s)
    assert np.array_equal(s_nv, s_ref) and g == g_ref
    with pytest.raises(nv.Nvfp4Error, match="MXFP4 block"):
        nv.check_device_errors()
    nv.check_device_errors()             # the count is cleared once read


@pytest.mark.parametrize("M,N,K,span", [(1, 17408, 5120, 13), (32, 1100, 2048, 13), (512, 600, 1024, 13),
                                        (32, 300, 1056, 13), (32, 700, 1024, 18), (512, 300, 2048, 18)])
def test_mx_weights_on_nvfp4_gemm(nv, M, N, K, span):
    """MXFP4 weights through the NVFP4 GEMV / GEMMs on the restated scales,
    against the oracle's MXFP4 product of the original scales.  span 18: block
    exponents over the whole 17-binade window, so the smallest blocks get the
    E4M3 subnormal scales 2^-9 .. 2^-7."""
    q, s = _mx_codes(N, K, M + N + K)
    if span != 13:
        s[:] = np.random.default_rng(N).integers(127 - span + 1, 128, s.shape, dtype=np.uint8)
        assert oracle.mx_to_nvfp4(q, s)[2] == 0
    x = workloads.random_bf16((M, K), 13 * M + K)
    s_nv, g = nv.mx_to_nvfp4(torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda())
    Y = nv.linear(x.cuda(), torch.from_numpy(q).cuda(), s_nv, g)
    torch.cuda.synchronize()
    if M * N * K > 2 ** 28:
        rng = np.random.default_rng(M)
        rows = rng.integers(0, M, 512)
        cols = rng.integers(0, N, 512)
        y_ref, bound = oracle.mx_linear(x, q, s, rows=rows, cols=cols)
        assert_within_tolerance(Y.cpu()[rows, cols], y_ref, bound, f"mx->nv M={M}")
    else:
        y_ref, bound = oracle.mx_linear(x, q, s)
        assert_within_tolerance(Y, y_ref, bound, f"mx->nv M={M} N={N} K={K}")
    nv.check_device_errors()


def test_mx_quantize_convert_gemm_full_size(nv):
    """The 27B decode layer quantized to MXFP4 on the GPU, restated, then the
    M=512 GEMM, sampled against the oracle on the oracle's own quantization."""
    cfg = workloads.CONFIGS["decode"]
    w = workloads.weight_bf16(cfg)
    q_ref, s_ref = oracle.mx_quantize(w)
    q, s = nv.mx_quantize_new(w.cuda())
    s_nv, g = nv.mx_to_nvfp4(q, s)
    X = workloads.random_bf16((512, cfg.K), 17)
    Y = nv.linear(X.cuda(), q, s_nv, g)
    torch.cuda.synchronize()
    rng = np.random.default_rng(18)
    rows = rng.integers(0, 512, 400)
    cols = rng.integers(0, cfg.N, 400)
    y_ref, bound = oracle.mx_linear(X, q_ref, s_ref, rows=rows, cols=cols)
    assert_within_tolerance(Y.cpu()[rows, cols], y_ref, bound, "mx quantize -> nvfp4 gemm")
    nv.check_device_errors()
