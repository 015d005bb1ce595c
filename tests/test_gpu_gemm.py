"""GPU tensor-core GEMM (nvfp4_gemm, M >= 2) against the oracle within
|y - y_ref| <= 1e-3 * sum|w x| + 1e-2 * |y_ref|, plus exact layout checks."""
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


def _run(nv, X_cpu, q_np, s_np, g, ldx=None, ldy=None, static_weights=False):
    M, K = X_cpu.shape
    N = q_np.shape[0]
    ldx = ldx or K
    ldy = ldy or N
    Xbuf = torch.zeros((M, ldx), dtype=torch.bfloat16)
    Xbuf[:, :K] = X_cpu
    X = Xbuf.cuda()[:, :K]
    q = torch.from_numpy(np.ascontiguousarray(q_np)).cuda()
    s = torch.from_numpy(np.ascontiguousarray(s_np)).cuda()
    gd = torch.tensor([float(np.float32(g))], dtype=torch.float32, device="cuda")
    Ybuf, check = guarded_empty((M, ldy), torch.bfloat16)
    Ybuf.fill_(float("nan"))
    Y = Ybuf[:, :N]
    n_ws = nv.gemm_workspace_size(M, N, K)
    ws, check_ws = guarded_empty((max(n_ws, 1),), torch.uint8)
    nv.gemm(X, q, s, gd, Y, workspace=ws if n_ws else None, static_weights=static_weights)
    check()
    check_ws()
    assert nv.lib.nvfp4_check_device_errors() == 0
    if ldy > N:  # padding columns untouched
        assert torch.isnan(Ybuf[:, N:].float()).all()
    return Y


@pytest.mark.parametrize("M,N,K", [(2, 128, 256), (5, 200, 512), (16, 384, 256), (17, 130, 1024),
                                   (32, 256, 512), (33, 128, 256), (64, 257, 768), (100, 128, 256),
                                   (128, 384, 512), (200, 256, 256), (256, 128, 1024), (300, 200, 512),
                                   (512, 384, 1024)])
def test_shapes_vs_oracle(nv, M, N, K):
    q, s = workloads.random_codes(N, K, M * 131 + N)
    X = workloads.random_bf16((M, K), M + 7 * N + K)
    g = np.float32(0.0071)
    y_ref, bound = oracle.linear(X, q.numpy(), s.numpy(), g)
    Y = _run(nv, X, q.numpy(), s.numpy(), g)
    assert_within_tolerance(Y, y_ref, bound, f"M={M} N={N} K={K}")


def test_one_hot_rows_exact_layout(nv):
    """X row m is one-hot at k = (37 m) mod K: Y[m, n] is exactly the
    dequantized weight W[n, k] (checks the swizzled operand layouts end to end)."""
    M, N, K = 64, 256, 512
    q, s = workloads.random_codes(N, K, 3)
    q, s = q.numpy(), s.numpy()
    ks = (37 * np.arange(M)) % K
    X = torch.zeros((M, K), dtype=torch.bfloat16)
    X[np.arange(M), ks] = 1.0
    Y = _run(nv, X, q, s, 1.0).float().cpu().double().numpy()
    deq = oracle.dequantize(q, s, 1.0)
    expect = deq[:, ks].T
    assert np.array_equal(Y, expect)


def test_strided_x_and_y(nv):
    M, N, K = 48, 200, 512
    q, s = workloads.random_codes(N, K, 4)
    X = workloads.random_bf16((M, K), 5)
    y_ref, bound = oracle.linear(X, q.numpy(), s.numpy(), 0.5)
    Y = _run(nv, X, q.numpy(), s.numpy(), 0.5, ldx=K + 64, ldy=N + 56)
    assert_within_tolerance(Y, y_ref, bound, "strided")


@pytest.mark.parametrize("M,K", [(3, 96), (7, 1040)])
def test_k_not_multiple_of_256_runs_row_gemvs(nv, M, K):
    N = 100
    q, s = workloads.random_codes(N, K, 6)
    X = workloads.random_bf16((M, K), 7)
    y_ref, bound = oracle.linear(X, q.numpy(), s.numpy(), 0.25)
    Y = _run(nv, X, q.numpy(), s.numpy(), 0.25)
    assert_within_tolerance(Y, y_ref, bound, f"K={K}")


def _sample_pairs(M, N, n, seed):
    r = np.random.default_rng(seed)
    rows = np.concatenate([[0, M - 1, M - 1], r.integers(0, M, n)])
    cols = np.concatenate([[0, N - 1, 0], r.integers(0, N, n)])
    return rows.astype(np.int64), cols.astype(np.int64)


@pytest.mark.parametrize("name", ["batch32", "prefill"])
def test_full_size_sampled(nv, name):
    cfg = workloads.CONFIGS[name]
    q, s, g = oracle.quantize(workloads.weight_bf16(cfg))
    X = workloads.activations(cfg.M, cfg.K, cfg.seed)
    Y = _run(nv, X, q, s, g).float().cpu().double().numpy()
    rows, cols = _sample_pairs(cfg.M, cfg.N, 4000, 2)
    y_ref, bound = oracle.linear(X, q, s, g, rows=rows, cols=cols)
    assert_within_tolerance(torch.from_numpy(Y[rows, cols]), y_ref, bound, name)


def test_gpu_quantize_then_gemm(nv):
    """Whole path on the GPU (quantizer output feeds the GEMM) vs the oracle."""
    M, N, K = 40, 384, 1024
    w = workloads.random_bf16((N, K), 8, 0.02)
    X = workloads.random_bf16((M, K), 9)
    q, s, g = nv.quantize_new(w.cuda())
    Y = nv.linear(X.cuda(), q, s, g)
    torch.cuda.synchronize()
    q_ref, s_ref, g_ref = oracle.quantize(w)
    assert np.array_equal(q.cpu().numpy(), q_ref) and np.array_equal(s.cpu().numpy(), s_ref)
    y_ref, bound = oracle.linear(X, q_ref, s_ref, g_ref)
    assert_within_tolerance(Y, y_ref, bound, "quantize->gemm")


def test_cuda_graph_replay(nv):
    M, N, K = 32, 512, 1024
    q, s = workloads.random_codes(N, K, 10)
    X = workloads.random_bf16((M, K), 11)
    y_ref, bound = oracle.linear(X, q.numpy(), s.numpy(), 0.125)
    Xd, qd, sd = X.cuda(), q.cuda(), s.cuda()
    gd = torch.tensor([0.125], device="cuda")
    Y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((nv.gemm_workspace_size(M, N, K),), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        nv.gemm(Xd, qd, sd, gd, Y, workspace=ws, static_weights=True)
    stream.synchronize()
    Y.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        nv.gemm(Xd, qd, sd, gd, Y, workspace=ws, static_weights=True)
    graph.replay()
    torch.cuda.synchronize()
    assert_within_tolerance(Y, y_ref, bound, "graph")


@pytest.mark.parametrize("M", [5, 40, 300])
def test_wide_range_rows_recomputed_exactly(nv, M):
    """Rows of X whose non-zero magnitudes span more than 2^32 (and rows of huge
    or tiny scale) must still match the oracle: the wide ones are recomputed in
    fp32 on CUDA cores, the others go through the scaled f16 MMA."""
    N, K = 256, 1024
    q, s = workloads.random_codes(N, K, 40 + M)
    X = workloads.random_bf16((M, K), 41 + M).float()
    X[0, 3] = 2.0 ** 90            # wide row
    X[0, 9] = 2.0 ** -70
    X[M - 1] *= 2.0 ** -125        # tiny but narrow row
    if M > 2:
        X[1] *= 2.0 ** 100         # huge but narrow row
        X[2, :] = 0.0              # all-zero row
    X = X.to(torch.bfloat16)
    y_ref, bound = oracle.linear(X, q.numpy(), s.numpy(), 0.3)
    Y = _run(nv, X, q.numpy(), s.numpy(), 0.3)
    assert_within_tolerance(Y, y_ref, bound, f"wide rows M={M}")


def test_static_weights_flag_matches(nv):
    M, N, K = 64, 384, 2048
    q, s = workloads.random_codes(N, K, 50)
    X = workloads.random_bf16((M, K), 51)
    y_ref, bound = oracle.linear(X, q.numpy(), s.numpy(), 0.5)
    Y = _run(nv, X, q.numpy(), s.numpy(), 0.5, static_weights=True)
    assert_within_tolerance(Y, y_ref, bound, "static weights")


def test_workspace_too_small_is_an_error(nv):
    M, N, K = 32, 128, 256
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    q = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    s = torch.zeros((N, K // 16), dtype=torch.uint8, device="cuda")
    g = torch.ones((1,), device="cuda")
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    need = nv.gemm_workspace_size(M, N, K)
    assert need > 0
    small = torch.empty((need - 16,), dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.Nvfp4Error) as ei:
        nv.gemm(X, q, s, g, Y, workspace=small)
    assert ei.value.status == 6
    with pytest.raises(nv.Nvfp4Error):
        nv.gemm(X, q, s, g, Y)
