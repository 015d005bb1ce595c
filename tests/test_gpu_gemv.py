"""GPU decode GEMV (nvfp4_gemv) against the oracle, within the stated
tolerance |y - y_ref| <= 1e-3 * sum|w x| + 1e-2 * |y_ref| per output, plus
exact cases where the fp32 result is exact."""
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


def _run(nv, x_cpu, q_np, s_np, g):
    N = q_np.shape[0]
    x = x_cpu.reshape(-1).cuda()
    q = torch.from_numpy(np.ascontiguousarray(q_np)).cuda()
    s = torch.from_numpy(np.ascontiguousarray(s_np)).cuda()
    gd = torch.tensor([float(np.float32(g))], dtype=torch.float32, device="cuda")
    y, check = guarded_empty((N,), torch.bfloat16)
    nv.gemv(x, q, s, gd, y)
    check()
    return y


def test_tiny_workload(nv):
    cfg = workloads.CONFIGS["tiny"]
    w = workloads.weight_bf16(cfg)
    x = workloads.activations(1, cfg.K, cfg.seed)
    q, s, g = oracle.quantize(w)
    y_ref, bound = oracle.linear(x, q, s, g)
    y = _run(nv, x, q, s, g)
    assert_within_tolerance(y, y_ref[0], bound[0], "tiny")


@pytest.mark.parametrize("N,K", [(1, 16), (5, 48), (31, 96), (33, 1024), (1000, 1040), (77, 5120),
                                 (300, 17408), (8, 49152)])
def test_ragged_shapes(nv, N, K):
    q, s = workloads.random_codes(N, K, N + K)
    x = workloads.random_bf16((1, K), N * 7 + K)
    g = np.float32(0.0037)
    y_ref, bound = oracle.linear(x, q.numpy(), s.numpy(), g)
    y = _run(nv, x, q.numpy(), s.numpy(), g)
    assert_within_tolerance(y, y_ref[0], bound[0], f"N={N} K={K}")


def test_every_packed_byte_one_hot(nv):
    """Row of bytes 0x00..0xFF (K = 512), x one-hot at each k: y is exactly the
    decoded element (low nibble for even k, high nibble for odd k)."""
    K = 512
    q = np.arange(256, dtype=np.uint8).reshape(1, 256).repeat(4, axis=0)
    s = np.full((4, K // 16), 0x38, np.uint8)   # scale 1.0
    s[1] = 0x40                                  # 2.0
    s[2] = 0x01                                  # 2^-9 (subnormal)
    s[3] = 0x7E                                  # 448
    deq = oracle.dequantize(q, s, 1.0)
    for k in range(K):
        x = torch.zeros((K,), dtype=torch.bfloat16)
        x[k] = 1.0
        y = _run(nv, x, q, s, 1.0).float().cpu().double().numpy()
        assert np.array_equal(y, deq[:, k]), (k, y, deq[:, k])


def test_all_ones_row_sums(nv):
    N, K = 64, 2048
    q, s = workloads.random_codes(N, K, 5)
    x = torch.ones((K,), dtype=torch.bfloat16)
    y_ref, bound = oracle.linear(x, q.numpy(), s.numpy(), 1.0)
    y = _run(nv, x, q.numpy(), s.numpy(), 1.0)
    assert_within_tolerance(y, y_ref[0], bound[0], "ones")


def test_exact_small_integers(nv):
    """Integer x times weights with few significant bits: every partial sum is
    exact in fp32, so the only rounding is the final BF16 one."""
    N, K = 48, 1024
    r = np.random.default_rng(2)
    q = r.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    s = np.full((N, K // 16), 0x38, np.uint8)
    x = torch.from_numpy(r.integers(-3, 4, size=K).astype(np.float32)).to(torch.bfloat16)
    y_ref, _ = oracle.linear(x, q, s, 1.0)
    y = _run(nv, x, q, s, 1.0).float().cpu().numpy()
    expect = torch.from_numpy(y_ref[0].astype(np.float32)).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(y, expect)


def _sample_rows(N, n, seed):
    r = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, N - 1], r.integers(0, N, n)]))
    return rows.astype(np.int64)


@pytest.mark.parametrize("name", ["decode", "merged"])
def test_full_size_sampled(nv, name):
    """Full 27B-class shapes, weights quantized by the oracle; outputs sampled."""
    cfg = workloads.CONFIGS[name]
    if cfg.weights == "merged":
        members = workloads.merged_members(cfg.seed, cfg.K)
        g = oracle.tensor_scale(max(oracle.amax(m) for m in members))
        parts = [oracle.quantize(m, g) for m in members]
        q = np.concatenate([p[0] for p in parts])
        s = np.concatenate([p[1] for p in parts])
    else:
        q, s, g = oracle.quantize(workloads.weight_bf16(cfg))
    x = workloads.activations(1, cfg.K, cfg.seed)
    y = _run(nv, x, q, s, g).float().cpu().double().numpy()
    rows = _sample_rows(cfg.N, 3000, 1)
    y_ref, bound = oracle.linear(x, q, s, g, rows=np.zeros_like(rows), cols=rows)
    assert_within_tolerance(torch.from_numpy(y[rows]), y_ref, bound, name)


def test_gemm_m1_routes_to_gemv(nv):
    N, K = 200, 512
    q, s = workloads.random_codes(N, K, 9)
    x = workloads.random_bf16((1, K), 10)
    y_ref, bound = oracle.linear(x, q.numpy(), s.numpy(), 0.5)
    Y = nv.linear(x.cuda(), q.cuda(), s.cuda(), torch.tensor([0.5], device="cuda"))
    torch.cuda.synchronize()
    assert_within_tolerance(Y, y_ref, bound, "gemm M=1")


def test_cuda_graph_replay(nv):
    N, K = 4096, 5120
    q, s = workloads.random_codes(N, K, 11)
    x = workloads.random_bf16((1, K), 12)
    y_ref, bound = oracle.linear(x, q.numpy(), s.numpy(), 0.25)
    xd, qd, sd = x.reshape(-1).cuda(), q.cuda(), s.cuda()
    gd = torch.tensor([0.25], device="cuda")
    y = torch.zeros((N,), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        nv.gemv(xd, qd, sd, gd, y)  # warm-up outside capture
    stream.synchronize()
    y.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        nv.gemv(xd, qd, sd, gd, y)
    graph.replay()
    torch.cuda.synchronize()
    assert_within_tolerance(y, y_ref[0], bound[0], "graph")


@pytest.mark.parametrize("N,K", [(600, 5120), (130, 17408), (40, 1040)])
@pytest.mark.parametrize("kind", ["wide", "tiny", "zero"])
def test_x_dynamic_range_paths(nv, N, K, kind):
    """x whose non-zero magnitudes span more than 2^32 takes the exact fp32
    path; tiny-but-narrow x takes the scaled f16 path; all-zero x gives 0."""
    q, s = workloads.random_codes(N, K, 13)
    x = workloads.random_bf16((1, K), 14).float()
    if kind == "wide":
        x[0, 0] = 2.0 ** 100
        x[0, 1] = -(2.0 ** -60)
        x[0, 7] = 3.0e-30
    elif kind == "tiny":
        x = x * 2.0 ** -120          # BF16 subnormals and tiny normals, narrow range
    else:
        x = x * 0.0
    x = x.to(torch.bfloat16)
    y_ref, bound = oracle.linear(x, q.numpy(), s.numpy(), 0.75)
    y = _run(nv, x, q.numpy(), s.numpy(), 0.75)
    assert_within_tolerance(y, y_ref[0], bound[0], f"{kind} N={N} K={K}")
    if kind == "zero":
        assert not y.float().abs().sum().item()


def test_static_weights_chain_in_graph(nv):
    """Eight GEMVs back to back in one CUDA graph with static weights (programmatic
    dependent launch), each feeding the next one's x: every output must match the
    oracle run on the previous output."""
    N = K = 5120
    q, s, g = oracle.quantize(workloads.to_bf16(workloads.plain_weight_f32(N, K, 31)))
    qd, sd = torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda()
    gd = torch.tensor([float(g)], device="cuda")
    x0 = workloads.random_bf16((K,), 32).cuda()
    ys = [torch.empty((N,), dtype=torch.bfloat16, device="cuda") for _ in range(8)]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        nv.gemv(x0, qd, sd, gd, ys[0], static_weights=True)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        prev = x0
        for y in ys:
            nv.gemv(prev, qd, sd, gd, y, static_weights=True)
            prev = y
    graph.replay()
    torch.cuda.synchronize()
    prev = x0.cpu()
    for i, y in enumerate(ys):
        y_ref, bound = oracle.linear(prev.reshape(1, -1), q, s, g)
        assert_within_tolerance(y, y_ref[0], bound[0], f"chain {i}")
        prev = y.cpu()


def test_quantize_then_gemv_same_stream(nv):
    """The quantizer writes q, s, g and the GEMV (no static-weights flag) reads them
    right after on the same stream: stream order must hold."""
    N, K = 2048, 5120
    w = workloads.random_bf16((N, K), 33, 0.02).cuda()
    x = workloads.random_bf16((K,), 34).cuda()
    q = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    s = torch.empty((N, K // 16), dtype=torch.uint8, device="cuda")
    g = torch.empty((1,), dtype=torch.float32, device="cuda")
    y = torch.empty((N,), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        q.fill_(0); s.fill_(0)
        nv.quantize(w, q, s, g)
        nv.gemv(x, q, s, g, y)
    torch.cuda.synchronize()
    q_ref, s_ref, g_ref = oracle.quantize(w.cpu())
    y_ref, bound = oracle.linear(x.cpu().reshape(1, -1), q_ref, s_ref, g_ref)
    assert_within_tolerance(y, y_ref[0], bound[0], "quantize->gemv")


@pytest.mark.parametrize("N,K", [(148 * 120 + 7, 2048),   # two row blocks per CTA
                                 (148 * 118 + 1, 1024),   # short last CTA
                                 (333, 1280),             # last 256-byte column half past K
                                 (3, 768), (1, 256),
                                 (500, 11520),            # largest K of the shared-memory ring
                                 (64, 11776)])            # next multiple of 256: register kernel
@pytest.mark.parametrize("static", [False, True])
def test_ring_shapes(nv, N, K, static):
    """Shapes at the edges of the TMA-ring GEMV (K a multiple of 256): rows
    split over the SMs in one or more blocks, ragged last blocks and columns,
    both weight-ordering flags; the device error counter stays clear."""
    q, s = workloads.random_codes(N, K, 3 * N + K)
    x = workloads.random_bf16((1, K), N + 5 * K)
    g = np.float32(0.011)
    y_ref, bound = oracle.linear(x, q.numpy(), s.numpy(), g)
    xd = x.reshape(-1).cuda()
    qd, sd = q.cuda(), s.cuda()
    gd = torch.tensor([float(g)], dtype=torch.float32, device="cuda")
    y, check = guarded_empty((N,), torch.bfloat16)
    nv.gemv(xd, qd, sd, gd, y, static_weights=static)
    check()
    assert_within_tolerance(y, y_ref[0], bound[0], f"N={N} K={K} static={static}")
    nv.check_device_errors()
