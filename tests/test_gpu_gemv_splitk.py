"""Split-K decode GEMV ("K-parallel" decode GEMV of imp docs/quantization.md,
"Dense layers" pipeline): the CTAs of a thread-block cluster each take a range
of 512-element columns of K for the same rows and add their fp32 partials in
rank order.  Checked against the oracle within |y - y_ref| <= 1e-3 * sum|w x|
+ 1e-2 * |y_ref| per output, for the library's own choice of split and for
every forced split on ragged shapes (uneven column shares, a half column at
the end of K, a last row block shorter than the others), both weight formats,
x on the exact fp32 path in some CTAs of a cluster and the scaled f16 path in
others, chained launches in a CUDA graph, and bit-for-bit repeatability."""
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


def _dev(q_np, s_np, g=None):
    q = torch.from_numpy(np.ascontiguousarray(q_np)).cuda()
    s = torch.from_numpy(np.ascontiguousarray(s_np)).cuda()
    gd = None if g is None else torch.tensor([float(np.float32(g))], dtype=torch.float32, device="cuda")
    return q, s, gd


def _gemv(nv, x_cpu, q_np, s_np, g, k_split=0, static=False):
    q, s, gd = _dev(q_np, s_np, g)
    y, check = guarded_empty((q_np.shape[0],), torch.bfloat16)
    nv.gemv(x_cpu.reshape(-1).cuda(), q, s, gd, y, k_split=k_split, static_weights=static)
    check()
    nv.check_device_errors()
    return y


def test_down_projection_full(nv):
    """The 27B MLP down projection N=5120, K=17408 (weights from the layer
    generator, quantized by the oracle), every output, with the library's
    own split and with each split that fits."""
    cfg = workloads.CONFIGS["down"]
    q, s, g = oracle.quantize(workloads.weight_bf16(cfg))
    x = workloads.activations(1, cfg.K, cfg.seed)
    y_ref, bound = oracle.linear(x, q, s, g)
    for k_split in (0, 2, 4, 8):
        y = _gemv(nv, x, q, s, g, k_split)
        assert_within_tolerance(y, y_ref[0], bound[0], f"down projection k_split={k_split}")


@pytest.mark.parametrize("N,K", [(130, 11520),    # 22.5 columns: ragged shares, half column at the end
                                 (1000, 4352),    # 8.5 columns
                                 (7, 40960),      # fewer rows than CTAs of a row block would want
                                 (148 * 70 + 3, 2048),  # last cluster with 3 rows
                                 (333, 4096)])
@pytest.mark.parametrize("k_split", [1, 2, 4, 8])
def test_forced_splits_ragged(nv, N, K, k_split):
    q, s = workloads.random_codes(N, K, 5 * N + K)
    x = workloads.random_bf16((1, K), N + 3 * K)
    g = np.float32(0.0093)
    y_ref, bound = oracle.linear(x, q.numpy(), s.numpy(), g)
    cols = -(-K // 512)
    if k_split > cols or (k_split > 1 and -(-cols // k_split) * 512 > 11520):
        pytest.skip("fewer 512-element columns than CTAs, or an x slice over 11520 elements per CTA")
    # (k_split=1 with K beyond one CTA's x slice runs the register kernel)
    y = _gemv(nv, x, q.numpy(), s.numpy(), g, k_split)
    assert_within_tolerance(y, y_ref[0], bound[0], f"N={N} K={K} k_split={k_split}")


@pytest.mark.parametrize("N,K", [(700, 8192), (5120, 17408)])
@pytest.mark.parametrize("k_split", [0, 2, 8])
def test_mxfp4_splits(nv, N, K, k_split):
    w = workloads.random_bf16((N, K), N + K, 0.02)
    q, s = oracle.mx_quantize(w)
    x = workloads.random_bf16((1, K), 2 * N + K)
    y_ref, bound = oracle.mx_linear(x, q, s)
    qd, sd, _ = _dev(q, s)
    y, check = guarded_empty((N,), torch.bfloat16)
    nv.mx_gemv(x.reshape(-1).cuda(), qd, sd, y, k_split=k_split)
    check()
    nv.check_device_errors()
    assert_within_tolerance(y, y_ref[0], bound[0], f"MXFP4 N={N} K={K} k_split={k_split}")


@pytest.mark.parametrize("kind", ["wide_first", "wide_last", "tiny", "zero"])
@pytest.mark.parametrize("k_split", [2, 4])
def test_x_paths_inside_a_cluster(nv, kind, k_split):
    """Each CTA decides on its own x slice: a wide range in the first (or last)
    slice sends that CTA to the exact fp32 path while the others stay on the
    scaled f16 path; their partials still add up."""
    N, K = 600, 16384
    q, s = workloads.random_codes(N, K, 41)
    x = workloads.random_bf16((1, K), 42).float()
    if kind == "wide_first":
        x[0, 3] = 2.0 ** 90
        x[0, 5] = -(2.0 ** -70)
    elif kind == "wide_last":
        x[0, K - 2] = -(2.0 ** 80)
        x[0, K - 9] = 2.0 ** -75
    elif kind == "tiny":
        x = x * 2.0 ** -118
    else:
        x = x * 0.0
    x = x.to(torch.bfloat16)
    y_ref, bound = oracle.linear(x, q.numpy(), s.numpy(), 0.5)
    y = _gemv(nv, x, q.numpy(), s.numpy(), 0.5, k_split)
    assert_within_tolerance(y, y_ref[0], bound[0], f"{kind} k_split={k_split}")
    if kind == "zero":
        assert not y.float().abs().sum().item()


def test_deterministic(nv):
    """The cluster adds partials in rank order: repeated calls agree bit for bit."""
    cfg = workloads.CONFIGS["down"]
    q, s = workloads.random_codes(cfg.N, cfg.K, 51)
    x = workloads.random_bf16((cfg.K,), 52).cuda()
    qd, sd, gd = _dev(q.numpy(), s.numpy(), 0.02)
    ys = []
    for _ in range(5):
        y = torch.empty((cfg.N,), dtype=torch.bfloat16, device="cuda")
        nv.gemv(x, qd, sd, gd, y, k_split=4)
        ys.append(y)
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y.view(torch.int16), ys[0].view(torch.int16))


def test_static_weights_chain_in_graph(nv):
    """Down projection then up projection and back, eight split-K and plain
    GEMVs alternating in one CUDA graph with programmatic dependent launch,
    each feeding the next one's x."""
    K1, N1 = 4096, 12288   # [12288, 4096] then [4096, 12288]: split-K on the second
    q1, s1, g1 = oracle.quantize(workloads.to_bf16(workloads.plain_weight_f32(N1, K1, 61)))
    q2, s2, g2 = oracle.quantize(workloads.to_bf16(workloads.plain_weight_f32(K1, N1, 62)))
    d1, d2 = _dev(q1, s1, g1), _dev(q2, s2, g2)
    x0 = workloads.random_bf16((K1,), 63).cuda()
    ys = [torch.empty((N1 if i % 2 == 0 else K1,), dtype=torch.bfloat16, device="cuda") for i in range(8)]
    stream = torch.cuda.Stream()

    def chain():
        prev = x0
        for i, y in enumerate(ys):
            q, s, g = d1 if i % 2 == 0 else d2
            nv.gemv(prev, q, s, g, y, static_weights=True, k_split=0 if i % 2 == 0 else 4)
            prev = y

    with torch.cuda.stream(stream):
        chain()
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        chain()
    for y in ys:
        y.zero_()
    graph.replay()
    torch.cuda.synchronize()
    nv.check_device_errors()
    prev = x0.cpu()
    for i, y in enumerate(ys):
        q, s, g = (q1, s1, g1) if i % 2 == 0 else (q2, s2, g2)
        y_ref, bound = oracle.linear(prev.reshape(1, -1), q, s, g)
        assert_within_tolerance(y, y_ref[0], bound[0], f"chain {i}")
        prev = y.cpu()


def test_split_that_does_not_fit_is_rejected(nv):
    """Forced splits with too few columns, with an x slice beyond one CTA's
    11520 elements, or with K % 256 != 0 are refused before any launch."""
    q, s = workloads.random_codes(64, 1024, 71)     # 2 columns of 512: a split of 4 cannot fit
    qd, sd, gd = _dev(q.numpy(), s.numpy(), 1.0)
    x = torch.zeros((1024,), dtype=torch.bfloat16, device="cuda")
    y = torch.full((64,), 7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.Nvfp4Error, match="NVFP4_ERR_SHAPE"):
        nv.gemv(x, qd, sd, gd, y, k_split=4)
    q2, s2 = workloads.random_codes(64, 1040, 72)   # K % 256 != 0: no split at all
    qd2, sd2, _ = _dev(q2.numpy(), s2.numpy())
    with pytest.raises(nv.Nvfp4Error, match="NVFP4_ERR_SHAPE"):
        nv.gemv(torch.zeros((1040,), dtype=torch.bfloat16, device="cuda"), qd2, sd2, gd, y, k_split=2)
    q3, s3 = workloads.random_codes(64, 40960, 73)  # a split of 2 leaves 20480 elements of x per CTA
    qd3, sd3, _ = _dev(q3.numpy(), s3.numpy())
    with pytest.raises(nv.Nvfp4Error, match="11520"):
        nv.gemv(torch.zeros((40960,), dtype=torch.bfloat16, device="cuda"), qd3, sd3, gd, y, k_split=2)
    torch.cuda.synchronize()
    assert bool((y.float() == 7.0).all())
