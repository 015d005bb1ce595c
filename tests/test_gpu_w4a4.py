"""GPU W4A4 (NVFP4 x NVFP4) prefill path against the oracle: the weight-scale
rearrangement and the activation quantizer bit-exact, the block-scaled FP4
GEMM within 1e-3 * sum|x_deq w_deq| + 1e-2 * |y_ref| of the oracle's W4A4
product (imp docs/quantization.md, dense-layer prefill "CUTLASS NVFP4 GEMM";
activations quantized by the weights' rule, g_x = amax / 2688)."""
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


def mma_layout(s: np.ndarray, pad: int) -> np.ndarray:
    """Row-major scales [R, K/16] -> the tensor-core scale layout stated in
    include/nvfp4_w4a4.h (rows padded with zeros to a multiple of `pad`)."""
    R, nb = s.shape
    Rp = (R + pad - 1) // pad * pad
    sp = np.zeros((Rp, nb), np.uint8)
    sp[:R] = s
    steps = nb // 4
    out = np.zeros(Rp * nb, np.uint8)
    r = np.arange(Rp)[:, None]
    b = np.arange(nb)[None, :]
    off = ((r // 128) * steps + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4
    out[off.ravel()] = sp.ravel()
    return out


def from_mma_layout(flat: np.ndarray, R: int, K: int, pad: int) -> np.ndarray:
    Rp = (R + pad - 1) // pad * pad
    nb = K // 16
    r = np.arange(Rp)[:, None]
    b = np.arange(nb)[None, :]
    off = ((r // 128) * (nb // 4) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4
    return flat[off]


def test_layout_helpers_are_inverse():
    s = np.random.default_rng(0).integers(0, 256, (300, 32), dtype=np.uint8)
    back = from_mma_layout(mma_layout(s, 256), 300, 512, 256)
    assert np.array_equal(back[:300], s) and not back[300:].any()


@pytest.mark.parametrize("N,K", [(17408, 5120), (300, 512), (1, 256), (128, 1024)])
def test_prepare_weights_layout(nv, N, K):
    s = np.random.default_rng(N + K).integers(0, 256, (N, K // 16), dtype=np.uint8)
    out = nv.w4a4_prepare_weights(torch.from_numpy(s).cuda(), K)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), mma_layout(s, 128))


@pytest.mark.parametrize("M,K", [(512, 5120), (300, 512), (1, 256), (257, 1024)])
def test_quantize_x_bit_exact(nv, M, K):
    X = workloads.activations(M, K, M + K)
    amax = torch.empty((nv.AMAX_FLOATS,), dtype=torch.float32, device="cuda")
    qx, sx = nv.w4a4_quantize_x(X.cuda(), amax)
    torch.cuda.synchronize()
    q_ref, s_ref, g_ref = oracle.quantize(X, oracle.tensor_scale(oracle.amax(X)))
    assert amax[0].item() == float(oracle.amax(X))
    assert np.array_equal(qx.cpu().numpy(), q_ref)
    got = from_mma_layout(sx.cpu().numpy(), M, K, 256)
    assert np.array_equal(got[:M], s_ref) and not got[M:].any()


def test_quantize_x_given_amax_and_strided_rows(nv):
    """A calibrated amax below max |X| (saturating codes) and rows of a wider tensor."""
    wide = workloads.activations(96, 1536, 3)
    X = wide[:, 256:256 + 1024]
    given = float(oracle.amax(X.contiguous())) / 3
    amax = torch.tensor([given], dtype=torch.float32, device="cuda")
    qx, sx = nv.w4a4_quantize_x(wide.cuda()[:, 256:256 + 1024], amax, given_amax=True)
    torch.cuda.synchronize()
    q_ref, s_ref, _ = oracle.quantize(X.contiguous(), oracle.tensor_scale(given))
    assert amax.item() == np.float32(given)
    assert np.array_equal(qx.cpu().numpy(), q_ref)
    assert np.array_equal(from_mma_layout(sx.cpu().numpy(), 96, 1024, 256)[:96], s_ref)


def _run(nv, X, q, s, g, x_amax=None, static=False, pair=False):
    M, K = X.shape
    N = q.shape[0]
    qd, sd = torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda()
    gd = torch.tensor([g], dtype=torch.float32, device="cuda")
    s_mma = nv.w4a4_prepare_weights(sd, K)
    ws = torch.empty((nv.w4a4_workspace_size(M, K),), dtype=torch.uint8, device="cuda")
    Y, check = guarded_empty((M, N), torch.bfloat16)
    am = None if x_amax is None else torch.tensor([x_amax], dtype=torch.float32, device="cuda")
    nv.w4a4_linear(X.cuda(), qd, s_mma, gd, Y, ws, x_amax=am, static_weights=static, pair=pair)
    check()
    nv.check_device_errors()
    return Y


@pytest.mark.parametrize("pair", [False, True], ids=["sm", "pair"])
@pytest.mark.parametrize("M,N,K", [(256, 256, 1024),   # one tile, four stages
                                   (300, 1000, 2048),  # ragged M and N tiles, a ring wrap
                                   (1, 130, 256),      # one token, one stage
                                   (40, 384, 1280),    # five stages on a four-stage ring
                                   (40, 1100, 1536),   # pairs: the last pair's odd CTA is past N
                                   (513, 128, 512)])   # three token tiles
def test_w4a4_gemm_vs_oracle(nv, M, N, K, pair):
    X = workloads.activations(M, K, 7 * M + K)
    q, s, g = oracle.quantize(workloads.random_bf16((N, K), N + K))
    Y = _run(nv, X, q, s, g, pair=pair)
    y_ref, bound, _ = oracle.w4a4_linear(X, q, s, g)
    assert_within_tolerance(Y, y_ref, bound, f"w4a4 M={M} N={N} K={K} pair={pair}")


@pytest.mark.parametrize("M,N,K", [(300, 1100, 2048), (512, 2048, 5120)])
def test_w4a4_pair_tiles_equal_single(nv, M, N, K):
    """Tiles on pairs of SMs form the same products and fp32 sums per output
    as tiles on one SM: the outputs agree bit for bit."""
    X = workloads.activations(M, K, M + 3 * K)
    q, s, g = oracle.quantize(workloads.random_bf16((N, K), N + 5))
    Y1 = _run(nv, X, q, s, g, pair=False)
    Y2 = _run(nv, X, q, s, g, pair=True)
    assert torch.equal(Y1, Y2)


@pytest.mark.parametrize("pair", [False, True], ids=["sm", "pair"])
def test_w4a4_full_size_sampled(nv, pair):
    """The 27B-class prefill layer: M = 512 tokens, W [17408, 5120]."""
    cfg = workloads.CONFIGS["prefill"]
    M, N, K = cfg.M, cfg.N, cfg.K
    w = workloads.weight_bf16(cfg)
    q, s, g = oracle.quantize(w)
    X = workloads.activations(M, K, cfg.seed + 1)
    Y = _run(nv, X, q, s, g, static=True, pair=pair)
    rng = np.random.default_rng(5)
    rows, cols = rng.integers(0, M, 600), rng.integers(0, N, 600)
    y_ref, bound, _ = oracle.w4a4_linear(X, q, s, g, rows=rows, cols=cols)
    assert_within_tolerance(Y.cpu()[rows, cols], y_ref, bound, "w4a4 512 x 17408 x 5120")


def test_w4a4_given_amax(nv):
    M, N, K = 64, 256, 512
    X = workloads.activations(M, K, 11)
    q, s, g = oracle.quantize(workloads.random_bf16((N, K), 12))
    given = float(oracle.amax(X)) * 0.5
    Y = _run(nv, X, q, s, g, x_amax=given)
    y_ref, bound, _ = oracle.w4a4_linear(X, q, s, g, x_amax=given)
    assert_within_tolerance(Y, y_ref, bound, "w4a4 calibrated amax")


def test_w4a4_exact_on_representable_inputs(nv):
    """X that NVFP4 holds exactly (g_x = 2^-6, block scales 64 and 448): the
    oracle's dequantized X is X itself, and the GEMM agrees with it."""
    rng = np.random.default_rng(13)
    M, N, K = 64, 128, 256
    e2m1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    x = rng.choice(e2m1, (M, K)) * rng.choice([-1.0, 1.0], (M, K))
    x[:, ::16] = 6.0
    x[0, 0] = 6.0 * 448.0 / 64.0      # tensor max 2688 / 64: g_x = 2^-6
    x[0, 1:16] = 0.0
    X = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    q, s, g = oracle.quantize(workloads.random_bf16((N, K), 14))
    Y = _run(nv, X, q, s, g)
    y_ref, bound, (qx, sx, g_x) = oracle.w4a4_linear(X, q, s, g)
    assert np.array_equal(oracle.dequantize(qx, sx, g_x), x)
    assert_within_tolerance(Y, y_ref, bound, "w4a4 representable")


def test_w4a4_graph_replay_and_static_flag(nv):
    M, N, K = 256, 512, 1024
    X = workloads.activations(M, K, 21).cuda()
    q, s, g = oracle.quantize(workloads.random_bf16((N, K), 22))
    qd, sd = torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda()
    gd = torch.tensor([g], dtype=torch.float32, device="cuda")
    s_mma = nv.w4a4_prepare_weights(sd, K)
    ws = torch.empty((nv.w4a4_workspace_size(M, K),), dtype=torch.uint8, device="cuda")
    Y0 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    nv.w4a4_linear(X, qd, s_mma, gd, Y0, ws)
    torch.cuda.synchronize()
    Y1 = torch.empty_like(Y0)
    st = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        nv.w4a4_linear(X, qd, s_mma, gd, Y1, ws, stream=st, static_weights=True)   # warm-up outside capture
        st.synchronize()
        with torch.cuda.graph(graph, stream=st):
            nv.w4a4_linear(X, qd, s_mma, gd, Y1, ws, stream=st, static_weights=True)
    Y1.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y0, Y1)
    nv.check_device_errors()
