"""Pins of the CPU oracle against facts the NVFP4 format fixes.

Nothing here compares the oracle with itself: each check uses the pages'
printed values (tests/golden), a library cast (ml_dtypes), a brute-force
restatement on tiny inputs, a closed form, or an exact round trip.
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
import workloads

F4 = ml_dtypes.float4_e2m1fn
F8 = ml_dtypes.float8_e4m3fn


def _read_golden(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ------------------------------------------------------------------ decode

def test_e2m1_table_matches_pages(golden_dir):
    rows = _read_golden(os.path.join(golden_dir, "e2m1_values.txt"))
    assert len(rows) == 16
    for code, val in rows:
        got = oracle.e2m1_decode(int(code))
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))
    lib_vals = np.arange(16, dtype=np.uint8).view(F4).astype(np.float64)
    for c in range(16):
        assert oracle.e2m1_decode(c) == lib_vals[c]
        assert math.copysign(1, oracle.e2m1_decode(c)) == math.copysign(1, lib_vals[c])
    mags = sorted({abs(oracle.e2m1_decode(c)) for c in range(16)})
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e4m3_decode_all_bytes():
    lib_vals = np.arange(256, dtype=np.uint8).view(F8).astype(np.float64)
    for b in range(256):
        got = oracle.e4m3_decode(b)
        if np.isnan(lib_vals[b]):
            assert math.isnan(got), hex(b)
        else:
            assert got == lib_vals[b], hex(b)
            assert math.copysign(1, got) == math.copysign(1, lib_vals[b])


def test_e4m3_facts(golden_dir):
    for byte, val in _read_golden(os.path.join(golden_dir, "e4m3_facts.txt")):
        got = oracle.e4m3_decode(int(byte, 16))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val), byte
    finite = [oracle.e4m3_decode(b) for b in range(256) if not math.isnan(oracle.e4m3_decode(b))]
    assert max(finite) == 448.0 and min(finite) == -448.0
    assert min(v for v in finite if v > 0) == 2.0 ** -9


def test_packed_byte_decode_all_256():
    """Every byte 0x00..0xFF as one row: low nibble is element 2b, high 2b+1."""
    q = np.arange(256, dtype=np.uint8).reshape(1, 256)
    s = np.full((1, 32), 0x38, np.uint8)  # E4M3 1.0
    w = oracle.dequantize(q, s, 1.0)
    lib_vals = np.arange(16, dtype=np.uint8).view(F4).astype(np.float64)
    for b in range(256):
        assert w[0, 2 * b] == lib_vals[b & 15]
        assert w[0, 2 * b + 1] == lib_vals[b >> 4]


# ---------------------------------------------------------------- rounding

def _near(values, ulps):
    """fp32 values within +-ulps of each given fp32 value (both signs of offset)."""
    v = np.asarray(values, np.float32).view(np.int32).astype(np.int64)
    off = np.arange(-ulps, ulps + 1, dtype=np.int64)
    out = (v[:, None] + off[None, :]).reshape(-1)
    out = out[(out >= 0) & (out < 0x7F800000)]
    return np.unique(out.astype(np.int32)).view(np.float32)


def test_e4m3_rounding_matches_library_cast():
    vals = np.arange(0x7F, dtype=np.uint8).view(F8).astype(np.float64)  # 0 .. 448
    mids = (vals[:-1] + vals[1:]) / 2
    pts = np.concatenate([_near(vals, 6), _near(mids, 6)])
    r = np.random.default_rng(11)
    pts = np.concatenate([pts, (2.0 ** r.uniform(-13, 8.8, 100000)).astype(np.float32)])
    pts = pts[pts <= 448.0]
    expect = pts.astype(F8).view(np.uint8)
    got = np.array([oracle.e4m3_rne_satfinite(float(p)) for p in pts], np.uint8)
    bad = np.nonzero(got != expect)[0]
    assert bad.size == 0, [(float(pts[i]), hex(got[i]), hex(expect[i])) for i in bad[:5]]


def test_e4m3_saturation():
    for v in [448.0, 448.5, 464.0, 465.0, 1e6, 3.0e38, float("inf")]:
        assert oracle.e4m3_rne_satfinite(v) == 0x7E
    assert oracle.e4m3_rne_satfinite(2.0 ** -10) == 0x00      # tie -> even (zero)
    assert oracle.e4m3_rne_satfinite(1.5 * 2.0 ** -9) == 0x02  # tie -> even


def test_e2m1_rounding_points(golden_dir):
    for v, code in _read_golden(os.path.join(golden_dir, "e2m1_rounding_points.txt")):
        assert oracle.e2m1_rne_satfinite(float(v)) == int(code), v


def test_e2m1_rounding_matches_library_cast():
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    mids = (mags[:-1] + mags[1:]) / 2
    pts = np.concatenate([_near(mags[1:], 8), _near(mids, 8)])
    r = np.random.default_rng(12)
    pts = np.concatenate([pts, r.uniform(0, 7, 100000).astype(np.float32),
                          (2.0 ** r.uniform(-30, 3, 20000)).astype(np.float32)])
    pts = np.concatenate([pts, -pts])
    expect = pts.astype(F4).view(np.uint8) & 15
    got = np.array([oracle.e2m1_rne_satfinite(float(p)) for p in pts], np.uint8)
    bad = np.nonzero(got != expect)[0]
    assert bad.size == 0, [(float(pts[i]), got[i], expect[i]) for i in bad[:5]]
    for v in [6.0, 6.01, 100.0, 3e38, float("inf")]:
        assert oracle.e2m1_rne_satfinite(v) == 7
        assert oracle.e2m1_rne_satfinite(-v) == 15


# ---------------------------------------------------------- quantizer pins

def _quantize_restated(w_bf16: torch.Tensor, g: np.float32):
    """Independent restatement of the quantizer with ml_dtypes casts doing the
    rounding (E4M3 cast after clipping at 448; the E2M1 cast saturates)."""
    w = w_bf16.float().numpy()
    N, K = w.shape
    blocks = w.reshape(N, K // 16, 16)
    amax_b = np.abs(blocks).max(axis=2).astype(np.float32)
    if g == 0:
        s = np.zeros((N, K // 16), np.uint8)
    else:
        s_f = (amax_b / np.float32(6.0)) / np.float32(g)
        s = np.minimum(s_f, np.float32(448.0)).astype(F8).view(np.uint8)
    d = s.view(F8).astype(np.float32) * np.float32(g)
    with np.errstate(divide="ignore"):
        r = np.float32(1.0) / d
    with np.errstate(invalid="ignore", over="ignore"):
        prod = blocks * r[:, :, None]
    codes = prod.astype(F4).view(np.uint8) & 15
    zero_in = blocks == 0
    codes = np.where(zero_in, np.where(np.signbit(blocks), 8, 0), codes)
    codes = np.where((d == 0)[:, :, None], 0, codes).astype(np.uint8).reshape(N, K)
    q = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return q, s


@pytest.mark.parametrize("seed,shape,std", [(0, (32, 256), 0.02), (1, (7, 96), 1.0),
                                            (2, (64, 64), 3e-5), (3, (16, 1024), 50.0)])
def test_quantize_matches_restatement(seed, shape, std):
    w = workloads.random_bf16(shape, seed, std)
    wf = w.float()
    # plant outliers, an all-zero block, negative zeros and a tiny block
    wf[0, 5] *= 40
    wf[1, 16:32] = 0.0
    wf[2, 0:16] = -0.0
    wf[3, 32:48] *= 1e-6
    w = wf.to(torch.bfloat16)
    q, s, g = oracle.quantize(w)
    q2, s2 = _quantize_restated(w, g)
    np.testing.assert_array_equal(s, s2)
    np.testing.assert_array_equal(q, q2)


def test_quantize_shared_g_restatement():
    w = workloads.random_bf16((24, 160), 5, 0.1)
    for g in [np.float32(1e-4), np.float32(3.3e-3), np.float32(0.0)]:
        q, s, _ = oracle.quantize(w, g)
        q2, s2 = _quantize_restated(w, g)
        np.testing.assert_array_equal(s, s2)
        np.testing.assert_array_equal(q, q2)


def test_amax_and_tensor_scale():
    w = workloads.random_bf16((33, 48), 7, 0.5)
    a = oracle.amax(w)
    assert a == np.float32(np.abs(w.float().numpy()).max())
    assert oracle.tensor_scale(a) == np.float32(a) / np.float32(2688.0)
    assert oracle.tensor_scale(0.0) == 0.0


def _exact_weights(N, K, seed, k_exp=12):
    """W whose every element is code * E4M3 * 2^-k_exp with a +-6 element in every
    block and a 448 scale in block (0, 0): quantizing it must give back exactly
    the codes and scales it was built from."""
    r = np.random.default_rng(seed)
    g = np.float32(2.0 ** -k_exp)
    codes = r.integers(0, 16, size=(N, K), dtype=np.uint8)
    scales = r.integers(1, 0x7F, size=(N, K // 16), dtype=np.uint8)  # finite, non-zero
    scales[0, 0] = 0x7E
    pos = r.integers(0, 16, size=(N, K // 16))
    for n in range(N):
        for b in range(K // 16):
            codes[n, b * 16 + pos[n, b]] = 7 if r.random() < 0.5 else 15
    cv = np.arange(16, dtype=np.uint8).view(F4).astype(np.float64)[codes]
    sv = scales.view(F8).astype(np.float64)
    w = cv * np.repeat(sv, 16, axis=1) * float(g)
    wt = torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(wt.double().numpy(), w)  # exactly representable in BF16
    q = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return wt, q, scales, g, w


def test_round_trip_exact():
    wt, q_ref, s_ref, g_ref, w = _exact_weights(12, 128, 3)
    q, s, g = oracle.quantize(wt)
    assert g == g_ref
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_array_equal(q, q_ref)
    deq = oracle.dequantize(q, s, g)
    assert np.array_equal(deq, w)


def test_shared_scale_merged_layer():
    """Merged q/k/v + gate/up share one tensor scale (model card, paragraph after
    the 'What is quantized' table): quantizing the stack equals stacking the
    members quantized with the shared g, and the shared g comes from the max of
    the members' amaxes."""
    K = 64
    members = workloads.merged_members(9, K=K, rows=(8, 8, 8, 16, 16))
    stack = torch.cat(members, 0)
    amaxes = [oracle.amax(m) for m in members]
    spread = max(amaxes) / min(amaxes)
    assert 3.5 < spread < 3.9
    g_shared = oracle.tensor_scale(max(amaxes))
    assert g_shared == oracle.tensor_scale(oracle.amax(stack))
    qs, ss, _ = oracle.quantize(stack, g_shared)
    parts = [oracle.quantize(m, g_shared) for m in members]
    np.testing.assert_array_equal(qs, np.concatenate([p[0] for p in parts]))
    np.testing.assert_array_equal(ss, np.concatenate([p[1] for p in parts]))

    # negative control: member k quantized against its own g, but dequantized
    # with the shared g (what an engine keeping one scale would do) fails
    x = workloads.random_bf16((1, K), 1)
    k_idx = 1
    qk, sk, gk = oracle.quantize(members[k_idx])
    assert gk != g_shared
    y_right, bound = oracle.linear(x, qk, sk, gk)
    y_wrong, _ = oracle.linear(x, qk, sk, g_shared)
    err = np.abs(y_wrong - y_right)
    assert np.any(err > oracle.tolerance(y_right, bound))


# ------------------------------------------------------- linear (GEMV/GEMM)

def _naive_linear(x_bf16, q, s, g):
    """Triple loop over values decoded by the library casts (not the oracle)."""
    f4 = np.arange(16, dtype=np.uint8).view(F4).astype(np.float64)
    f8 = np.arange(256, dtype=np.uint8).view(F8).astype(np.float64)
    x = x_bf16.double().numpy()
    M, K = x.shape
    N = q.shape[0]
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                byte = int(q[n, k // 2])
                code = byte & 15 if k % 2 == 0 else byte >> 4
                acc += float(g) * f8[s[n, k // 16]] * f4[code] * x[m, k]
            y[m, n] = acc
    return y


@pytest.mark.parametrize("M,N,K,seed", [(1, 5, 16, 0), (3, 7, 48, 1), (4, 16, 64, 2), (2, 33, 32, 3)])
def test_linear_brute_force(M, N, K, seed):
    q, s = workloads.random_codes(N, K, seed)
    q, s = q.numpy(), s.numpy()
    x = workloads.random_bf16((M, K), seed + 100)
    g = np.float32(0.0123)
    y, bound = oracle.linear(x, q, s, g)
    y_naive = _naive_linear(x, q, s, g)
    np.testing.assert_allclose(y, y_naive, rtol=1e-12, atol=1e-12)
    assert np.all(bound >= np.abs(y) - 1e-12)
    # sampled-output entry point agrees with the full one
    rows = np.array([M - 1, 0], np.int64)
    cols = np.array([0, N - 1], np.int64)
    ys, bs = oracle.linear(x, q, s, g, rows, cols)
    np.testing.assert_array_equal(ys, y[rows, cols])
    np.testing.assert_array_equal(bs, bound[rows, cols])


def test_linear_one_hot_and_ones():
    N, K = 9, 64
    q, s = workloads.random_codes(N, K, 4)
    q, s = q.numpy(), s.numpy()
    g = np.float32(0.5)
    deq = oracle.dequantize(q, s, g)
    eye = torch.eye(K, dtype=torch.bfloat16)
    y, _ = oracle.linear(eye, q, s, g)
    np.testing.assert_array_equal(y, deq.T)  # one-hot x returns a column of W
    ones = torch.ones((1, K), dtype=torch.bfloat16)
    y1, _ = oracle.linear(ones, q, s, g)
    np.testing.assert_array_equal(y1[0], deq.sum(axis=1))


def test_linear_exact_small_integers():
    wt, q, s, g, w = _exact_weights(6, 64, 8, k_exp=0)
    x = torch.from_numpy(np.random.default_rng(3).integers(-8, 9, size=(2, 64)).astype(np.float32)).to(torch.bfloat16)
    y, _ = oracle.linear(x, q, s, g)
    # every product and partial sum is an exact dyadic rational -> exact in fp64
    y_exact = x.double().numpy() @ w.T
    assert np.array_equal(y, y_exact)


def test_tolerance_form():
    y = np.array([1.0, -2.0])
    b = np.array([10.0, 4.0])
    np.testing.assert_allclose(oracle.tolerance(y, b), [1e-2 + 1e-2, 4e-3 + 2e-2])
