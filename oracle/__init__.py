"""CPU oracle for the NVFP4 W4A16 linear layer (ctypes wrapper of nvfp4_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product library (``gemm_decode_nvfp4_b200``) never imports it and
has no CPU fallback.

The C file states what each function follows on the pages and the readings
taken where the pages are silent.  Every function here is pinned by the
``-m "not gpu"`` tests against facts the format fixes (the sixteen E2M1
values, E4M3 bit fields, library casts in ml_dtypes, brute force on tiny
inputs, exact round trips, the shared-scale identity).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB = os.path.join(_HERE, "libnvfp4_oracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp32 kept strict: no contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        c_i64, c_f, c_p = ctypes.c_int64, ctypes.c_float, ctypes.c_void_p
        L.oracle_e2m1_decode.argtypes = [ctypes.c_int]
        L.oracle_e2m1_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_int]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_rne_satfinite.argtypes = [c_f]
        L.oracle_e4m3_rne_satfinite.restype = ctypes.c_int
        L.oracle_e2m1_rne_satfinite.argtypes = [c_f]
        L.oracle_e2m1_rne_satfinite.restype = ctypes.c_int
        L.oracle_amax.argtypes = [c_p, c_i64, c_i64, c_i64]
        L.oracle_amax.restype = c_f
        L.oracle_tensor_scale.argtypes = [c_f]
        L.oracle_tensor_scale.restype = c_f
        L.oracle_quantize.argtypes = [c_p, c_i64, c_i64, c_i64, c_f, c_p, c_p]
        L.oracle_quantize.restype = None
        L.oracle_quantize_mse.argtypes = [c_p, c_i64, c_i64, c_i64, c_f, ctypes.c_int, c_p, c_p]
        L.oracle_quantize_mse.restype = None
        L.oracle_dequantize.argtypes = [c_p, c_p, c_f, c_i64, c_i64, c_p]
        L.oracle_dequantize.restype = None
        L.oracle_linear.argtypes = [c_p, c_i64, c_p, c_p, c_f, c_i64, c_i64, c_i64,
                                    c_p, c_p, c_i64, c_p, c_p]
        L.oracle_linear.restype = None
        L.oracle_e8m0_decode.argtypes = [ctypes.c_int]
        L.oracle_e8m0_decode.restype = ctypes.c_double
        L.oracle_mx_quantize.argtypes = [c_p, c_i64, c_i64, c_i64, c_p, c_p]
        L.oracle_mx_quantize.restype = None
        L.oracle_mx_dequantize.argtypes = [c_p, c_p, c_i64, c_i64, c_p]
        L.oracle_mx_dequantize.restype = None
        L.oracle_mx_linear.argtypes = [c_p, c_i64, c_p, c_p, c_i64, c_i64, c_i64,
                                       c_p, c_p, c_i64, c_p, c_p]
        L.oracle_mx_linear.restype = None
        L.oracle_num_threads.argtypes = []
        L.oracle_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(w) -> np.ndarray:
    """BF16 torch tensor (or uint16 array) -> contiguous uint16 numpy view."""
    if isinstance(w, np.ndarray):
        assert w.dtype == np.uint16
        return np.ascontiguousarray(w)
    import torch
    assert w.dtype == torch.bfloat16
    return np.ascontiguousarray(w.contiguous().view(torch.int16).numpy().view(np.uint16))


# ----------------------------------------------------------- scalar helpers

def e2m1_decode(code: int) -> float:
    return lib().oracle_e2m1_decode(int(code))


def e4m3_decode(byte: int) -> float:
    return lib().oracle_e4m3_decode(int(byte))


def e4m3_rne_satfinite(v: float) -> int:
    return lib().oracle_e4m3_rne_satfinite(float(np.float32(v)))


def e2m1_rne_satfinite(v: float) -> int:
    return lib().oracle_e2m1_rne_satfinite(float(np.float32(v)))


def num_threads() -> int:
    return lib().oracle_num_threads()


# ----------------------------------------------------------- tensor helpers

def amax(w) -> np.float32:
    """max |w| of a BF16 matrix (2-D) or vector."""
    b = _bf16_bits(w)
    if b.ndim == 1:
        b = b.reshape(1, -1)
    rows, cols = b.shape
    return np.float32(lib().oracle_amax(_ptr(b), rows, cols, cols))


def tensor_scale(a) -> np.float32:
    """g = amax / (6 * 448) in fp32."""
    return np.float32(lib().oracle_tensor_scale(float(np.float32(a))))


def quantize(w, g=None):
    """RTN NVFP4 of a BF16 [N, K] matrix.  Returns (q [N, K/2] u8, s [N, K/16] u8,
    g fp32).  g defaults to this tensor's own amax / 2688; pass the shared g of
    a merged layer to quantize one member."""
    b = _bf16_bits(w)
    N, K = b.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    if g is None:
        g = tensor_scale(amax(b))
    g = np.float32(g)
    q = np.empty((N, K // 2), np.uint8)
    s = np.empty((N, K // 16), np.uint8)
    lib().oracle_quantize(_ptr(b), N, K, K, float(g), _ptr(q), _ptr(s))
    return q, s, g


def quantize_mse(w, g=None, window: int = 8):
    """NVFP4 with each micro-scale chosen by the least squared reconstruction
    error over the E4M3 codes within `window` codes of the round-to-nearest
    one (imp docs/quantization.md, micro-scale search paragraph; readings in
    nvfp4_oracle.c).  Returns (q, s, g) like quantize; window 0 is quantize."""
    b = _bf16_bits(w)
    N, K = b.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    if g is None:
        g = tensor_scale(amax(b))
    g = np.float32(g)
    q = np.empty((N, K // 2), np.uint8)
    s = np.empty((N, K // 16), np.uint8)
    lib().oracle_quantize_mse(_ptr(b), N, K, K, float(g), int(window), _ptr(q), _ptr(s))
    return q, s, g


def dequantize(q: np.ndarray, s: np.ndarray, g) -> np.ndarray:
    """W_deq [N, K] in fp64."""
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    N, K = q.shape[0], q.shape[1] * 2
    out = np.empty((N, K), np.float64)
    lib().oracle_dequantize(_ptr(q), _ptr(s), float(np.float32(g)), N, K, _ptr(out))
    return out


def linear(x, q: np.ndarray, s: np.ndarray, g, rows=None, cols=None):
    """y = x . W^T in fp64 with the per-element magnitude bound sum |w x|.

    x is BF16 [M, K] (or [K]).  With rows/cols (equal-length index arrays) only
    those outputs are computed and 1-D arrays are returned; otherwise [M, N]."""
    xb = _bf16_bits(x)
    if xb.ndim == 1:
        xb = xb.reshape(1, -1)
    M, K = xb.shape
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    N = q.shape[0]
    assert q.shape[1] * 2 == K and s.shape == (N, K // 16)
    if rows is None:
        y = np.empty((M, N), np.float64)
        bound = np.empty((M, N), np.float64)
        lib().oracle_linear(_ptr(xb), K, _ptr(q), _ptr(s), float(np.float32(g)), M, N, K,
                            None, None, -1, _ptr(y), _ptr(bound))
        return y, bound
    ri = np.ascontiguousarray(rows, np.int64)
    ci = np.ascontiguousarray(cols, np.int64)
    assert ri.shape == ci.shape and ri.ndim == 1
    y = np.empty(ri.shape, np.float64)
    bound = np.empty(ri.shape, np.float64)
    lib().oracle_linear(_ptr(xb), K, _ptr(q), _ptr(s), float(np.float32(g)), M, N, K,
                        _ptr(ri), _ptr(ci), len(ri), _ptr(y), _ptr(bound))
    return y, bound


def tolerance(y_ref: np.ndarray, bound: np.ndarray) -> np.ndarray:
    """Acceptance bound per output: 1e-3 * sum|w x| + 1e-2 * |y_ref|."""
    return 1e-3 * bound + 1e-2 * np.abs(y_ref)


# ------------------------------------------------------------------ MXFP4

def e8m0_decode(byte: int) -> float:
    return lib().oracle_e8m0_decode(int(byte))


def mx_quantize(w):
    """Round-to-nearest MXFP4 of a BF16 [N, K] matrix (K % 32 == 0).
    Returns (q [N, K/2] u8, s [N, K/32] u8 UE8M0)."""
    b = _bf16_bits(w)
    N, K = b.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    q = np.empty((N, K // 2), np.uint8)
    s = np.empty((N, K // 32), np.uint8)
    lib().oracle_mx_quantize(_ptr(b), N, K, K, _ptr(q), _ptr(s))
    return q, s


def mx_dequantize(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """W_deq [N, K] in fp64."""
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    N, K = q.shape[0], q.shape[1] * 2
    out = np.empty((N, K), np.float64)
    lib().oracle_mx_dequantize(_ptr(q), _ptr(s), N, K, _ptr(out))
    return out


def mx_linear(x, q: np.ndarray, s: np.ndarray, rows=None, cols=None):
    """MXFP4 y = x . W^T in fp64 with the bound sum |w x| (as ``linear``)."""
    xb = _bf16_bits(x)
    if xb.ndim == 1:
        xb = xb.reshape(1, -1)
    M, K = xb.shape
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    N = q.shape[0]
    assert q.shape[1] * 2 == K and s.shape == (N, K // 32)
    if rows is None:
        y = np.empty((M, N), np.float64)
        bound = np.empty((M, N), np.float64)
        lib().oracle_mx_linear(_ptr(xb), K, _ptr(q), _ptr(s), M, N, K, None, None, -1, _ptr(y), _ptr(bound))
        return y, bound
    ri = np.ascontiguousarray(rows, np.int64)
    ci = np.ascontiguousarray(cols, np.int64)
    assert ri.shape == ci.shape and ri.ndim == 1
    y = np.empty(ri.shape, np.float64)
    bound = np.empty(ri.shape, np.float64)
    lib().oracle_mx_linear(_ptr(xb), K, _ptr(q), _ptr(s), M, N, K, _ptr(ri), _ptr(ci), len(ri),
                           _ptr(y), _ptr(bound))
    return y, bound


# ------------------------------------------------------ grouped (MoE) GEMV

def linear_grouped(X, q: np.ndarray, s: np.ndarray, g: np.ndarray, expert_ids, token_ids):
    """Grouped decode GEMV over stacked experts (imp docs/quantization.md, MoE
    layers: one contiguous [ne, N, K_packed] buffer per projection, per-expert
    scales).  For problem p: y[p] = x[token_ids[p]] . W[expert_ids[p]]^T with
    expert e's codes q[e], scales s[e] and tensor scale g[e].  Returns
    (y [P, N], bound [P, N]) in fp64, each row from ``linear``."""
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    g = np.asarray(g, np.float32).reshape(-1)
    xb = _bf16_bits(X)
    if xb.ndim == 1:
        xb = xb.reshape(1, -1)
    E, N = q.shape[0], q.shape[1]
    ids_e = np.asarray(expert_ids, np.int64).reshape(-1)
    ids_t = np.asarray(token_ids, np.int64).reshape(-1)
    assert ids_e.shape == ids_t.shape and s.shape[:2] == (E, N) and g.shape == (E,)
    y = np.empty((len(ids_e), N), np.float64)
    bound = np.empty((len(ids_e), N), np.float64)
    for p, (e, t) in enumerate(zip(ids_e, ids_t)):
        yp, bp = linear(xb[t:t + 1], q[e], s[e], g[e])
        y[p], bound[p] = yp[0], bp[0]
    return y, bound


# ------------------------------------------- MXFP4 scales as NVFP4 scales

def _e4m3_byte_of_pow2(j: int) -> int:
    """E4M3 code of 2^j for j in [-9, 8] (subnormals below 2^-6)."""
    assert -9 <= j <= 8
    return (j + 7) << 3 if j >= -6 else 1 << (j + 9)


def mx_to_nvfp4(q: np.ndarray, s_mx: np.ndarray):
    """The same weights in NVFP4 form: the codes stay, each UE8M0 block scale
    2^k (32 elements) becomes the E4M3 scale 2^(k - G) of its two 16-element
    halves, with the tensor scale g = 2^G, G = (largest k of a block with a
    non-zero code) - 8.  Exact when every such block has k - G >= -9 (E4M3
    holds the powers 2^-9 .. 2^8); blocks whose codes are all zero get scale 0.
    A block with scale byte 255 decodes to NaN (e8m0_decode), which no finite
    NVFP4 scale holds: it takes no part in G and is counted like a block
    outside the window.  Returns (s_nv [N, K/16], g, number of counted blocks,
    which get scale 0)."""
    q = np.ascontiguousarray(q, np.uint8)
    s_mx = np.ascontiguousarray(s_mx, np.uint8)
    N, nb = s_mx.shape
    mags = np.stack([q & 7, (q >> 4) & 7], axis=-1).reshape(N, nb, 32)
    nan_block = s_mx == 255
    nonzero = mags.any(axis=2) & ~nan_block
    k = s_mx.astype(np.int64) - 127
    if nonzero.any():
        G = int(k[nonzero].max()) - 8
    else:
        G = 0
    s_nv = np.zeros((N, nb), np.uint8)
    bad = int(nan_block.sum())
    for n in range(N):
        for b in range(nb):
            if not nonzero[n, b]:
                continue
            j = int(k[n, b]) - G
            if j < -9:
                bad += 1
                continue
            s_nv[n, b] = _e4m3_byte_of_pow2(j)
    g = np.float32(np.ldexp(1.0, G))
    return np.repeat(s_nv, 2, axis=1), g, bad


def w4a4_linear(x, q: np.ndarray, s: np.ndarray, g, x_amax=None, rows=None, cols=None):
    """W4A4 product (the pages' NVFP4 x NVFP4 prefill GEMM, imp
    docs/quantization.md, dense-layer pipeline and the Modelopt row of the
    tools table).  The pages give no activation rule; the reading taken is the
    weights' own: X is quantized round-to-nearest to NVFP4 with the tensor
    scale g_x = x_amax / 2688 (x_amax = max |X| when not given, as a calibrated
    input scale would be), then y = X_deq . W_deq^T in fp64 with the bound
    sum |x_deq w_deq|.

    x is BF16 [M, K]; with rows/cols only those outputs are computed (1-D
    results).  Returns (y, bound, (qx, sx, g_x))."""
    xb = _bf16_bits(x)
    if xb.ndim == 1:
        xb = xb.reshape(1, -1)
    g_x = tensor_scale(amax(xb) if x_amax is None else x_amax)
    qx, sx, g_x = quantize(xb, g_x)
    xd = dequantize(qx, sx, g_x)
    if rows is None:
        wd = dequantize(q, s, g)
        return xd @ wd.T, np.abs(xd) @ np.abs(wd).T, (qx, sx, g_x)
    ri = np.asarray(rows, np.int64)
    ci = np.asarray(cols, np.int64)
    wd = dequantize(np.asarray(q)[ci], np.asarray(s)[ci], g)
    xr = xd[ri]
    return (xr * wd).sum(axis=1), (np.abs(xr) * np.abs(wd)).sum(axis=1), (qx, sx, g_x)
