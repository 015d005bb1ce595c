"""Python binding of libnvfp4 (include/nvfp4.h): the NVFP4 W4A16 linear layer on B200.

Argument marshalling only: every entry point takes torch CUDA tensors, checks
dtypes and shapes, and passes raw device pointers, leading dimensions and the
current CUDA stream to the C ABI.  All arithmetic runs in the library's CUDA
kernels; there is no CPU path.  Importing fails loudly if the library has not
been built (``python gemm_decode_nvfp4_b200/build.py``).

Layouts follow the NVFP4 format of the pages (imp docs/quantization.md, format
table: packed nibbles, E4M3 micro-scales per 16, FP32 tensor scale):
q uint8 [N, K/2] (low nibble = even k), s uint8 [N, K/16], g float32 [1].
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

__all__ = [
    "Nvfp4Error", "LIB_PATH", "lib", "version", "amax", "quantize", "quantize_mse", "gemv", "gemm",
    "gemm_workspace_size", "quantize_new", "linear", "declared_symbols", "check_device_errors",
    "FLAG_STATIC_WEIGHTS", "gemm_noalloc", "GEMM_NOALLOC_SCRATCH_BYTES",
    "mx_quantize", "mx_quantize_new", "mx_gemv", "gemv_grouped", "mx_to_nvfp4",
    "GIVEN_AMAX", "w4a4_prepare_weights", "w4a4_quantize_x", "w4a4_gemm", "w4a4_linear",
    "w4a4_workspace_size", "AMAX_FLOATS",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "nvfp4.h")
MX_HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "mxfp4.h")
W4A4_HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "nvfp4_w4a4.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python gemm_decode_nvfp4_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)

_p, _i64, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
lib.nvfp4_version.argtypes, lib.nvfp4_version.restype = [], ctypes.c_int
lib.nvfp4_last_error.argtypes, lib.nvfp4_last_error.restype = [], ctypes.c_char_p
lib.nvfp4_status_string.argtypes, lib.nvfp4_status_string.restype = [ctypes.c_int], ctypes.c_char_p
lib.nvfp4_amax.argtypes = [_p, _i64, _i64, _i64, _p, _p]
lib.nvfp4_quantize.argtypes = [_p, _i64, _i64, _i64, _p, _p, _p, _p, _p]
lib.nvfp4_quantize_mse.argtypes = [_p, _i64, _i64, _i64, _p, ctypes.c_int32, _p, _p, _p, _p]
lib.nvfp4_gemv.argtypes = [_p, _p, _p, _p, _p, _i64, _i64, _p]
lib.nvfp4_gemm.argtypes = [_p, _i64, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _sz, _p]
lib.nvfp4_gemv_ex.argtypes = [_p, _p, _p, _p, _p, _i64, _i64, ctypes.c_uint32, _p]
lib.nvfp4_gemm_ex.argtypes = [_p, _i64, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _sz, ctypes.c_uint32, _p]
lib.nvfp4_gemm_noalloc.argtypes = [_p, _i64, _p, _p, _p, _p, _i64, _i64, _i64, _i64, ctypes.c_uint32, _p]
lib.nvfp4_gemm_workspace_size.argtypes = [_i64, _i64, _i64]
lib.nvfp4_gemv_grouped.argtypes = [_p, _i64, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _i64, _i64,
                                   ctypes.c_uint32, _p]
lib.mxfp4_quantize.argtypes = [_p, _i64, _i64, _i64, _p, _p, _p]
lib.mxfp4_to_nvfp4_scales.argtypes = [_p, _p, _i64, _i64, _p, _p, _p]
lib.nvfp4_w4a4_weight_scales_bytes.argtypes, lib.nvfp4_w4a4_weight_scales_bytes.restype = [_i64, _i64], _sz
lib.nvfp4_w4a4_x_scales_bytes.argtypes, lib.nvfp4_w4a4_x_scales_bytes.restype = [_i64, _i64], _sz
lib.nvfp4_w4a4_workspace_size.argtypes, lib.nvfp4_w4a4_workspace_size.restype = [_i64, _i64], _sz
lib.nvfp4_w4a4_prepare_weights.argtypes = [_p, _i64, _i64, _p, _p]
lib.nvfp4_w4a4_quantize_x.argtypes = [_p, _i64, _i64, _i64, _p, _p, _p, ctypes.c_uint32, _p]
lib.nvfp4_w4a4_gemm.argtypes = [_p, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, ctypes.c_uint32, _p]
lib.nvfp4_w4a4_linear.argtypes = [_p, _i64, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _sz, ctypes.c_uint32, _p]
lib.mxfp4_gemv.argtypes = [_p, _p, _p, _p, _i64, _i64, _p]
lib.mxfp4_gemv_ex.argtypes = [_p, _p, _p, _p, _i64, _i64, ctypes.c_uint32, _p]
lib.nvfp4_gemm_workspace_size.restype = _sz
lib.nvfp4_check_device_errors.argtypes = []
for _f in (lib.nvfp4_amax, lib.nvfp4_quantize, lib.nvfp4_quantize_mse, lib.nvfp4_gemv, lib.nvfp4_gemm, lib.nvfp4_gemv_ex, lib.nvfp4_gemm_ex,
           lib.nvfp4_gemm_noalloc, lib.nvfp4_check_device_errors, lib.mxfp4_quantize, lib.mxfp4_gemv,
           lib.mxfp4_gemv_ex, lib.nvfp4_gemv_grouped, lib.mxfp4_to_nvfp4_scales,
           lib.nvfp4_w4a4_prepare_weights, lib.nvfp4_w4a4_quantize_x, lib.nvfp4_w4a4_gemm,
           lib.nvfp4_w4a4_linear):
    _f.restype = ctypes.c_int


class Nvfp4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        name = lib.nvfp4_status_string(status).decode()
        msg = lib.nvfp4_last_error().decode()
        super().__init__(f"{fn}: {name}: {msg}")


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise Nvfp4Error(fn, status)


def check_device_errors() -> None:
    """Raise if a tensor-core GEMM CTA gave up on a bounded pipeline wait."""
    _check("nvfp4_check_device_errors", lib.nvfp4_check_device_errors())


def version() -> int:
    return lib.nvfp4_version()


def declared_symbols() -> list[str]:
    """Names of the entry points include/nvfp4.h, mxfp4.h and nvfp4_w4a4.h declare."""
    names = []
    for path in (HEADER_PATH, MX_HEADER_PATH, W4A4_HEADER_PATH):
        with open(path) as f:
            names += re.findall(r"NVFP4_API\s+[\w\s\*]+?\b((?:nvfp4|mxfp4)_\w+)\s*\(", f.read())
    return names


def _device(*tensors) -> torch.device:
    """The one CUDA device all the given tensors (None skipped) live on."""
    devs = {t.device for t in tensors if t is not None}
    if len(devs) != 1:
        raise ValueError(f"tensors must all be on one CUDA device, got {sorted(str(d) for d in devs)}")
    return devs.pop()


def _stream(stream, dev: torch.device) -> int:
    """The raw stream handle for a call on `dev`: the given stream (which must
    belong to `dev`) or that device's current stream."""
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    if s.device != dev:
        raise ValueError(f"stream is on {s.device}, the tensors on {dev}")
    return s.cuda_stream


def _call(fn: str, dev: torch.device, *args) -> None:
    """Call lib.<fn>(*args) with `dev` current (the library launches on the
    current device) and raise on a non-zero status."""
    with torch.cuda.device(dev):
        _check(fn, getattr(lib, fn)(*args))


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dtype, what: str, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{what} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{what} must be {ndim}-D, got shape {tuple(t.shape)}")
    if t.dim() >= 1 and t.numel() > 0 and t.stride(-1) != 1:
        raise ValueError(f"{what} must be contiguous in its last dimension")


def _rows_ld(t: torch.Tensor):
    return (t.shape[0], t.stride(0)) if t.dim() == 2 else (1, t.shape[-1])


def amax(w: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """out = max(out, max|w|) for a BF16 matrix w (out: float32 [1] on the device)."""
    _need(w, torch.bfloat16, "w")
    _need(out, torch.float32, "out")
    w2 = w if w.dim() == 2 else w.reshape(1, -1)
    dev = _device(w, out)
    _call("nvfp4_amax", dev, _ptr(w2), w2.shape[0], w2.shape[1], w2.stride(0), _ptr(out), _stream(stream, dev))


def quantize(w: torch.Tensor, q: torch.Tensor, s: torch.Tensor, g_out: torch.Tensor | None,
             amax: torch.Tensor | None = None, stream=None) -> None:
    """RTN NVFP4 of BF16 w [N, K] into q [N, K/2] u8 and s [N, K/16] u8; g_out gets
    g = amax / 2688.  With amax=None the tensor's own amax is used."""
    _need(w, torch.bfloat16, "w", 2)
    _need(q, torch.uint8, "q", 2)
    _need(s, torch.uint8, "s", 2)
    N, K = w.shape
    if q.shape != (N, K // 2) or s.shape != (N, K // 16) or not q.is_contiguous() or not s.is_contiguous():
        raise ValueError("q/s must be contiguous [N, K/2] / [N, K/16]")
    if g_out is not None:
        _need(g_out, torch.float32, "g_out")
    if amax is not None:
        _need(amax, torch.float32, "amax")
    dev = _device(w, q, s, g_out, amax)
    _call("nvfp4_quantize", dev, _ptr(w), N, K, w.stride(0), _ptr(amax), _ptr(q), _ptr(s), _ptr(g_out),
          _stream(stream, dev))


def quantize_mse(w: torch.Tensor, q: torch.Tensor, s: torch.Tensor, g_out: torch.Tensor | None,
                 amax: torch.Tensor | None = None, window: int = 8, stream=None) -> None:
    """NVFP4 of BF16 w [N, K] with each micro-scale chosen by the least fp64
    reconstruction error among the E4M3 codes within `window` of the
    round-to-nearest one (nvfp4_quantize_mse); otherwise as quantize()."""
    _need(w, torch.bfloat16, "w", 2)
    _need(q, torch.uint8, "q", 2)
    _need(s, torch.uint8, "s", 2)
    N, K = w.shape
    if q.shape != (N, K // 2) or s.shape != (N, K // 16) or not q.is_contiguous() or not s.is_contiguous():
        raise ValueError("q/s must be contiguous [N, K/2] / [N, K/16]")
    if g_out is not None:
        _need(g_out, torch.float32, "g_out")
    if amax is not None:
        _need(amax, torch.float32, "amax")
    dev = _device(w, q, s, g_out, amax)
    _call("nvfp4_quantize_mse", dev, _ptr(w), N, K, w.stride(0), _ptr(amax), int(window), _ptr(q), _ptr(s),
          _ptr(g_out), _stream(stream, dev))


FLAG_STATIC_WEIGHTS = 1
FLAG_W4A4_PAIR = 1 << 12


def _ksplit_flag(k_split: int) -> int:
    """NVFP4_FLAG_KSPLIT(k_split): 0 = the library's choice, else 1, 2, 4 or 8."""
    if k_split not in (0, 1, 2, 4, 8):
        raise ValueError(f"k_split must be 0, 1, 2, 4 or 8, got {k_split}")
    return k_split << 8


def gemv(x: torch.Tensor, q: torch.Tensor, s: torch.Tensor, g: torch.Tensor, y: torch.Tensor,
         stream=None, static_weights: bool = False, k_split: int = 0) -> None:
    """y[N] = bf16(g * W_deq . x) for BF16 x [K] (or [1, K]).  static_weights: q, s, g
    are not written by work still running on the stream (see NVFP4_FLAG_STATIC_WEIGHTS).
    k_split: CTAs of a cluster that split K (NVFP4_FLAG_KSPLIT); 0 = chosen per shape."""
    _need(x, torch.bfloat16, "x")
    _need(q, torch.uint8, "q", 2)
    _need(s, torch.uint8, "s", 2)
    _need(g, torch.float32, "g")
    _need(y, torch.bfloat16, "y")
    N, K = q.shape[0], q.shape[1] * 2
    if x.numel() != K or y.numel() != N or not x.is_contiguous() or not y.is_contiguous():
        raise ValueError("x must hold K and y N contiguous elements")
    if not q.is_contiguous() or not s.is_contiguous() or s.shape != (N, K // 16):
        raise ValueError("q/s must be contiguous [N, K/2] / [N, K/16]")
    flags = (FLAG_STATIC_WEIGHTS if static_weights else 0) | _ksplit_flag(k_split)
    dev = _device(x, q, s, g, y)
    _call("nvfp4_gemv_ex", dev, _ptr(x), _ptr(q), _ptr(s), _ptr(g), _ptr(y), N, K, flags, _stream(stream, dev))


def gemm_workspace_size(M: int, N: int, K: int) -> int:
    return lib.nvfp4_gemm_workspace_size(M, N, K)


def gemm(X: torch.Tensor, q: torch.Tensor, s: torch.Tensor, g: torch.Tensor, Y: torch.Tensor,
         workspace: torch.Tensor | None = None, stream=None, static_weights: bool = False) -> None:
    """Y [M, N] = bf16(g * X . W_deq^T) for BF16 X [M, K]."""
    _need(X, torch.bfloat16, "X", 2)
    _need(q, torch.uint8, "q", 2)
    _need(s, torch.uint8, "s", 2)
    _need(g, torch.float32, "g")
    _need(Y, torch.bfloat16, "Y", 2)
    M, K = X.shape
    N = q.shape[0]
    if q.shape[1] * 2 != K or Y.shape != (M, N):
        raise ValueError(f"shape mismatch: X {tuple(X.shape)}, q {tuple(q.shape)}, Y {tuple(Y.shape)}")
    if not q.is_contiguous() or not s.is_contiguous() or s.shape != (N, K // 16):
        raise ValueError("q/s must be contiguous [N, K/2] / [N, K/16]")
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, torch.uint8, "workspace")
        ws_bytes = workspace.numel()
    flags = FLAG_STATIC_WEIGHTS if static_weights else 0
    dev = _device(X, q, s, g, Y, workspace)
    _call("nvfp4_gemm_ex", dev, _ptr(X), X.stride(0), _ptr(q), _ptr(s), _ptr(g), _ptr(Y), Y.stride(0), M, N, K,
          _ptr(workspace), ws_bytes, flags, _stream(stream, dev))


def _header_constant(name: str) -> int:
    with open(HEADER_PATH) as f:
        m = re.search(r"#define\s+" + name + r"\s+\(\(\(size_t\)(\d+) << (\d+)\) \+ (\d+)\)", f.read())
    if not m:
        raise ImportError(f"{name} not found in {HEADER_PATH}")
    return (int(m.group(1)) << int(m.group(2))) + int(m.group(3))


# Bytes of the scratch array built into the library for gemm_noalloc.
GEMM_NOALLOC_SCRATCH_BYTES = _header_constant("NVFP4_GEMM_NOALLOC_SCRATCH_BYTES")


def gemm_noalloc(X: torch.Tensor, q: torch.Tensor, s: torch.Tensor, g: torch.Tensor, Y: torch.Tensor,
                 stream=None, static_weights: bool = False) -> None:
    """gemm() with the library's built-in scratch instead of a workspace
    (nvfp4_gemm_noalloc): allocates nothing, for callers that cannot.  Calls on
    one device share the scratch and must be ordered (one stream)."""
    _need(X, torch.bfloat16, "X", 2)
    _need(q, torch.uint8, "q", 2)
    _need(s, torch.uint8, "s", 2)
    _need(g, torch.float32, "g")
    _need(Y, torch.bfloat16, "Y", 2)
    M, K = X.shape
    N = q.shape[0]
    if q.shape[1] * 2 != K or Y.shape != (M, N):
        raise ValueError(f"shape mismatch: X {tuple(X.shape)}, q {tuple(q.shape)}, Y {tuple(Y.shape)}")
    if not q.is_contiguous() or not s.is_contiguous() or s.shape != (N, K // 16):
        raise ValueError("q/s must be contiguous [N, K/2] / [N, K/16]")
    flags = FLAG_STATIC_WEIGHTS if static_weights else 0
    dev = _device(X, q, s, g, Y)  # the built-in scratch of this device is used
    _call("nvfp4_gemm_noalloc", dev, _ptr(X), X.stride(0), _ptr(q), _ptr(s), _ptr(g), _ptr(Y), Y.stride(0), M, N,
          K, flags, _stream(stream, dev))


# ------------------------------------------------------ allocating helpers

def quantize_new(w: torch.Tensor, amax: torch.Tensor | None = None, stream=None):
    """Allocate q, s, g on w's device and quantize into them."""
    N, K = w.shape
    q = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    s = torch.empty((N, K // 16), dtype=torch.uint8, device=w.device)
    g = torch.empty((1,), dtype=torch.float32, device=w.device)
    quantize(w, q, s, g, amax=amax, stream=stream)
    return q, s, g


def linear(X: torch.Tensor, q: torch.Tensor, s: torch.Tensor, g: torch.Tensor, stream=None) -> torch.Tensor:
    """Allocate Y and run the GEMM (the GEMV when X has one row)."""
    X2 = X if X.dim() == 2 else X.reshape(1, -1)
    Y = torch.empty((X2.shape[0], q.shape[0]), dtype=torch.bfloat16, device=X.device)
    n_ws = gemm_workspace_size(X2.shape[0], q.shape[0], X2.shape[1])
    ws = torch.empty((n_ws,), dtype=torch.uint8, device=X.device) if n_ws else None
    gemm(X2, q, s, g, Y, workspace=ws, stream=stream)
    return Y if X.dim() == 2 else Y.reshape(-1)


# ---------------------------------------------------------------------- MXFP4
# imp docs/quantization.md, MXFP4 paragraph: NVFP4's nibble layout with one UE8M0
# micro-scale per 32 elements and no tensor scale (include/mxfp4.h).

def mx_quantize(w: torch.Tensor, q: torch.Tensor, s: torch.Tensor, stream=None) -> None:
    """Round-to-nearest MXFP4 of BF16 w [N, K] into q [N, K/2] and s [N, K/32]."""
    _need(w, torch.bfloat16, "w", 2)
    _need(q, torch.uint8, "q", 2)
    _need(s, torch.uint8, "s", 2)
    N, K = w.shape
    if w.stride(1) != 1 or not q.is_contiguous() or not s.is_contiguous():
        raise ValueError("w rows and q, s must be contiguous")
    if q.shape != (N, K // 2) or s.shape != (N, K // 32):
        raise ValueError("q/s must be [N, K/2] / [N, K/32]")
    dev = _device(w, q, s)
    _call("mxfp4_quantize", dev, _ptr(w), N, K, w.stride(0), _ptr(q), _ptr(s), _stream(stream, dev))


def mx_quantize_new(w: torch.Tensor, stream=None):
    """Allocate q, s on w's device and MXFP4-quantize into them."""
    N, K = w.shape
    q = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    s = torch.empty((N, K // 32), dtype=torch.uint8, device=w.device)
    mx_quantize(w, q, s, stream=stream)
    return q, s


def mx_gemv(x: torch.Tensor, q: torch.Tensor, s: torch.Tensor, y: torch.Tensor, stream=None,
            static_weights: bool = False, k_split: int = 0) -> None:
    """y[N] = bf16(W_deq . x) for MXFP4 weights and BF16 x [K]; k_split as for gemv()."""
    _need(x, torch.bfloat16, "x")
    _need(q, torch.uint8, "q", 2)
    _need(s, torch.uint8, "s", 2)
    _need(y, torch.bfloat16, "y")
    N, K = q.shape[0], q.shape[1] * 2
    if x.numel() != K or y.numel() != N or not x.is_contiguous() or not y.is_contiguous():
        raise ValueError("x must hold K and y N contiguous elements")
    if not q.is_contiguous() or not s.is_contiguous() or s.shape != (N, K // 32):
        raise ValueError("q/s must be contiguous [N, K/2] / [N, K/32]")
    flags = (FLAG_STATIC_WEIGHTS if static_weights else 0) | _ksplit_flag(k_split)
    dev = _device(x, q, s, y)
    _call("mxfp4_gemv_ex", dev, _ptr(x), _ptr(q), _ptr(s), _ptr(y), N, K, flags, _stream(stream, dev))


# ------------------------------------------------------------ grouped (MoE) GEMV

def gemv_grouped(X: torch.Tensor, q: torch.Tensor, s: torch.Tensor, g: torch.Tensor, expert_ids: torch.Tensor,
                 token_ids: torch.Tensor, Y: torch.Tensor, stream=None) -> None:
    """Y[p] = bf16(g[e] * W_deq[e] . X[t]) for e = expert_ids[p], t = token_ids[p]
    with stacked experts q [E, N, K/2], s [E, N, K/16], g [E] (imp docs/quantization.md,
    MoE layers: one contiguous [ne, N, K_packed] buffer per projection)."""
    _need(X, torch.bfloat16, "X", 2)
    _need(q, torch.uint8, "q", 3)
    _need(s, torch.uint8, "s", 3)
    _need(g, torch.float32, "g")
    _need(expert_ids, torch.int32, "expert_ids")
    _need(token_ids, torch.int32, "token_ids")
    _need(Y, torch.bfloat16, "Y", 2)
    E, N, K = q.shape[0], q.shape[1], q.shape[2] * 2
    T, P = X.shape[0], expert_ids.numel()
    if X.shape[1] != K or X.stride(1) != 1 or Y.stride(1) != 1 or Y.shape != (P, N):
        raise ValueError("X must be [T, K] and Y [P, N] with unit column stride")
    if not q.is_contiguous() or not s.is_contiguous() or s.shape != (E, N, K // 16) or g.numel() != E:
        raise ValueError("q/s/g must be contiguous [E, N, K/2] / [E, N, K/16] / [E]")
    if token_ids.numel() != P or not expert_ids.is_contiguous() or not token_ids.is_contiguous():
        raise ValueError("expert_ids and token_ids must be contiguous [P]")
    dev = _device(X, q, s, g, expert_ids, token_ids, Y)
    _call("nvfp4_gemv_grouped", dev,
          _ptr(X), X.stride(0), _ptr(q), _ptr(s), _ptr(g), _ptr(expert_ids), _ptr(token_ids), _ptr(Y), Y.stride(0),
          P, E, T, N, K, 0, _stream(stream, dev))


def mx_to_nvfp4(q: torch.Tensor, s_mx: torch.Tensor, stream=None):
    """MXFP4 scales s_mx [N, K/32] restated as NVFP4 scales [N, K/16] and a
    power-of-two tensor scale g [1] (exact within 17 binades; see
    include/mxfp4.h), so that (q, s_nv, g) runs on gemv/gemm."""
    _need(q, torch.uint8, "q", 2)
    _need(s_mx, torch.uint8, "s_mx", 2)
    N, K = q.shape[0], q.shape[1] * 2
    if not q.is_contiguous() or not s_mx.is_contiguous() or s_mx.shape != (N, K // 32):
        raise ValueError("q/s_mx must be contiguous [N, K/2] / [N, K/32]")
    s_nv = torch.empty((N, K // 16), dtype=torch.uint8, device=q.device)
    g = torch.empty((1,), dtype=torch.float32, device=q.device)
    dev = _device(q, s_mx)
    _call("mxfp4_to_nvfp4_scales", dev, _ptr(q), _ptr(s_mx), N, K, _ptr(s_nv), _ptr(g), _stream(stream, dev))
    return s_nv, g


# ----------------------------------------------------------------------- W4A4
# NVFP4 x NVFP4 prefill (include/nvfp4_w4a4.h): activations quantized by the
# weights' rule, block-scaled FP4 tensor-core GEMM.

GIVEN_AMAX = 2  # NVFP4_W4A4_GIVEN_AMAX
AMAX_FLOATS = 260  # NVFP4_W4A4_AMAX_FLOATS: the x_amax buffer of a dynamic quantize


def w4a4_prepare_weights(s: torch.Tensor, K: int, stream=None) -> torch.Tensor:
    """Row-major weight scales [N, K/16] -> the tensor-core scale layout (u8)."""
    _need(s, torch.uint8, "s", 2)
    N = s.shape[0]
    if not s.is_contiguous() or s.shape[1] * 16 != K:
        raise ValueError("s must be contiguous [N, K/16]")
    out = torch.empty((lib.nvfp4_w4a4_weight_scales_bytes(N, K),), dtype=torch.uint8, device=s.device)
    dev = _device(s)
    _call("nvfp4_w4a4_prepare_weights", dev, _ptr(s), N, K, _ptr(out), _stream(stream, dev))
    return out


def w4a4_quantize_x(X: torch.Tensor, x_amax: torch.Tensor, given_amax: bool = False, stream=None):
    """X [M, K] -> (qx [M, K/2], sx in the tensor-core scale layout).  x_amax:
    given_amax: [1] (or longer), read; else [AMAX_FLOATS], x_amax[0] receives
    max |X|."""
    _need(X, torch.bfloat16, "X", 2)
    _need(x_amax, torch.float32, "x_amax")
    if not given_amax and x_amax.numel() < AMAX_FLOATS:
        raise ValueError(f"x_amax needs {AMAX_FLOATS} floats for a dynamic amax")
    M, K = X.shape
    if X.stride(1) != 1:
        raise ValueError("X rows must be contiguous")
    ldx = X.stride(0)
    qx = torch.empty((M, K // 2), dtype=torch.uint8, device=X.device)
    sx = torch.empty((lib.nvfp4_w4a4_x_scales_bytes(M, K),), dtype=torch.uint8, device=X.device)
    dev = _device(X, x_amax)
    _call("nvfp4_w4a4_quantize_x", dev, _ptr(X), ldx, M, K, _ptr(qx), _ptr(sx), _ptr(x_amax),
          GIVEN_AMAX if given_amax else 0, _stream(stream, dev))
    return qx, sx


def _need_w4a4_weights(q: torch.Tensor, s_mma: torch.Tensor, g: torch.Tensor):
    """q [N, K/2] contiguous, s_mma holding the rearranged scales of [N, K/16]
    (w4a4_prepare_weights), g an fp32 tensor scale.  Returns (N, K)."""
    _need(q, torch.uint8, "q", 2)
    _need(s_mma, torch.uint8, "s_mma")
    _need(g, torch.float32, "g")
    if not q.is_contiguous() or not s_mma.is_contiguous():
        raise ValueError("q and s_mma must be contiguous")
    N, K = q.shape[0], q.shape[1] * 2
    if s_mma.numel() < lib.nvfp4_w4a4_weight_scales_bytes(N, K):
        raise ValueError(f"s_mma holds {s_mma.numel()} bytes, [{N}, {K}] needs "
                         f"{lib.nvfp4_w4a4_weight_scales_bytes(N, K)} (w4a4_prepare_weights)")
    return N, K


def w4a4_gemm(qx, sx, x_amax, q, s_mma, g, Y, stream=None, static_weights: bool = False, pair: bool = False) -> None:
    """Y [M, N] = bf16(g * (x_amax[0] / 2688) * Xq . Wq^T) from quantized
    activations (qx, sx, x_amax from w4a4_quantize_x) and weights (q, s_mma
    from w4a4_prepare_weights, g).  pair: tiles of 256 weight rows on pairs
    of SMs (NVFP4_FLAG_W4A4_PAIR)."""
    _need(Y, torch.bfloat16, "Y", 2)
    _need(qx, torch.uint8, "qx", 2)
    _need(sx, torch.uint8, "sx")
    _need(x_amax, torch.float32, "x_amax")
    N, K = _need_w4a4_weights(q, s_mma, g)
    M = Y.shape[0]
    if qx.shape != (M, K // 2) or Y.shape[1] != N or not qx.is_contiguous() or not sx.is_contiguous():
        raise ValueError(f"shape mismatch: qx {tuple(qx.shape)}, q {tuple(q.shape)}, Y {tuple(Y.shape)}")
    if sx.numel() < lib.nvfp4_w4a4_x_scales_bytes(M, K):
        raise ValueError(f"sx holds {sx.numel()} bytes, [{M}, {K}] needs {lib.nvfp4_w4a4_x_scales_bytes(M, K)}")
    flags = (FLAG_STATIC_WEIGHTS if static_weights else 0) | (FLAG_W4A4_PAIR if pair else 0)
    dev = _device(qx, sx, x_amax, q, s_mma, g, Y)
    _call("nvfp4_w4a4_gemm", dev, _ptr(qx), _ptr(sx), _ptr(x_amax), _ptr(q), _ptr(s_mma), _ptr(g), _ptr(Y),
          Y.stride(0), M, N, K, flags, _stream(stream, dev))


def w4a4_workspace_size(M: int, K: int) -> int:
    return lib.nvfp4_w4a4_workspace_size(M, K)


def w4a4_linear(X: torch.Tensor, q: torch.Tensor, s_mma: torch.Tensor, g: torch.Tensor, Y: torch.Tensor,
                workspace: torch.Tensor, x_amax: torch.Tensor | None = None, stream=None,
                static_weights: bool = False, pair: bool = False) -> None:
    """Y [M, N] = W4A4 product of BF16 X [M, K] (quantized on the fly into the
    workspace) and NVFP4 weights (q, s_mma from w4a4_prepare_weights, g)."""
    _need(X, torch.bfloat16, "X", 2)
    _need(Y, torch.bfloat16, "Y", 2)
    _need(workspace, torch.uint8, "workspace")
    if x_amax is not None:
        _need(x_amax, torch.float32, "x_amax")
    N, Kq = _need_w4a4_weights(q, s_mma, g)
    M, K = X.shape
    if Kq != K or Y.shape != (M, N):
        raise ValueError(f"shape mismatch: X {tuple(X.shape)}, q {tuple(q.shape)}, Y {tuple(Y.shape)}")
    flags = (FLAG_STATIC_WEIGHTS if static_weights else 0) | (FLAG_W4A4_PAIR if pair else 0)
    if X.stride(1) != 1:
        raise ValueError("X rows must be contiguous")
    dev = _device(X, x_amax, q, s_mma, g, Y, workspace)
    _call("nvfp4_w4a4_linear", dev, _ptr(X), X.stride(0), _ptr(x_amax), _ptr(q), _ptr(s_mma), _ptr(g), _ptr(Y),
          Y.stride(0), M, N, K, _ptr(workspace), workspace.numel(), flags, _stream(stream, dev))
