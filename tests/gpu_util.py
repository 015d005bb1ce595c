"""Helpers shared by the GPU tests (not collected as tests)."""
import numpy as np
import torch

CANARY_BYTE = 0xA5
GUARD_BYTES = 256


def guarded_empty(shape, dtype, device="cuda"):
    """A tensor of `shape` inside a larger buffer whose 256-byte guard bands on both
    sides are filled with a canary byte.  Returns (view, check) where check()
    asserts that no byte of the guards changed."""
    esize = torch.empty((), dtype=dtype).element_size()
    numel = int(np.prod(shape)) if len(shape) else 1
    nbytes = numel * esize
    total = GUARD_BYTES * 2 + ((nbytes + 255) // 256) * 256
    base = torch.full((total,), CANARY_BYTE, dtype=torch.uint8, device=device)
    view = base[GUARD_BYTES:GUARD_BYTES + nbytes].view(dtype).view(shape)

    def check():
        torch.cuda.synchronize()
        head = base[:GUARD_BYTES]
        tail = base[GUARD_BYTES + nbytes:]
        assert bool((head == CANARY_BYTE).all()), "write before the start of the output"
        assert bool((tail == CANARY_BYTE).all()), "write past the end of the output"

    return view, check


def assert_within_tolerance(y_gpu: torch.Tensor, y_ref: np.ndarray, bound: np.ndarray, what=""):
    """|y_gpu - y_ref| <= 1e-3 * sum|w x| + 1e-2 * |y_ref| per element."""
    import oracle
    y = y_gpu.detach().float().cpu().double().numpy().reshape(y_ref.shape)
    tol = oracle.tolerance(y_ref, bound)
    err = np.abs(y - y_ref)
    bad = np.nonzero(~(err <= tol))
    if bad[0].size:
        i = tuple(b[0] for b in bad)
        raise AssertionError(f"{what}: {bad[0].size} outputs out of tolerance; first at {i}: "
                             f"gpu={y[i]!r} ref={y_ref[i]!r} tol={tol[i]!r}")
    return float(np.max(err / np.maximum(tol, 1e-300))) if err.size else 0.0
