"""Shared helpers for the MBOK tests (device buffers, oracle comparisons)."""
from __future__ import annotations

import numpy as np

from oracle import mbok_oracle as O

GEMV_REL = 1e-3
GEMV_ABS = 1e-6
GEMV_REL_L2 = 1e-5


# Guarded outputs: every output buffer of the GPU tests sits between two guard
# regions filled with one byte pattern.  A kernel that writes past either end
# of its output (a masking slip on a ragged shape) changes a guard byte, which
# check_guards() reports after the test (run by the fixture in conftest.py).
GUARD_BYTES = 512          # keeps the buffer's 256-byte alignment
GUARD_BYTE = 0xA5
_LIVE_GUARDS = []


def guarded(shape, dtype):
    """A CUDA tensor of `shape` and `dtype` between two guard regions (its own
    contents start as the guard pattern, so every element must be written)."""
    import torch
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    raw = torch.full((2 * GUARD_BYTES + n,), GUARD_BYTE, dtype=torch.uint8, device="cuda")
    _LIVE_GUARDS.append((raw, n))
    return raw[GUARD_BYTES:GUARD_BYTES + n].view(dtype).view(*shape)


def check_guards():
    """Assert that the guard regions of every buffer from guarded() since the
    last check still hold the pattern; forget those buffers."""
    import torch
    if not _LIVE_GUARDS:
        return
    torch.cuda.synchronize()
    bad = []
    for raw, n in _LIVE_GUARDS:
        head, tail = raw[:GUARD_BYTES], raw[GUARD_BYTES + n:]
        if not (bool((head == GUARD_BYTE).all()) and bool((tail == GUARD_BYTE).all())):
            bad.append(n)
    _LIVE_GUARDS.clear()
    assert not bad, f"bytes written outside output buffers of {bad} bytes"


def guarded_packed(K, M, N):
    import torch
    import boolean_weight_matmul_b200 as mb
    return guarded((mb.packed_bytes(K, M, N) // 4,), torch.int32)


def guarded_alpha(K, M, N):
    import torch
    import boolean_weight_matmul_b200 as mb
    return guarded((mb.alpha_elems(K, M, N),), torch.float16)


def ensure_built():
    from boolean_weight_matmul_b200 import build
    return build.build()


def to_dev(a: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.cuda()


def packed_from_signs_gpu(signs: np.ndarray):
    """GPU packing (the product) of int8 signs [K][M][N]."""
    import boolean_weight_matmul_b200 as mb
    K, M, N = signs.shape
    packed = guarded_packed(K, M, N)
    mb.pack_bits(to_dev(signs), K, M, N, packed)
    return packed


def alpha_blocked_gpu(alpha_mgk: np.ndarray, K: int, M: int, N: int):
    """GPU blocking (the product) of logical fp16 scales [M][G][K]."""
    import torch
    import boolean_weight_matmul_b200 as mb
    a = to_dev(np.ascontiguousarray(alpha_mgk, dtype=np.float16).view(np.int16)).view(torch.float16)
    out = guarded_alpha(K, M, N)
    mb.pack_alpha(a, K, M, N, out)
    return out


def x_dev(x: np.ndarray, dtype: str):
    import torch
    if dtype == "f32":
        return to_dev(x.astype(np.float32))
    return to_dev(x.view(np.int16)).view(torch.bfloat16)


def gemv_gpu(packed, alpha_blk, K, M, N, x_np, x_dtype):
    import torch
    import boolean_weight_matmul_b200 as mb
    batch = x_np.shape[0]
    x = x_dev(x_np, x_dtype)
    y = guarded((batch, M), torch.float32)
    ws = mb.zeros_workspace(K, M, N, batch)
    mb.gemv(packed, alpha_blk, K, M, N, 128, x, mb.F32 if x_dtype == "f32" else mb.BF16, batch, y, ws)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def gemm_gpu(packed, alpha_blk, K, M, N, X_bits: np.ndarray, precision=None):
    import torch
    import boolean_weight_matmul_b200 as mb
    T = X_bits.shape[0]
    X = x_dev(X_bits, "bf16")
    Y = guarded((T, M), torch.bfloat16)
    mb.gemm(packed, alpha_blk, K, M, N, 128, X, T, Y, precision=precision)
    torch.cuda.synchronize()
    return Y.float().cpu().numpy()


# A bf16 output differs from the exact value by up to half a bf16 ulp
# (2^-9 relative) from its own final rounding; the GEMM bound adds one bf16
# ulp of the exact value on top of the accumulation bound.
BF16_OUT_REL = 2.0 ** -8


def assert_close(y, y_ref, E, rel_l2=None, what="", out_rel=0.0):
    """Per-element |y - y_ref| <= 1e-3 E + out_rel |y_ref| + 1e-6, optionally rel-L2."""
    ok = O.within_tolerance(y, y_ref, E + (out_rel / GEMV_REL) * np.abs(y_ref), GEMV_REL, GEMV_ABS)
    if not ok.all():
        bad = np.argwhere(~ok)[:5]
        raise AssertionError(f"{what}: {int((~ok).sum())} elements out of tolerance, e.g. "
                             + ", ".join(f"{tuple(b)} got {float(y[tuple(b)])} want {float(y_ref[tuple(b)])} "
                                         f"bound {GEMV_REL * float(E[tuple(b)]) + GEMV_ABS}" for b in bad))
    if rel_l2 is not None:
        e = O.rel_l2(y, y_ref)
        assert e <= rel_l2, f"{what}: relative L2 error {e} > {rel_l2}"
