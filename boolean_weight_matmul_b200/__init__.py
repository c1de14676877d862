"""Python binding of libmbok, the B200 library for the multi-Boolean-kernel
(MBOK) linear layer y = W x with W = sum_k alpha_k * B_k.

This module only marshals arguments: every call below forwards device
pointers, sizes and the current CUDA stream to the C ABI declared in
include/mbok.h, where all work runs in the library's kernels.  There is no
CPU fallback: a missing library or a CPU tensor raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmbok.so")

OK = 0
F32 = 0
BF16 = 1
GROUP = 128
MAX_K = 4
MAX_BATCH = 16
GEMV_AUTO = 0
GEMV_LOOKUP = 1
GEMV_TENSOR = 2
GEMV_LOOKUP_SLABS = 3
GEMV_LOOKUP_ROWS = 4
GEMM_AUTO = 0
GEMM_BF16 = 1
GEMM_SPLIT = 2

_lib = None


class MbokError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded libmbok.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m boolean_weight_matmul_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        sigs = {
            "mbok_status_string": ([i], ctypes.c_char_p),
            "mbok_layout_version": ([], i),
            "mbok_packed_bytes": ([i, i, i], sz),
            "mbok_alpha_elems": ([i, i, i], sz),
            "mbok_gemv_workspace_bytes": ([i, i, i, i], sz),
            "mbok_pack_bits": ([vp, i, i, i, vp, vp], i),
            "mbok_pack_alpha": ([vp, i, i, i, vp, vp], i),
            "mbok_residual_binarize": ([vp, i, i, i, i, vp, vp, vp, vp], i),
            "mbok_gemv": ([vp, vp, i, i, i, i, vp, i, i, vp, vp, sz, vp], i),
            "mbok_gemm": ([vp, vp, i, i, i, i, vp, i, vp, vp], i),
            "mbok_gemm_ex": ([vp, vp, i, i, i, i, vp, i, vp, i, vp], i),
            "mbok_gemv_ex": ([vp, vp, i, i, i, i, vp, i, i, vp, vp, sz, i, i, vp], i),
            "mbok_gemv_noalloc": ([vp, vp, i, i, i, i, vp, i, i, vp, vp], i),
            "mbok_read_device_errors": ([ctypes.POINTER(ctypes.c_uint)], i),
            "mbok_check_wait_timeout": ([ctypes.c_uint, vp], i),
            "mbok_gemv_set_kernel": ([i], i),
            "mbok_gemv_set_static_weights": ([i], i),
            "mbok_gemv_svid_workspace_bytes": ([i, i, i, i], sz),
            "mbok_gemv_svid": ([vp, vp, vp, i, i, i, vp, i, i, vp, vp, sz, vp], i),
            "mbok_refit_alpha": ([vp, vp, i, i, i, i, vp, vp], i),
            "mbok_svid_workspace_bytes": ([i, i], sz),
            "mbok_svid_binarize": ([vp, i, i, i, i, vp, vp, vp, vp, vp, sz, vp], i),
            "mbok_gemv_multi_workspace_bytes": ([i, vp, vp, i], sz),
            "mbok_gemv_multi": ([i, vp, vp, vp, vp, i, i, vp, i, i, vp, vp, sz, vp], i),
        }
        for name, (args, res) in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().mbok_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != OK:
        raise MbokError(what, status)


def _ptrs(*ts) -> list:
    """Device pointers of the arguments (None stays None, an int is taken as a
    raw device pointer).  Every tensor must be a contiguous CUDA tensor on the
    current device: the library launches there, and a pointer into another
    GPU's memory would be dereferenced by its kernels."""
    dev = None
    out = []
    for t in ts:
        if t is None or isinstance(t, int):
            out.append(t)
            continue
        if not t.is_cuda:
            raise ValueError("MBOK operates on CUDA tensors only")
        if not t.is_contiguous():
            raise ValueError("MBOK needs contiguous tensors")
        if dev is None:
            dev = torch.cuda.current_device()
        if t.device.index != dev:
            raise ValueError(f"tensor on {t.device} but the current device is cuda:{dev}; "
                             "MBOK launches on the current device")
        out.append(t.data_ptr())
    return out


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


# ---- sizes ---------------------------------------------------------------

def layout_version() -> int:
    return lib().mbok_layout_version()


def packed_bytes(K: int, M: int, N: int) -> int:
    return lib().mbok_packed_bytes(K, M, N)


def alpha_elems(K: int, M: int, N: int) -> int:
    return lib().mbok_alpha_elems(K, M, N)


def gemv_workspace_bytes(K: int, M: int, N: int, batch: int = 1) -> int:
    return lib().mbok_gemv_workspace_bytes(K, M, N, batch)


# ---- allocation helpers (torch owns the memory) --------------------------

def empty_packed(K: int, M: int, N: int, device="cuda") -> torch.Tensor:
    n = packed_bytes(K, M, N)
    if n == 0:
        raise MbokError("packed_bytes", 2)
    return torch.empty(n // 4, dtype=torch.int32, device=device)


def empty_alpha(K: int, M: int, N: int, device="cuda") -> torch.Tensor:
    n = alpha_elems(K, M, N)
    if n == 0:
        raise MbokError("alpha_elems", 2)
    return torch.empty(n, dtype=torch.float16, device=device)


def zeros_workspace(K: int, M: int, N: int, batch: int = 1, device="cuda") -> torch.Tensor:
    n = max(gemv_workspace_bytes(K, M, N, batch), 256)
    return torch.zeros(n, dtype=torch.uint8, device=device)


# ---- the calls ------------------------------------------------------------

def pack_bits(signs, K, M, N, packed, stream=None) -> None:
    ps, pp = _ptrs(signs, packed)
    _check(lib().mbok_pack_bits(ps, K, M, N, pp, _stream(stream)), "mbok_pack_bits")


def pack_alpha(alpha_mgk, K, M, N, alpha_out, stream=None) -> None:
    pa, po = _ptrs(alpha_mgk, alpha_out)
    _check(lib().mbok_pack_alpha(pa, K, M, N, po, _stream(stream)), "mbok_pack_alpha")


def residual_binarize(W, M, N, K, group, packed, alpha, residual=None, stream=None) -> None:
    pw, pp, pa, pr = _ptrs(W, packed, alpha, residual)
    _check(lib().mbok_residual_binarize(pw, M, N, K, group, pp, pa, pr, _stream(stream)), "mbok_residual_binarize")


def svid_binarize(W, M, N, K, iters, packed, s_in, s_out, residual, workspace=None, stream=None) -> None:
    """Successive SVID (see include/mbok.h); allocates its workspace if none is given."""
    if workspace is None:
        workspace = torch.empty(int(lib().mbok_svid_workspace_bytes(M, N)), dtype=torch.uint8, device=W.device)
    pw, pp, pi, po, pr, pws = _ptrs(W, packed, s_in, s_out, residual, workspace)
    _check(lib().mbok_svid_binarize(pw, M, N, K, iters, pp, pi, po, pr, pws,
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "mbok_svid_binarize")


def refit_alpha(W, packed, K, M, N, group, alpha_out, stream=None) -> None:
    """Least-squares scales for fixed kernels (see include/mbok.h)."""
    pw, pp, po = _ptrs(W, packed, alpha_out)
    _check(lib().mbok_refit_alpha(pw, pp, K, M, N, group, po, _stream(stream)), "mbok_refit_alpha")


def gemv(packed, alpha, K, M, N, group, x, x_dtype, batch, y, workspace, stream=None, kernel=None,
         weights_static=None) -> None:
    """mbok_gemv; mbok_gemv_ex when a kernel choice or a static-weights flag
    is given (the other then takes its default: GEMV_AUTO, static)."""
    ws_bytes = 0 if workspace is None else (workspace.numel() * workspace.element_size()
                                            if isinstance(workspace, torch.Tensor) else 0)
    pp, pa, px, py, pws = _ptrs(packed, alpha, x, y, workspace)
    if kernel is None and weights_static is None:
        _check(lib().mbok_gemv(pp, pa, K, M, N, group, px, x_dtype, batch, py, pws, ws_bytes, _stream(stream)),
               "mbok_gemv")
    else:
        k = GEMV_AUTO if kernel is None else int(kernel)
        ws_flag = 1 if weights_static is None or weights_static else 0
        _check(lib().mbok_gemv_ex(pp, pa, K, M, N, group, px, x_dtype, batch, py, pws, ws_bytes, k, ws_flag,
                                  _stream(stream)), "mbok_gemv_ex")


def _int_array(vals):
    arr = (ctypes.c_int * len(vals))(*[int(v) for v in vals])
    return arr, ctypes.cast(arr, ctypes.c_void_p)


def gemv_multi_workspace_bytes(K_list, M_list, N: int) -> int:
    ka, kp = _int_array(K_list)
    ma, mp = _int_array(M_list)
    return int(lib().mbok_gemv_multi_workspace_bytes(len(K_list), kp, mp, N))


def zeros_multi_workspace(K_list, M_list, N: int, device="cuda") -> torch.Tensor:
    n = max(gemv_multi_workspace_bytes(K_list, M_list, N), 256)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def gemv_multi(packed_list, alpha_list, K_list, M_list, N, group, x, x_dtype, batch, y, workspace,
               stream=None) -> None:
    """Several matrices sharing x, each with its own K and M, in one launch per
    vector; y holds their outputs one after another (see include/mbok.h)."""
    n = len(packed_list)
    if not (len(alpha_list) == len(K_list) == len(M_list) == n):
        raise ValueError("gemv_multi: one packed, alpha, K and M per matrix")
    ptrs = _ptrs(*packed_list, *alpha_list, x, y, workspace)
    pp = (ctypes.c_void_p * n)(*ptrs[:n])
    pa = (ctypes.c_void_p * n)(*ptrs[n:2 * n])
    px, py, pws = ptrs[2 * n:]
    ka, kp = _int_array(K_list)
    ma, mp = _int_array(M_list)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().mbok_gemv_multi(n, ctypes.cast(pp, ctypes.c_void_p), ctypes.cast(pa, ctypes.c_void_p), kp, mp,
                                 N, group, px, x_dtype, batch, py, pws, ws_bytes, _stream(stream)),
           "mbok_gemv_multi")


def gemv_svid_workspace_bytes(K: int, M: int, N: int, batch: int = 1) -> int:
    return int(lib().mbok_gemv_svid_workspace_bytes(K, M, N, batch))


def zeros_svid_workspace(K: int, M: int, N: int, batch: int = 1, device="cuda") -> torch.Tensor:
    n = max(gemv_svid_workspace_bytes(K, M, N, batch), 256)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def gemv_svid(packed, s_in, s_out, K, M, N, x, x_dtype, batch, y, workspace, stream=None) -> None:
    """Rank-1-scaled layer: y = sum_k s_out[k] * (B_k (s_in[k] * x)) (see include/mbok.h)."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    pp, pi, po, px, py, pws = _ptrs(packed, s_in, s_out, x, y, workspace)
    _check(lib().mbok_gemv_svid(pp, pi, po, K, M, N, px, x_dtype, batch, py, pws, ws_bytes, _stream(stream)),
           "mbok_gemv_svid")


def gemv_noalloc(packed, alpha, K, M, N, group, x, x_dtype, batch, y, stream=None) -> None:
    """mbok_gemv for callers that cannot allocate: scratch comes from the
    library's built-in array (see include/mbok.h)."""
    pp, pa, px, py = _ptrs(packed, alpha, x, y)
    _check(lib().mbok_gemv_noalloc(pp, pa, K, M, N, group, px, x_dtype, batch, py, _stream(stream)),
           "mbok_gemv_noalloc")


def gemv_set_kernel(kernel: int) -> None:
    """Process-wide kernel choice of gemv / gemv_noalloc (GEMV_AUTO,
    GEMV_LOOKUP, GEMV_TENSOR, GEMV_LOOKUP_SLABS or GEMV_LOOKUP_ROWS)."""
    _check(lib().mbok_gemv_set_kernel(kernel), "mbok_gemv_set_kernel")


def gemv_set_static_weights(on: bool) -> None:
    """Promise that GEMV weights are never written by work still running
    when a GEMV launches (see include/mbok.h)."""
    _check(lib().mbok_gemv_set_static_weights(1 if on else 0), "mbok_gemv_set_static_weights")


class gemv_kernel:
    """Context manager: run the enclosed gemv calls on one kernel, then
    return to GEMV_AUTO."""

    def __init__(self, kernel: int):
        self.kernel = kernel

    def __enter__(self):
        gemv_set_kernel(self.kernel)
        return self

    def __exit__(self, *exc):
        gemv_set_kernel(GEMV_AUTO)
        return False


def gemm(packed, alpha, K, M, N, group, X, T, Y, stream=None, precision=None) -> None:
    """mbok_gemm, or mbok_gemm_ex when a weight precision (GEMM_AUTO,
    GEMM_BF16, GEMM_SPLIT) is given."""
    pp, pa, px, py = _ptrs(packed, alpha, X, Y)
    if precision is None:
        _check(lib().mbok_gemm(pp, pa, K, M, N, group, px, T, py, _stream(stream)), "mbok_gemm")
    else:
        _check(lib().mbok_gemm_ex(pp, pa, K, M, N, group, px, T, py, int(precision), _stream(stream)),
               "mbok_gemm_ex")


def read_device_errors() -> int:
    """Flags of kernels whose bounded waits gave up since the last read (0 = none)."""
    f = ctypes.c_uint(0)
    _check(lib().mbok_read_device_errors(ctypes.byref(f)), "mbok_read_device_errors")
    return f.value


def check_wait_timeout(timeout_us: int = 20000, stream=None) -> None:
    """Run the bounded-wait self-check (see include/mbok.h)."""
    _check(lib().mbok_check_wait_timeout(timeout_us, _stream(stream)), "mbok_check_wait_timeout")


def dtype_code(x: torch.Tensor) -> int:
    if x.dtype == torch.float32:
        return F32
    if x.dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported activation dtype {x.dtype}")
