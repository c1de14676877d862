"""Host-side checks of the C ABI (no GPU work): the library loads, exports
every function include/mbok.h declares, sizes are right, and argument errors
are reported before anything is launched."""
import ctypes
import os
import re

import pytest

from helpers import ensure_built

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mbok.h")

FAKE = 1 << 20          # a 16-byte aligned non-null address; never dereferenced
FAKE_ODD = FAKE + 1     # misaligned


@pytest.fixture(scope="module")
def L():
    ensure_built()
    import boolean_weight_matmul_b200 as mb
    return mb.lib()


def header_functions():
    text = open(HEADER).read()
    return re.findall(r"^\s*(?:const\s+char\s*\*|int|size_t)\s+(mbok_\w+)\s*\(", text, re.M)


def test_header_declares_the_calls():
    names = set(header_functions())
    for n in ("mbok_pack_bits", "mbok_residual_binarize", "mbok_gemv", "mbok_gemm",
              "mbok_pack_alpha", "mbok_packed_bytes", "mbok_alpha_elems",
              "mbok_gemv_workspace_bytes", "mbok_status_string", "mbok_layout_version"):
        assert n in names


def test_library_exports_every_declared_function(L):
    names = header_functions()
    assert names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/mbok.h but not exported"


def test_sizes(L):
    assert L.mbok_layout_version() == 1
    assert L.mbok_packed_bytes(3, 4096, 4096) == 512 * 3 * 4096
    assert L.mbok_packed_bytes(1, 13, 384) == 2 * 1 * 384
    assert L.mbok_alpha_elems(3, 4096, 4096) == 4096 * 32 * 3
    assert L.mbok_alpha_elems(2, 13, 256) == 16 * 2 * 2
    assert L.mbok_packed_bytes(0, 8, 128) == 0
    assert L.mbok_packed_bytes(1, 8, 100) == 0
    assert L.mbok_gemv_workspace_bytes(3, 4096, 512, 1) == 0       # one slab: no workspace
    assert L.mbok_gemv_workspace_bytes(3, 4096, 4096, 1) >= 8 * 4096 * 4
    assert L.mbok_gemv_workspace_bytes(3, 4096, 4096, 17) == 0


def test_status_strings(L):
    for s in range(8):
        assert L.mbok_status_string(s).decode() not in ("", "unknown status")
    assert L.mbok_status_string(99).decode() == "unknown status"


def test_gemv_argument_errors(L):
    g = lambda **kw: L.mbok_gemv(*[kw.get(k, v) for k, v in dict(
        packed=FAKE, alpha=FAKE, K=3, M=64, N=1024, group=128, x=FAKE, dt=1, batch=1, y=FAKE,
        ws=FAKE, wsb=1 << 20, stream=None).items()])
    assert g(K=0) == 1 and g(K=5) == 1
    assert g(M=0) == 2 and g(N=100) == 2 and g(N=0) == 2
    assert g(group=64) == 4
    assert g(packed=None) == 1 and g(x=None) == 1 and g(y=None) == 1
    assert g(dt=7) == 1
    assert g(batch=0) == 1 and g(batch=17) == 1
    assert g(x=FAKE_ODD) == 3 and g(packed=FAKE + 4) == 3
    assert g(ws=None) == 6 and g(wsb=16) == 6


def test_gemm_and_pack_argument_errors(L):
    assert L.mbok_read_device_errors(None) == 1
    assert L.mbok_gemm(FAKE, FAKE, 3, 64, 256, 128, FAKE, 0, FAKE, None) == 2
    assert L.mbok_gemm(FAKE, FAKE, 3, 64, 256, 256, FAKE, 8, FAKE, None) == 4
    assert L.mbok_gemm(FAKE, FAKE, 3, 64, 256, 128, FAKE_ODD, 8, FAKE, None) == 3
    assert L.mbok_gemm(None, FAKE, 3, 64, 256, 128, FAKE, 8, FAKE, None) == 1
    assert L.mbok_pack_bits(None, 1, 8, 128, FAKE, None) == 1
    assert L.mbok_pack_bits(FAKE, 1, 8, 130, FAKE, None) == 2
    assert L.mbok_pack_bits(FAKE_ODD, 1, 8, 128, FAKE, None) == 3
    assert L.mbok_pack_alpha(FAKE, 5, 8, 128, FAKE, None) == 1
    assert L.mbok_residual_binarize(FAKE, 8, 128, 2, 64, FAKE, FAKE, None, None) == 4
    assert L.mbok_residual_binarize(FAKE, 8, 128, 2, 128, FAKE, FAKE, FAKE_ODD, None) == 3
    assert L.mbok_residual_binarize(FAKE, 0, 128, 2, 128, FAKE, FAKE, None, None) == 2


def test_binding_refuses_cpu_tensors(L):
    import torch
    import boolean_weight_matmul_b200 as mb
    s = torch.ones(1, 8, 128, dtype=torch.int8)
    with pytest.raises(ValueError):
        mb.pack_bits(s, 1, 8, 128, torch.empty(64, dtype=torch.int32))


def test_gemv_kernel_choice(L):
    import boolean_weight_matmul_b200 as mb
    assert L.mbok_gemv_set_kernel(-1) == 1 and L.mbok_gemv_set_kernel(5) == 1
    for k in (mb.GEMV_LOOKUP, mb.GEMV_TENSOR, mb.GEMV_LOOKUP_SLABS, mb.GEMV_LOOKUP_ROWS, mb.GEMV_AUTO):
        assert L.mbok_gemv_set_kernel(k) == 0
    with mb.gemv_kernel(mb.GEMV_TENSOR):
        pass
    with pytest.raises(mb.MbokError):
        mb.gemv_set_kernel(7)


def test_gemv_static_weights_switch(L):
    assert L.mbok_gemv_set_static_weights(2) == 1 and L.mbok_gemv_set_static_weights(-1) == 1
    assert L.mbok_gemv_set_static_weights(0) == 0
    assert L.mbok_gemv_set_static_weights(1) == 0      # the default


def test_gemv_svid_argument_errors(L):
    g = lambda **kw: L.mbok_gemv_svid(*[kw.get(k, v) for k, v in dict(
        packed=FAKE, s_in=FAKE, s_out=FAKE, K=3, M=64, N=1024, x=FAKE, dt=1, batch=1, y=FAKE,
        ws=FAKE, wsb=1 << 20, stream=None).items()])
    assert g(K=0) == 1 and g(K=5) == 1
    assert g(M=0) == 2 and g(N=100) == 2
    assert g(s_in=None) == 1 and g(s_out=None) == 1 and g(x=None) == 1
    assert g(batch=0) == 1 and g(batch=17) == 1 and g(dt=5) == 1
    assert g(s_in=FAKE + 8) == 3 and g(s_out=FAKE_ODD) == 3
    assert g(ws=None) == 6 and g(wsb=16) == 6
    assert L.mbok_gemv_svid_workspace_bytes(3, 4096, 4096, 1) > L.mbok_gemv_workspace_bytes(3, 4096, 4096, 1)
    assert L.mbok_gemv_svid_workspace_bytes(1, 4096, 512, 1) == 0


def test_refit_argument_errors(L):
    assert L.mbok_refit_alpha(FAKE, FAKE, 3, 64, 256, 64, FAKE, None) == 4
    assert L.mbok_refit_alpha(None, FAKE, 3, 64, 256, 128, FAKE, None) == 1
    assert L.mbok_refit_alpha(FAKE_ODD, FAKE, 3, 64, 256, 128, FAKE, None) == 3
    assert L.mbok_refit_alpha(FAKE, FAKE, 0, 64, 256, 128, FAKE, None) == 1
    assert L.mbok_refit_alpha(FAKE, FAKE, 3, 64, 200, 128, FAKE, None) == 2


def test_svid_binarize_argument_errors(L):
    g = lambda **kw: L.mbok_svid_binarize(*[kw.get(k, v) for k, v in dict(
        W=FAKE, M=64, N=256, K=3, iters=6, packed=FAKE, s_in=FAKE, s_out=FAKE, R=FAKE, ws=FAKE,
        wsb=1 << 24, stream=None).items()])
    assert g(K=0) == 1 and g(iters=0) == 1 and g(W=None) == 1 and g(R=None) == 1
    assert g(N=100) == 2 and g(M=0) == 2
    assert g(W=FAKE_ODD) == 3 and g(R=FAKE + 4) == 3
    assert g(ws=None) == 6 and g(wsb=16) == 6
    assert L.mbok_svid_workspace_bytes(64, 256) >= (64 + 2 * 256 + 256) * 4


def test_wait_timeout_check_argument_errors(L):
    assert L.mbok_check_wait_timeout(0, None) == 1
    assert L.mbok_check_wait_timeout(2000000, None) == 1


def test_pointer_marshalling_checks_device(monkeypatch):
    # The binding passes raw device pointers to kernels launched on the
    # current device, so it refuses CPU, non-contiguous and other-device
    # tensors before anything reaches the library.  Stand-in tensors keep this
    # a host-only test.
    import types
    import torch
    import boolean_weight_matmul_b200 as mb

    class Fake:
        def __init__(self, dev, contiguous=True, cuda=True, ptr=0x1000):
            self.is_cuda = cuda
            self.device = types.SimpleNamespace(index=dev, type="cuda" if cuda else "cpu")
            self._c = contiguous
            self._p = ptr

        def is_contiguous(self):
            return self._c

        def data_ptr(self):
            return self._p

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)
    assert mb._ptrs(Fake(1, ptr=16), None, 7) == [16, None, 7]
    with pytest.raises(ValueError, match="current device"):
        mb._ptrs(Fake(1), Fake(0))
    with pytest.raises(ValueError, match="CUDA tensors only"):
        mb._ptrs(Fake(None, cuda=False))
    with pytest.raises(ValueError, match="contiguous"):
        mb._ptrs(Fake(1, contiguous=False))
    with pytest.raises(ValueError, match="CUDA tensors only"):
        mb.gemv(torch.zeros(4, dtype=torch.int32), None, 1, 8, 128, 128, None, mb.BF16, 1, None, None)


def test_gemv_multi_sizes_and_argument_errors(L):
    # mbok_gemv_multi: several matrices sharing x, each with its own K and M.
    # Sizes and argument errors are host-side (nothing launches on an error).
    import ctypes
    import boolean_weight_matmul_b200 as mb
    O = lambda M: (M + 7) // 8
    # one region of [N/512 slabs][O_s * 8] fp32 partials per matrix
    assert mb.gemv_multi_workspace_bytes([4, 2, 3], [5120, 136, 77], 5120) == \
        10 * 4 * 8 * (O(5120) + O(136) + O(77))
    assert mb.gemv_multi_workspace_bytes([4, 2], [64, 64], 512) == 0          # one slab: no workspace
    assert mb.gemv_multi_workspace_bytes([5], [8], 1024) == 0                 # K out of range
    assert mb.gemv_multi_workspace_bytes([1] * 9, [8] * 9, 1024) == 0         # more than 8 matrices
    assert mb.gemv_multi_workspace_bytes([1, 1], [8, 1 << 22], 1024) == 0    # more than 2^22 rows in all

    ia = lambda v: (ctypes.c_int * len(v))(*v)
    dummy = (ctypes.c_void_p * 2)(0x1000, 0x2000)
    call = lambda nseg, K, M, N=1024, group=128, dtype=1, batch=1, x=0x3000, y=0x4000: L.mbok_gemv_multi(
        nseg, ctypes.cast(dummy, ctypes.c_void_p), ctypes.cast(dummy, ctypes.c_void_p),
        ctypes.cast(ia(K), ctypes.c_void_p), ctypes.cast(ia(M), ctypes.c_void_p), N, group, x, dtype, batch, y,
        None, 0, None)
    assert call(0, [1], [8]) == 1                       # no matrix
    assert call(9, [1] * 9, [8] * 9) == 1               # too many
    assert call(2, [1, 5], [8, 8]) == 1                 # K out of range
    assert call(2, [1, 2], [8, 0]) == 2                 # M < 1
    assert call(2, [1, 2], [8, 8], N=1000) == 2         # N not a multiple of 128
    assert call(2, [1, 2], [8, 8], group=64) == 4       # group != 128
    assert call(2, [1, 2], [8, 8], dtype=7) == 1        # bad dtype
    assert call(2, [1, 2], [8, 8], batch=17) == 1       # batch out of range
    assert call(2, [1, 2], [8, 8], x=0x3008) == 3       # x not 16-byte aligned
    assert call(2, [1, 2], [8, 8]) == 6                 # N > 512 needs a workspace


def test_gemv_ex_argument_checks(L):
    # Per-call kernel choice and static-weights flag: invalid values are
    # refused on the host before anything is launched (the pointers are never
    # dereferenced).
    P = 1 << 20
    assert L.mbok_gemv_ex(P, P, 3, 64, 512, 128, P, 1, 1, P, P, 1 << 20, 5, 1, None) == 1
    assert L.mbok_gemv_ex(P, P, 3, 64, 512, 128, P, 1, 1, P, P, 1 << 20, -1, 1, None) == 1
    assert L.mbok_gemv_ex(P, P, 3, 64, 512, 128, P, 1, 1, P, P, 1 << 20, 1, 2, None) == 1
    assert L.mbok_gemv_ex(P, P, 3, 64, 500, 128, P, 1, 1, P, P, 1 << 20, 1, 1, None) == 2
