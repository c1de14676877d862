"""mbok_gemv_noalloc: the decode GEMV for callers that cannot allocate device
memory (allocator-free serving loops, plugins whose host framework owns every
device buffer, C callers without an allocator).  Its scratch comes from an
array built into the library instead of a caller workspace.

Checked through the C ABI against mbok_gemv on the same inputs, within the
GEMV tolerance of the other tests, for two calls in a row (two shapes, so the
second call starts from what the first left in the shared array).  This file
is collected last on purpose."""
import ctypes

import numpy as np
import pytest

from oracle import mbok_oracle as O
from boolean_weight_matmul_b200 import workloads as wl
from helpers import alpha_blocked_gpu, ensure_built, packed_from_signs_gpu, x_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ensure_built()


def _inputs(K, M, N, batch, seed):
    s = wl.random_signs(K, M, N, seed)
    a = wl.alpha_decaying(K, M, N, seed + 1)
    x = wl.x_normal(batch, N, seed + 2)
    return packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N), x_dev(x, "bf16")


def _both(K, M, N, batch, seed):
    import torch
    import boolean_weight_matmul_b200 as mb
    L = mb.lib()
    packed, alpha, x = _inputs(K, M, N, batch, seed)
    stream = torch.cuda.current_stream().cuda_stream
    y_ref = torch.empty(batch, M, dtype=torch.float32, device="cuda")
    ws = mb.zeros_workspace(K, M, N, batch)
    st = L.mbok_gemv(packed.data_ptr(), alpha.data_ptr(), K, M, N, 128, x.data_ptr(), mb.BF16,
                     batch, y_ref.data_ptr(), ws.data_ptr(), ws.numel(), stream)
    assert st == 0, mb.status_string(st)
    y = torch.full((batch, M), float("nan"), dtype=torch.float32, device="cuda")
    st = L.mbok_gemv_noalloc(packed.data_ptr(), alpha.data_ptr(), K, M, N, 128, x.data_ptr(),
                             mb.BF16, batch, y.data_ptr(), stream)
    assert st == 0, mb.status_string(st)
    torch.cuda.synchronize()
    return y.cpu().numpy(), y_ref.cpu().numpy()


def test_noalloc_matches_gemv_two_calls_in_a_row():
    for (K, M, N, batch, seed) in ((3, 4096, 4096, 1, 901), (4, 1000, 5120, 2, 902)):
        y, y_ref = _both(K, M, N, batch, seed)
        E = np.abs(y_ref).astype(np.float64) + np.abs(y).astype(np.float64)
        assert np.isfinite(y).all()
        assert O.within_tolerance(y, y_ref.astype(np.float64), E).all()
        assert O.rel_l2(y, y_ref.astype(np.float64)) <= 1e-5


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import boolean_weight_matmul_b200 as mb
    L = mb.lib()
    # (4 << 20) bytes of scratch; 32768 x 131072 needs far more.
    st = L.mbok_gemv_noalloc(1 << 20, 1 << 20, 1, 32768, 131072, 128, 1 << 20, mb.BF16, 1,
                             1 << 20, None)
    assert st == 7 and "scratch" in mb.status_string(st)
