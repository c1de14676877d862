"""mbok_gemv_noalloc: the decode GEMV for callers that cannot allocate device
memory -- serving loops that must not call cudaMalloc once they run, plugins
whose host framework owns every device buffer, C callers with no allocator.
Its scratch (the partial sums of the 8-bit slab lookup kernel, the one GEMV
kernel that needs scratch) comes from an array built into the library
instead of a caller workspace.

Checked through the C ABI on the calls that do use the scratch: the slab
kernel at batch 1 over eight slabs, the same kernel at batch 4 (four launches
sharing the array one after another), and a shape whose rows are too wide for
the whole-row tables, so that the default choice takes the slab kernel.  Each
output must be bit-identical to mbok_gemv's with the same kernel and inputs,
and both must meet the GEMV tolerance against the oracle.  The calls run back
to back, so each one starts from what the previous left in the shared array.
This file is collected last on purpose."""
import numpy as np
import pytest

from oracle import mbok_oracle as O
from boolean_weight_matmul_b200 import workloads as wl
from helpers import (GEMV_REL_L2, alpha_blocked_gpu, assert_close, ensure_built, guarded, packed_from_signs_gpu,
                     x_dev)

pytestmark = pytest.mark.gpu

SLABS = 3   # MBOK_GEMV_LOOKUP_SLABS
AUTO = 0    # MBOK_GEMV_AUTO


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ensure_built()


def _case(K, M, N, batch, seed, kernel):
    """(y from mbok_gemv_noalloc, y from mbok_gemv, y_ref, E) for one case."""
    import torch
    import boolean_weight_matmul_b200 as mb
    L = mb.lib()
    s = wl.random_signs(K, M, N, seed)
    a = wl.alpha_decaying(K, M, N, seed + 1)
    x = wl.x_normal(batch, N, seed + 2)
    packed, alpha, xd = packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N), x_dev(x, "bf16")
    stream = torch.cuda.current_stream().cuda_stream
    assert L.mbok_gemv_set_kernel(kernel) == 0
    try:
        assert L.mbok_gemv_workspace_bytes(K, M, N, batch) > 0, "this case must need scratch"
        y_ws = guarded((batch, M), torch.float32).fill_(float("nan"))
        ws = mb.zeros_workspace(K, M, N, batch)
        st = L.mbok_gemv(packed.data_ptr(), alpha.data_ptr(), K, M, N, 128, xd.data_ptr(), mb.BF16,
                         batch, y_ws.data_ptr(), ws.data_ptr(), ws.numel(), stream)
        assert st == 0, mb.status_string(st)
        y = guarded((batch, M), torch.float32).fill_(float("nan"))
        st = L.mbok_gemv_noalloc(packed.data_ptr(), alpha.data_ptr(), K, M, N, 128, xd.data_ptr(),
                                 mb.BF16, batch, y.data_ptr(), stream)
        assert st == 0, mb.status_string(st)
        torch.cuda.synchronize()
    finally:
        L.mbok_gemv_set_kernel(AUTO)
    y_ref, E = O.linear(O.pack_signs(s), a, K, M, N, x, "bf16")
    return y.cpu().numpy(), y_ws.cpu().numpy(), y_ref, E


def test_noalloc_equals_gemv_and_oracle_calls_in_a_row():
    cases = ((3, 4096, 4096, 1, 901, SLABS),    # batch 1, eight 512-column slabs
             (4, 1000, 5120, 4, 902, SLABS),    # batch 4: four launches share the array in turn
             (2, 512, 11008, 1, 903, AUTO))     # too wide for whole rows: the default is the slab kernel
    for (K, M, N, batch, seed, kernel) in cases:
        y, y_ws, y_ref, E = _case(K, M, N, batch, seed, kernel)
        what = f"noalloc K={K} M={M} N={N} batch={batch}"
        assert np.array_equal(y.view(np.uint32), y_ws.view(np.uint32)), what + ": differs from mbok_gemv"
        assert_close(y, y_ref, E, GEMV_REL_L2, what)
        assert_close(y_ws, y_ref, E, GEMV_REL_L2, what + " (mbok_gemv)")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import boolean_weight_matmul_b200 as mb
    L = mb.lib()
    # (4 << 20) bytes of scratch; 32768 x 131072 needs far more.
    st = L.mbok_gemv_noalloc(1 << 20, 1 << 20, 1, 32768, 131072, 128, 1 << 20, mb.BF16, 1,
                             1 << 20, None)
    assert st == 7 and "scratch" in mb.status_string(st)
