"""GPU parity: every call of the C ABI against the CPU oracle on the same
seeded inputs.  Packing, scale blocking and residual binarisation must match
bit for bit; matrix products must meet the stated tolerance
(|y - y_ref| <= 1e-3 * sum_j |W x| + 1e-6 per element; relative L2 <= 1e-5
for the fp32-output GEMV)."""
import numpy as np
import pytest

from oracle import mbok_oracle as O
from boolean_weight_matmul_b200 import workloads as wl
from helpers import (BF16_OUT_REL, GEMV_REL_L2, alpha_blocked_gpu, assert_close, ensure_built, gemm_gpu, x_dev,
                     guarded, guarded_alpha, guarded_packed, check_guards,
                     gemv_gpu, packed_from_signs_gpu, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ensure_built()


def _words_u32(t) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


# --------------------------------------------------------------------------
# Packing
# --------------------------------------------------------------------------

@pytest.mark.parametrize("K,M,N", [(1, 1, 128), (3, 13, 384), (4, 129, 256), (2, 256, 512),
                                   (3, 4096, 4096)])
def test_pack_bits_bit_exact(K, M, N):
    s = wl.random_signs(K, M, N, 200 + K + M, p_zero=0.05)
    got = _words_u32(packed_from_signs_gpu(s))
    assert np.array_equal(got, O.pack_signs(s))


@pytest.mark.parametrize("K,M,N", [(1, 1, 128), (3, 13, 384), (4, 4096, 4096)])
def test_pack_alpha_bit_exact(K, M, N):
    a = wl.alpha_decaying(K, M, N, 300 + K)
    got = alpha_blocked_gpu(a, K, M, N).cpu().numpy()
    assert np.array_equal(got.view(np.uint16), O.block_alpha(a, K, M, N).view(np.uint16))


# --------------------------------------------------------------------------
# Residual binarisation (bit-exact)
# --------------------------------------------------------------------------

def _residual_gpu(W: np.ndarray, K: int):
    import torch
    import boolean_weight_matmul_b200 as mb
    M, N = W.shape
    Wd = to_dev(W)
    packed = guarded_packed(K, M, N)
    alpha = guarded_alpha(K, M, N)
    R = guarded((M, N), torch.float32)
    mb.residual_binarize(Wd, M, N, K, 128, packed, alpha, R)
    torch.cuda.synchronize()
    return _words_u32(packed), alpha.cpu().numpy(), R.cpu().numpy()


def _check_residual(W, K):
    M, N = W.shape
    pw, pa, pr = _residual_gpu(W, K)
    s, a, R = O.residual_binarize(W, K)
    assert np.array_equal(pw, O.pack_signs(s)), "packed kernels differ"
    assert np.array_equal(pa.view(np.uint16), O.block_alpha(a, K, M, N).view(np.uint16)), "scales differ"
    assert np.array_equal(pr.view(np.uint32), R.view(np.uint32)), "residual differs"


@pytest.mark.parametrize("K,M,N", [(1, 256, 512), (3, 256, 512), (4, 13, 384), (2, 1, 128)])
def test_residual_bit_exact_small(K, M, N):
    _check_residual(wl.w_normal(M, N, wl.seed_of(1, K, 3)), K)


def test_residual_edge_cases():
    # zero and negative-zero groups (sign(0) = +1, alpha = 0), and a group whose
    # mean sits just above an fp16 midpoint (single rounding from fp64).
    W = wl.w_normal(9, 384, 77)
    W[0, :128] = 0.0
    W[1, 128:256] = -0.0
    W[2, :] = 1.0
    W[2, 5] = 1 + 2.0 ** -4
    W[2, 77] = 1 + 2.0 ** -23
    for K in (1, 3):
        _check_residual(W, K)


@pytest.mark.parametrize("K,M,N", [(3, 11008, 4096), (2, 4096, 11008)])
def test_residual_bit_exact_llama7b_mlp(K, M, N):
    _check_residual(wl.w_normal(M, N, wl.seed_of(3, 0 if M > N else 2, 3)), K)


# --------------------------------------------------------------------------
# Decode / small-batch GEMV
# --------------------------------------------------------------------------

def _gemv_case(K, M, N, batch, x_dtype, seed, alpha_kind="abs_normal", rows=None, p_zero=0.0):
    s = wl.random_signs(K, M, N, seed, p_zero=p_zero)
    a = (wl.alpha_abs_normal if alpha_kind == "abs_normal" else wl.alpha_decaying)(K, M, N, seed + 1)
    x = wl.x_normal(batch, N, seed + 2, x_dtype)
    y = gemv_gpu(packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N), K, M, N, x, x_dtype)
    y_ref, E = O.linear(O.pack_signs(s), a, K, M, N, x, x_dtype, rows=rows)
    if rows is not None:
        y = y[:, rows]
    return y, y_ref, E


@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("M,N", [(1, 128), (7, 256), (13, 640), (128, 512), (129, 1024), (64, 1536)])
def test_gemv_small_shapes(K, M, N):
    for x_dtype in ("f32", "bf16"):
        y, y_ref, E = _gemv_case(K, M, N, 1, x_dtype, 1000 + 17 * K + M + N)
        assert_close(y, y_ref, E, GEMV_REL_L2, f"K={K} M={M} N={N} {x_dtype}")


@pytest.mark.parametrize("batch", [2, 3, 4, 16])
def test_gemv_small_batch(batch):
    y, y_ref, E = _gemv_case(3, 200, 1152, batch, "bf16", 4000 + batch, "decaying")
    assert_close(y, y_ref, E, GEMV_REL_L2, f"batch={batch}")


def test_gemv_toy_workload_f32():
    w = wl.TOY_GEMV
    s = wl.random_signs(w.K, w.M, w.N, wl.seed_of(1, 0, 4))
    a = wl.alpha_abs_normal(w.K, w.M, w.N, wl.seed_of(1, 0, 1))
    x = wl.x_normal(1, w.N, wl.seed_of(1, 0, 2), "f32")
    y = gemv_gpu(packed_from_signs_gpu(s), alpha_blocked_gpu(a, w.K, w.M, w.N), w.K, w.M, w.N, x, "f32")
    y_ref, E = O.linear(O.pack_signs(s), a, w.K, w.M, w.N, x, "f32")
    assert_close(y, y_ref, E, GEMV_REL_L2, w.name)


def test_gemv_q_proj_full_random_words():
    # LLaMA-7B q_proj, K=3, batch 1, Bernoulli(0.5) words as drawn (layout-free),
    # decaying scales; every output row checked.
    import torch
    w = wl.Q_PROJ_7B
    K, M, N = w.K, w.M, w.N
    words = wl.random_words(O.packed_bytes(K, M, N) // 4, wl.seed_of(2, 0, 0))
    a = wl.alpha_decaying(K, M, N, wl.seed_of(2, 0, 1))
    x = wl.x_normal(1, N, wl.seed_of(2, 0, 2))
    packed = to_dev(words.view(np.int32))
    y = gemv_gpu(packed, alpha_blocked_gpu(a, K, M, N), K, M, N, x, "bf16")
    y_ref, E = O.linear(words, a, K, M, N, x, "bf16")
    assert_close(y, y_ref, E, GEMV_REL_L2, w.name)
    del packed
    torch.cuda.empty_cache()


@pytest.mark.parametrize("which,K,batch", [("gate", 3, 1), ("down", 2, 4), ("up", 3, 16)])
def test_gemv_llama7b_mlp_residual_weights(which, K, batch):
    # Weights from the GPU residual binarisation of W ~ N(0, 0.02^2) (the
    # workload recipe); oracle on 384 sampled rows.
    import torch
    import boolean_weight_matmul_b200 as mb
    w = wl.mlp_7b(K, which, batch)
    M, N = w.M, w.N
    W = wl.w_normal(M, N, wl.seed_of(3, 1, 3))
    packed = guarded_packed(K, M, N)
    alpha = guarded_alpha(K, M, N)
    mb.residual_binarize(to_dev(W), M, N, K, 128, packed, alpha)
    x = wl.x_normal(batch, N, wl.seed_of(3, 1, 2))
    y = gemv_gpu(packed, alpha, K, M, N, x, "bf16")
    words = _words_u32(packed)
    a_mgk = O.unblock_alpha(alpha.cpu().numpy(), K, M, N)
    rows = np.sort(np.random.default_rng(9).choice(M, 384, replace=False))
    y_ref, E = O.linear(words, a_mgk, K, M, N, x, "bf16", rows=rows)
    assert_close(y[:, rows], y_ref, E, GEMV_REL_L2, w.name)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,M,N", [("q", 5120, 5120), ("gate", 13824, 5120), ("down", 5120, 13824)])
def test_gemv_llama13b_shapes_k4_sampled(name, M, N):
    y, y_ref, E = _gemv_case(4, M, N, 1, "bf16", 5000 + M + N, "decaying",
                             rows=np.sort(np.random.default_rng(M).choice(M, 256, replace=False)))
    assert_close(y, y_ref, E, GEMV_REL_L2, f"llama13b {name}")


def test_gemv_flip_invariance_bitwise():
    # Flipping every bit of kernel k and negating its scales gives the same y
    # bit for bit (each lookup negates exactly).
    K, M, N = 3, 300, 1536
    s = wl.random_signs(K, M, N, 61)
    a = wl.alpha_decaying(K, M, N, 62)
    x = wl.x_normal(1, N, 63)
    y0 = gemv_gpu(packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N), K, M, N, x, "bf16")
    for k in range(K):
        s2, a2 = s.copy(), a.copy()
        s2[k] = -s2[k]
        a2[:, :, k] = -a2[:, :, k]
        y1 = gemv_gpu(packed_from_signs_gpu(s2), alpha_blocked_gpu(a2, K, M, N), K, M, N, x, "bf16")
        assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32))


def test_no_kernel_wait_gave_up():
    # Bounded waits inside the kernels never expired during the runs above.
    import boolean_weight_matmul_b200 as mb
    y, y_ref, E = _gemv_case(3, 1000, 4096, 1, "bf16", 77)
    assert_close(y, y_ref, E, GEMV_REL_L2, "after-run check")
    assert mb.read_device_errors() == 0


def test_gemv_deterministic():
    K, M, N = 3, 4096, 4096
    s = wl.random_signs(K, M, N, 71)
    a = wl.alpha_decaying(K, M, N, 72)
    x = wl.x_normal(1, N, 73)
    p, al = packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N)
    y0 = gemv_gpu(p, al, K, M, N, x, "bf16")
    y1 = gemv_gpu(p, al, K, M, N, x, "bf16")
    assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32))


# --------------------------------------------------------------------------
# The two GEMV kernels, each forced for every batch size
# --------------------------------------------------------------------------

# lookup: the default lookup kernel (slabs); tensor: MMAs; lookup_rows: whole
# rows with 4-bit tables where they fit (else slabs).
KERNELS = {"lookup": 1, "tensor": 2, "lookup_rows": 4}


@pytest.mark.parametrize("kernel", ["lookup", "tensor", "lookup_rows"])
@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("M,N,batch", [(1, 128, 1), (7, 256, 3), (13, 640, 5), (129, 1024, 2),
                                       (64, 1536, 16), (24, 384, 6)])
def test_gemv_kernel_small_shapes(kernel, K, M, N, batch):
    import boolean_weight_matmul_b200 as mb
    with mb.gemv_kernel(KERNELS[kernel]):
        for x_dtype in ("f32", "bf16"):
            y, y_ref, E = _gemv_case(K, M, N, batch, x_dtype, 6000 + 17 * K + M + N + batch)
            assert_close(y, y_ref, E, GEMV_REL_L2, f"{kernel} K={K} M={M} N={N} b={batch} {x_dtype}")


@pytest.mark.parametrize("batch", [1, 5, 6, 11, 16])
def test_gemv_tensor_f32_batches(batch):
    # fp32 activations take three bf16 columns each: 5 vectors per launch.
    import boolean_weight_matmul_b200 as mb
    with mb.gemv_kernel(mb.GEMV_TENSOR):
        y, y_ref, E = _gemv_case(3, 40, 768, batch, "f32", 6500 + batch, "decaying")
    assert_close(y, y_ref, E, GEMV_REL_L2, f"tensor f32 batch={batch}")


@pytest.mark.parametrize("batch", [1, 16])
def test_gemv_tensor_q_proj_full(batch):
    # LLaMA-7B q_proj K=3 on the tensor-core kernel, every output row checked.
    import torch
    import boolean_weight_matmul_b200 as mb
    w = wl.Q_PROJ_7B
    K, M, N = w.K, w.M, w.N
    words = wl.random_words(O.packed_bytes(K, M, N) // 4, wl.seed_of(2, 0, 0))
    a = wl.alpha_decaying(K, M, N, wl.seed_of(2, 0, 1))
    x = wl.x_normal(batch, N, wl.seed_of(2, 0, 2))
    packed = to_dev(words.view(np.int32))
    with mb.gemv_kernel(mb.GEMV_TENSOR):
        y = gemv_gpu(packed, alpha_blocked_gpu(a, K, M, N), K, M, N, x, "bf16")
    y_ref, E = O.linear(words, a, K, M, N, x, "bf16")
    assert_close(y, y_ref, E, GEMV_REL_L2, f"{w.name} tensor b{batch}")
    del packed
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,M,N,batch", [("gate", 11008, 4096, 4), ("down", 4096, 11008, 16),
                                            ("gate13b", 13824, 5120, 16)])
def test_gemv_tensor_mlp_sampled(name, M, N, batch):
    K = 3 if name == "gate" else (2 if name == "down" else 4)
    rows = np.sort(np.random.default_rng(M + batch).choice(M, 256, replace=False))
    y, y_ref, E = _gemv_case(K, M, N, batch, "bf16", 7000 + M + N, "decaying", rows=rows)
    assert_close(y, y_ref, E, GEMV_REL_L2, f"tensor {name} b{batch}")


@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("batch", [3, 12])
def test_gemv_tensor_long_rows(K, batch):
    # Rows of 8 or more 1024-column slices take the tensor kernel's deep copy
    # ring: N = 8320 is nine slices, the last one partial (one 128-column
    # group); ragged M; one (batch 3) and two (batch 12) 8-column tiles of B;
    # bf16 and fp32 activations; every output checked.
    import boolean_weight_matmul_b200 as mb
    M, N = 72, 8320
    with mb.gemv_kernel(mb.GEMV_TENSOR):
        for x_dtype in ("bf16", "f32"):
            y, y_ref, E = _gemv_case(K, M, N, batch, x_dtype, 6800 + 10 * K + batch, "decaying")
            assert_close(y, y_ref, E, GEMV_REL_L2, f"tensor long rows K={K} b={batch} {x_dtype}")


@pytest.mark.parametrize("kernel", ["lookup", "tensor", "lookup_rows"])
def test_gemv_kernel_flip_invariance_bitwise(kernel):
    # Negated signs (exact) times negated scales: the same y bit for bit.
    import boolean_weight_matmul_b200 as mb
    K, M, N, batch = 3, 136, 1536, 4
    s = wl.random_signs(K, M, N, 81)
    a = wl.alpha_decaying(K, M, N, 82)
    x = wl.x_normal(batch, N, 83)
    with mb.gemv_kernel(KERNELS[kernel]):
        y0 = gemv_gpu(packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N), K, M, N, x, "bf16")
        for k in range(K):
            s2, a2 = s.copy(), a.copy()
            s2[k] = -s2[k]
            a2[:, :, k] = -a2[:, :, k]
            y1 = gemv_gpu(packed_from_signs_gpu(s2), alpha_blocked_gpu(a2, K, M, N), K, M, N, x, "bf16")
            assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32))


@pytest.mark.parametrize("kernel", ["lookup", "lookup_rows"])
@pytest.mark.parametrize("M,N", [(4096, 4096), (300, 1536), (5120, 13824)])
def test_gemv_static_weights_same_bits(M, N, kernel):
    # Copying weights into shared memory before the dependency wait changes
    # no result: bit-identical outputs, also for a chain of launches whose
    # inputs the previous launch wrote.
    import torch
    import boolean_weight_matmul_b200 as mb
    K = 3
    s = wl.random_signs(K, M, N, 101)
    a = wl.alpha_decaying(K, M, N, 102)
    x = wl.x_normal(1, N, 103)
    p, al = packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N)
    with mb.gemv_kernel(KERNELS[kernel]):
        mb.gemv_set_static_weights(False)
        y0 = gemv_gpu(p, al, K, M, N, x, "bf16")
        mb.gemv_set_static_weights(True)
        try:
            y1 = gemv_gpu(p, al, K, M, N, x, "bf16")
            # chain: y of one launch (bf16) is the x of the next, no host sync between
            xs = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
            ws = mb.zeros_workspace(K, M, N, 1)
            ys = []
            cur = xs
            for _ in range(3):
                y = guarded((1, M), torch.float32)
                mb.gemv(p, al, K, M, N, 128, cur, mb.BF16, 1, y, ws)
                ys.append(y)
                if M == N:
                    cur = (y * 0.05).to(torch.bfloat16)
            torch.cuda.synchronize()
        finally:
            mb.gemv_set_static_weights(True)   # the default
    assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32))
    assert_close(y1, *O.linear(O.pack_signs(s), a, K, M, N, x, "bf16"), GEMV_REL_L2, "static weights")
    if M == N:
        # each link of the chain against the oracle on the activations it actually read
        cur = x
        for y in ys:
            yn = y.cpu().numpy()
            y_ref, E = O.linear(O.pack_signs(s), a, K, M, N, cur, "bf16")
            assert_close(yn, y_ref, E, GEMV_REL_L2, "static weights chain")
            cur = wl.f32_to_bf16_bits((yn * np.float32(0.05)).astype(np.float32))


def test_gemv_tensor_deterministic_and_batch_independent():
    # Same bits run to run; a vector's result does not depend on its batch
    # neighbours (columns of B never mix) among batches that use the same
    # launch shape (up to 8 vectors: one 8-column MMA tile; 9..16: two).
    import boolean_weight_matmul_b200 as mb
    K, M, N = 3, 1000, 4096
    s = wl.random_signs(K, M, N, 91)
    a = wl.alpha_decaying(K, M, N, 92)
    x = wl.x_normal(16, N, 93)
    p, al = packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N)
    with mb.gemv_kernel(mb.GEMV_TENSOR):
        y0 = gemv_gpu(p, al, K, M, N, x, "bf16")
        y1 = gemv_gpu(p, al, K, M, N, x, "bf16")
        y9 = gemv_gpu(p, al, K, M, N, x[:9], "bf16")
        y8 = gemv_gpu(p, al, K, M, N, x[:8], "bf16")
        y_one = gemv_gpu(p, al, K, M, N, x[5:6], "bf16")
    assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32))
    assert np.array_equal(y0[:9].view(np.uint32), y9.view(np.uint32))
    assert np.array_equal(y8[5].view(np.uint32), y_one[0].view(np.uint32))


@pytest.mark.parametrize("kernel", ["lookup", "tensor", "lookup_rows"])
def test_gemv_ex_per_call_choice_equals_process_wide(kernel):
    # mbok_gemv_ex with a kernel and static-weights flag per call gives, bit for
    # bit, what mbok_gemv gives under the same process-wide choices.
    import torch
    import boolean_weight_matmul_b200 as mb
    K, M, N, batch = 3, 264, 1536, 3
    s = wl.random_signs(K, M, N, 71)
    a = wl.alpha_decaying(K, M, N, 72)
    x = x_dev(wl.x_normal(batch, N, 73), "bf16")
    p, al = packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N)
    ws = mb.zeros_workspace(K, M, N, batch)
    for static in (True, False):
        y0 = guarded((batch, M), torch.float32)
        with mb.gemv_kernel(KERNELS[kernel]):
            mb.gemv_set_static_weights(static)
            try:
                mb.gemv(p, al, K, M, N, 128, x, mb.BF16, batch, y0, ws)
            finally:
                mb.gemv_set_static_weights(True)
        y1 = guarded((batch, M), torch.float32)
        mb.gemv(p, al, K, M, N, 128, x, mb.BF16, batch, y1, ws, kernel=KERNELS[kernel], weights_static=static)
        torch.cuda.synchronize()
        assert torch.equal(y0.view(torch.int32), y1.view(torch.int32))


@pytest.mark.parametrize("K,M,N", [
    (3, 20000, 4096),    # 68 row pairs per CTA: more octets than ring slots, the ring wraps
    (2, 40000, 512),     # more than 128 row pairs per CTA would be needed: a second wave of CTAs
    (4, 1000, 10240),    # the widest rows the 4-bit tables cover (20 blocks of 512 columns)
    (1, 333, 10368),     # one unit block more: the slab kernel takes over
])
def test_gemv_lookup_whole_rows_geometry(K, M, N):
    # Row ranges that start and end inside octets, sampled around every CTA
    # boundary of the whole-row lookup kernel plus random rows.
    import boolean_weight_matmul_b200 as mb
    pairs = (M + 1) // 2
    ncta = min(148, pairs)
    if -(-pairs // ncta) > 128:
        ncta = -(-pairs // 128)
    edges = np.array([2 * (c * pairs // ncta) for c in range(ncta)])
    rows = np.unique(np.clip(np.concatenate([edges - 1, edges, edges + 1, [M - 1],
                                             np.random.default_rng(M).choice(M, 200, replace=False)]), 0, M - 1))
    with mb.gemv_kernel(mb.GEMV_LOOKUP_ROWS):
        y, y_ref, E = _gemv_case(K, M, N, 1, "bf16", 8800 + M + N, "decaying", rows=rows)
    assert_close(y, y_ref, E, GEMV_REL_L2, f"whole-row lookup K={K} M={M} N={N}")
    assert mb.read_device_errors() == 0


def _multi_case(Ks, Ms, N, batch, x_dtype, seed):
    """mbok_gemv_multi over matrices with their own K and M, the separate
    slab lookup-kernel calls, and the oracle (per matrix, concatenated)."""
    import torch
    import boolean_weight_matmul_b200 as mb
    signs = [wl.random_signs(K, M, N, seed + 10 * i) for i, (K, M) in enumerate(zip(Ks, Ms))]
    alphas = [wl.alpha_decaying(K, M, N, seed + 10 * i + 1) for i, (K, M) in enumerate(zip(Ks, Ms))]
    x = wl.x_normal(batch, N, seed + 99, x_dtype)
    packed = [packed_from_signs_gpu(sg) for sg in signs]
    alpha = [alpha_blocked_gpu(a, K, M, N) for a, K, M in zip(alphas, Ks, Ms)]
    xd = x_dev(x, x_dtype)
    dt = mb.F32 if x_dtype == "f32" else mb.BF16
    y = guarded((batch, sum(Ms)), torch.float32)
    mb.gemv_multi(packed, alpha, Ks, Ms, N, 128, xd, dt, batch, y, mb.zeros_multi_workspace(Ks, Ms, N))
    torch.cuda.synchronize()
    with mb.gemv_kernel(mb.GEMV_LOOKUP_SLABS):
        sep = np.concatenate([gemv_gpu(p, a, K, M, N, x, x_dtype) for p, a, K, M in zip(packed, alpha, Ks, Ms)],
                             axis=1)
    refs = [O.linear(O.pack_signs(sg), a, K, M, N, x, x_dtype) for sg, a, K, M in zip(signs, alphas, Ks, Ms)]
    y_ref = np.concatenate([r[0] for r in refs], axis=1)
    E = np.concatenate([r[1] for r in refs], axis=1)
    return y.cpu().numpy(), sep, y_ref, E


@pytest.mark.parametrize("Ks,Ms,N,batch,x_dtype", [
    ((4, 2, 3), (136, 64, 77), 1536, 1, "bf16"),     # mixed K, ragged M, 3 slabs
    ((3, 1), (40, 8), 512, 2, "f32"),                 # one slab: outputs stored directly, two vectors
    ((2,), (300,), 1024, 1, "bf16"),                  # a single matrix
    ((1, 2, 3, 4, 1, 2, 3, 4), (8, 16, 24, 32, 40, 48, 56, 64), 640, 1, "bf16"),   # eight matrices, ragged slab
    ((3, 1), (40, 24), 9216, 1, "bf16"),              # 18 slabs: the combine's batch of 16 and its remainder
])
def test_gemv_multi_equals_separate_calls(Ks, Ms, N, batch, x_dtype):
    # Each row is computed as in its own matrix's launch (same tables, same
    # octet order, slabs added in order), so the fused outputs equal the
    # separate slab lookup-kernel calls bit for bit, and the oracle within tolerance.
    y, sep, y_ref, E = _multi_case(Ks, Ms, N, batch, x_dtype, 12000 + N + sum(Ms))
    assert np.array_equal(y.view(np.uint32), sep.view(np.uint32))
    assert_close(y, y_ref, E, GEMV_REL_L2, f"multi K={Ks} M={Ms} N={N}")


def test_gemv_multi_llama13b_qkv_mixed_k():
    # LLaMA-13B q, k, v (5120 x 5120 each) with K = 4, 2, 3 in one launch.
    y, sep, y_ref, E = _multi_case((4, 2, 3), (5120, 5120, 5120), 5120, 1, "bf16", 13000)
    assert np.array_equal(y.view(np.uint32), sep.view(np.uint32))
    assert_close(y, y_ref, E, GEMV_REL_L2, "13B qkv mixed K")


def test_gemv_fused_projections_equal_separate_calls():
    # Matrices with the same K and N whose M are multiples of 8 fuse along M by
    # concatenating their packed bytes and blocked scales (octet-major storage):
    # one call gives, row for row, the bits of the separate calls.
    import torch
    import boolean_weight_matmul_b200 as mb
    K, N = 3, 1280
    Ms = (320, 64, 64)
    parts = []
    for i, M in enumerate(Ms):
        s = wl.random_signs(K, M, N, 9300 + i)
        a = wl.alpha_decaying(K, M, N, 9310 + i)
        parts.append((packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N), M))
    for batch in (1, 4):
        x = wl.x_normal(batch, N, 9320 + batch)
        ys = [gemv_gpu(p, al, K, M, N, x, "bf16") for (p, al, M) in parts]
        packed = torch.cat([p for (p, _, _) in parts])
        alpha = torch.cat([al for (_, al, _) in parts])
        y = gemv_gpu(packed, alpha, K, sum(Ms), N, x, "bf16")
        assert np.array_equal(y.view(np.uint32), np.concatenate(ys, axis=1).view(np.uint32))


# --------------------------------------------------------------------------
# Rank-1 (SVID) scaled kernels
# --------------------------------------------------------------------------

def _svid_gpu(signs, s_in, s_out, x, x_dtype, s_out_offset=0):
    import torch
    import boolean_weight_matmul_b200 as mb
    K, M, N = signs.shape
    batch = x.shape[0]
    packed = packed_from_signs_gpu(signs) if signs.dtype == np.int8 else signs
    si = to_dev(np.ascontiguousarray(s_in, dtype=np.float16).view(np.int16)).view(torch.float16)
    so = to_dev(np.ascontiguousarray(s_out, dtype=np.float16).view(np.int16)).view(torch.float16)
    if s_out_offset:
        # the same scales at an element offset inside a larger buffer
        buf = torch.zeros(so.numel() + s_out_offset, dtype=torch.float16, device=so.device)
        buf[s_out_offset:].copy_(so.reshape(-1))
        so = buf[s_out_offset:].view(K, M)
    xd = x_dev(x, x_dtype)
    y = guarded((batch, M), torch.float32)
    ws = mb.zeros_svid_workspace(K, M, N, batch)
    mb.gemv_svid(packed, si, so, K, M, N, xd, mb.F32 if x_dtype == "f32" else mb.BF16, batch, y, ws)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("M,N,batch", [(1, 128, 1), (13, 640, 3), (129, 1024, 1), (64, 1536, 2)])
def test_gemv_svid_small_shapes(K, M, N, batch):
    for x_dtype in ("f32", "bf16"):
        s = wl.random_signs(K, M, N, 8000 + K + M, p_zero=0.05)
        s_in, s_out = wl.svid_scales(K, M, N, 8001 + K + M)
        x = wl.x_normal(batch, N, 8002 + K + M, x_dtype)
        y = _svid_gpu(s, s_in, s_out, x, x_dtype)
        y_ref, E = O.linear_svid(O.pack_signs(s), s_in, s_out, K, M, N, x, x_dtype)
        assert_close(y, y_ref, E, GEMV_REL_L2, f"svid K={K} M={M} N={N} b={batch} {x_dtype}")


@pytest.mark.parametrize("K,M,N,offset", [(3, 64, 1536, 1), (2, 256, 4096, 4), (4, 136, 1024, 8)])
def test_gemv_svid_output_scale_alignment(K, M, N, offset):
    """s_out at a 2-, 8- or 16-byte offset with M % 8 == 0: the kernel copies
    each octet's scales with its bits only from a 16-byte-aligned s_out, and
    loads them one by one otherwise; both give the oracle's result."""
    s = wl.random_signs(K, M, N, 8300 + K + M)
    s_in, s_out = wl.svid_scales(K, M, N, 8301 + K + M)
    x = wl.x_normal(2, N, 8302 + K + M)
    y = _svid_gpu(s, s_in, s_out, x, "bf16", s_out_offset=offset)
    y_ref, E = O.linear_svid(O.pack_signs(s), s_in, s_out, K, M, N, x, "bf16")
    assert_close(y, y_ref, E, GEMV_REL_L2, f"svid K={K} M={M} N={N} s_out offset {offset}")


@pytest.mark.parametrize("K,M,N,sample", [(3, 4096, 4096, None), (4, 13824, 5120, 256), (2, 4096, 11008, 256)])
def test_gemv_svid_llama_shapes(K, M, N, sample):
    s = wl.random_signs(K, M, N, 8100 + M)
    s_in, s_out = wl.svid_scales(K, M, N, 8101 + M)
    x = wl.x_normal(1, N, 8102 + M)
    rows = None if sample is None else np.sort(np.random.default_rng(M).choice(M, sample, replace=False))
    y = _svid_gpu(s, s_in, s_out, x, "bf16")
    y_ref, E = O.linear_svid(O.pack_signs(s), s_in, s_out, K, M, N, x, "bf16", rows=rows)
    if rows is not None:
        y = y[:, rows]
    assert_close(y, y_ref, E, GEMV_REL_L2, f"svid {M}x{N} K={K}")


def test_gemv_svid_flip_invariance_and_determinism():
    K, M, N = 3, 136, 1536
    s = wl.random_signs(K, M, N, 8201)
    s_in, s_out = wl.svid_scales(K, M, N, 8202)
    x = wl.x_normal(1, N, 8203)
    y0 = _svid_gpu(s, s_in, s_out, x, "bf16")
    assert np.array_equal(y0.view(np.uint32), _svid_gpu(s, s_in, s_out, x, "bf16").view(np.uint32))
    for k in range(K):
        s2, so2 = s.copy(), s_out.copy()
        s2[k] = -s2[k]
        so2[k] = -so2[k]
        y1 = _svid_gpu(s2, s_in, so2, x, "bf16")
        assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32))


# --------------------------------------------------------------------------
# Closed-form scale refit (bit-exact)
# --------------------------------------------------------------------------

def _refit_gpu(W, packed, K):
    import torch
    import boolean_weight_matmul_b200 as mb
    M, N = W.shape
    out = guarded_alpha(K, M, N)
    mb.refit_alpha(to_dev(W), packed, K, M, N, 128, out)
    torch.cuda.synchronize()
    return O.unblock_alpha(out.cpu().numpy(), K, M, N)


@pytest.mark.parametrize("K,M,N", [(1, 13, 384), (2, 64, 256), (3, 37, 512), (4, 16, 1024)])
def test_refit_bit_exact_random_kernels(K, M, N):
    W = wl.w_normal(M, N, 9000 + K)
    signs = wl.random_signs(K, M, N, 9001 + K, p_zero=0.02)
    packed = packed_from_signs_gpu(signs)
    got = _refit_gpu(W, packed, K)
    want = O.refit_alpha(W, O.pack_signs(signs), K, M, N)
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


def test_refit_bit_exact_on_greedy_kernels_and_dependent_kernels():
    # Kernels from the GPU residual binarisation; then kernel 2 replaced by
    # kernel 0 negated on half the rows (exactly dependent: scale 0).
    import boolean_weight_matmul_b200 as mb
    K, M, N = 3, 40, 768
    W = wl.w_normal(M, N, 9100)
    packed = guarded_packed(K, M, N)
    alpha = guarded_alpha(K, M, N)
    mb.residual_binarize(to_dev(W), M, N, K, 128, packed, alpha)
    words = _words_u32(packed)
    signs = O.unpack_bits(words, K, M, N)
    got = _refit_gpu(W, packed, K)
    assert np.array_equal(got.view(np.uint16), O.refit_alpha(W, words, K, M, N).view(np.uint16))
    s2 = signs.copy()
    s2[2, : M // 2] = -s2[0, : M // 2]
    got2 = _refit_gpu(W, packed_from_signs_gpu(s2.astype(np.int8)), K)
    want2 = O.refit_alpha(W, O.pack_signs(s2.astype(np.int8)), K, M, N)
    assert np.array_equal(got2.view(np.uint16), want2.view(np.uint16))
    assert np.all(want2[: M // 2, :, 2] == 0)


def test_refit_llama7b_gate_sampled():
    import boolean_weight_matmul_b200 as mb
    K, M, N = 3, 11008, 4096
    W = wl.w_normal(M, N, 9200)
    packed = guarded_packed(K, M, N)
    alpha = guarded_alpha(K, M, N)
    mb.residual_binarize(to_dev(W), M, N, K, 128, packed, alpha)
    got = _refit_gpu(W, packed, K)
    rows = np.sort(np.random.default_rng(3).choice(M, 64, replace=False))
    want = O.refit_alpha(W, _words_u32(packed), K, M, N, rows=rows)
    assert np.array_equal(got[rows].view(np.uint16), want.view(np.uint16))


# --------------------------------------------------------------------------
# Successive SVID: signs and residual bit-exact given the scales; scales
# within one fp16 rounding of the SVD's
# --------------------------------------------------------------------------

def _svid_binarize_gpu(W, K, iters=6):
    import torch
    import boolean_weight_matmul_b200 as mb
    M, N = W.shape
    packed = guarded_packed(K, M, N)
    s_in = guarded((K, N), torch.float16)
    s_out = guarded((K, M), torch.float16)
    R = guarded((M, N), torch.float32)
    mb.svid_binarize(to_dev(W), M, N, K, iters, packed, s_in, s_out, R)
    torch.cuda.synchronize()
    return _words_u32(packed), s_in.cpu().numpy(), s_out.cpu().numpy(), R.cpu().numpy()


def _check_svid_steps(W, K, words, s_in, s_out, R_gpu, rows=None):
    # Replay the steps in the oracle with the GPU's fp16 scales: each kernel's
    # signs and the final residual must match bit for bit; each scale must be
    # within one fp16 ulp of the rank-1 SVD of |R| (which the oracle computes).
    M, N = W.shape
    signs = O.unpack_bits(words, K, M, N)
    R = W.astype(np.float32)
    for k in range(K):
        so_ref, si_ref = O.svid_scales_of(np.abs(R.astype(np.float64)))
        for got, ref in ((s_out[k], so_ref), (s_in[k], si_ref)):
            ulp = np.spacing(np.abs(ref)).astype(np.float64)
            assert np.all(np.abs(got.astype(np.float64) - ref.astype(np.float64)) <= ulp), f"kernel {k} scales"
        b, R = O.svid_step(R, s_out[k], s_in[k])
        assert np.array_equal(signs[k], b), f"kernel {k} signs"
    assert np.array_equal(R_gpu.view(np.uint32), R.view(np.uint32))


@pytest.mark.parametrize("K,M,N", [(1, 8, 128), (3, 300, 768), (4, 77, 1024), (2, 512, 2048)])
def test_svid_binarize_stepwise(K, M, N):
    W = wl.w_normal(M, N, 9400 + K + M)
    words, s_in, s_out, R = _svid_binarize_gpu(W, K)
    _check_svid_steps(W, K, words, s_in, s_out, R)


def test_svid_binarize_exact_rank1_and_zero_residual():
    # |W| constant: the first kernel is exact, the residual is 0, and the next
    # kernel's scales are 0 (no NaN from the all-zero residual).
    M, N, c = 16, 256, 0.0625
    W = (np.where(wl.random_signs(1, M, N, 5)[0] >= 0, 1.0, -1.0) * c).astype(np.float32)
    words, s_in, s_out, R = _svid_binarize_gpu(W, 2)
    assert np.all(s_out[0] == 0.5) and np.all(s_in[0] == 0.125)
    assert np.all(s_out[1] == 0) and np.all(s_in[1] == 0) and np.all(R == 0)


def test_svid_binarize_then_gemv_matches_oracle():
    # The kernels and scales it produces drive mbok_gemv_svid.
    K, M, N = 3, 1024, 4096
    W = wl.w_normal(M, N, 9500)
    words, s_in, s_out, R = _svid_binarize_gpu(W, K)
    _check_svid_steps(W, K, words, s_in, s_out, R)
    x = wl.x_normal(1, N, 9501)
    import torch
    import boolean_weight_matmul_b200 as mb
    packed = to_dev(words.view(np.int32))
    si = to_dev(s_in.view(np.int16)).view(torch.float16)
    so = to_dev(s_out.view(np.int16)).view(torch.float16)
    yd = guarded((1, M), torch.float32)
    mb.gemv_svid(packed, si, so, K, M, N, x_dev(x, "bf16"), mb.BF16, 1, yd, mb.zeros_svid_workspace(K, M, N))
    torch.cuda.synchronize()
    y_ref, E = O.linear_svid(words, s_in, s_out, K, M, N, x, "bf16")
    assert_close(yd.cpu().numpy(), y_ref, E, GEMV_REL_L2, "svid_binarize -> gemv_svid")


def test_bounded_wait_gives_up_and_context_stays_usable():
    # A wait that nothing completes ends after its limit with an error flag
    # the host reads; the flag clears on read and the next call works.
    import boolean_weight_matmul_b200 as mb
    assert mb.read_device_errors() == 0
    mb.check_wait_timeout(20000)
    assert mb.read_device_errors() == 4
    assert mb.read_device_errors() == 0
    y, y_ref, E = _gemv_case(3, 64, 512, 2, "bf16", 9600)
    assert_close(y, y_ref, E, GEMV_REL_L2, "after the timeout check")


# --------------------------------------------------------------------------
# Prefill GEMM
# --------------------------------------------------------------------------

@pytest.mark.parametrize("K,M,N,T", [(1, 128, 128, 1), (3, 200, 384, 37), (4, 129, 512, 130),
                                     (2, 64, 1024, 256)])
def test_gemm_small(K, M, N, T):
    s = wl.random_signs(K, M, N, 800 + T)
    a = wl.alpha_decaying(K, M, N, 801 + T)
    X = wl.x_normal(T, N, 802 + T)
    Y = gemm_gpu(packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N), K, M, N, X)
    Y_ref, E = O.linear(O.pack_signs(s), a, K, M, N, X, "bf16")
    assert_close(Y, Y_ref, E, None, f"gemm K={K} M={M} N={N} T={T}", out_rel=BF16_OUT_REL)


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_gemm_weight_tile_is_each_level_rounded_once(K, split):
    # With X the identity (token t = unit vector e_t) every output is one
    # weight of the tile: Y[t][r] = Wt[r][t] (one nonzero product per tile
    # term, fp32 accumulation).  With one rounding it must be the exact weight
    # W[r][t] = sum_k alpha_k b_k rounded once to bf16, bit for bit; with the
    # split, RN_bf16(hi + lo) where hi = RN_bf16(W) and lo = RN_bf16(W - hi),
    # i.e. again RN_bf16(W) after the output's rounding.  Rows and columns span
    # two row tiles, two groups and every column of a stage.
    import boolean_weight_matmul_b200 as mb
    M, N = 256, 256
    s = wl.random_signs(K, M, N, 870 + K)
    a = wl.alpha_decaying(K, M, N, 875 + K)
    eye = np.zeros((N, N), dtype=np.float32)
    np.fill_diagonal(eye, 1.0)
    X = (eye.view(np.uint32) >> 16).astype(np.uint16)   # bf16 bit patterns of 0 and 1
    Y = gemm_gpu(packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N), K, M, N, X,
                 precision=mb.GEMM_SPLIT if split else mb.GEMM_BF16)
    W = O.reconstruct_W(O.pack_signs(s), a, K, M, N)
    want = O.round_bf16(W).T
    bad = np.argwhere(Y != want)
    assert bad.size == 0, (f"{len(bad)} weights differ from RN_bf16(W), e.g. token {bad[0][0]} row {bad[0][1]}: "
                           f"got {Y[tuple(bad[0])]} want {want[tuple(bad[0])]}")


@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("N", [128, 256, 512, 1024])
def test_gemm_small_n_every_output(K, N):
    # Small N is where the accumulation bound 1e-3 * sum|W x| is tightest
    # against the weight tile's rounding: 4096 tokens, every output checked,
    # with mbok_gemm's own choice (the split up to N = 512, one rounding above).
    M, T = 256, 4096
    s = wl.random_signs(K, M, N, 850 + 10 * K + N)
    a = wl.alpha_decaying(K, M, N, 851 + 10 * K + N)
    X = wl.x_normal(T, N, 852 + 10 * K + N)
    Y = gemm_gpu(packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N), K, M, N, X)
    Y_ref, E = O.linear(O.pack_signs(s), a, K, M, N, X, "bf16")
    assert_close(Y, Y_ref, E, None, f"gemm K={K} N={N} T={T}", out_rel=BF16_OUT_REL)


@pytest.mark.parametrize("K", [1, 3])
def test_gemm_split_at_prefill_width(K):
    # The split asked for explicitly at N = 4096: same bound, sampled rows.
    import boolean_weight_matmul_b200 as mb
    M, N, T = 512, 4096, 1024
    s = wl.random_signs(K, M, N, 860 + K)
    a = wl.alpha_decaying(K, M, N, 861 + K)
    X = wl.x_normal(T, N, 862 + K)
    Y = gemm_gpu(packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N), K, M, N, X, precision=mb.GEMM_SPLIT)
    rows = np.sort(np.random.default_rng(863).choice(M, 64, replace=False))
    Y_ref, E = O.linear(O.pack_signs(s), a, K, M, N, X, "bf16", rows=rows)
    assert_close(Y[:, rows], Y_ref, E, None, f"gemm split K={K}", out_rel=BF16_OUT_REL)


def test_gemm_prefill_q_proj_sampled():
    # LLaMA-7B q_proj prefill: K=3, 4096 x 4096, 2048 tokens; 128 sampled rows.
    w = wl.PREFILL_7B
    K, M, N, T = w.K, w.M, w.N, w.tokens
    words = wl.random_words(O.packed_bytes(K, M, N) // 4, wl.seed_of(4, 0, 0))
    a = wl.alpha_decaying(K, M, N, wl.seed_of(4, 0, 1))
    X = wl.x_normal(T, N, wl.seed_of(4, 0, 2))
    Y = gemm_gpu(to_dev(words.view(np.int32)), alpha_blocked_gpu(a, K, M, N), K, M, N, X)
    rows = np.sort(np.random.default_rng(4).choice(M, 128, replace=False))
    Y_ref, E = O.linear(words, a, K, M, N, X, "bf16", rows=rows)
    assert_close(Y[:, rows], Y_ref, E, None, w.name, out_rel=BF16_OUT_REL)


def test_gemm_several_tiles_per_cta():
    # More tiles than SMs (4096 rows = 16 row tiles x 18 token tiles of 4096
    # tokens): persistent CTAs take a second tile and reuse their tensor-memory
    # accumulators after the epilogue drains them.  Sampled rows from every
    # row tile, every token.
    import boolean_weight_matmul_b200 as mb
    K, M, N, T = 3, 4096, 4096, 4096
    s = wl.random_signs(K, M, N, 881)
    a = wl.alpha_decaying(K, M, N, 882)
    X = wl.x_normal(T, N, 883)
    Y = gemm_gpu(packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N), K, M, N, X)
    rows = np.sort(np.concatenate([np.random.default_rng(884 + t).choice(256, 8, replace=False) + 256 * t
                                   for t in range(M // 256)]))
    Y_ref, E = O.linear(O.pack_signs(s), a, K, M, N, X, "bf16", rows=rows)
    assert_close(Y[:, rows], Y_ref, E, None, "gemm several tiles per CTA", out_rel=BF16_OUT_REL)
    assert mb.read_device_errors() == 0


@pytest.mark.parametrize("precision", ["auto", "bf16"])
def test_gemm_many_short_tiles_per_cta(precision):
    # N = 128 is two 64-column stages per tile, fewer than the copy ring's
    # slots, and 4096 rows x 8192 tokens make 16 x 32 tiles, so persistent CTAs
    # take three or four tiles each: the last one is drained by all 20 warps
    # only once it is in the accumulator.  Every output checked, for the split
    # (mbok_gemm's choice at N = 128) and for the single bf16 tile.
    import boolean_weight_matmul_b200 as mb
    K, M, N, T = 2, 4096, 128, 8192
    s = wl.random_signs(K, M, N, 891)
    a = wl.alpha_decaying(K, M, N, 892)
    X = wl.x_normal(T, N, 893)
    prec = None if precision == "auto" else mb.GEMM_BF16
    Y = gemm_gpu(packed_from_signs_gpu(s), alpha_blocked_gpu(a, K, M, N), K, M, N, X, precision=prec)
    Y_ref, E = O.linear(O.pack_signs(s), a, K, M, N, X, "bf16")
    if precision == "auto":
        assert_close(Y, Y_ref, E, None, "gemm many short tiles", out_rel=BF16_OUT_REL)
    else:
        # A single bf16 tile: each weight rounded once (|dW| <= 2^-9 |W|, so
        # |dy| <= 2^-9 sum|W x| = 2^-9 E) plus the output's own rounding,
        # each bound taken with a factor 2 of margin, per element.
        assert np.isfinite(Y).all()
        bad = np.abs(Y - Y_ref) > 2.0 ** -8 * E + 2.0 ** -8 * np.abs(Y_ref) + 1e-6
        assert not bad.any(), f"{int(bad.sum())} outputs outside the bf16-tile bound"
    assert mb.read_device_errors() == 0


def test_gemm_no_wait_gave_up():
    import boolean_weight_matmul_b200 as mb
    s = wl.random_signs(2, 256, 512, 991)
    a = wl.alpha_decaying(2, 256, 512, 992)
    X = wl.x_normal(300, 512, 993)
    Y = gemm_gpu(packed_from_signs_gpu(s), alpha_blocked_gpu(a, 2, 256, 512), 2, 256, 512, X)
    Y_ref, E = O.linear(O.pack_signs(s), a, 2, 256, 512, X, "bf16")
    assert_close(Y, Y_ref, E, None, "gemm after-run check", out_rel=BF16_OUT_REL)
    assert mb.read_device_errors() == 0


def test_output_guards_catch_a_write_past_the_end():
    # The guard check itself: a byte written just past an output (here by the
    # host, through torch) must be reported.
    import torch
    y = guarded((3, 5), torch.float32)
    y.fill_(1.0)
    base = y.view(-1).view(torch.uint8)
    raw = torch.as_strided(base, (base.numel() + 1,), (1,))   # one byte beyond the end
    raw[-1] = 0
    with pytest.raises(AssertionError):
        check_guards()
