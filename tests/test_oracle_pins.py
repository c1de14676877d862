"""Pins for the CPU oracle, each against something other than the oracle itself.

Every check cites the fact it rests on.  A plausible slip in the oracle (a
dropped kernel, a wrong sign, a transposed index, a wrong word or bit order, a
double rounding of the scale) fails at least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import mbok_oracle as O
from boolean_weight_matmul_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _signs_alpha_x(K, M, N, seed, x_dtype="f32"):
    s = wl.random_signs(K, M, N, seed)
    a = wl.alpha_abs_normal(K, M, N, seed + 1)
    x = wl.x_normal(1, N, seed + 2, x_dtype)
    return s, a, x


# --------------------------------------------------------------------------
# Layout (O6): hand-worked words, scalar addressing, round trip
# --------------------------------------------------------------------------

def test_layout_hand_worked_example():
    # tests/golden/layout_k2_2x128.txt: words derived by hand from the format rules.
    with open(os.path.join(GOLDEN, "layout_k2_2x128.txt")) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]
    assert lines[0] == "K=2 M=2 N=128"
    expect = [int(t, 16) for t in lines[1].split(":")[1].split()]
    j = np.arange(128)
    signs = np.stack([
        np.stack([np.where(j % 3 == 0, 1, -1), np.where((j == 5) | (j == 100), 1, -1)]),
        np.stack([np.where(j < 40, 1, -1), -np.ones(128, dtype=int)]),
    ]).astype(np.int8)                                  # [K=2][M=2][N=128]
    packed = O.pack_signs(signs)
    assert packed.shape == (O.packed_bytes(2, 2, 128) // 4,) == (64,)
    assert [int(v) for v in packed[0::4]] == expect
    assert not np.delete(packed, np.arange(0, 64, 4)).any()
    idx = dict(t.split("=") for t in lines[2].split(":")[1].split())
    for k in range(2):
        for r in range(2):
            assert O.alpha_index(2, 2, 128, k, r, 0) == int(idx[f"k{k}r{r}"])
    assert O.alpha_elems(2, 2, 128) == int(idx["total"])
    a = np.arange(4, dtype=np.float16).reshape(2, 1, 2)            # [M][G][K]
    blk = O.block_alpha(a, 2, 2, 128)
    assert blk.shape == (16,)
    assert [float(blk[i]) for i in (0, 1, 8, 9)] == [0.0, 2.0, 1.0, 3.0]
    assert np.array_equal(O.unblock_alpha(blk, 2, 2, 128), a)


def test_layout_scalar_addressing_ragged():
    # The vectorised packer agrees bit by bit with the scalar address rule, for
    # a ragged last octet (M=13) and three groups.
    K, M, N = 3, 13, 384
    s = wl.random_signs(K, M, N, 11, p_zero=0.05)
    by = O.pack_signs(s).view(np.uint8)
    r = np.random.default_rng(5)
    for _ in range(3000):
        k, row, col = int(r.integers(K)), int(r.integers(M)), int(r.integers(N))
        byte, bit = O.byte_and_bit(K, M, N, k, row, col)
        assert (int(by[byte]) >> bit) & 1 == int(s[k, row, col] >= 0)


def test_layout_round_trip_and_zero_maps_to_plus_one():
    K, M, N = 4, 129, 256
    s = wl.random_signs(K, M, N, 12, p_zero=0.1)
    b = O.unpack_bits(O.pack_signs(s), K, M, N)
    assert np.array_equal(b, np.where(s >= 0, 1, -1))
    a = wl.alpha_decaying(K, M, N, 13)
    assert np.array_equal(O.unblock_alpha(O.block_alpha(a, K, M, N), K, M, N), a)


# --------------------------------------------------------------------------
# The linear op (O1 brute force, O2 flips, O3 levels, O5 XNOR, O7 dense)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("K", [1, 2, 3])
def test_brute_force_exact_rational(K):
    # y_r = sum_j (sum_k alpha_{k,r,g(j)} s_{k,r,j}) x_j in exact rational
    # arithmetic, straight from the int8 signs (Paper-Notes 关键设计:
    # W ~= sum_k alpha_k B_k with group-wise scales).
    M, N = 3, 256
    s, a, x = _signs_alpha_x(K, M, N, 100 + K)
    y, E = O.linear(O.pack_signs(s), a, K, M, N, x, "f32")
    xf = [Fraction(float(v)) for v in x[0]]
    for r in range(M):
        acc = Fraction(0)
        for j in range(N):
            w = sum(Fraction(float(a[r, j // 128, k])) * int(s[k, r, j] >= 0 and 1 or -1) for k in range(K))
            acc += w * xf[j]
        assert abs(y[0, r] - float(acc)) <= 1e-14 * E[0, r] + 1e-300


def test_per_kernel_decomposition_agrees():
    # The pages' form "Wx = K Boolean mat-vecs" (Paper-Notes 关键设计):
    # sum_k alpha_k (B_k x), evaluated kernel by kernel and group by group.
    K, M, N = 3, 5, 384
    s, a, x = _signs_alpha_x(K, M, N, 7)
    y, E = O.linear(O.pack_signs(s), a, K, M, N, x, "f32")
    xf = x[0].astype(np.float64)
    y2 = np.zeros(M)
    for k in range(K):
        for g in range(N // 128):
            sl = slice(128 * g, 128 * g + 128)
            y2 += a[:, g, k].astype(np.float64) * (s[k][:, sl].astype(np.float64) @ xf[sl])
    assert np.all(np.abs(y[0] - y2) <= 1e-13 * E[0])


def test_flip_invariance_bitwise():
    # Negating alpha_k and flipping every sign of B_k leaves W, hence y,
    # unchanged exactly (IEEE negation is exact).
    K, M, N = 3, 7, 256
    s, a, x = _signs_alpha_x(K, M, N, 21)
    y0, _ = O.linear(O.pack_signs(s), a, K, M, N, x, "f32")
    for k in range(K):
        s2, a2 = s.copy(), a.copy()
        s2[k] = -s2[k]
        a2[:, :, k] = -a2[:, :, k]
        y1, _ = O.linear(O.pack_signs(s2), a2, K, M, N, x, "f32")
        assert np.array_equal(y0, y1)


# --------------------------------------------------------------------------
# Rank-1 (SVID) scales: W = sum_k B_k (.) (s_out^k s_in^k^T)
# (Italian 2A/2B, Dutch "Methodologie" 2, Spanish 2B)
# --------------------------------------------------------------------------

def _svid_case(K, M, N, seed):
    s = wl.random_signs(K, M, N, seed, p_zero=0.05)
    s_in, s_out = wl.svid_scales(K, M, N, seed + 1)
    x = wl.x_normal(2, N, seed + 2, "f32")
    return s, s_in, s_out, x


@pytest.mark.parametrize("K", [1, 2, 3])
def test_svid_brute_force_exact_rational(K):
    # y_r = sum_j (sum_k b_krj s_out_kr s_in_kj) x_j in exact rational arithmetic.
    M, N = 3, 128
    s, s_in, s_out, x = _svid_case(K, M, N, 400 + K)
    y, E = O.linear_svid(O.pack_signs(s), s_in, s_out, K, M, N, x, "f32")
    for b in range(2):
        xf = [Fraction(float(v)) for v in x[b]]
        for r in range(M):
            acc = Fraction(0)
            for j in range(N):
                w = sum(Fraction(float(s_out[k, r])) * Fraction(float(s_in[k, j])) * (1 if s[k, r, j] >= 0 else -1)
                        for k in range(K))
                acc += w * xf[j]
            assert abs(y[b, r] - float(acc)) <= 1e-14 * E[b, r] + 1e-300


def test_svid_with_unit_input_scale_is_the_grouped_form():
    # s_in = 1: W = sum_k s_out_k B_k, i.e. the grouped form with
    # alpha_{k,r,g} = s_out_k[r] for every group.
    K, M, N = 3, 11, 384
    s, _, s_out, x = _svid_case(K, M, N, 31)
    s_in = np.ones((K, N), dtype=np.float16)
    y, _ = O.linear_svid(O.pack_signs(s), s_in, s_out, K, M, N, x, "f32")
    alpha = np.repeat(s_out.T[:, None, :], N // 128, axis=1)          # [M][G][K]
    y2, _ = O.linear(O.pack_signs(s), alpha, K, M, N, x, "f32")
    assert np.allclose(y, y2, rtol=1e-12, atol=0)


def test_svid_unit_output_scale_scales_the_input():
    # K = 1, s_out = 1: y = B (s_in (.) x), the grouped form with alpha = 1 on
    # the scaled input (bf16 x times fp16 s_in is exact in fp32).
    K, M, N = 1, 9, 256
    s = wl.random_signs(K, M, N, 41)
    s_in, _ = wl.svid_scales(K, M, N, 42)
    s_out = np.ones((K, M), dtype=np.float16)
    xb = wl.x_normal(1, N, 43, "bf16")
    y, _ = O.linear_svid(O.pack_signs(s), s_in, s_out, K, M, N, xb, "bf16")
    xs = (O.as_f64(xb, "bf16") * s_in[0].astype(np.float64)).astype(np.float32)
    assert np.array_equal(xs.astype(np.float64), O.as_f64(xb, "bf16") * s_in[0].astype(np.float64))
    ones = np.ones((M, N // 128, K), dtype=np.float16)
    y2, _ = O.linear(O.pack_signs(s), ones, K, M, N, xs, "f32")
    assert np.allclose(y, y2, rtol=1e-12, atol=0)


def test_svid_rank1_closed_form():
    # All bits set, K = 1: W = s_out s_in^T, so y = s_out * (s_in . x).
    K, M, N = 1, 6, 256
    s = np.ones((K, M, N), dtype=np.int8)
    s_in, s_out = wl.svid_scales(K, M, N, 51)
    x = wl.x_normal(1, N, 52, "f32")
    y, _ = O.linear_svid(O.pack_signs(s), s_in, s_out, K, M, N, x, "f32")
    dot = float(np.dot(s_in[0].astype(np.float64), x[0].astype(np.float64)))
    assert np.allclose(y[0], s_out[0].astype(np.float64) * dot, rtol=1e-12, atol=0)


def test_svid_flip_invariance_bitwise():
    # Flipping B_k and negating s_out^k leaves every W entry, hence y, unchanged.
    K, M, N = 3, 7, 256
    s, s_in, s_out, x = _svid_case(K, M, N, 61)
    s = np.where(s == 0, 1, s).astype(np.int8)   # a 0 entry means +1 and would not flip
    y0, _ = O.linear_svid(O.pack_signs(s), s_in, s_out, K, M, N, x, "f32")
    for k in range(K):
        s2, so2 = s.copy(), s_out.copy()
        s2[k] = -s2[k]
        so2[k] = -so2[k]
        y1, _ = O.linear_svid(O.pack_signs(s2), s_in, so2, K, M, N, x, "f32")
        assert np.array_equal(y0, y1)


@pytest.mark.parametrize("K", [1, 2, 3, 4])
def test_at_most_2_pow_K_levels(K):
    # Paper-Notes 关键设计: K kernels give 2^K weight levels.
    M, N = 4, 256
    s = wl.random_signs(K, M, N, 30 + K)
    a = wl.alpha_decaying(K, M, N, 40 + K)
    W = O.reconstruct_W(O.pack_signs(s), a, K, M, N)
    for r in range(M):
        for g in range(N // 128):
            vals = set(W[r, 128 * g:128 * g + 128].tolist())
            lev = O.levels(K, a[r, g, :])
            assert vals <= lev
            assert len(vals) <= 2 ** K
            if K <= 3:  # 128 random columns hit all 2^K sign patterns
                assert vals == lev


def test_xnor_popcount_identity():
    # K=1, alpha=1, x in {-1,+1}^N: b.x = 2*popcount(XNOR(b, x)) - N
    # (the XNOR+popcount form named on the Paper-Notes page, 关键设计).
    M, N = 6, 512
    s = wl.random_signs(1, M, N, 50)
    a = np.ones((M, N // 128, 1), dtype=np.float16)
    xs = np.where(np.random.default_rng(51).random(N) < 0.5, -1.0, 1.0).astype(np.float32)
    y, _ = O.linear(O.pack_signs(s), a, 1, M, N, xs[None, :], "f32")
    xbits = sum(1 << j for j in range(N) if xs[j] > 0)
    for r in range(M):
        bbits = sum(1 << j for j in range(N) if s[0, r, j] >= 0)
        xnor = ~(bbits ^ xbits) & ((1 << N) - 1)
        assert y[0, r] == 2 * bin(xnor).count("1") - N


def test_dense_special_case():
    # K=1 with one scale a for every group: y = a * (B x), B x by a naive loop.
    M, N = 4, 256
    s = wl.random_signs(1, M, N, 60)
    aval = np.float16(0.037)
    a = np.full((M, N // 128, 1), aval, dtype=np.float16)
    x = wl.x_normal(1, N, 61, "f32")
    y, E = O.linear(O.pack_signs(s), a, 1, M, N, x, "f32")
    for r in range(M):
        acc = 0.0
        for j in range(N):
            acc += (1.0 if s[0, r, j] >= 0 else -1.0) * float(x[0, j])
        assert abs(y[0, r] - float(aval) * acc) <= 1e-12 * E[0, r]


def test_bf16_activations_exact_widening():
    # bf16 bit pattern 0x3FC0 is 1.5, 0xC020 is -2.5; fp64 widening is exact.
    x = np.array([[0x3FC0, 0xC020]], dtype=np.uint16)
    assert O.as_f64(x, "bf16").tolist() == [[1.5, -2.5]]


# --------------------------------------------------------------------------
# Residual binarisation (O4)
# --------------------------------------------------------------------------

def test_residual_k1_closed_form_least_squares():
    # Paper-Notes 关键设计 (closed-form least squares for alpha given B):
    # for B = sign(W) the optimum is a* = mean|W| over the group; the stored
    # fp16 scale is the fp16 value nearest to it, so it beats both fp16 neighbours.
    M, N = 8, 256
    W = wl.w_normal(M, N, 70)
    s, a, R = O.residual_binarize(W, 1)
    assert np.array_equal(s[0], np.where(W >= 0, 1, -1))
    for r in range(M):
        for g in range(N // 128):
            w = W[r, 128 * g:128 * g + 128].astype(np.float64)
            exact_mean = math.fsum(abs(v) for v in w) / 128.0
            assert a[r, g, 0] == np.float16(exact_mean)
            b = np.where(w >= 0, 1.0, -1.0)

            def f(al):
                return float(np.sum((w - al * b) ** 2))
            h = a[r, g, 0]
            up = np.nextafter(h, np.float16(np.inf))
            dn = np.nextafter(h, np.float16(-np.inf))
            assert f(float(h)) <= f(float(up)) and f(float(h)) <= f(float(dn))


def test_sign_and_scale_jointly_optimal_brute_force():
    # On an 8-entry toy group, over all 2^8 sign vectors with their optimal
    # scale <w,b>/8, the best fit is b = sign(w) with scale mean|w|.
    r = np.random.default_rng(71)
    for _ in range(20):
        w = r.standard_normal(8)
        best = None
        for m in range(256):
            b = np.array([1.0 if (m >> i) & 1 else -1.0 for i in range(8)])
            al = float(w @ b) / 8.0
            err = float(np.sum((w - al * b) ** 2))
            if best is None or err < best[0] - 1e-15:
                best = (err, b, al)
        assert np.array_equal(best[1], np.where(w >= 0, 1.0, -1.0)) or np.array_equal(best[1], -np.where(w >= 0, 1.0, -1.0))
        assert abs(abs(best[2]) - float(np.mean(np.abs(w)))) < 1e-12


def test_residual_norm_identity_and_monotone():
    # Each kernel fits the residual of the previous ones (Dutch technical
    # summary, Successive SVID; Spanish 2B).  Per group, with S = sum|R_{k-1}|:
    #   ||R_k||^2 = ||R_{k-1}||^2 - 2 alpha S + 128 alpha^2   (exact algebra; the
    # fp32 rounding of R_k is the only slack), and ||R_k|| never grows.
    K, M, N = 3, 16, 512
    W = wl.w_normal(M, N, 72)
    s, a, RK = O.residual_binarize(W, K)
    R = W.astype(np.float64)
    prev = None
    for k in range(K):
        for r in range(M):
            for g in range(N // 128):
                seg = R[r, 128 * g:128 * g + 128]
                S = float(np.sum(np.abs(seg)))
                al = float(a[r, g, k])
                b = s[k, r, 128 * g:128 * g + 128].astype(np.float64)
                assert np.array_equal(b, np.where(seg >= 0, 1.0, -1.0))
                assert a[r, g, k] == np.float16(S / 128.0)
                new = seg - al * b
                pred = float(np.sum(seg ** 2)) - 2 * al * S + 128 * al * al
                assert abs(float(np.sum(new ** 2)) - pred) <= 1e-12 * max(1.0, float(np.sum(seg ** 2)))
        R = (R.astype(np.float32) - np.repeat(a[:, :, k].astype(np.float32), 128, axis=1) * s[k].astype(np.float32)).astype(np.float64)
        nrm = float(np.linalg.norm(R))
        assert prev is None or nrm <= prev
        prev = nrm
    assert np.array_equal(R.astype(np.float32), RK)
    # the kernels reconstruct W up to the final residual (fp32 steps only)
    Wk = O.reconstruct_W(O.pack_signs(s), a, K, M, N)
    assert np.max(np.abs(W.astype(np.float64) - Wk - RK.astype(np.float64))) <= 4 * 2.0 ** -24 * 0.2


def test_residual_scale_rounds_once_from_fp64():
    # Reading: the group mean is rounded once, fp64 -> fp16 nearest-even.
    # Group: 126 x 1.0, 1 + 2^-4, 1 + 2^-23  ->  mean = 1 + 2^-11 + 2^-30,
    # just above the fp16 midpoint 1 + 2^-11, so it rounds up to 1 + 2^-10;
    # rounding through fp32 first would land on the midpoint and give 1.0.
    assert np.float16(1 + 2.0 ** -11 + 2.0 ** -40) == np.float16(1 + 2.0 ** -10)
    W = np.ones((1, 128), dtype=np.float32)
    W[0, 5] = 1 + 2.0 ** -4
    W[0, 77] = 1 + 2.0 ** -23
    s, a, R = O.residual_binarize(W, 1)
    assert a[0, 0, 0] == np.float16(1 + 2.0 ** -10)
    assert np.float16(np.float32(1 + 2.0 ** -11 + 2.0 ** -30)) == np.float16(1.0)


def test_residual_zero_group_and_sign_of_zero():
    # sign(0) = +1 (also for -0.0); an all-zero group gets alpha = 0 and keeps R.
    W = np.zeros((2, 256), dtype=np.float32)
    W[0, 128:] = -0.0
    W[1, :128] = np.linspace(-1, 1, 128, dtype=np.float32)
    s, a, R = O.residual_binarize(W, 2)
    assert (s[:, 0, :] == 1).all()
    assert a[0, 0, 0] == 0 and a[0, 1, 0] == 0
    assert np.array_equal(R[0], W[0])


# --------------------------------------------------------------------------
# Tolerance (O8)
# --------------------------------------------------------------------------

def test_tolerance_sanity():
    K, M, N = 2, 32, 256
    s, a, x = _signs_alpha_x(K, M, N, 80)
    y, E = O.linear(O.pack_signs(s), a, K, M, N, x, "f32")
    bound = 1e-3 * E + 1e-6
    assert O.within_tolerance(y + 0.5 * bound, y, E).all()
    assert not O.within_tolerance(y + 2.0 * bound, y, E).any()
    assert O.rel_l2(y, y) == 0.0


# --------------------------------------------------------------------------
# Closed-form scale refit for fixed kernels (Paper-Notes 关键设计,
# 缩放因子的高效优化: least squares once B is fixed)
# --------------------------------------------------------------------------

def test_refit_k1_equals_the_greedy_closed_form():
    # K = 1 with B = sign(w): the least-squares scale is mean|w|, which the
    # greedy residual step computes (same fp64 sum, same single rounding).
    W = wl.w_normal(5, 384, 71)
    signs, alpha, _ = O.residual_binarize(W, 1)
    a2 = O.refit_alpha(W, O.pack_signs(signs), 1, 5, 384)
    assert np.array_equal(a2.view(np.uint16), alpha.view(np.uint16))


@pytest.mark.parametrize("K", [2, 3, 4])
def test_refit_matches_library_least_squares(K):
    # Against numpy's lstsq on each group (a library routine): within fp16
    # rounding of the fp64 solution, and the normal equations hold.
    M, N = 4, 256
    W = wl.w_normal(M, N, 80 + K)
    signs = wl.random_signs(K, M, N, 90 + K)
    a = O.refit_alpha(W, O.pack_signs(signs), K, M, N).astype(np.float64)
    for r in range(M):
        for g in range(N // 128):
            B = signs[:, r, 128 * g:128 * g + 128].astype(np.float64).T        # [128][K]
            B = np.where(B == 0, 1.0, B)
            w = W[r, 128 * g:128 * g + 128].astype(np.float64)
            ref = np.linalg.lstsq(B, w, rcond=None)[0]
            ulp = np.abs(ref) * 2.0 ** -10 + 2.0 ** -24
            assert np.all(np.abs(a[r, g] - ref) <= ulp)
            assert np.all(np.abs(B.T @ (w - B @ ref)) <= 1e-12 * np.abs(B.T @ np.abs(w)).max())


def test_refit_lowers_the_error_of_the_greedy_scales():
    # Refitting all K scales jointly can only lower the squared error of the
    # greedy (one kernel at a time) scales, up to the fp16 rounding.
    K, M, N = 3, 6, 512
    W = wl.w_normal(M, N, 95)
    signs, alpha, _ = O.residual_binarize(W, K)
    a2 = O.refit_alpha(W, O.pack_signs(signs), K, M, N)
    Wg = O.reconstruct_W(O.pack_signs(signs), alpha, K, M, N)
    Wr = O.reconstruct_W(O.pack_signs(signs), a2, K, M, N)
    err_g = ((W.astype(np.float64) - Wg) ** 2).sum()
    err_r = ((W.astype(np.float64) - Wr) ** 2).sum()
    assert err_r <= err_g * (1 + 1e-3)


def test_refit_dependent_kernel_gets_zero():
    # A kernel equal (or opposite) to an earlier one on a group is dropped:
    # scale 0, the earlier kernel takes the one-kernel least-squares scale.
    N = 128
    w = wl.w_normal(1, N, 97)[0]
    b0 = np.where(wl.random_signs(1, 1, N, 98)[0, 0] >= 0, 1, -1).astype(np.int8)
    b = np.stack([b0, -b0, np.where(w >= 0, 1, -1).astype(np.int8)])
    a = O.refit_alpha_group(b, w).astype(np.float64)
    assert a[1] == 0.0
    B = np.stack([b[0], b[2]]).astype(np.float64).T
    ref = np.linalg.lstsq(B, w.astype(np.float64), rcond=None)[0]
    assert np.all(np.abs(a[[0, 2]] - ref) <= np.abs(ref) * 2.0 ** -10 + 2.0 ** -24)


# --------------------------------------------------------------------------
# Successive SVID (Dutch "Methodologie" 2, Italian 2A, Spanish 2B)
# --------------------------------------------------------------------------

def test_svid_constant_magnitude_is_exact():
    # |W| = c everywhere is exactly rank 1: sigma = c sqrt(MN), u, v constant,
    # so one kernel reproduces W and leaves R_1 = 0 (c, sqrt(M), sqrt(N) chosen
    # so the scales are exact in fp16).
    M, N, c = 16, 256, 0.0625     # sigma = c sqrt(MN) = 4: s_out = 0.5, s_in = 0.125
    W = (np.where(wl.random_signs(1, M, N, 5)[0] >= 0, 1.0, -1.0) * c).astype(np.float32)
    signs, s_in, s_out, R = O.svid_binarize(W, 1)
    assert np.all(np.abs(R) <= 1e-9)
    assert np.array_equal(signs[0], np.where(W >= 0, 1, -1))
    prod = s_out[0].astype(np.float64)[:, None] * s_in[0].astype(np.float64)[None, :]
    assert np.all(prod == c)


def test_svid_recovers_a_rank1_scaled_sign_matrix():
    # W = b (.) (p q^T) with positive p, q: sign(W) = b and |W| = p q^T is rank 1,
    # so the first kernel recovers W up to the fp16 rounding of the scales.
    M, N = 24, 384
    b = np.where(wl.random_signs(1, M, N, 6)[0] >= 0, 1.0, -1.0)
    g = np.random.default_rng(7)
    p, q = g.uniform(0.5, 2.0, M), g.uniform(0.01, 0.05, N)
    W = (b * np.outer(p, q)).astype(np.float32)
    signs, s_in, s_out, R = O.svid_binarize(W, 1)
    assert np.array_equal(signs[0].astype(np.float64), b)
    assert np.max(np.abs(R)) <= 2 * 2.0 ** -11 * np.max(np.abs(W))


def test_svid_beats_the_plain_rank1_of_w():
    # The pages' claim: sign(W) (.) rank1(|W|) approximates W better than the
    # rank-1 approximation of W itself.
    W = wl.w_normal(64, 512, 8).astype(np.float64)
    _, _, _, R = O.svid_binarize(W.astype(np.float32), 1)
    U, S, Vt = np.linalg.svd(W, full_matrices=False)
    plain = W - S[0] * np.outer(U[:, 0], Vt[0])
    assert np.linalg.norm(R.astype(np.float64)) < np.linalg.norm(plain)


def test_svid_residual_shrinks_and_signs_of_zero():
    W = wl.w_normal(32, 256, 9)
    W[0, :5] = 0.0
    W[1, 3] = -0.0
    signs, _, _, R = O.svid_binarize(W, 3)
    assert np.all(signs[0][0, :5] == 1) and signs[0][1, 3] == 1
    norms = [np.linalg.norm(W.astype(np.float64))]
    R = W.copy()
    for k in range(3):
        so, si = O.svid_scales_of(np.abs(R.astype(np.float64)))
        _, R = O.svid_step(R, so, si)
        norms.append(np.linalg.norm(R.astype(np.float64)))
    assert all(a > b for a, b in zip(norms, norms[1:]))


def test_round_bf16_pins():
    """The bf16 rounding used for the GEMM's weight tile, pinned without
    restating it: representable values are fixed points, midpoints go to the
    even neighbour, fp64 inputs just past a midpoint round up (a detour
    through fp32 would round them down), and on fp32 inputs it agrees with
    torch's float32 -> bfloat16 conversion."""
    import torch
    # representable: 8 significant bits
    rep = np.array([1.0, -1.0, 1.0 + 2.0 ** -7, 3.0, 0.0, 2.0 ** -126, -(2.0 ** 100), 1.9921875])
    assert np.array_equal(O.round_bf16(rep), rep)
    # ties to even: spacing at 1.0 is 2^-7
    assert O.round_bf16(1.0 + 2.0 ** -8) == 1.0
    assert O.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert O.round_bf16(-(1.0 + 2.0 ** -8)) == -1.0
    # single rounding from fp64: just above the midpoint rounds up
    assert O.round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 1.0 + 2.0 ** -7
    assert np.float32(1.0 + 2.0 ** -8 + 2.0 ** -40) == np.float32(1.0 + 2.0 ** -8)
    # agreement with a library conversion on fp32 values (normal and subnormal)
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        rng.standard_normal(2000) * 2.0 ** -130]).astype(np.float32)
    lib = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_bf16(v.astype(np.float64)), lib)
