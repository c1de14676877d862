"""CPU oracle for the multi-Boolean-kernel (MBOK) linear layer.

TEST INFRASTRUCTURE.  Only the tests, the smoke check of the package entry
point and the CPU-baseline leg of the benchmark may import or run this module.
The product (the C ABI and its Python binding) never calls it, and it shares
no code with the CUDA path: it reads only the layout definition restated
below and the seeded inputs.

What it computes, and where the method defines it
-------------------------------------------------
Source pages: "Highly Efficient and Effective LLMs with Multi-Boolean
Architectures" (ICLR 2026; arXiv 2505.22811) as summarised by the Paper-Notes
page (section "方法详解 / 关键设计") and by the gist.science technical summaries
(Italian 2A-2D, Dutch "Methodologie", Spanish 2A-2D).

* Representation (Paper-Notes, 关键设计, "多核布尔参数表示"): a weight matrix
  is approximated by a weighted sum of K Boolean matrices,
  W ~= sum_k alpha_k * B_k with B_k in {-1,+1}^{M x N}.
* Grouping (Paper-Notes, 关键设计, "分组量化策略"; ablation table: group
  size 128 is the usual choice): every 128-column group of a row has its own
  scale, so alpha_{k,r,g} multiplies B_k[r, 128g:128g+128].
* The linear op (Paper-Notes, 关键设计: "Wx decomposes into K Boolean
  matrix-vector products"): y = W x with that W.  The oracle reconstructs W in
  fp64 (exact: each entry is a sum of at most four fp16 values times +-1) and
  multiplies with a float64 BLAS product.
* Scale for a fixed sign matrix (Paper-Notes, 关键设计, "缩放因子的高效优化":
  closed-form least squares): for B = sign(R) the least-squares scale of a
  group is mean|R| over the group.
* Kernel k fits what kernels 1..k-1 left (Dutch technical summary,
  "Successive SVID"; Spanish 2B "Extracción Sucesiva": each later kernel
  approximates the residual of the previous approximation; Paper-Notes,
  训练策略: greedy initialisation).  Here: R_0 = W, B_k = sign(R_{k-1}),
  alpha_k = mean|R_{k-1}| per (row, group), R_k = R_{k-1} - alpha_k B_k.

Readings where the pages are silent (each one is listed in the design notes):
  sign(0) = +1 (and -0.0 >= 0 so also +1); packer input 0 also maps to +1;
  a stored bit 1 means +1;
  the greedy residual keeps R in fp32, sums |R| over a group in fp64 in column
  order j = 0..127, divides by 128 (exact), rounds once from fp64 to fp16
  (nearest, ties to even), and updates R <- R - alpha_hat * b with the fp16
  value, as one fp32 subtraction;
  N must be a multiple of 128 (no ragged group).

Storage format, version 1 (the pages give none; this is the library's format):
  rows are cut into octets of 8 (the last octet is padded; pad rows are
  ignored).  The packed kernels are bytes ordered
      [octet o][kernel k][unit q][row i in octet][2 bytes]
  where unit q covers columns 16q..16q+15: the little-endian 16-bit halfword
  for row 8o+i holds column 16q+b in bit b.  A set bit means +1.
  Scales alpha are fp16; logically [M][N/128][K], stored blocked as
      [octet o][group g][kernel k][row i in octet].

Rank-1 scales (SVID form).  The technical summaries also write each kernel
with its own rank-1 scale, W ~= sum_k B_k (.) (s_out^k s_in^k^T) (Italian 2A/2B,
Dutch "Methodologie" 2, Spanish 2B): s_in^k has one value per column and
s_out^k one per row, so y = sum_k s_out^k (.) (B_k (s_in^k (.) x)).  The
oracle for that form (linear_svid) reconstructs W_rj = sum_k b_krj s_out_kr
s_in_kj in fp64 (each product of two fp16 values is exact; the sum over k is
rounded in fp64) and multiplies as above.  Scales are fp16, s_in [K][N] and
s_out [K][M].

Parity pins: see tests/test_oracle_pins.py (brute force in exact rational
arithmetic, flip invariance, level count, least-squares closed form, residual
norm identity, the XNOR/popcount identity, a hand-worked layout example, the
dense special case and a rounding case for the fp64->fp16 step).
"""
from __future__ import annotations

import math

import numpy as np

GROUP = 128        # columns per scale group
OCTET = 8          # rows per storage block
UNIT = 16          # columns per 16-bit unit


# --------------------------------------------------------------------------
# Layout sizes and addressing (restated from the format definition above)
# --------------------------------------------------------------------------

def n_groups(N: int) -> int:
    if N % GROUP or N <= 0:
        raise ValueError("N must be a positive multiple of 128")
    return N // GROUP


def n_octets(M: int) -> int:
    return (M + OCTET - 1) // OCTET


def packed_bytes(K: int, M: int, N: int) -> int:
    n_groups(N)
    return n_octets(M) * K * N


def alpha_elems(K: int, M: int, N: int) -> int:
    return n_octets(M) * OCTET * n_groups(N) * K


def byte_and_bit(K: int, M: int, N: int, k: int, r: int, j: int) -> tuple[int, int]:
    """Byte offset and bit position that hold kernel k, row r, column j."""
    o, i = divmod(r, OCTET)
    q, b = divmod(j, UNIT)
    byte = ((o * K + k) * (N // UNIT) + q) * UNIT + 2 * i + b // 8
    return byte, b % 8


def alpha_index(K: int, M: int, N: int, k: int, r: int, g: int) -> int:
    o, i = divmod(r, OCTET)
    return ((o * n_groups(N) + g) * K + k) * OCTET + i


# --------------------------------------------------------------------------
# Packing and unpacking
# --------------------------------------------------------------------------

def pack_signs(signs: np.ndarray) -> np.ndarray:
    """int8 signs [K][M][N] -> packed bytes viewed as uint32 words.
    An entry >= 0 is stored as a set bit (+1)."""
    K, M, N = signs.shape
    n_groups(N)
    O = n_octets(M)
    bits = np.zeros((K, O * OCTET, N), dtype=np.uint16)
    bits[:, :M, :] = signs >= 0
    b = bits.reshape(K, O, OCTET, N // UNIT, UNIT)
    half = np.zeros((K, O, OCTET, N // UNIT), dtype=np.uint16)
    for t in range(UNIT):
        half |= b[..., t] << np.uint16(t)
    # storage order [o][k][q][i], little-endian halfwords
    h = np.ascontiguousarray(half.transpose(1, 0, 3, 2)).astype("<u2").ravel()
    return h.view("<u4").astype(np.uint32)


def unpack_rows(packed: np.ndarray, K: int, M: int, N: int, rows) -> np.ndarray:
    """Packed words -> b in {-1,+1}, int8 [K][len(rows)][N], for the listed rows."""
    O = n_octets(M)
    rows = np.asarray(rows, dtype=np.int64)
    h = np.ascontiguousarray(packed, dtype="<u4").view("<u2").reshape(O, K, N // UNIT, OCTET)
    sel = h[rows // OCTET, :, :, rows % OCTET]                       # [R][K][N/16]
    shifts = np.arange(UNIT, dtype=np.uint16)
    bits = (sel[..., None] >> shifts) & np.uint16(1)                  # [R][K][N/16][16]
    bits = bits.reshape(len(rows), K, N).transpose(1, 0, 2)           # [K][R][N]
    return np.where(bits == 1, 1, -1).astype(np.int8)


def unpack_bits(packed: np.ndarray, K: int, M: int, N: int) -> np.ndarray:
    return unpack_rows(packed, K, M, N, np.arange(M))


def block_alpha(alpha_mgk: np.ndarray, K: int, M: int, N: int) -> np.ndarray:
    """fp16 [M][G][K] -> the stored order [o][g][k][i] (pad rows 0)."""
    G, O = n_groups(N), n_octets(M)
    a = np.zeros((O * OCTET, G, K), dtype=np.float16)
    a[:M] = np.asarray(alpha_mgk, dtype=np.float16).reshape(M, G, K)
    return np.ascontiguousarray(a.reshape(O, OCTET, G, K).transpose(0, 2, 3, 1)).ravel()


def unblock_alpha(alpha_blk: np.ndarray, K: int, M: int, N: int) -> np.ndarray:
    """The stored order -> fp16 [M][G][K]."""
    G, O = n_groups(N), n_octets(M)
    a = np.asarray(alpha_blk, dtype=np.float16).reshape(O, G, K, OCTET).transpose(0, 3, 1, 2)
    return np.ascontiguousarray(a.reshape(O * OCTET, G, K)[:M])


# --------------------------------------------------------------------------
# The weight and the linear op
# --------------------------------------------------------------------------

def reconstruct_rows(packed, alpha, K: int, M: int, N: int, rows) -> np.ndarray:
    """fp64 W[rows, :] with W_rj = sum_k alpha_{k,r,floor(j/128)} * b_{k,r,j}."""
    G = n_groups(N)
    rows = np.asarray(rows, dtype=np.int64)
    b = unpack_rows(packed, K, M, N, rows).astype(np.float64)        # [K][R][N]
    a = np.asarray(alpha, dtype=np.float16).reshape(M, G, K)[rows].astype(np.float64)  # [R][G][K]
    a_cols = np.repeat(a, GROUP, axis=1)                             # [R][N][K]
    W = np.zeros((len(rows), N), dtype=np.float64)
    for k in range(K):
        W += a_cols[:, :, k] * b[k]
    return W


def reconstruct_W(packed, alpha, K: int, M: int, N: int) -> np.ndarray:
    return reconstruct_rows(packed, alpha, K, M, N, np.arange(M))


def as_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Activations to fp64 (exact for fp32 and bf16)."""
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        return (np.asarray(x, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def linear(packed, alpha, K: int, M: int, N: int, x, x_dtype: str, rows=None):
    """y[b][r] = sum_j W_rj x[b][j] and E[b][r] = sum_j |W_rj x[b][j]| in fp64.

    x is [batch][N] (fp32, or bf16 bit patterns).  rows selects output rows
    (default all).  E feeds the per-element tolerance |y - y_ref| <= 1e-3 E + 1e-6.
    """
    rows = np.arange(M) if rows is None else np.asarray(rows, dtype=np.int64)
    W = reconstruct_rows(packed, alpha, K, M, N, rows)
    xf = as_f64(x, x_dtype).reshape(-1, N)
    y = xf @ W.T
    E = np.abs(xf) @ np.abs(W).T
    return y, E


# --------------------------------------------------------------------------
# Rank-1 (SVID) scales
# --------------------------------------------------------------------------

def reconstruct_svid_rows(packed, s_in, s_out, K: int, M: int, N: int, rows) -> np.ndarray:
    """fp64 W[rows, :] with W_rj = sum_k b_{k,r,j} * s_out[k][r] * s_in[k][j]."""
    rows = np.asarray(rows, dtype=np.int64)
    b = unpack_rows(packed, K, M, N, rows).astype(np.float64)                  # [K][R][N]
    si = np.asarray(s_in, dtype=np.float16).reshape(K, N).astype(np.float64)    # [K][N]
    so = np.asarray(s_out, dtype=np.float16).reshape(K, M).astype(np.float64)   # [K][M]
    W = np.zeros((len(rows), N), dtype=np.float64)
    for k in range(K):
        W += (so[k, rows][:, None] * si[k][None, :]) * b[k]
    return W


def linear_svid(packed, s_in, s_out, K: int, M: int, N: int, x, x_dtype: str, rows=None):
    """y[b][r] = sum_j W_rj x[b][j] and E[b][r] = sum_j |W_rj x[b][j]| in fp64 for
    the rank-1-scaled kernels W = sum_k B_k (.) (s_out^k s_in^k^T)."""
    rows = np.arange(M) if rows is None else np.asarray(rows, dtype=np.int64)
    W = reconstruct_svid_rows(packed, s_in, s_out, K, M, N, rows)
    xf = as_f64(x, x_dtype).reshape(-1, N)
    return xf @ W.T, np.abs(xf) @ np.abs(W).T


# --------------------------------------------------------------------------
# Greedy residual binarisation
# --------------------------------------------------------------------------

def residual_binarize(W: np.ndarray, K: int):
    """fp32 W [M][N] -> (signs int8 [K][M][N], alpha fp16 [M][G][K], R_K fp32 [M][N]).

    For k = 1..K, per (row r, group g):
      b     = sign(R_{k-1}), sign(0) = +1
      alpha = RN_fp16( (sum_{j=0..127} |R_{k-1}|, fp64, in column order) / 128 )
      R_k   = R_{k-1} - alpha * b     (fp32, alpha the fp16 value, one rounding)
    """
    W = np.asarray(W, dtype=np.float32)
    M, N = W.shape
    G = n_groups(N)
    R = W.copy()
    signs = np.empty((K, M, N), dtype=np.int8)
    alpha = np.empty((M, G, K), dtype=np.float16)
    for k in range(K):
        b = np.where(R >= np.float32(0), np.int8(1), np.int8(-1))
        A = np.abs(R).astype(np.float64).reshape(M, G, GROUP)
        acc = np.zeros((M, G), dtype=np.float64)
        for j in range(GROUP):          # the prescribed summation order
            acc = acc + A[:, :, j]
        a16 = (acc / 128.0).astype(np.float16)
        a32 = np.repeat(a16.astype(np.float32), GROUP, axis=1)      # [M][N]
        R = (R - a32 * b.astype(np.float32)).astype(np.float32)
        signs[k] = b
        alpha[:, :, k] = a16
    return signs, alpha, R


# --------------------------------------------------------------------------
# Tolerance
# --------------------------------------------------------------------------

# --------------------------------------------------------------------------
# Successive SVID (rank-1 scales extracted kernel by kernel)
# --------------------------------------------------------------------------
# Dutch technical summary, "Methodologie" 2 (Successive SVID), Italian 2A and
# Spanish 2B: take a rank-1 approximation of the absolute values (via SVD) to
# get the scale vectors, the signs as the Boolean matrix, and give the
# residual to the next kernel:
#     B_k = sign(R_{k-1}),  |R_{k-1}| ~ sigma u v^T,
#     s_out^k = sqrt(sigma) u,  s_in^k = sqrt(sigma) v   (u, v >= 0),
#     R_k = R_{k-1} - B_k (.) (s_out^k s_in^k^T).
# Readings (listed in the design notes): sign(0) = +1; the top singular
# triple of the nonnegative |R| is taken with u, v >= 0 (its Perron vectors);
# the product is split evenly (sqrt(sigma) on each side); s_out and s_in are
# rounded once to fp16 (nearest even) from fp64, and the residual update uses
# those fp16 values: R <- R - b * (s_out_r * s_in_j) as one fp32 product
# (exact: two 11-bit significands) and one fp32 subtraction.

def svid_scales_of(A: np.ndarray):
    """Rank-1 scales of a nonnegative matrix: fp16 (s_out [M], s_in [N])."""
    U, S, Vt = np.linalg.svd(np.asarray(A, dtype=np.float64), full_matrices=False)
    u, v, sigma = U[:, 0], Vt[0], S[0]
    if u.sum() < 0:
        u, v = -u, -v
    u, v = np.abs(u), np.abs(v)      # Perron vectors of a nonnegative matrix
    root = math.sqrt(sigma)
    return (root * u).astype(np.float16), (root * v).astype(np.float16)


def svid_step(R: np.ndarray, s_out: np.ndarray, s_in: np.ndarray):
    """One update with given fp16 scales: (signs int8 [M][N], R_next fp32)."""
    R = np.asarray(R, dtype=np.float32)
    b = np.where(R >= 0, 1, -1).astype(np.int8)
    prod = np.asarray(s_out, dtype=np.float16).astype(np.float32)[:, None] * \
        np.asarray(s_in, dtype=np.float16).astype(np.float32)[None, :]
    R_next = (R - np.where(b > 0, prod, -prod)).astype(np.float32)
    return b, R_next


def svid_binarize(W: np.ndarray, K: int):
    """fp32 W [M][N] -> (signs int8 [K][M][N], s_in fp16 [K][N], s_out fp16 [K][M], R_K fp32)."""
    R = np.asarray(W, dtype=np.float32).copy()
    M, N = R.shape
    signs = np.zeros((K, M, N), dtype=np.int8)
    s_in = np.zeros((K, N), dtype=np.float16)
    s_out = np.zeros((K, M), dtype=np.float16)
    for k in range(K):
        s_out[k], s_in[k] = svid_scales_of(np.abs(R.astype(np.float64)))
        signs[k], R = svid_step(R, s_out[k], s_in[k])
    return signs, s_in, s_out, R


# --------------------------------------------------------------------------
# Closed-form scale refit for fixed kernels
# --------------------------------------------------------------------------
# Paper-Notes page, 关键设计 "缩放因子的高效优化": once the Boolean matrices
# are fixed, the scales have a closed-form least-squares solution, and the
# method alternates (fixed alpha -> update B, fixed B -> update alpha).  Per
# (row r, group g) the scales minimise ||w - sum_k alpha_k b_k||^2 over the
# group's 128 columns, i.e. solve G alpha = c with the Gram matrix
# G_kl = sum_j b_kj b_lj (integers) and c_k = sum_j b_kj w_j.
# Readings (listed in the design notes): c_k is summed in fp64 in column order;
# the solution is adj(G) c / det(G) with the adjugate and determinant exact
# integers, the numerator summed in fp64 over the kernels in order and
# divided once, then rounded once fp64 -> fp16 (nearest even).  Kernels whose
# signs on the group are linearly dependent on earlier ones (a zero
# determinant, detected exactly) are left out in kernel order and get 0.

def _int_det(a) -> int:
    n = len(a)
    if n == 0:
        return 1
    if n == 1:
        return a[0][0]
    total = 0
    for col in range(n):
        minor = [row[:col] + row[col + 1:] for row in a[1:]]
        total += (-1) ** col * a[0][col] * _int_det(minor)
    return total


def _int_adjugate(a):
    n = len(a)
    if n == 1:
        return [[1]]
    adj = [[0] * n for _ in range(n)]
    for i in range(n):
        for j in range(n):
            minor = [row[:j] + row[j + 1:] for k, row in enumerate(a) if k != i]
            adj[j][i] = (-1) ** (i + j) * _int_det(minor)     # transpose of the cofactors
    return adj


def refit_alpha_group(b: np.ndarray, w: np.ndarray) -> np.ndarray:
    """b: int signs [K][128] (+-1), w: fp32 [128] -> fp16 [K] least-squares scales."""
    K = b.shape[0]
    bi = [[int(v) for v in b[k]] for k in range(K)]
    G = [[sum(x * y for x, y in zip(bi[k], bi[l])) for l in range(K)] for k in range(K)]
    c = []
    for k in range(K):
        acc = 0.0
        for j in range(len(w)):
            acc = acc + (float(w[j]) if bi[k][j] > 0 else -float(w[j]))
        c.append(acc)
    active = []
    for k in range(K):
        trial = active + [k]
        if _int_det([[G[i][j] for j in trial] for i in trial]) != 0:
            active = trial
    out = np.zeros(K, dtype=np.float16)
    if not active:
        return out
    Ga = [[G[i][j] for j in active] for i in active]
    det = _int_det(Ga)
    adj = _int_adjugate(Ga)
    for a_idx, k in enumerate(active):
        num = 0.0
        for i_idx in range(len(active)):
            num = num + float(adj[a_idx][i_idx]) * c[active[i_idx]]
        out[k] = np.float16(num / float(det))
    return out


def refit_alpha(W: np.ndarray, packed, K: int, M: int, N: int, rows=None) -> np.ndarray:
    """Least-squares scales for fixed kernels: fp16 [len(rows)][G][K]."""
    W = np.asarray(W, dtype=np.float32)
    rows = np.arange(M) if rows is None else np.asarray(rows, dtype=np.int64)
    b = unpack_rows(packed, K, M, N, rows)
    G = n_groups(N)
    out = np.zeros((len(rows), G, K), dtype=np.float16)
    for ri, r in enumerate(rows):
        for g in range(G):
            sl = slice(GROUP * g, GROUP * g + GROUP)
            out[ri, g] = refit_alpha_group(b[:, ri, sl], W[r, sl])
    return out


def within_tolerance(y, y_ref, E, rel: float = 1e-3, abs_: float = 1e-6) -> np.ndarray:
    """Per-element bound |y - y_ref| <= rel * E + abs_ (boolean mask)."""
    y = np.asarray(y, dtype=np.float64)
    return np.abs(y - y_ref) <= rel * E + abs_


def rel_l2(y, y_ref) -> float:
    y = np.asarray(y, dtype=np.float64)
    den = float(np.linalg.norm(y_ref))
    return float(np.linalg.norm(y - y_ref)) / (den if den > 0 else 1.0)


def round_bf16(v) -> np.ndarray:
    """Round fp64 values once to bfloat16 (8 significant bits, the fp32
    exponent range), nearest with ties to even; returned as fp64.

    The prefill GEMM multiplies a bfloat16 weight tile: every weight W_rj,
    exact in fp64 (reconstruct_rows), rounded once.  Written from the format's
    definition: x = m * 2^e with 1/2 <= |m| < 1 (frexp), m scaled to 8 bits
    and rounded half-to-even (numpy rint), the quantum fixed at 2^-133 below
    the smallest normal 2^-126.  Finite inputs within the bf16 range only."""
    x = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(x)
    normal = np.rint(m * 256.0) * np.exp2(e.astype(np.float64) - 8.0)
    sub = np.rint(x * 2.0 ** 133) * 2.0 ** -133
    return np.where(np.abs(x) < 2.0 ** -126, sub, normal)


def levels(K: int, alphas) -> set:
    """The set {sum_k s_k alpha_k : s in {-1,+1}^K} (at most 2^K weight levels)."""
    out = set()
    for m in range(1 << K):
        out.add(math.fsum((1.0 if (m >> k) & 1 else -1.0) * float(alphas[k]) for k in range(K)))
    return out
