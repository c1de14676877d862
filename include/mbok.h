/*
 * mbok.h - C ABI of the multi-Boolean-kernel (MBOK) linear layer on B200.
 *
 * The method ("Highly Efficient and Effective LLMs with Multi-Boolean
 * Architectures", ICLR 2026) stores a weight matrix as K Boolean kernels with
 * group-wise scales,
 *
 *     W[r][j] = sum_{k<K} alpha[k][r][g(j)] * B_k[r][j],   B_k in {-1,+1},
 *     g(j) = j / 128,
 *
 * (Paper-Notes page, section 方法详解 / 关键设计: multi-kernel Boolean
 * parameters, group-wise scaling with groups of 128) and evaluates y = W x as
 * K Boolean matrix-vector products (same section).
 *
 * Conventions for every call
 *  - All data pointers are DEVICE pointers owned by the caller, in memory of
 *    the current device (cudaSetDevice): kernels launch there and the library
 *    does not check where a pointer lives.  The library
 *    allocates nothing and never synchronises (except
 *    mbok_read_device_errors); between calls it keeps only cached kernel
 *    attributes and two process-wide switches (mbok_gemv_set_kernel,
 *    mbok_gemv_set_static_weights).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued on it; results are ready when the stream reaches them.
 *  - Return value: an mbok_status.  Argument errors are detected on the host
 *    and returned before anything is launched; a launch error returns
 *    MBOK_ERR_CUDA.  No call aborts, traps or throws.
 *  - Group size: `group` arguments must equal MBOK_GROUP (128); N must be a
 *    positive multiple of 128.  1 <= K <= MBOK_MAX_K.  M >= 1.
 *
 * Storage format MBOK_LAYOUT_VERSION 1 (the pages define none):
 *  - Rows are cut into octets of 8 (O = ceil(M/8); rows of the last octet at
 *    or beyond M are padding and are ignored by every reader).
 *  - packed: O*K*N bits as bytes ordered [octet o][kernel k][unit q][row i][2],
 *    where unit q holds columns 16q..16q+15 of rows 8o..8o+7 in 16 bytes:
 *    the 16-bit little-endian halfword i of the unit is row 8o+i, and its bit b
 *    is column 16q+b.  A set bit means +1, a clear bit means -1.
 *  - alpha: fp16 (IEEE binary16 bit patterns) ordered [octet o][group g]
 *    [kernel k][row i], i.e. element ((o*G + g)*K + k)*8 + i is the scale of
 *    kernel k, row 8o+i, group g (G = N/128).  Pad rows are ignored.
 *  - packed must be 16-byte aligned, alpha 16-byte aligned.
 */
#ifndef MBOK_H
#define MBOK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MBOK_OK = 0,
  MBOK_ERR_INVALID_ARG = 1,   /* NULL pointer, K / batch / dtype out of range */
  MBOK_ERR_SHAPE = 2,         /* M < 1, N not a positive multiple of 128, T < 1 */
  MBOK_ERR_ALIGN = 3,         /* a pointer lacks its required alignment */
  MBOK_ERR_UNSUPPORTED = 4,   /* group != 128 */
  MBOK_ERR_CUDA = 5,          /* a kernel launch failed */
  MBOK_ERR_WORKSPACE = 6,     /* workspace NULL or smaller than required */
  MBOK_ERR_SCRATCH_LIMIT = 7  /* problem needs more than MBOK_NOALLOC_SCRATCH_BYTES */
} mbok_status;

typedef enum { MBOK_F32 = 0, MBOK_BF16 = 1 } mbok_dtype;

#define MBOK_GROUP 128
#define MBOK_LAYOUT_VERSION 1
#define MBOK_MAX_K 4
#define MBOK_MAX_BATCH 16
/* Values of mbok_gemv_set_kernel. */
#define MBOK_GEMV_AUTO 0
#define MBOK_GEMV_LOOKUP 1
#define MBOK_GEMV_TENSOR 2
#define MBOK_GEMV_LOOKUP_SLABS 3
#define MBOK_GEMV_LOOKUP_ROWS 4
/* Size of the scratch array built into the library for mbok_gemv_noalloc. */
#define MBOK_NOALLOC_SCRATCH_BYTES (4u << 20)

/* Human-readable name of a status code (static string, never NULL). */
const char* mbok_status_string(int status);

/* The storage-format version this library reads and writes (1). */
int mbok_layout_version(void);

/* Bytes of the packed kernels for (K, M, N): ceil(M/8)*K*N.  0 on bad shape. */
size_t mbok_packed_bytes(int K, int M, int N);

/* fp16 elements of the blocked scales: ceil(M/8)*8*(N/128)*K.  0 on bad shape. */
size_t mbok_alpha_elems(int K, int M, int N);

/* Bytes of device workspace mbok_gemv needs for (K, M, N, batch), whichever
 * kernel the call takes.  The caller allocates it (256-byte aligned; no
 * initialisation needed) and may reuse it for any later call with the same or
 * smaller requirement.  Only the 8-bit slab lookup kernel uses it: it holds
 * the per-CTA partial sums of one call, which a second, small launch of the
 * same call adds up in a fixed order.  Calls that share one workspace must
 * not run concurrently (calls in one stream are fine). */
size_t mbok_gemv_workspace_bytes(int K, int M, int N, int batch);

/* Pack K sign matrices into layout 1.
 *   signs  : int8 [K][M][N], row-major; an entry >= 0 means +1 (so 0 -> +1),
 *            an entry < 0 means -1.  (B_k in {-1,+1}: Paper-Notes 关键设计.)
 *   packed : mbok_packed_bytes(K,M,N) bytes, 16-byte aligned; every byte is
 *            written (pad rows as 0 bits). */
int mbok_pack_bits(const int8_t* signs, int K, int M, int N, uint32_t* packed, void* stream);

/* Reorder scales from the logical fp16 [M][N/128][K] (kernel fastest) into
 * the blocked order of layout 1.  alpha_out holds mbok_alpha_elems(K,M,N)
 * elements; pad rows are written as 0.  Both pointers 16-byte aligned. */
int mbok_pack_alpha(const uint16_t* alpha_mgk, int K, int M, int N, uint16_t* alpha_out,
                    void* stream);

/* Greedy residual binarisation, producing K kernels from a dense weight.
 * Each later kernel fits the residual the earlier ones leave (Dutch and
 * Spanish technical summaries, "Successive SVID" / "Extracción Sucesiva");
 * for a fixed sign matrix the least-squares group scale is mean|R|
 * (Paper-Notes 关键设计, closed-form scale).  Per row r and group g,
 * for k = 0..K-1:
 *     b      = sign(R) with sign(0) = +1 (also for -0.0),
 *     alpha  = fp16( (sum over the group's 128 columns of |R|, accumulated in
 *              fp64 in column order) / 128 ), rounded once, nearest-even,
 *     R      = R - alpha*b   (fp32, with the fp16 alpha, one rounding),
 * starting from R = W.  Results are bit-exact and deterministic.
 *   W        : fp32 [M][N] row-major (16-byte aligned).
 *   packed   : layout 1, mbok_packed_bytes(K,M,N) bytes.
 *   alpha    : layout 1, mbok_alpha_elems(K,M,N) fp16 elements.
 *   residual : fp32 [M][N] receiving R after the K-th kernel, or NULL.
 * NaN in W yields unspecified bits and NaN scales for its group. */
int mbok_residual_binarize(const float* W, int M, int N, int K, int group, uint32_t* packed,
                           uint16_t* alpha, float* residual, void* stream);

/* Bytes of device workspace mbok_svid_binarize needs for an M x N matrix. */
size_t mbok_svid_workspace_bytes(int M, int N);

/* Successive SVID: K kernels with rank-1 scales extracted one after another
 * (Dutch technical summary "Methodologie" 2, Italian 2A, Spanish 2B: the
 * signs of the residual, a rank-1 approximation of its absolute values as
 * the scale vectors, the residual passed on).  Starting from R = W, for
 * k = 0..K-1:
 *     B_k     = sign(R), sign(0) = +1,
 *     |R| ~ sigma u v^T with u, v >= 0: the top singular pair by `iters`
 *              power iterations from the uniform vector (u = |R| v,
 *              v = |R|^T u / ||.||), then u = |R| v, sigma = ||u||,
 *     s_out[k] = fp16(u / sqrt(sigma)),  s_in[k] = fp16(sqrt(sigma) v),
 *     R       = R - b * (s_out[k][r] * s_in[k][j])  (fp32, the fp16 scales).
 * All sums run in a fixed order, so results are deterministic.  Evaluate the
 * result with mbok_gemv_svid.
 *   W        : fp32 [M][N] (16-byte aligned), not modified.
 *   iters    : power iterations per kernel, 1..1000 (6 is ample for
 *              weight-like matrices, whose |R| has a dominant singular value).
 *   packed   : out, layout 1.   s_in: out, fp16 [K][N].   s_out: out, fp16 [K][M].
 *   residual : out, fp32 [M][N] = R after the K-th kernel (also the working
 *              buffer; 16-byte aligned).
 *   workspace: mbok_svid_workspace_bytes(M, N) bytes, 16-byte aligned. */
int mbok_svid_binarize(const float* W, int M, int N, int K, int iters, uint32_t* packed, uint16_t* s_in,
                       uint16_t* s_out, float* residual, void* workspace, size_t workspace_bytes, void* stream);

/* Least-squares scales for fixed kernels: the scale step of the alternating
 * optimisation (Paper-Notes 关键设计: once the B_k are fixed the scales have a
 * closed-form least-squares solution).  Per row r and group g the K scales
 * minimise sum over the group's 128 columns of (W[r][j] - sum_k alpha_k b_kj)^2:
 *     G alpha = c,  G_kl = sum_j b_kj b_lj (exact integers),
 *     c_k = sum_j b_kj W[r][j] (fp64, column order),
 *     alpha = adj(G) c / det(G) with exact integer adjugate and determinant,
 *     the numerator summed in fp64 in kernel order, one division, one
 *     rounding fp64 -> fp16 (nearest even).
 * A kernel whose signs on the group depend linearly on earlier kernels (exact
 * zero determinant) is left out, in kernel order, with scale 0.  Bit-exact and
 * deterministic.
 *   W      : fp32 [M][N] row-major (16-byte aligned).
 *   packed : the K kernels, layout 1.
 *   alpha  : out, layout 1, mbok_alpha_elems(K,M,N) fp16 elements (pad rows 0). */
int mbok_refit_alpha(const float* W, const uint32_t* packed, int K, int M, int N, int group, uint16_t* alpha,
                     void* stream);

/* Fusing projections that share an input (q/k/v, gate/up): matrices with the
 * same K and N whose M are multiples of 8 concatenate along M by
 * concatenating their packed bytes and their blocked scales (both are
 * octet-major), and one mbok_gemv over the concatenation gives, row for row,
 * exactly the results of the separate calls (tested).  Matrices with
 * different K (each layer's matrices may get their own number of kernels:
 * Italian technical summary, 2D, kernel allocation) or any M fuse with
 * mbok_gemv_multi below. */

/* y[b][r] = sum_j W[r][j] * x[b][j] for b < batch (decode / small batch).
 * Evaluated as sum over groups and kernels of alpha[k][r][g] times the
 * +-1 dot product of B_k's group slice with x (Paper-Notes 关键设计: Wx as
 * K Boolean matrix-vector products), accumulated in fp32.
 *   packed, alpha : layout 1.
 *   x       : [batch][N], fp32 (x_dtype MBOK_F32) or bf16 bit patterns
 *             (MBOK_BF16); 16-byte aligned.
 *   batch   : 1..MBOK_MAX_BATCH.
 *   y       : fp32 [batch][M] (4-byte aligned), fully overwritten.
 *   workspace, workspace_bytes : see mbok_gemv_workspace_bytes.
 * Accuracy: |y - y_exact| <= 1e-3 * sum_j |W[r][j] x[b][j]| + 1e-6 per
 * element and relative L2 error <= 1e-5 (fp32 accumulation).  For a given
 * (shape, batch, kernel choice) the result is deterministic run to run.
 * Kernels (see mbok_gemv_set_kernel): by default one vector runs on the
 * lookup-table kernel and two or more on the tensor-core kernel, which
 * forms each +-1 dot product as an exact bf16 MMA (fp32 activations are
 * split exactly into three bf16 parts) and scales it per group in fp32. */
int mbok_gemv(const uint32_t* packed, const uint16_t* alpha, int K, int M, int N, int group,
              const void* x, int x_dtype, int batch, float* y, void* workspace,
              size_t workspace_bytes, void* stream);

/* mbok_gemv with the two process-wide choices given per call instead:
 *   kernel         : MBOK_GEMV_AUTO, _LOOKUP, _TENSOR, _LOOKUP_SLABS or
 *                    _LOOKUP_ROWS, as for mbok_gemv_set_kernel;
 *   weights_static : 1 or 0, as for mbok_gemv_set_static_weights.
 * Other arguments, results and accuracy as mbok_gemv; mbok_gemv is this call
 * with the process-wide values.  Nothing process-wide is read or written, so
 * host threads may issue calls with different choices concurrently.
 * MBOK_ERR_INVALID_ARG for any other kernel or weights_static value. */
int mbok_gemv_ex(const uint32_t* packed, const uint16_t* alpha, int K, int M, int N, int group,
                 const void* x, int x_dtype, int batch, float* y, void* workspace, size_t workspace_bytes,
                 int kernel, int weights_static, void* stream);

/* Bytes of device workspace mbok_gemv_svid needs (same rules as
 * mbok_gemv_workspace_bytes; one workspace may serve both calls if it has
 * the larger of the two sizes). */
size_t mbok_gemv_svid_workspace_bytes(int K, int M, int N, int batch);

/* The rank-1-scaled form of the layer (Italian technical summary 2A/2B,
 * Dutch "Methodologie" 2, Spanish 2B: each kernel carries its own rank-1
 * scale, W = sum_k B_k (.) (s_out^k s_in^k^T)):
 *     y[b][r] = sum_k s_out[k][r] * sum_j b_{k,r,j} * s_in[k][j] * x[b][j].
 *   packed : the K sign matrices in layout 1 (as for mbok_gemv).
 *   s_in   : fp16 [K][N] input scales, 16-byte aligned.
 *   s_out  : fp16 [K][M] output scales; any 2-byte alignment.  With M a
 *            multiple of 8 and s_out 16-byte aligned, each 8-row octet's
 *            scales are copied into shared memory with its bits (faster).
 *   x, x_dtype, batch, y, workspace, workspace_bytes, stream: as mbok_gemv
 *            (workspace sized by mbok_gemv_svid_workspace_bytes).
 * Each product s_in * x is formed in fp32 (exact for bf16 x), the +-1 sums
 * come from lookup tables of those products (one launch per vector; each
 * kernel k of a 512-column slab is its own CTA), and the row totals are
 * scaled by s_out in fp32.  Accuracy and determinism as for mbok_gemv, with
 * W the rank-1-scaled matrix above. */
int mbok_gemv_svid(const uint32_t* packed, const uint16_t* s_in, const uint16_t* s_out, int K, int M, int N,
                   const void* x, int x_dtype, int batch, float* y, void* workspace, size_t workspace_bytes,
                   void* stream);

/* Bytes of device workspace mbok_gemv_multi needs (same rules as
 * mbok_gemv_workspace_bytes): the matrices' partial sums, one region per
 * matrix.  0 if N <= 512 or on a bad argument. */
size_t mbok_gemv_multi_workspace_bytes(int nseg, const int* K, const int* M, int N);

/* Several matrices that read the same x, e.g. a layer's q, k and v or its
 * gate and up projections, each with its own number of kernels K[s] and rows
 * M[s], in one launch per vector:
 *     y[b][R_s + r] = sum_j W_s[r][j] * x[b][j],   R_s = M[0] + ... + M[s-1],
 * i.e. the matrices' outputs one after another in each output row of y
 * (fp32 [batch][M[0] + ... + M[nseg-1]]).  The lookup-table kernel of
 * mbok_gemv (any batch: one launch, plus the small launch that adds the
 * slabs' partials, per vector); every output equals, bit for bit, that of
 * mbok_gemv on the matrix alone with the lookup kernel (tested).
 *   nseg       : 1..8 matrices.
 *   packed[s], alpha[s] : matrix s in layout 1 with K[s] kernels (host arrays
 *                of device pointers, each 16-byte aligned).
 *   K[s], M[s] : host arrays; each (K[s], M[s], N) must be a valid shape and
 *                the M[s] sum to at most 2^22.
 *   N, group, x, x_dtype, batch, workspace, workspace_bytes, stream: as
 *                mbok_gemv (workspace sized by mbok_gemv_multi_workspace_bytes).
 * Calls sharing one workspace must not run concurrently. */
int mbok_gemv_multi(int nseg, const uint32_t* const* packed, const uint16_t* const* alpha, const int* K,
                    const int* M, int N, int group, const void* x, int x_dtype, int batch, float* y,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Kernel choice of mbok_gemv and mbok_gemv_noalloc for this process (all
 * devices, all later calls):
 *   MBOK_GEMV_AUTO (default): lookup tables for one vector, tensor cores for
 *     more;
 *   MBOK_GEMV_LOOKUP: lookup tables, once per vector: 8-bit tables over
 *     512-column slabs, whose partial sums a second small launch adds
 *     through the workspace;
 *   MBOK_GEMV_TENSOR: tensor cores for any batch;
 *   MBOK_GEMV_LOOKUP_SLABS: the slab lookup kernel (as MBOK_GEMV_LOOKUP);
 *   MBOK_GEMV_LOOKUP_ROWS: whole rows per CTA with 4-bit tables, one launch
 *     and no workspace, where those tables fit one CTA's shared memory
 *     (N <= 10240; wider rows take the slab kernel).
 * All kernels meet the accuracy stated for mbok_gemv; results differ in
 * rounding.  Atomic, but calls already issued keep the kernel they chose.
 * Returns MBOK_ERR_INVALID_ARG for any other value. */
int mbok_gemv_set_kernel(int kernel);

/* Whether the GEMV kernels may read their weights (packed bits and scales:
 * alpha, or s_in and s_out for mbok_gemv_svid) before waiting for the
 * preceding launch in the stream.  GEMV launches use
 * programmatic dependent launch: a GEMV may start while the kernel before it
 * finishes, if that kernel signalled early (griddepcontrol.launch_dependents);
 * everything it reads after its wait is ordered after that kernel.  With
 * on = 1 (the default) the first weight tiles are copied into shared memory
 * before the wait, hiding their DRAM latency behind the preceding kernel's
 * tail -- by the tensor-core kernel always, by the lookup kernels for
 * launches of up to 16 MB of packed bits (larger launches measured faster
 * reading nothing ahead of the wait); activations, outputs and the
 * workspace are always touched after the wait.  This is safe unless a kernel
 * that signals early writes the weights right before a GEMV -- no kernel of
 * this library does (the ones that write weights never signal early, so a
 * GEMV after them starts only when they are complete).  on = 0 keeps every
 * read after the wait.  Results do not change.  Process-wide; returns
 * MBOK_ERR_INVALID_ARG for other values. */
int mbok_gemv_set_static_weights(int on);

/* mbok_gemv without a workspace argument, for callers that cannot allocate
 * device memory: code that must not call cudaMalloc after start-up (an
 * allocator-free or real-time serving loop), code that runs where allocation
 * is forbidden or would break the caller's memory accounting (a plugin inside
 * a host framework that owns every device buffer), or a C caller with no
 * allocator of its own.  (The method's pages have no counterpart; this is a
 * property of the library, not of the method.)
 *
 * Same arguments, results and accuracy as mbok_gemv, minus the workspace.
 * The scratch mbok_gemv would take from the workspace (the partial sums of
 * the 8-bit slab lookup kernel; the whole-row lookup and tensor-core kernels
 * need none) comes instead from one array of MBOK_NOALLOC_SCRATCH_BYTES
 * (4 MiB) compiled into the library; every GPU that loads the library holds
 * that array until the process exits.  This entry point calls no allocating
 * routine (no cudaMalloc / cudaFree).
 *  - Limit: shapes whose mbok_gemv_workspace_bytes exceeds
 *    MBOK_NOALLOC_SCRATCH_BYTES are rejected with MBOK_ERR_SCRATCH_LIMIT
 *    (roughly M * N > 500 million weights).
 *  - The first call on a device looks up the array's device address (once
 *    per device, with that device current); make that first call before any
 *    CUDA stream capture on that device.
 *  - Nothing in the array outlives a call (each call writes its partial sums
 *    before reading them), so it needs no clearing.
 *  - All calls in the process share the one array: calls that may overlap on
 *    the GPU (different streams without ordering, or several host threads)
 *    race and give wrong results.  Order them on one stream. */
int mbok_gemv_noalloc(const uint32_t* packed, const uint16_t* alpha, int K, int M, int N,
                      int group, const void* x, int x_dtype, int batch, float* y, void* stream);

/* Diagnostic: waits inside the library's kernels are bounded (about a second);
 * a kernel that gives up records a flag and returns early instead of hanging.
 * Writes the flags accumulated on the current device since the last call to
 * *flags (0 = none; bit 0 = a whole-row lookup GEMV copy wait gave up, in
 * which case that CTA stored none of its rows of y; bit 1 = a prefill-GEMM
 * pipeline wait gave up; bit 2 = a tensor-core GEMV copy wait gave up, in
 * which case that launch stored no outputs) and clears them.  Synchronises
 * the device.  Returns MBOK_ERR_CUDA if the flags cannot be read. */
int mbok_read_device_errors(unsigned* flags);

/* Self-check of the bounded waits that the pipelined kernels use: launches
 * one warp that waits, with the same bounded-wait code, on an mbarrier that
 * nothing completes.  After timeout_us microseconds (1..1000000) the wait
 * gives up and records bit 2 of mbok_read_device_errors, exactly as a copy
 * that never landed would; the context stays usable.  No fault, no hang. */
int mbok_check_wait_timeout(unsigned timeout_us, void* stream);

/* Weight precision of the prefill GEMM (argument `precision` of mbok_gemm_ex). */
#define MBOK_GEMM_AUTO 0      /* MBOK_GEMM_SPLIT when N <= MBOK_GEMM_SPLIT_MAX_N, else MBOK_GEMM_BF16 */
#define MBOK_GEMM_BF16 1      /* each weight rounded once to bf16: one MMA per tile */
#define MBOK_GEMM_SPLIT 2     /* each weight as two bf16 terms: two MMAs per tile */
#define MBOK_GEMM_SPLIT_MAX_N 512

/* Y[t][r] = sum_j Wt[r][j] * X[t][j] for t < T (prefill) on the tensor cores
 * (tcgen05, fp32 accumulation in tensor memory).  K Boolean kernels give at
 * most 2^K weight levels per (row, group) (Paper-Notes page, 关键设计); the
 * kernel forms each level v = sum_k s_k alpha_k (s_k = +-1) in fp32 in kernel
 * order -- exactly W[r][j] whenever a group's K scales lie within a factor
 * 2^11 of one another -- and the tile Wt it multiplies is
 *   MBOK_GEMM_BF16:  RN_bf16(v), one rounding: |Wt - W| <= 2^-8 |W|;
 *   MBOK_GEMM_SPLIT: RN_bf16(v) + RN_bf16(v - RN_bf16(v)), two bf16 terms that
 *                    both pass through the MMAs into the same accumulator:
 *                    |Wt - W| <= 2^-16 |W|, at twice the tensor work.
 * Y is rounded to bf16.  X: bf16 [T][N]; Y: bf16 [T][M]; both 16-byte
 * aligned; 1 <= T <= 2^23.
 * Accuracy: |Y - Y_exact| <= u * sum_j |W x| + (fp32 accumulation) + half a
 * bf16 ulp of Y, with u = 2^-16 (split) or 2^-8 (bf16).  The split meets
 * 1e-3 * sum_j |W x| + 2^-8 * |Y_exact| + 1e-6 for every output.  With one
 * rounding the error of a group's weights shares the rounding of its few
 * levels, so the bound above holds only on average: the tests hold every
 * output to it for N >= 1024 (at N = 128 a few outputs in 10^5 miss), which
 * is why MBOK_GEMM_AUTO splits for N <= 512.  Waits inside the kernel are
 * bounded: see mbok_read_device_errors. */
int mbok_gemm_ex(const uint32_t* packed, const uint16_t* alpha, int K, int M, int N, int group,
                 const uint16_t* X, int T, uint16_t* Y, int precision, void* stream);

/* mbok_gemm_ex with MBOK_GEMM_AUTO. */
int mbok_gemm(const uint32_t* packed, const uint16_t* alpha, int K, int M, int N, int group,
              const uint16_t* X, int T, uint16_t* Y, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MBOK_H */
