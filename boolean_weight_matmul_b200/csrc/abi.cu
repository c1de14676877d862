// C ABI of the MBOK library: argument checks on the host, then launches on
// the caller's stream.  Nothing here allocates, synchronises or keeps state
// beyond cached kernel attributes.
#include <atomic>

#include "mbok_common.cuh"

namespace mbok {
cudaError_t launch_pack_bits(const int8_t*, const Shape&, uint8_t*, cudaStream_t);
cudaError_t launch_pack_alpha(const uint16_t*, const Shape&, uint16_t*, cudaStream_t);
cudaError_t launch_residual_binarize(const float*, const Shape&, uint8_t*, __half*, float*,
                                     cudaStream_t);
cudaError_t launch_refit_alpha(const float*, const uint8_t*, const Shape&, __half*, cudaStream_t);
size_t svid_workspace_bytes(int, int);
cudaError_t launch_svid_binarize(const float*, const Shape&, int, uint8_t*, __half*, __half*, float*, void*,
                                 cudaStream_t);
cudaError_t launch_gemv_lut(const uint8_t*, const uint16_t*, const Shape&, const void*, bool,
                            float*, void*, cudaStream_t, bool);
cudaError_t launch_gemv_lut4(const uint8_t*, const uint16_t*, const Shape&, const void*, bool, float*,
                             cudaStream_t, bool);
bool gemv_lut4_supported(const Shape&);
unsigned gemv_lut4_error_flags();
size_t gemv_lut_workspace_bytes(const Shape&);
size_t gemv_svid_workspace_bytes(const Shape&);
cudaError_t launch_gemv_svid(const uint8_t*, const uint16_t*, const uint16_t*, const Shape&, const void*, bool,
                             float*, void*, cudaStream_t, bool);
unsigned gemv_mma_error_flags();
cudaError_t launch_wait_timeout_probe(unsigned, cudaStream_t);
cudaError_t launch_gemv_mma(const uint8_t*, const uint16_t*, const Shape&, const void*, bool, int,
                            float*, cudaStream_t, bool);
cudaError_t launch_gemv(const uint8_t*, const uint16_t*, const Shape&, const void*, bool, int, float*,
                        void*, cudaStream_t);

cudaError_t launch_gemv_lut_multi(int, const uint8_t* const*, const uint16_t* const*, const int*, const int*, int,
                                  const void*, bool, float*, void*, cudaStream_t, bool);
size_t gemv_multi_workspace_bytes(int, const int*, const int*, int);

cudaError_t launch_gemm_tc(const uint8_t*, const uint16_t*, const Shape&, const uint16_t*, int,
                           uint16_t*, bool, cudaStream_t);
unsigned gemm_error_flags();

// Process-wide kernel choice of mbok_gemv / mbok_gemv_noalloc (atomic: host
// threads may set and read it concurrently; a call reads it once).
std::atomic<int> gemv_kernel_choice{MBOK_GEMV_AUTO};
// Process-wide: GEMV weights may be read before the grid dependency wait
// (see mbok_gemv_set_static_weights).
std::atomic<bool> gemv_weights_static{true};

// One decode GEMV call with kernel choice `choice` (MBOK_GEMV_*): a
// lookup-table kernel once per vector -- 512-column slabs with 8-bit tables
// and a combine launch, or, when asked for, whole rows with 4-bit tables in
// one launch where they fit one CTA (N <= 10240) -- or the tensor-core kernel
// over the whole batch.  The slab kernel is the default lookup kernel: on B200
// it measured faster at the LLaMA shapes (the whole-row kernel saves the
// combine launch but does twice the lookups).
cudaError_t launch_gemv(const uint8_t* packed, const uint16_t* alpha, const Shape& s, const void* x,
                        bool x_f32, int batch, float* y, void* workspace, cudaStream_t stream, int choice,
                        bool weights_static) {
  bool tensor = batch > 1;
  if (choice == MBOK_GEMV_LOOKUP || choice == MBOK_GEMV_LOOKUP_SLABS || choice == MBOK_GEMV_LOOKUP_ROWS)
    tensor = false;
  if (choice == MBOK_GEMV_TENSOR) tensor = true;
  if (tensor) return launch_gemv_mma(packed, alpha, s, x, x_f32, batch, y, stream, weights_static);
  const bool rows = choice == MBOK_GEMV_LOOKUP_ROWS && gemv_lut4_supported(s);
  const size_t xbytes = x_f32 ? 4 : 2;
  for (int b = 0; b < batch; ++b) {
    const void* xb = static_cast<const char*>(x) + size_t(b) * s.N * xbytes;
    const cudaError_t e =
        rows ? launch_gemv_lut4(packed, alpha, s, xb, x_f32, y + size_t(b) * s.M, stream, weights_static)
             : launch_gemv_lut(packed, alpha, s, xb, x_f32, y + size_t(b) * s.M, workspace, stream, weights_static);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// The same with the process-wide choices (mbok_gemv_set_kernel,
// mbok_gemv_set_static_weights), read once.
cudaError_t launch_gemv(const uint8_t* packed, const uint16_t* alpha, const Shape& s, const void* x,
                        bool x_f32, int batch, float* y, void* workspace, cudaStream_t stream) {
  return launch_gemv(packed, alpha, s, x, x_f32, batch, y, workspace, stream,
                     gemv_kernel_choice.load(std::memory_order_relaxed),
                     gemv_weights_static.load(std::memory_order_relaxed));
}
}  // namespace mbok

using namespace mbok;

namespace {

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Common shape checks; returns MBOK_OK or the first failing status.
int check_shape(int K, int M, int N) {
  if (K < 1 || K > MBOK_MAX_K) return MBOK_ERR_INVALID_ARG;
  if (M < 1 || N < MBOK_GROUP || N % MBOK_GROUP != 0) return MBOK_ERR_SHAPE;
  // keep every grid dimension and 32-bit unit index in range
  if (M > (1 << 22) || N > (1 << 20)) return MBOK_ERR_SHAPE;
  return MBOK_OK;
}

inline int from_cuda(cudaError_t e) { return e == cudaSuccess ? MBOK_OK : MBOK_ERR_CUDA; }

}  // namespace

extern "C" {

const char* mbok_status_string(int status) {
  switch (status) {
    case MBOK_OK: return "ok";
    case MBOK_ERR_INVALID_ARG: return "invalid argument";
    case MBOK_ERR_SHAPE: return "unsupported shape";
    case MBOK_ERR_ALIGN: return "misaligned pointer";
    case MBOK_ERR_UNSUPPORTED: return "unsupported option";
    case MBOK_ERR_CUDA: return "CUDA launch error";
    case MBOK_ERR_WORKSPACE: return "workspace missing or too small";
    case MBOK_ERR_SCRATCH_LIMIT: return "problem exceeds the built-in scratch of mbok_gemv_noalloc";
    default: return "unknown status";
  }
}

int mbok_layout_version(void) { return MBOK_LAYOUT_VERSION; }

size_t mbok_packed_bytes(int K, int M, int N) {
  if (check_shape(K, M, N) != MBOK_OK) return 0;
  const Shape s = make_shape(K, M, N);
  return size_t(s.O) * K * N;
}

size_t mbok_alpha_elems(int K, int M, int N) {
  if (check_shape(K, M, N) != MBOK_OK) return 0;
  const Shape s = make_shape(K, M, N);
  return size_t(s.O) * kOctet * s.G * K;
}

size_t mbok_gemv_workspace_bytes(int K, int M, int N, int batch) {
  if (check_shape(K, M, N) != MBOK_OK || batch < 1 || batch > MBOK_MAX_BATCH) return 0;
  return gemv_lut_workspace_bytes(make_shape(K, M, N));
}

int mbok_pack_bits(const int8_t* signs, int K, int M, int N, uint32_t* packed, void* stream) {
  const int st = check_shape(K, M, N);
  if (st != MBOK_OK) return st;
  if (signs == nullptr || packed == nullptr) return MBOK_ERR_INVALID_ARG;
  if (!aligned(signs, 16) || !aligned(packed, 16)) return MBOK_ERR_ALIGN;
  return from_cuda(launch_pack_bits(signs, make_shape(K, M, N), reinterpret_cast<uint8_t*>(packed),
                                    as_stream(stream)));
}

int mbok_pack_alpha(const uint16_t* alpha_mgk, int K, int M, int N, uint16_t* alpha_out,
                    void* stream) {
  const int st = check_shape(K, M, N);
  if (st != MBOK_OK) return st;
  if (alpha_mgk == nullptr || alpha_out == nullptr) return MBOK_ERR_INVALID_ARG;
  if (!aligned(alpha_mgk, 16) || !aligned(alpha_out, 16)) return MBOK_ERR_ALIGN;
  return from_cuda(launch_pack_alpha(alpha_mgk, make_shape(K, M, N), alpha_out, as_stream(stream)));
}

int mbok_residual_binarize(const float* W, int M, int N, int K, int group, uint32_t* packed,
                           uint16_t* alpha, float* residual, void* stream) {
  const int st = check_shape(K, M, N);
  if (st != MBOK_OK) return st;
  if (group != MBOK_GROUP) return MBOK_ERR_UNSUPPORTED;
  if (W == nullptr || packed == nullptr || alpha == nullptr) return MBOK_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(alpha, 16) ||
      (residual != nullptr && !aligned(residual, 16)))
    return MBOK_ERR_ALIGN;
  const Shape s = make_shape(K, M, N);
  if (s.O > 65535) return MBOK_ERR_SHAPE;
  return from_cuda(launch_residual_binarize(W, s, reinterpret_cast<uint8_t*>(packed),
                                            reinterpret_cast<__half*>(alpha), residual,
                                            as_stream(stream)));
}

size_t mbok_svid_workspace_bytes(int M, int N) {
  if (check_shape(1, M, N) != MBOK_OK) return 0;
  return svid_workspace_bytes(M, N);
}

int mbok_svid_binarize(const float* W, int M, int N, int K, int iters, uint32_t* packed, uint16_t* s_in,
                       uint16_t* s_out, float* residual, void* workspace, size_t workspace_bytes, void* stream) {
  const int st = check_shape(K, M, N);
  if (st != MBOK_OK) return st;
  if (iters < 1 || iters > 1000) return MBOK_ERR_INVALID_ARG;
  if (W == nullptr || packed == nullptr || s_in == nullptr || s_out == nullptr || residual == nullptr)
    return MBOK_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(s_in, 2) || !aligned(s_out, 2) || !aligned(residual, 16))
    return MBOK_ERR_ALIGN;
  if (workspace == nullptr || workspace_bytes < svid_workspace_bytes(M, N) || !aligned(workspace, 16))
    return MBOK_ERR_WORKSPACE;
  return from_cuda(launch_svid_binarize(W, make_shape(K, M, N), iters, reinterpret_cast<uint8_t*>(packed),
                                        reinterpret_cast<__half*>(s_in), reinterpret_cast<__half*>(s_out), residual,
                                        workspace, as_stream(stream)));
}

int mbok_refit_alpha(const float* W, const uint32_t* packed, int K, int M, int N, int group, uint16_t* alpha,
                     void* stream) {
  const int st = check_shape(K, M, N);
  if (st != MBOK_OK) return st;
  if (group != MBOK_GROUP) return MBOK_ERR_UNSUPPORTED;
  if (W == nullptr || packed == nullptr || alpha == nullptr) return MBOK_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(alpha, 16)) return MBOK_ERR_ALIGN;
  const Shape s = make_shape(K, M, N);
  if (s.O > 65535) return MBOK_ERR_SHAPE;
  return from_cuda(launch_refit_alpha(W, reinterpret_cast<const uint8_t*>(packed), s,
                                      reinterpret_cast<__half*>(alpha), as_stream(stream)));
}

int mbok_gemv_ex(const uint32_t* packed, const uint16_t* alpha, int K, int M, int N, int group,
                 const void* x, int x_dtype, int batch, float* y, void* workspace, size_t workspace_bytes,
                 int kernel, int weights_static, void* stream) {
  const int st = check_shape(K, M, N);
  if (st != MBOK_OK) return st;
  if (group != MBOK_GROUP) return MBOK_ERR_UNSUPPORTED;
  if (packed == nullptr || alpha == nullptr || x == nullptr || y == nullptr)
    return MBOK_ERR_INVALID_ARG;
  if (x_dtype != MBOK_F32 && x_dtype != MBOK_BF16) return MBOK_ERR_INVALID_ARG;
  if (batch < 1 || batch > MBOK_MAX_BATCH) return MBOK_ERR_INVALID_ARG;
  if (kernel < MBOK_GEMV_AUTO || kernel > MBOK_GEMV_LOOKUP_ROWS) return MBOK_ERR_INVALID_ARG;
  if (weights_static != 0 && weights_static != 1) return MBOK_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(alpha, 16) || !aligned(x, 16) || !aligned(y, 4))
    return MBOK_ERR_ALIGN;
  const Shape s = make_shape(K, M, N);
  const size_t need = gemv_lut_workspace_bytes(s);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 16)))
    return MBOK_ERR_WORKSPACE;
  return from_cuda(launch_gemv(reinterpret_cast<const uint8_t*>(packed), alpha, s, x, x_dtype == MBOK_F32,
                               batch, y, workspace, as_stream(stream), kernel, weights_static == 1));
}

int mbok_gemv(const uint32_t* packed, const uint16_t* alpha, int K, int M, int N, int group,
              const void* x, int x_dtype, int batch, float* y, void* workspace,
              size_t workspace_bytes, void* stream) {
  return mbok_gemv_ex(packed, alpha, K, M, N, group, x, x_dtype, batch, y, workspace, workspace_bytes,
                      gemv_kernel_choice.load(std::memory_order_relaxed),
                      gemv_weights_static.load(std::memory_order_relaxed) ? 1 : 0, stream);
}

// Argument checks of the multi-matrix GEMV's shape arrays; MBOK_OK or the
// first failing status, and the total row count in *rows.
static int check_multi(int nseg, const int* K, const int* M, int N, long long* rows) {
  if (nseg < 1 || nseg > 8 || K == nullptr || M == nullptr) return MBOK_ERR_INVALID_ARG;
  long long total = 0;
  for (int i = 0; i < nseg; ++i) {
    const int st = check_shape(K[i], M[i], N);
    if (st != MBOK_OK) return st;
    total += M[i];
  }
  if (total > (1 << 22)) return MBOK_ERR_SHAPE;
  *rows = total;
  return MBOK_OK;
}

size_t mbok_gemv_multi_workspace_bytes(int nseg, const int* K, const int* M, int N) {
  long long rows = 0;
  if (check_multi(nseg, K, M, N, &rows) != MBOK_OK) return 0;
  return gemv_multi_workspace_bytes(nseg, K, M, N);
}

int mbok_gemv_multi(int nseg, const uint32_t* const* packed, const uint16_t* const* alpha, const int* K,
                    const int* M, int N, int group, const void* x, int x_dtype, int batch, float* y,
                    void* workspace, size_t workspace_bytes, void* stream) {
  long long rows = 0;
  const int st = check_multi(nseg, K, M, N, &rows);
  if (st != MBOK_OK) return st;
  if (group != MBOK_GROUP) return MBOK_ERR_UNSUPPORTED;
  if (packed == nullptr || alpha == nullptr || x == nullptr || y == nullptr) return MBOK_ERR_INVALID_ARG;
  if (x_dtype != MBOK_F32 && x_dtype != MBOK_BF16) return MBOK_ERR_INVALID_ARG;
  if (batch < 1 || batch > MBOK_MAX_BATCH) return MBOK_ERR_INVALID_ARG;
  for (int i = 0; i < nseg; ++i) {
    if (packed[i] == nullptr || alpha[i] == nullptr) return MBOK_ERR_INVALID_ARG;
    if (!aligned(packed[i], 16) || !aligned(alpha[i], 16)) return MBOK_ERR_ALIGN;
  }
  if (!aligned(x, 16) || !aligned(y, 4)) return MBOK_ERR_ALIGN;
  const size_t need = gemv_multi_workspace_bytes(nseg, K, M, N);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 16)))
    return MBOK_ERR_WORKSPACE;
  const uint8_t* p8[8];
  for (int i = 0; i < nseg; ++i) p8[i] = reinterpret_cast<const uint8_t*>(packed[i]);
  const size_t xbytes = (x_dtype == MBOK_F32) ? 4 : 2;
  for (int b = 0; b < batch; ++b) {
    const void* xb = static_cast<const char*>(x) + size_t(b) * N * xbytes;
    const cudaError_t e = launch_gemv_lut_multi(nseg, p8, alpha, K, M, N, xb, x_dtype == MBOK_F32,
                                                y + size_t(b) * size_t(rows), workspace, as_stream(stream),
                                                gemv_weights_static.load(std::memory_order_relaxed));
    if (e != cudaSuccess) return MBOK_ERR_CUDA;
  }
  return MBOK_OK;
}

int mbok_gemv_set_static_weights(int on) {
  if (on != 0 && on != 1) return MBOK_ERR_INVALID_ARG;
  gemv_weights_static.store(on == 1, std::memory_order_relaxed);
  return MBOK_OK;
}

int mbok_gemv_set_kernel(int kernel) {
  if (kernel < MBOK_GEMV_AUTO || kernel > MBOK_GEMV_LOOKUP_ROWS) return MBOK_ERR_INVALID_ARG;
  gemv_kernel_choice.store(kernel, std::memory_order_relaxed);
  return MBOK_OK;
}

size_t mbok_gemv_svid_workspace_bytes(int K, int M, int N, int batch) {
  if (check_shape(K, M, N) != MBOK_OK || batch < 1 || batch > MBOK_MAX_BATCH) return 0;
  return gemv_svid_workspace_bytes(make_shape(K, M, N));
}

int mbok_gemv_svid(const uint32_t* packed, const uint16_t* s_in, const uint16_t* s_out, int K, int M, int N,
                   const void* x, int x_dtype, int batch, float* y, void* workspace, size_t workspace_bytes,
                   void* stream) {
  const int st = check_shape(K, M, N);
  if (st != MBOK_OK) return st;
  if (packed == nullptr || s_in == nullptr || s_out == nullptr || x == nullptr || y == nullptr)
    return MBOK_ERR_INVALID_ARG;
  if (x_dtype != MBOK_F32 && x_dtype != MBOK_BF16) return MBOK_ERR_INVALID_ARG;
  if (batch < 1 || batch > MBOK_MAX_BATCH) return MBOK_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(s_in, 16) || !aligned(s_out, 2) || !aligned(x, 16) || !aligned(y, 4))
    return MBOK_ERR_ALIGN;
  const Shape s = make_shape(K, M, N);
  const size_t need = gemv_svid_workspace_bytes(s);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 16)))
    return MBOK_ERR_WORKSPACE;
  const size_t xbytes = (x_dtype == MBOK_F32) ? 4 : 2;
  for (int b = 0; b < batch; ++b) {
    const void* xb = static_cast<const char*>(x) + size_t(b) * N * xbytes;
    const cudaError_t e = launch_gemv_svid(reinterpret_cast<const uint8_t*>(packed), s_in, s_out, s, xb,
                                           x_dtype == MBOK_F32, y + size_t(b) * M, workspace, as_stream(stream),
                                           gemv_weights_static.load(std::memory_order_relaxed));
    if (e != cudaSuccess) return MBOK_ERR_CUDA;
  }
  return MBOK_OK;
}

int mbok_check_wait_timeout(unsigned timeout_us, void* stream) {
  if (timeout_us < 1 || timeout_us > 1000000) return MBOK_ERR_INVALID_ARG;
  return from_cuda(launch_wait_timeout_probe(timeout_us, as_stream(stream)));
}

int mbok_read_device_errors(unsigned* flags) {
  if (flags == nullptr) return MBOK_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return MBOK_ERR_CUDA;
  const unsigned g = gemv_lut4_error_flags();
  const unsigned m = gemm_error_flags();
  const unsigned t = gemv_mma_error_flags();
  if (g == ~0u || m == ~0u || t == ~0u) return MBOK_ERR_CUDA;
  *flags = (g ? 1u : 0u) | (m ? 2u : 0u) | (t ? 4u : 0u);
  return MBOK_OK;
}

int mbok_gemm_ex(const uint32_t* packed, const uint16_t* alpha, int K, int M, int N, int group,
                 const uint16_t* X, int T, uint16_t* Y, int precision, void* stream) {
  const int st = check_shape(K, M, N);
  if (st != MBOK_OK) return st;
  if (group != MBOK_GROUP) return MBOK_ERR_UNSUPPORTED;
  if (T < 1 || T > (1 << 23)) return MBOK_ERR_SHAPE;
  if (packed == nullptr || alpha == nullptr || X == nullptr || Y == nullptr)
    return MBOK_ERR_INVALID_ARG;
  if (precision < MBOK_GEMM_AUTO || precision > MBOK_GEMM_SPLIT) return MBOK_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(alpha, 16) || !aligned(X, 16) || !aligned(Y, 16))
    return MBOK_ERR_ALIGN;
  const bool split = precision == MBOK_GEMM_SPLIT || (precision == MBOK_GEMM_AUTO && N <= MBOK_GEMM_SPLIT_MAX_N);
  return from_cuda(launch_gemm_tc(reinterpret_cast<const uint8_t*>(packed), alpha, make_shape(K, M, N), X,
                                  T, Y, split, as_stream(stream)));
}

int mbok_gemm(const uint32_t* packed, const uint16_t* alpha, int K, int M, int N, int group,
              const uint16_t* X, int T, uint16_t* Y, void* stream) {
  return mbok_gemm_ex(packed, alpha, K, M, N, group, X, T, Y, MBOK_GEMM_AUTO, stream);
}

}  // extern "C"
