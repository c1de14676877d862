// Successive SVID on the GPU: K Boolean kernels with rank-1 scales.
//
// Each kernel takes the signs of the current residual and a rank-1
// approximation of its absolute values (via the SVD) as the scale vectors;
// the residual passes to the next kernel (Dutch technical summary,
// "Methodologie" 2, Successive SVID; Italian 2A; Spanish 2B):
//     B_k = sign(R_{k-1}),  |R_{k-1}| ~ sigma u v^T,
//     s_out^k = sqrt(sigma) u,  s_in^k = sqrt(sigma) v,
//     R_k = R_{k-1} - B_k (.) (s_out^k s_in^k^T).
// The top singular pair of the nonnegative |R| comes from power iteration
// started at the uniform vector (it stays nonnegative and converges to the
// Perron vectors; the second singular value of |R| is a few percent of the
// first for weight-like matrices, so a few iterations reach fp16 accuracy):
//     u = |R| v,  w = |R|^T u,  v = w / ||w||   (iters times), then
//     u = |R| v,  sigma = ||u||,  s_out = u / sqrt(sigma),  s_in = sqrt(sigma) v.
// Every sum runs in a fixed order (a warp per row; per-block column partials
// summed in block order; norms in one CTA), so results are deterministic.  The
// scales are rounded once to fp16 and the residual update uses those values:
// R <- R - b * (s_out_r * s_in_j), one exact fp32 product and one fp32
// subtraction, the signs packed into storage format 1 in the same pass.
#include "mbok_common.cuh"

namespace mbok {

constexpr int kSvThreads = 256;
constexpr int kSvRowBlock = 64;          // rows per column-partial block
constexpr int kSvColsPerThread = 4;

struct SvidWork {
  float* u;        // [M]
  float* v;        // [N]
  float* w;        // [N]
  float* partial;  // [nblk][N]
  int nblk;
};

// u[r] = sum_j |R[r][j]| v[j]: one warp per row, lanes stride the row in
// float4s, then a fixed shuffle tree.
__global__ void __launch_bounds__(kSvThreads) svid_rows_kernel(const float* __restrict__ R, const float* __restrict__ v,
                                                               float* __restrict__ u, int M, int N) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * (kSvThreads / 32) + (threadIdx.x >> 5);
  if (r >= M) return;
  const float4* row = reinterpret_cast<const float4*>(R + size_t(r) * N);
  const float4* vv = reinterpret_cast<const float4*>(v);
  float acc = 0.f;
  for (int c = lane; c < N / 4; c += 32) {
    const float4 a = row[c], b = vv[c];
    acc = __fmaf_rn(fabsf(a.x), b.x, acc);
    acc = __fmaf_rn(fabsf(a.y), b.y, acc);
    acc = __fmaf_rn(fabsf(a.z), b.z, acc);
    acc = __fmaf_rn(fabsf(a.w), b.w, acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) u[r] = acc;
}

// partial[blk][j] = sum over the block's rows r (in order) of |R[r][j]| u[r].
__global__ void __launch_bounds__(kSvThreads) svid_cols_kernel(const float* __restrict__ R, const float* __restrict__ u,
                                                               float* __restrict__ partial, int M, int N) {
  const int j0 = (blockIdx.x * kSvThreads + threadIdx.x) * kSvColsPerThread;
  if (j0 >= N) return;
  const int r0 = blockIdx.y * kSvRowBlock, r1 = min(r0 + kSvRowBlock, M);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int r = r0; r < r1; ++r) {
    const float4 a = *reinterpret_cast<const float4*>(R + size_t(r) * N + j0);
    const float ur = u[r];
    acc.x = __fmaf_rn(fabsf(a.x), ur, acc.x);
    acc.y = __fmaf_rn(fabsf(a.y), ur, acc.y);
    acc.z = __fmaf_rn(fabsf(a.z), ur, acc.z);
    acc.w = __fmaf_rn(fabsf(a.w), ur, acc.w);
  }
  *reinterpret_cast<float4*>(partial + size_t(blockIdx.y) * N + j0) = acc;
}

// w[j] = sum over blocks (in order) of partial[blk][j].
__global__ void __launch_bounds__(kSvThreads) svid_colsum_kernel(const float* __restrict__ partial, float* __restrict__ w,
                                                                 int N, int nblk) {
  const int j = blockIdx.x * kSvThreads + threadIdx.x;
  if (j >= N) return;
  float acc = 0.f;
  for (int b = 0; b < nblk; ++b) acc += partial[size_t(b) * N + j];
  w[j] = acc;
}

// Fixed-order block reduction of sum x^2 over n values (one CTA).
__device__ __forceinline__ float block_sumsq(const float* __restrict__ x, int n) {
  __shared__ float red[kSvThreads];
  float acc = 0.f;
  for (int i = threadIdx.x; i < n; i += kSvThreads) acc = __fmaf_rn(x[i], x[i], acc);
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = kSvThreads / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  const float total = red[0];
  __syncthreads();
  return total;
}

// v = w / ||w|| (one CTA).
// (An all-zero w, from an all-zero residual, leaves v as it is.)
__global__ void __launch_bounds__(kSvThreads) svid_normalize_kernel(const float* __restrict__ w, float* __restrict__ v,
                                                                    int n) {
  const float norm = sqrtf(block_sumsq(w, n));
  if (norm == 0.f) return;
  const float inv = 1.f / norm;
  for (int i = threadIdx.x; i < n; i += kSvThreads) v[i] = w[i] * inv;
}

__global__ void svid_fill_kernel(float* __restrict__ v, int n, float value) {
  const int i = blockIdx.x * kSvThreads + threadIdx.x;
  if (i < n) v[i] = value;
}

// sigma = ||u||; s_out = u / sqrt(sigma), s_in = sqrt(sigma) v, rounded to fp16 (one CTA).
__global__ void __launch_bounds__(kSvThreads) svid_scales_kernel(const float* __restrict__ u, const float* __restrict__ v,
                                                                 __half* __restrict__ s_out, __half* __restrict__ s_in,
                                                                 int M, int N) {
  const float sigma = sqrtf(block_sumsq(u, M));
  const float root = sqrtf(sigma);
  const float inv_root = sigma > 0.f ? 1.f / root : 0.f;   // all-zero residual: zero scales
  for (int i = threadIdx.x; i < M; i += kSvThreads) s_out[i] = __float2half_rn(u[i] * inv_root);
  for (int j = threadIdx.x; j < N; j += kSvThreads) s_in[j] = __float2half_rn(root * v[j]);
}

// Signs of R for kernel k into layout 1, and R <- R - b * (s_out_r * s_in_j).
// One thread per (octet, 16-column unit).
__global__ void __launch_bounds__(kSvThreads) svid_sign_update_kernel(float* __restrict__ R, const __half* __restrict__ s_out,
                                                                      const __half* __restrict__ s_in, Shape s, int k,
                                                                      uint8_t* __restrict__ packed) {
  const long long idx = (long long)blockIdx.x * kSvThreads + threadIdx.x;
  if (idx >= (long long)s.O * s.Q) return;
  const int o = int(idx / s.Q), q = int(idx % s.Q);
  float sin_f[kUnit];
#pragma unroll
  for (int b = 0; b < kUnit; ++b) sin_f[b] = __half2float(s_in[q * kUnit + b]);
  // The unit's 16 residuals of a row are 64 contiguous bytes (16-byte aligned:
  // R is, and N is a multiple of 128): four 16-byte loads and stores, for four
  // rows at a time, instead of 16 scalar accesses per row (the same
  // arithmetic per element).  The scalar form ran at 1.0 TB/s (355 us per
  // kernel at 11008 x 4096); this one took the whole K = 3 conversion from
  // 2.49 to 1.60 ms.
  uint32_t h[kOctet];
#pragma unroll
  for (int i0 = 0; i0 < kOctet; i0 += 4) {
    float4 v[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = o * kOctet + i0 + i;
      const float4* src = reinterpret_cast<const float4*>(R + size_t(r) * s.N + size_t(q) * kUnit);
#pragma unroll
      for (int c = 0; c < 4; ++c) v[i][c] = r < s.M ? src[c] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = o * kOctet + i0 + i;
      h[i0 + i] = 0;
      if (r >= s.M) continue;
      const float so = __half2float(s_out[r]);
      float4* dst = reinterpret_cast<float4*>(R + size_t(r) * s.N + size_t(q) * kUnit);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float e[4] = {v[i][c].x, v[i][c].y, v[i][c].z, v[i][c].w};
#pragma unroll
        for (int d = 0; d < 4; ++d) {
          const int b = 4 * c + d;
          const bool pos = e[d] >= 0.f;
          h[i0 + i] |= uint32_t(pos) << b;
          const float p = __fmul_rn(so, sin_f[b]);
          e[d] = __fsub_rn(e[d], pos ? p : -p);
        }
        dst[c] = make_float4(e[0], e[1], e[2], e[3]);
      }
    }
  }
  uint4 out;
  out.x = h[0] | (h[1] << 16);
  out.y = h[2] | (h[3] << 16);
  out.z = h[4] | (h[5] << 16);
  out.w = h[6] | (h[7] << 16);
  *reinterpret_cast<uint4*>(packed + unit_offset(s, o, k, q)) = out;
}

static size_t round4(size_t n) { return (n + 3) / 4 * 4; }

size_t svid_workspace_bytes(int M, int N) {
  const size_t nblk = (size_t(M) + kSvRowBlock - 1) / kSvRowBlock;
  return (round4(M) + 2 * size_t(N) + nblk * size_t(N)) * sizeof(float);
}

// W (fp32 [M][N]) -> K kernels in layout 1, s_in fp16 [K][N], s_out fp16
// [K][M], residual fp32 [M][N] = R_K; the workspace as sized above.
cudaError_t launch_svid_binarize(const float* W, const Shape& s, int iters, uint8_t* packed, __half* s_in,
                                 __half* s_out, float* R, void* workspace, cudaStream_t stream) {
  const int M = s.M, N = s.N;
  char* base = static_cast<char*>(workspace);
  SvidWork wk;
  wk.nblk = (M + kSvRowBlock - 1) / kSvRowBlock;
  wk.u = reinterpret_cast<float*>(base);
  wk.v = wk.u + round4(M);   // 16-byte aligned for the float4 reads
  wk.w = wk.v + N;
  wk.partial = wk.w + N;
  // R starts as W.
  cudaError_t e = cudaMemcpyAsync(R, W, size_t(M) * N * sizeof(float), cudaMemcpyDeviceToDevice, stream);
  if (e != cudaSuccess) return e;
  const dim3 rows_grid((M + kSvThreads / 32 - 1) / (kSvThreads / 32));
  const dim3 cols_grid((N / kSvColsPerThread + kSvThreads - 1) / kSvThreads, wk.nblk);
  const dim3 vec_grid((N + kSvThreads - 1) / kSvThreads);
  const long long units = (long long)s.O * s.Q;
  const dim3 upd_grid(unsigned((units + kSvThreads - 1) / kSvThreads));
  for (int k = 0; k < s.K; ++k) {
    svid_fill_kernel<<<vec_grid, kSvThreads, 0, stream>>>(wk.v, N, 1.f / sqrtf(float(N)));
    for (int t = 0; t < iters; ++t) {
      svid_rows_kernel<<<rows_grid, kSvThreads, 0, stream>>>(R, wk.v, wk.u, M, N);
      svid_cols_kernel<<<cols_grid, kSvThreads, 0, stream>>>(R, wk.u, wk.partial, M, N);
      svid_colsum_kernel<<<vec_grid, kSvThreads, 0, stream>>>(wk.partial, wk.w, N, wk.nblk);
      svid_normalize_kernel<<<1, kSvThreads, 0, stream>>>(wk.w, wk.v, N);
    }
    svid_rows_kernel<<<rows_grid, kSvThreads, 0, stream>>>(R, wk.v, wk.u, M, N);
    svid_scales_kernel<<<1, kSvThreads, 0, stream>>>(wk.u, wk.v, s_out + size_t(k) * M, s_in + size_t(k) * N, M, N);
    svid_sign_update_kernel<<<upd_grid, kSvThreads, 0, stream>>>(R, s_out + size_t(k) * M, s_in + size_t(k) * N, s, k,
                                                                  packed);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace mbok
