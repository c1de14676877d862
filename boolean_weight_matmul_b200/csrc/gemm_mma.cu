// Prefill GEMM Y = X Wt^T with warp-level mma.sync (bf16 in, fp32 accumulate).
//
// Wt is W = sum_k alpha_k B_k
// (Paper-Notes page, 方法详解 / 关键设计) rounded to bf16 element-wise while it is
// unpacked into shared memory.
//
// CTA tile: 128 tokens x 128 weight rows, K-step 32 columns, 8 warps as
// 2 (tokens) x 4 (rows), each warp 64 x 32.  Operands staged in padded shared
// memory (80-byte rows) and read with ldmatrix.
#include "mbok_common.cuh"

namespace mbok {

constexpr int kMmaBT = 128;   // tokens per CTA
constexpr int kMmaBR = 128;   // weight rows per CTA
constexpr int kMmaBK = 32;    // columns per step
constexpr int kMmaPitch = kMmaBK + 8;   // bf16 elements per smem row
constexpr int kMmaThreads = 256;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
  const int n = pred ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)), "l"(gmem), "r"(n));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t r[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void mma_bf16(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Unpack 16 columns (one unit) of row r for all kernels into bf16:
// w_j = sum_k (bit ? alpha_k : -alpha_k), fp32 sum, then rounded to bf16.
__device__ __forceinline__ void unpack_unit_bf16(const uint8_t* packed, const uint16_t* alpha,
                                                 const Shape& s, int r, int q, uint32_t out[8]) {
  if (r >= s.M) {
#pragma unroll
    for (int i = 0; i < 8; ++i) out[i] = 0;
    return;
  }
  const int o = r / kOctet, i = r % kOctet, g = q / kUnitsPerGroup;
  float w[16];
#pragma unroll
  for (int b = 0; b < 16; ++b) w[b] = 0.f;
  for (int k = 0; k < s.K; ++k) {
    const uint32_t h = *reinterpret_cast<const uint16_t*>(packed + unit_offset(s, o, k, q) + 2 * i);
    const float a = __half2float(__ushort_as_half(alpha[alpha_offset(s, o, g, k) + i]));
#pragma unroll
    for (int b = 0; b < 16; ++b) w[b] += ((h >> b) & 1u) ? a : -a;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(w[2 * e], w[2 * e + 1]);
    out[e] = *reinterpret_cast<const uint32_t*>(&v);
  }
}

__global__ void __launch_bounds__(kMmaThreads)
gemm_mma_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ alpha, Shape s,
                const uint16_t* __restrict__ X, int T, int x_pitch, uint16_t* __restrict__ Y,
                float* __restrict__ Yf, int y_pitch) {
  __shared__ __align__(128) uint16_t Xs[2][kMmaBT][kMmaPitch];
  __shared__ __align__(128) uint16_t Ws[2][kMmaBR][kMmaPitch];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.y * kMmaBT, r0 = blockIdx.x * kMmaBR;
  const int wt = (warp >> 2) * 64, wr = (warp & 3) * 32;

  float acc[4][4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.f;

  auto stage = [&](int buf, int step) {
    const int c0 = step * kMmaBK;
    // X: 128 tokens x 32 columns = 512 chunks of 16 bytes, 2 per thread
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int chunk = tid + u * kMmaThreads;
      const int row = chunk >> 2, part = chunk & 3;
      const int t = t0 + row;
      const bool ok = t < T;
      const uint16_t* src = X + size_t(ok ? t : 0) * x_pitch + c0 + part * 8;
      cp_async16(&Xs[buf][row][part * 8], src, ok);
    }
    // W: 128 rows x 2 units, one (row, unit) per thread
    {
      const int row = tid >> 1, u = tid & 1;
      uint32_t v[8];
      unpack_unit_bf16(packed, alpha, s, r0 + row, c0 / kUnit + u, v);
      uint4* dst = reinterpret_cast<uint4*>(&Ws[buf][row][u * 16]);
      dst[0] = make_uint4(v[0], v[1], v[2], v[3]);
      dst[1] = make_uint4(v[4], v[5], v[6], v[7]);
    }
    asm volatile("cp.async.commit_group;\n" ::);
  };

  const int steps = s.N / kMmaBK;
  stage(0, 0);
  for (int step = 0; step < steps; ++step) {
    const int buf = step & 1;
    if (step + 1 < steps) {
      stage(buf ^ 1, step + 1);
      asm volatile("cp.async.wait_group 1;\n" ::);
    } else {
      asm volatile("cp.async.wait_group 0;\n" ::);
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kMmaBK; kk += 16) {
      uint32_t af[4][4], bfr[2][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
        ldmatrix_x4(af[mt], &Xs[buf][wt + mt * 16 + (lane & 15)][kk + (lane >> 4) * 8]);
#pragma unroll
      for (int np = 0; np < 2; ++np)
        ldmatrix_x4(bfr[np], &Ws[buf][wr + np * 16 + (lane & 7) + ((lane >> 4) << 3)][kk + ((lane >> 3) & 1) * 8]);
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
          mma_bf16(acc[mt][nt], af[mt], bfr[nt >> 1][(nt & 1) * 2], bfr[nt >> 1][(nt & 1) * 2 + 1]);
    }
    __syncthreads();
  }

  const int g = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = t0 + wt + mt * 16 + g + h * 8;
        if (t >= T) continue;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = r0 + wr + nt * 8 + tq * 2 + e;
          if (r >= s.M) continue;
          const float v = acc[mt][nt][h * 2 + e];
          if (Yf != nullptr) {
            Yf[size_t(t) * y_pitch + r] = v;
          } else {
            Y[size_t(t) * y_pitch + r] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
          }
        }
      }
}

cudaError_t launch_gemm_mma(const uint8_t* packed, const uint16_t* alpha, const Shape& s,
                            const uint16_t* X, int T, uint16_t* Y, float* Yf,
                            cudaStream_t stream) {
  dim3 grid((s.M + kMmaBR - 1) / kMmaBR, (T + kMmaBT - 1) / kMmaBT);
  gemm_mma_kernel<<<grid, kMmaThreads, 0, stream>>>(packed, alpha, s, X, T, s.N, Y, Yf, s.M);
  return cudaGetLastError();
}

}  // namespace mbok
