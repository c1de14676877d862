// Greedy residual binarisation on the GPU, bit-exact by construction.
//
// Each later kernel approximates what the earlier ones leave (Dutch technical
// summary, "Successive SVID"; Spanish technical summary 2B, "Extracción
// Sucesiva"), starting from the greedy initialisation named on the Paper-Notes
// page (训练策略).  For a fixed sign matrix the least-squares group scale is
// mean|R| (Paper-Notes 关键设计, closed-form scale).  Per (row, group), for
// k = 0..K-1:
//     b     = sign(R), sign(0) = +1
//     alpha = fp16(sum_{j=0..127} |R_j| / 128): fp64 sum in column order,
//             one round-to-nearest-even from fp64 to fp16
//     R     = R - alpha * b   (fp32, one rounding, using the fp16 alpha)
// One thread owns one (row, group) and keeps its 128 residuals in registers,
// so the summation order is exactly the column order.
#include "mbok_common.cuh"

namespace mbok {

constexpr int kResidualThreads = 256;            // 32 groups x 8 rows
constexpr int kResidualGroupsPerBlock = kResidualThreads / kOctet;

template <int K>
__global__ void __launch_bounds__(kResidualThreads)
residual_binarize_kernel(const float* __restrict__ W, Shape s, uint8_t* __restrict__ packed,
                         __half* __restrict__ alpha, float* __restrict__ residual) {
  const int i = threadIdx.x % kOctet;                                  // row in octet
  const int g = blockIdx.x * kResidualGroupsPerBlock + threadIdx.x / kOctet;
  const int o = blockIdx.y;
  if (g >= s.G) return;
  const int r = o * kOctet + i;
  const bool valid = r < s.M;

  float R[kGroup];
  if (valid) {
    const float4* src = reinterpret_cast<const float4*>(W + size_t(r) * s.N + size_t(g) * kGroup);
#pragma unroll
    for (int v = 0; v < kGroup / 4; ++v) {
      const float4 t = src[v];
      R[4 * v] = t.x; R[4 * v + 1] = t.y; R[4 * v + 2] = t.z; R[4 * v + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < kGroup; ++j) R[j] = 0.f;
  }

#pragma unroll
  for (int k = 0; k < K; ++k) {
    double acc = 0.0;
#pragma unroll
    for (int j = 0; j < kGroup; ++j) acc = __dadd_rn(acc, double(fabsf(R[j])));
    const __half ah = valid ? __double2half(acc * (1.0 / kGroup)) : __float2half(0.f);
    const float a = __half2float(ah);

    uint8_t* unit0 = packed + unit_offset(s, o, k, g * kUnitsPerGroup) + 2 * i;
#pragma unroll
    for (int u = 0; u < kUnitsPerGroup; ++u) {
      uint32_t h = 0;
#pragma unroll
      for (int b = 0; b < kUnit; ++b) {
        const int j = u * kUnit + b;
        const bool pos = R[j] >= 0.f;
        h |= uint32_t(pos) << b;
        R[j] = __fsub_rn(R[j], pos ? a : -a);
      }
      *reinterpret_cast<uint16_t*>(unit0 + size_t(u) * 16) = valid ? uint16_t(h) : uint16_t(0);
    }
    alpha[alpha_offset(s, o, g, k) + i] = ah;
  }

  if (residual != nullptr && valid) {
    float4* dst = reinterpret_cast<float4*>(residual + size_t(r) * s.N + size_t(g) * kGroup);
#pragma unroll
    for (int v = 0; v < kGroup / 4; ++v)
      dst[v] = make_float4(R[4 * v], R[4 * v + 1], R[4 * v + 2], R[4 * v + 3]);
  }
}

cudaError_t launch_residual_binarize(const float* W, const Shape& s, uint8_t* packed,
                                     __half* alpha, float* residual, cudaStream_t stream) {
  dim3 grid((s.G + kResidualGroupsPerBlock - 1) / kResidualGroupsPerBlock, s.O);
  switch (s.K) {
    case 1: residual_binarize_kernel<1><<<grid, kResidualThreads, 0, stream>>>(W, s, packed, alpha, residual); break;
    case 2: residual_binarize_kernel<2><<<grid, kResidualThreads, 0, stream>>>(W, s, packed, alpha, residual); break;
    case 3: residual_binarize_kernel<3><<<grid, kResidualThreads, 0, stream>>>(W, s, packed, alpha, residual); break;
    default: residual_binarize_kernel<4><<<grid, kResidualThreads, 0, stream>>>(W, s, packed, alpha, residual); break;
  }
  return cudaGetLastError();
}

}  // namespace mbok
