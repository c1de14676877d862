// Packing of sign matrices and scales into storage format 1.
//
// The method's weights are K Boolean matrices B_k in {-1,+1} with one scale
// per (kernel, row, 128-column group) (Paper-Notes page, 方法详解 / 关键设计:
// multi-kernel Boolean parameters, group-wise scales).  These kernels only
// move data; they hold no arithmetic of the method.
#include "mbok_common.cuh"

namespace mbok {

// One thread per 16-byte unit (octet o, kernel k, unit q): reads the 16 int8
// signs of each of the unit's 8 rows and writes 8 halfwords.  An int8 >= 0
// becomes a set bit (+1); pad rows (r >= M) become 0.
__global__ void pack_bits_kernel(const int8_t* __restrict__ signs, Shape s,
                                 uint8_t* __restrict__ packed) {
  const size_t total = size_t(s.O) * s.K * s.Q;
  const size_t idx = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int q = int(idx % s.Q);
  const size_t t = idx / s.Q;
  const int k = int(t % s.K);
  const int o = int(t / s.K);
  uint32_t half[kOctet];
#pragma unroll
  for (int i = 0; i < kOctet; ++i) {
    const int r = o * kOctet + i;
    uint32_t h = 0;
    if (r < s.M) {
      const uint4 v = *reinterpret_cast<const uint4*>(
          signs + (size_t(k) * s.M + r) * s.N + size_t(q) * kUnit);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t neg = 0;  // bit b set when signs[b] < 0 (its byte's top bit)
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int b = 0; b < 4; ++b) neg |= ((w[c] >> (8 * b + 7)) & 1u) << (4 * c + b);
      h = (~neg) & 0xFFFFu;
    }
    half[i] = h;
  }
  uint4 out;
  out.x = half[0] | (half[1] << 16);
  out.y = half[2] | (half[3] << 16);
  out.z = half[4] | (half[5] << 16);
  out.w = half[6] | (half[7] << 16);
  *reinterpret_cast<uint4*>(packed + unit_offset(s, o, k, q)) = out;
}

// One thread per stored scale: the blocked element ((o*G + g)*K + k)*8 + i
// takes the logical element (r*G + g)*K + k of row r = 8o + i (0 for pad rows).
__global__ void pack_alpha_kernel(const uint16_t* __restrict__ in, Shape s,
                                  uint16_t* __restrict__ out) {
  const size_t total = size_t(s.O) * kOctet * s.G * s.K;
  const size_t e = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= total) return;
  const int i = int(e % kOctet);
  size_t t = e / kOctet;
  const int k = int(t % s.K);
  t /= s.K;
  const int g = int(t % s.G);
  const int o = int(t / s.G);
  const int r = o * kOctet + i;
  out[e] = (r < s.M) ? in[(size_t(r) * s.G + g) * s.K + k] : uint16_t(0);
}

cudaError_t launch_pack_bits(const int8_t* signs, const Shape& s, uint8_t* packed,
                             cudaStream_t stream) {
  const size_t total = size_t(s.O) * s.K * s.Q;
  const int threads = 256;
  const unsigned blocks = unsigned((total + threads - 1) / threads);
  pack_bits_kernel<<<blocks, threads, 0, stream>>>(signs, s, packed);
  return cudaGetLastError();
}

cudaError_t launch_pack_alpha(const uint16_t* in, const Shape& s, uint16_t* out,
                              cudaStream_t stream) {
  const size_t total = size_t(s.O) * kOctet * s.G * s.K;
  const int threads = 256;
  const unsigned blocks = unsigned((total + threads - 1) / threads);
  pack_alpha_kernel<<<blocks, threads, 0, stream>>>(in, s, out);
  return cudaGetLastError();
}

}  // namespace mbok
