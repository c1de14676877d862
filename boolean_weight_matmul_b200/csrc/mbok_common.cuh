// Shared definitions for the MBOK kernels (sm_100a).
//
// Storage format 1 (see include/mbok.h): rows in octets of 8; packed bits
// ordered [octet][kernel][16-column unit][row in octet] as 16-bit halfwords
// (bit b of a halfword = column 16*unit + b, set = +1); scales fp16 ordered
// [octet][group][kernel][row in octet].
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/mbok.h"

namespace mbok {

constexpr int kGroup = 128;   // columns per scale group
constexpr int kOctet = 8;     // rows per storage block
constexpr int kUnit = 16;     // columns per 16-bit unit
constexpr int kUnitsPerGroup = kGroup / kUnit;

struct Shape {
  int K, M, N;
  int O;   // row octets
  int G;   // groups
  int Q;   // 16-column units per row
};

inline Shape make_shape(int K, int M, int N) {
  Shape s;
  s.K = K; s.M = M; s.N = N;
  s.O = (M + kOctet - 1) / kOctet;
  s.G = N / kGroup;
  s.Q = N / kUnit;
  return s;
}

// Byte offset of the 16-byte unit (octet o, kernel k, unit q).
__host__ __device__ inline size_t unit_offset(const Shape& s, int o, int k, int q) {
  return ((size_t(o) * s.K + k) * s.Q + q) * 16;
}

// Element offset of the 8 scales (octet o, group g, kernel k).
__host__ __device__ inline size_t alpha_offset(const Shape& s, int o, int g, int k) {
  return ((size_t(o) * s.G + g) * s.K + k) * kOctet;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) {
  return __uint_as_float(b << 16);
}

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t h2) {
  __half2 h = *reinterpret_cast<__half2*>(&h2);
  return __half22float2(h);
}

// SM count of the current device (queried once per process per device index).
inline int device_sm_count() {
  static int cached[64] = {0};
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] > 0) return cached[dev];
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  cached[dev] = n;
  return n;
}

}  // namespace mbok
