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
#include "device_once.h"

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

// The current device index, or -1 if the runtime cannot say.
inline int current_device() {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

// SM count of the current device (queried once per device index).
inline int device_sm_count() {
  static PerDeviceValue<int> cache;
  const int dev = current_device();
  const int n = cache.get(dev, [dev]() -> int {
    int v = 0;
    if (dev < 0 || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return v > 0 ? v : 0;
  });
  return n > 0 ? n : 148;
}

// Dynamic shared-memory size (and, if asked, the largest shared-memory
// carveout) of kernel `fn`, set once per device for the flag set `once`:
// the runtime keeps these attributes per device context.
inline cudaError_t set_smem_attr_once(PerDeviceOnce& once, const void* fn, int bytes, bool max_carveout = false) {
  return static_cast<cudaError_t>(run_once_for_device(once, current_device(), [&]() -> int {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && max_carveout)
      e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    return static_cast<int>(e);
  }));
}

}  // namespace mbok
