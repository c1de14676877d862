// Device helpers shared by the lookup-table GEMV kernels (sm_100a): async
// copies, L2 prefetch, programmatic-dependent-launch control, the table read
// and the cross-lane reduction of an octet's partial sums.
#pragma once

#include "mbok_common.cuh"

namespace mbok {

// ---------------------------------------------------------------------------
// PTX helpers: async copies, L2 prefetch, grid dependency control
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p));
}

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// ---------------------------------------------------------------------------
// Table reads and reductions
// ---------------------------------------------------------------------------

// A lookup: the fp32 table entry at byte offset `off` from `base`.
__device__ __forceinline__ float lut(const unsigned char* base, uint32_t off) {
  return *reinterpret_cast<const float*>(base + off);
}

// Sum acc (8 rows) over the 32 lanes; returns, in every lane, the total of row
// ((lane >> 2) & 7).  Fixed order, hence deterministic.
__device__ __forceinline__ float octet_reduce(const float2 acc2[4], int lane) {
  const float acc[8] = {acc2[0].x, acc2[0].y, acc2[1].x, acc2[1].y,
                        acc2[2].x, acc2[2].y, acc2[3].x, acc2[3].y};
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  float r1[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float keep = b4 ? acc[i + 4] : acc[i];
    const float send = b4 ? acc[i] : acc[i + 4];
    r1[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  float r2[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float keep = b3 ? r1[i + 2] : r1[i];
    const float send = b3 ? r1[i] : r1[i + 2];
    r2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  const float keep = b2 ? r2[1] : r2[0];
  const float send = b2 ? r2[0] : r2[1];
  float r3 = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  r3 += __shfl_xor_sync(0xffffffffu, r3, 2);
  r3 += __shfl_xor_sync(0xffffffffu, r3, 1);
  return r3;
}

}  // namespace mbok
