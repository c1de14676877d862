// Small-batch GEMV Y = W X (2..16 activation vectors) on the sm_100a tensor
// cores: tcgen05.mma with the sign tiles in tensor memory.
//
// The layer is y_r = sum_g sum_k alpha_{k,r,g} * s_{k,r,g} with
// s_{k,r,g} = sum_{j in g} b_{k,r,j} x_j, b in {-1,+1} (Paper-Notes page,
// 方法详解 / 关键设计: W x as K Boolean products, one scale per group).  Each
// s_{k,.,g} for a 128-row tile is one exact tensor-core product:
//
//  * A = the +-1 signs of kernel k on the tile's 128 rows x the group's 128
//    columns as bf16 (0x3F80 = +1, 0xBF80 = -1), built in registers (a pair
//    of columns is one shift and one three-input logic op on the bit
//    pattern) and stored straight into tensor memory with tcgen05.st: thread
//    = row = tensor-memory lane, two bf16 per column.  The MMA reads A from
//    there (the tcgen05 "A in tensor memory" form), so the signs never pass
//    through shared memory.
//  * B = the activations of the group, NB rows (vectors; for fp32 input the
//    three exact bf16 parts hi, mid, lo of each vector) x 128 columns,
//    brought into shared memory by TMA with 128-byte swizzle (rows past the
//    batch are zero-filled by the copy).
//  * D = s_{k,.,g} for the NB rows of B, fp32 in tensor memory; every product
//    is exact, so each s is an fp32 sum of exact terms.  Four read-back warps
//    load D (tcgen05.ld), add the parts of an fp32 vector (hi + mid, + lo),
//    and apply the fp16 group scale with one fp32 FMA per (row, vector),
//    groups and kernels in order.
//  * Work units are (row tile, group) pairs in tile-major order; a
//    persistent grid of at most one CTA per SM takes equal contiguous runs
//    of units (stream-K), so every SM gets the same number of groups.  A CTA
//    stores one partial row sum per tile it touches; a second small grid
//    adds the partials of each tile in CTA order: deterministic.
//  * Warp roles: warp 0 issues the TMA loads of a unit (activations, the
//    tile's bits of the group: 16 octets x K lines of 128 bytes, 128-byte
//    swizzle, and its scales) into a 6-stage ring; warp 1 (one thread)
//    issues the MMAs, 8 x (M=128, N=NB, K=16) per (unit, kernel), and
//    commits them to mbarriers; warps 2-5 read the accumulators back; warps
//    6-21 build the sign tiles, four per tensor-memory lane quarter, two
//    16-column chunks each.  Tensor memory holds two accumulator sets (one
//    unit read back while the next accumulates) and a ring of sign slots.
//  * Every mbarrier wait is bounded (1 s); on timeout the CTA records an
//    error flag (bit 2 of mbok_read_device_errors), drains what it issued
//    (bounded), frees its tensor memory and exits.
#include "tc_common.cuh"

namespace mbok {

constexpr int kGtRows = 128;                              // rows per tile: MMA M, one lane per row
constexpr int kGtOctets = kGtRows / kOctet;               // 16
constexpr int kGtChunks = kGroup / kUnit;                 // 8 MMAs (K = 16) per (unit, kernel)
constexpr int kGtProdPerQuad = 4;                         // sign-building warps per lane quarter
constexpr int kGtProdWarps = 4 * kGtProdPerQuad;          // 16
constexpr int kGtChunksPerProd = kGtChunks / kGtProdPerQuad;   // 2
constexpr int kGtReadWarp0 = 2;                           // warps 2..5: accumulator read-back
constexpr int kGtProdWarp0 = 6;                           // warps 6..21: sign tiles
constexpr int kGtThreads = (kGtProdWarp0 + kGtProdWarps) * 32;
constexpr int kGtStages = 6;
constexpr int kGtMaxCtas = 160;                           // grid bound (sizes the workspace)
constexpr unsigned kGtTmemCols = 512;
// At least this much shared memory per CTA, so that no two CTAs of these
// kernels share an SM: each allocates all 512 tensor-memory columns.
constexpr int kGtSmemFloor = 120 * 1024;

static_assert(kGtChunksPerProd == 2, "a sign-building warp stores two chunks (16 columns) at once");

template <int K, int NB>
struct GtGeom {
  static constexpr int kXBytes = 2 * NB * 128;              // two 64-column atoms of NB rows
  static constexpr int kBitsBytes = kGtOctets * K * 128;    // lines (octet, kernel) of 128 bytes
  static constexpr int kAlphaBytes = kGtOctets * K * 16;    // [octet][kernel][8 rows] fp16
  static constexpr int kTx = kXBytes + kBitsBytes + kAlphaBytes;
  static constexpr int kStage = (kTx + 1023) / 1024 * 1024;
  static constexpr int kDCols = K * NB;                     // one accumulator set
  static constexpr int kASlotsFit = (int(kGtTmemCols) - 2 * kDCols) / 64;
  static constexpr int kASlots = kASlotsFit > 6 ? 6 : kASlotsFit;   // sign slots of 64 columns
  static constexpr int kACol0 = 2 * kDCols;
  // Kernels whose sign slots are written, handed over and multiplied together
  // (all K when tensor memory holds them twice over).
  static constexpr int kKGroup = 2 * K <= kASlots ? K : (kASlots / 2 >= 1 ? kASlots / 2 : 1);
  static constexpr int kBarBytes = 8 * (2 * kGtStages + 2 * kASlots + 4) + 16;
  static constexpr int kSmemNeed = kGtStages * kStage + 1024 + kBarBytes;
  static constexpr int kSmem = kSmemNeed > kGtSmemFloor ? kSmemNeed : kGtSmemFloor;
  static_assert(kASlots >= 2, "tensor memory must hold two accumulator sets and two sign slots");
  static_assert(kXBytes % 1024 == 0 && kBitsBytes % 1024 == 0, "swizzled buffers start 1024-byte aligned");
};

struct GtParams {
  float* partial;   // [ncta + T - 1][batch][128] row sums per (CTA, tile)
  Shape s;
  int batch;
  int T;            // row tiles
  int U;            // units = T * G
  int ncta;
  uint32_t idesc;
};

__device__ unsigned int g_gemv_tc_error;

__device__ __forceinline__ void gt_grid_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void gt_allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// Warp-uniform bounded wait: every lane polls (and so acquires), the warp
// agrees on the outcome.
__device__ __forceinline__ bool gt_wait_warp(uint64_t* bar, unsigned parity) {
  return __all_sync(0xffffffffu, tc_wait(bar, parity)) != 0;
}

// First unit of CTA c: floor(c U / ncta); CTA owning unit u: the largest c
// with first(c) <= u.
__host__ __device__ __forceinline__ int gt_first_unit(int c, int U, int ncta) {
  return int((long long)c * U / ncta);
}
__host__ __device__ __forceinline__ int gt_cta_of(int u, int U, int ncta) {
  return int(((long long)(u + 1) * ncta + U - 1) / U) - 1;
}

// bf16 pair for columns (2I, 2I+1) of a 16-column unit: u = h | h << 15 holds
// bit b at b and at b + 15, so a shift by 15 - 2I brings bit 2I to 15 and bit
// 2I+1 to 31; a set bit is +1: word = (~s & 0x80008000) | 0x3F803F80.
template <int I>
__device__ __forceinline__ uint32_t gt_sign_pair(uint32_t u) {
  const uint32_t s = u << (15 - 2 * I);
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xAE;\n" : "=r"(r) : "r"(s), "r"(0x80008000u), "r"(0x3F803F80u));
  return r;
}

__device__ __forceinline__ void gt_sign_unit(uint32_t h, uint32_t* w) {
  const uint32_t u = h | (h << 15);
  w[0] = gt_sign_pair<0>(u);
  w[1] = gt_sign_pair<1>(u);
  w[2] = gt_sign_pair<2>(u);
  w[3] = gt_sign_pair<3>(u);
  w[4] = gt_sign_pair<4>(u);
  w[5] = gt_sign_pair<5>(u);
  w[6] = gt_sign_pair<6>(u);
  w[7] = gt_sign_pair<7>(u);
}

__device__ __forceinline__ void gt_tmem_st16(uint32_t taddr, const uint32_t* w) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(
          taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]), "r"(w[8]),
      "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
      : "memory");
}

__device__ __forceinline__ void gt_tmem_ld16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

// Part `part` (0 = hi, 1 = mid, 2 = lo) of the exact three-way bf16 split of v:
// hi = bf16(v), mid = bf16(v - hi), lo = bf16(v - hi - mid); each difference is
// exact in fp32 and lo carries the last 8 significant bits.
__device__ __forceinline__ uint16_t gt_bf16_part(float v, int part) {
  const uint16_t h = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  if (part == 0) return h;
  const float r = __fsub_rn(v, __uint_as_float(uint32_t(h) << 16));
  const uint16_t m = __bfloat16_as_ushort(__float2bfloat16_rn(r));
  if (part == 1) return m;
  return __bfloat16_as_ushort(__float2bfloat16_rn(__fsub_rn(r, __uint_as_float(uint32_t(m) << 16))));
}

// fp32 X [batch][N] -> bf16 parts [3 * batch][N], row 3n + part.
__global__ void __launch_bounds__(256) gemv_tc_split_kernel(const float* __restrict__ x, uint16_t* __restrict__ xs,
                                                            int N, int batch) {
  gt_allow_dependents();
  gt_grid_wait();
  const long long i = (long long)blockIdx.x * 256 + threadIdx.x;
  if (i >= (long long)batch * N) return;
  const int n = int(i / N), j = int(i % N);
  const float v = x[i];
#pragma unroll
  for (int part = 0; part < 3; ++part) xs[size_t(3 * n + part) * N + j] = gt_bf16_part(v, part);
}

template <int K, int NB, bool XF32>
__global__ void __launch_bounds__(kGtThreads, 1)
gemv_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap bmap,
               const __grid_constant__ CUtensorMap amap, GtParams p) {
  using G = GtGeom<K, NB>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGtStages * G::kStage);   // unit's TMA data landed
  uint64_t* empty = full + kGtStages;          // unit's stage consumed (signs built, scales read, MMAs done)
  uint64_t* afull = empty + kGtStages;         // sign slot written
  uint64_t* aempty = afull + G::kASlots;       // sign slot's MMAs done
  uint64_t* dfull = aempty + G::kASlots;       // accumulator set holds a finished unit
  uint64_t* dempty = dfull + 2;                // accumulator set read back
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dempty + 2);
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int u0 = gt_first_unit(cta, p.U, p.ncta);
  const int n_units = gt_first_unit(cta + 1, p.U, p.ncta) - u0;
  const int Gn = p.s.G;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGtStages; ++s) {
      tc_mbar_init(&full[s], 1);
      tc_mbar_init(&empty[s], kGtProdWarps + 4 + 1);
    }
    for (int a = 0; a < G::kASlots; ++a) {
      tc_mbar_init(&afull[a], kGtProdWarps);
      tc_mbar_init(&aempty[a], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc_mbar_init(&dfull[b], 1);
      tc_mbar_init(&dempty[b], 4 * 32);
    }
    s_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(tc_smem(tmem_slot)),
                 "r"(kGtTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Activations (and everything else) only after the previous grid.
  gt_grid_wait();
  gt_allow_dependents();
  bool ok = true;

  if (warp == 0) {
    // ---- TMA producer ----
    if (lane == 0) {
      for (int i = 0; i < n_units; ++i) {
        const int u = u0 + i, t = u / Gn, g = u % Gn, s = i % kGtStages;
        if (i >= kGtStages && !tc_wait(&empty[s], unsigned(i / kGtStages - 1) & 1u)) { ok = false; break; }
        unsigned char* st = smem + s * G::kStage;
        tc_arrive_expect_tx(&full[s], unsigned(G::kTx));
        tc_tma_load_2d(st, &xmap, g * kGroup, 0, &full[s]);
        tc_tma_load_2d(st + NB * 128, &xmap, g * kGroup + 64, 0, &full[s]);
        tc_tma_load_2d(st + G::kXBytes, &bmap, g * kGroup, t * kGtOctets * K, &full[s]);
        tc_tma_load_2d(st + G::kXBytes + G::kBitsBytes, &amap, g * K * kOctet, t * kGtOctets, &full[s]);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      for (int i = 0; i < n_units && ok; ++i) {
        const int s = i % kGtStages, b = i & 1;
        if (!tc_wait(&full[s], unsigned(i / kGtStages) & 1u)) { ok = false; break; }
        if (i >= 2 && !tc_wait(&dempty[b], unsigned((i >> 1) - 1) & 1u)) { ok = false; break; }
        tc_fence_after();
        const uint32_t xs = tc_smem(smem + s * G::kStage);
        for (int k0 = 0; k0 < K && ok; k0 += G::kKGroup) {
          const int kn = K - k0 < G::kKGroup ? K - k0 : G::kKGroup;
          for (int kk = 0; kk < kn; ++kk) {
            const int j = i * K + k0 + kk;
            if (!tc_wait(&afull[j % G::kASlots], unsigned(j / G::kASlots) & 1u)) { ok = false; break; }
          }
          if (!ok) break;
          tc_fence_after();
          // the group's accumulator chains interleaved, chunk by chunk
#pragma unroll
          for (int cc = 0; cc < kGtChunks; ++cc) {
            const uint64_t bdesc = tc_desc_sw128(xs + (cc >> 2) * (NB * 128) + (cc & 3) * 32);
            for (int kk = 0; kk < kn; ++kk) {
              const int j = i * K + k0 + kk;
              tc_mma_ts(tmem + uint32_t(b * G::kDCols + (k0 + kk) * NB),
                        tmem + uint32_t(G::kACol0 + (j % G::kASlots) * 64 + 8 * cc), bdesc, p.idesc,
                        cc > 0 ? 1u : 0u);
            }
          }
          for (int kk = 0; kk < kn; ++kk) tc_commit(&aempty[(i * K + k0 + kk) % G::kASlots]);
        }
        if (!ok) break;
        tc_commit(&dfull[b]);
        tc_commit(&empty[s]);
      }
    }
  } else if (warp < kGtProdWarp0) {
    // ---- accumulator read-back: lane quarter (warp & 3), one row per thread ----
    const int quad = warp & 3;
    const int m = 32 * quad + lane, o = m >> 3, ir = m & 7;
    const uint32_t lane_addr = uint32_t(32 * quad) << 16;
    // vectors one accumulator set can hold: NB (bf16) or NB / 3 (fp32, three parts each)
    constexpr int kVec = XF32 ? NB / 3 : NB;
    float acc[kVec];
    int cur = -1;
    auto store = [&](int t) {
      const int row = t * kGtRows + m;
      if (row >= p.s.M) return;   // (a partial row is never read)
      float* dst = p.partial + size_t(cta + t) * p.batch * kGtRows + m;
#pragma unroll
      for (int n = 0; n < kVec; ++n)
        if (n < p.batch) dst[size_t(n) * kGtRows] = acc[n];
    };
    for (int i = 0; i < n_units; ++i) {
      const int u = u0 + i, t = u / Gn, s = i % kGtStages, b = i & 1;
      if (t != cur) {
        if (cur >= 0) store(cur);
        cur = t;
#pragma unroll
        for (int n = 0; n < kVec; ++n) acc[n] = 0.f;
      }
      if (!gt_wait_warp(&dfull[b], unsigned(i >> 1) & 1u)) { ok = false; break; }
      tc_fence_after();
      const uint16_t* al = reinterpret_cast<const uint16_t*>(smem + s * G::kStage + G::kXBytes + G::kBitsBytes);
      auto apply = [&](int k, const uint32_t* v) {
        const float a = __half2float(__ushort_as_half(al[(o * K + k) * kOctet + ir]));
#pragma unroll
        for (int n = 0; n < kVec; ++n) {
          if (n < p.batch) {
            const float dsum = XF32 ? __fadd_rn(__fadd_rn(__uint_as_float(v[3 * n]), __uint_as_float(v[3 * n + 1])),
                                                __uint_as_float(v[3 * n + 2]))
                                    : __uint_as_float(v[n]);
            acc[n] = __fmaf_rn(a, dsum, acc[n]);
          }
        }
      };
      if constexpr (NB == 16 && K <= 3) {
        // all K accumulators of the unit in flight at once, one wait
        uint32_t v[K][16];
#pragma unroll
        for (int k = 0; k < K; ++k) gt_tmem_ld16(tmem + lane_addr + uint32_t(b * G::kDCols + k * NB), v[k]);
        asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
        for (int k = 0; k < K; ++k) apply(k, v[k]);
      } else {
#pragma unroll 1
        for (int k = 0; k < K; ++k) {
          uint32_t v[NB];
#pragma unroll
          for (int h = 0; h < NB / 16; ++h)
            gt_tmem_ld16(tmem + lane_addr + uint32_t(b * G::kDCols + k * NB + 16 * h), v + 16 * h);
          asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
          apply(k, v);
        }
      }
      tc_fence_before();
      tc_arrive(&dempty[b]);
      __syncwarp();
      if (lane == 0) tc_arrive(&empty[s]);
    }
    if (ok && cur >= 0) store(cur);
  } else {
    // ---- sign tiles: lane quarter (warp & 3), chunks 2pj and 2pj + 1 ----
    const int quad = warp & 3, pj = (warp - kGtProdWarp0) >> 2;
    const int m = 32 * quad + lane, o = m >> 3, ir = m & 7;
    const uint32_t lane_addr = uint32_t(32 * quad) << 16;
    for (int i = 0; i < n_units && ok; ++i) {
      const int s = i % kGtStages;
      if (!gt_wait_warp(&full[s], unsigned(i / kGtStages) & 1u)) { ok = false; break; }
      const unsigned char* bits = smem + s * G::kStage + G::kXBytes;
      for (int k0 = 0; k0 < K && ok; k0 += G::kKGroup) {
        const int kn = K - k0 < G::kKGroup ? K - k0 : G::kKGroup;
        for (int kk = 0; kk < kn; ++kk) {
          const int j = i * K + k0 + kk;
          if (j >= G::kASlots && !gt_wait_warp(&aempty[j % G::kASlots], unsigned(j / G::kASlots - 1) & 1u)) {
            ok = false;
            break;
          }
        }
        if (!ok) break;
        tc_fence_after();
        for (int kk = 0; kk < kn; ++kk) {
          const int k = k0 + kk, a = (i * K + k) % G::kASlots;
          // line (octet, kernel) of the swizzled bits: 16-byte chunk q sits at q ^ (line & 7)
          const int line = o * K + k;
          const unsigned char* lp = bits + line * 128 + 2 * ir;
          const uint32_t h0 = *reinterpret_cast<const uint16_t*>(lp + (((2 * pj) ^ (line & 7)) << 4));
          const uint32_t h1 = *reinterpret_cast<const uint16_t*>(lp + (((2 * pj + 1) ^ (line & 7)) << 4));
          uint32_t w[16];
          gt_sign_unit(h0, w);
          gt_sign_unit(h1, w + 8);
          gt_tmem_st16(tmem + lane_addr + uint32_t(G::kACol0 + a * 64 + 16 * pj), w);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
          for (int kk = 0; kk < kn; ++kk) tc_arrive(&afull[(i * K + k0 + kk) % G::kASlots]);
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) tc_arrive(&empty[s]);
    }
  }

  if (!ok) atomicOr(&s_fail, 1);
  tc_fence_before();
  __syncthreads();
  if (s_fail != 0 && threadIdx.x == 0) {
    // Record the failure and let every copy and MMA this CTA issued complete
    // (bounded) before its shared and tensor memory are released.
    atomicOr(&g_gemv_tc_error, 1u);
    for (int s = 0; s < kGtStages; ++s) {
      (void)tc_wait(&full[s], 0u, kTcDrainNs);
      (void)tc_wait(&full[s], 1u, kTcDrainNs);
    }
    for (int a = 0; a < G::kASlots; ++a) {
      (void)tc_wait(&aempty[a], 0u, kTcDrainNs);
      (void)tc_wait(&aempty[a], 1u, kTcDrainNs);
    }
    for (int b = 0; b < 2; ++b) {
      (void)tc_wait(&dfull[b], 0u, kTcDrainNs);
      (void)tc_wait(&dfull[b], 1u, kTcDrainNs);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kGtTmemCols));
  }
}

// y[n][r] = sum, in CTA order, of the partials of the CTAs that cover row
// tile r / 128.
__global__ void __launch_bounds__(256) gemv_tc_combine_kernel(const float* __restrict__ partial, float* __restrict__ y,
                                                              int M, int batch, int T, int Gn, int U, int ncta) {
  gt_allow_dependents();
  gt_grid_wait();
  const long long idx = (long long)blockIdx.x * 256 + threadIdx.x;
  if (idx >= (long long)T * batch * kGtRows) return;
  const int m = int(idx % kGtRows);
  const int n = int((idx / kGtRows) % batch);
  const int t = int(idx / ((long long)kGtRows * batch));
  const int row = t * kGtRows + m;
  if (row >= M) return;
  const int c_lo = gt_cta_of(t * Gn, U, ncta), c_hi = gt_cta_of((t + 1) * Gn - 1, U, ncta);
  float sum = 0.f;
  for (int c = c_lo; c <= c_hi; ++c) sum += partial[(size_t(c + t) * batch + n) * kGtRows + m];
  y[size_t(n) * M + row] = sum;
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

static size_t round256(size_t n) { return (n + 255) / 256 * 256; }

static size_t gt_partial_bytes(const Shape& s, int batch) {
  const size_t T = size_t((s.M + kGtRows - 1) / kGtRows);
  return round256((size_t(kGtMaxCtas) + T - 1) * size_t(batch) * kGtRows * sizeof(float));
}

// Partials, then (fp32 input) the bf16 parts of X.
size_t gemv_tc_workspace_bytes(const Shape& s, int batch) {
  return gt_partial_bytes(s, batch) + round256(size_t(3) * batch * s.N * sizeof(uint16_t));
}

unsigned gemv_tc_error_flags() {
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_gemv_tc_error, sizeof(v)) != cudaSuccess) return ~0u;
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(g_gemv_tc_error, &zero, sizeof(zero)) != cudaSuccess) return ~0u;
  return v;
}

static cudaLaunchAttribute pdl_attr() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

template <int K, int NB, bool XF32>
static cudaError_t launch_gt(const CUtensorMap& xm, const CUtensorMap& bm, const CUtensorMap& am,
                             const GtParams& p, cudaStream_t stream) {
  using G = GtGeom<K, NB>;
  auto fn = gemv_tc_kernel<K, NB, XF32>;
  static bool attr_set = false;   // set once, outside any stream capture
  if (!attr_set) {
    const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, G::kSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchAttribute attr[1] = {pdl_attr()};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.ncta);
  cfg.blockDim = dim3(kGtThreads);
  cfg.dynamicSmemBytes = G::kSmem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, xm, bm, am, p);
}

template <bool XF32>
static cudaError_t launch_gt_nb(int K, int NB, const CUtensorMap& xm, const CUtensorMap& bm, const CUtensorMap& am,
                                const GtParams& p, cudaStream_t stream) {
#define MBOK_GT_CASE(KK, NN) \
  if (K == KK && NB == NN) return launch_gt<KK, NN, XF32>(xm, bm, am, p, stream);
  if constexpr (!XF32) {
    MBOK_GT_CASE(1, 16) MBOK_GT_CASE(2, 16) MBOK_GT_CASE(3, 16) MBOK_GT_CASE(4, 16)
  } else {
    MBOK_GT_CASE(1, 16) MBOK_GT_CASE(2, 16) MBOK_GT_CASE(3, 16) MBOK_GT_CASE(4, 16)
    MBOK_GT_CASE(1, 32) MBOK_GT_CASE(2, 32) MBOK_GT_CASE(3, 32) MBOK_GT_CASE(4, 32)
    MBOK_GT_CASE(1, 48) MBOK_GT_CASE(2, 48) MBOK_GT_CASE(3, 48) MBOK_GT_CASE(4, 48)
  }
#undef MBOK_GT_CASE
  return cudaErrorInvalidValue;
}

// Y [batch][M] fp32 = W X for X [batch][N] (bf16, or fp32 when x_f32), batch
// 1..16; workspace as sized by gemv_tc_workspace_bytes.  Returns
// cudaErrorNotSupported when the tensor-map encoder is unavailable.
cudaError_t launch_gemv_tc(const uint8_t* packed, const uint16_t* alpha, const Shape& s, const void* x, bool x_f32,
                           int batch, float* y, void* workspace, cudaStream_t stream) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  const int rows_x = x_f32 ? 3 * batch : batch;
  const int NB = (rows_x + 15) / 16 * 16;
  const int T = (s.M + kGtRows - 1) / kGtRows;
  const int U = T * s.G;
  int ncta = device_sm_count();
  if (ncta > kGtMaxCtas) ncta = kGtMaxCtas;
  if (ncta > U) ncta = U;

  float* partial = static_cast<float*>(workspace);
  uint16_t* xs = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) + gt_partial_bytes(s, batch));
  cudaLaunchAttribute attr[1] = {pdl_attr()};
  const void* xsrc = x;
  if (x_f32) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned((size_t(batch) * s.N + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_tc_split_kernel, static_cast<const float*>(x), xs, s.N, batch);
    if (e != cudaSuccess) return e;
    xsrc = xs;
  }

  const cuuint32_t ones[2] = {1, 1};
  CUtensorMap xm, bm, am;
  {  // activations: bf16 [rows_x][N], box 64 columns x NB rows (rows past rows_x read as 0)
    const cuuint64_t dims[2] = {cuuint64_t(s.N), cuuint64_t(rows_x)};
    const cuuint64_t strides[1] = {cuuint64_t(s.N) * 2};
    const cuuint32_t box[2] = {64u, cuuint32_t(NB)};
    if (enc(&xm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(xsrc), dims, strides, box, ones,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {  // bits: bytes [O*K][N] (one row = one (octet, kernel)), box one group (128 bytes) x 16K rows
    const cuuint64_t dims[2] = {cuuint64_t(s.N), cuuint64_t(s.O) * s.K};
    const cuuint64_t strides[1] = {cuuint64_t(s.N)};
    const cuuint32_t box[2] = {cuuint32_t(kGroup), cuuint32_t(kGtOctets * s.K)};
    if (enc(&bm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed), dims, strides, box, ones,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {  // scales: fp16 [O][G*K*8], box K*8 values x 16 octets
    const cuuint64_t dims[2] = {cuuint64_t(s.G) * s.K * kOctet, cuuint64_t(s.O)};
    const cuuint64_t strides[1] = {cuuint64_t(s.G) * s.K * kOctet * 2};
    const cuuint32_t box[2] = {cuuint32_t(s.K * kOctet), cuuint32_t(kGtOctets)};
    if (enc(&am, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(alpha), dims, strides, box, ones,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }

  GtParams p;
  p.partial = partial;
  p.s = s;
  p.batch = batch;
  p.T = T;
  p.U = U;
  p.ncta = ncta;
  p.idesc = tc_idesc_bf16(kGtRows, NB);
  cudaError_t e = x_f32 ? launch_gt_nb<true>(s.K, NB, xm, bm, am, p, stream)
                        : launch_gt_nb<false>(s.K, NB, xm, bm, am, p, stream);
  if (e != cudaSuccess) return e;

  cudaLaunchConfig_t c2 = {};
  c2.gridDim = dim3(unsigned((size_t(T) * batch * kGtRows + 255) / 256));
  c2.blockDim = dim3(256);
  c2.stream = stream;
  c2.attrs = attr;
  c2.numAttrs = 1;
  e = cudaLaunchKernelEx(&c2, gemv_tc_combine_kernel, static_cast<const float*>(partial), y, s.M, batch, T, s.G, U,
                         ncta);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mbok
