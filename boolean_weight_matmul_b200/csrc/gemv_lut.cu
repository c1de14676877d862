// Decode GEMV y = W x for one activation vector (batch 1), sm_100a.
//
// The method evaluates W x as K Boolean matrix-vector products scaled by the
// group scales (Paper-Notes page, 方法详解 / 关键设计).  With b in {-1,+1},
//     y_r = sum_g sum_k alpha_{k,r,g} * s_{k,r,g},   s_{k,r,g} = sum_{j in g} b_{k,r,j} x_j.
// The prior-art operator on the FluxBin page (算子创新: LUT-based GEMV that
// streams uint32 weight words, extracts pattern indices with bit operations
// and fetches precomputed partial sums) motivates a lookup table; this kernel
// is laid out for the B200 shared-memory pipe and HBM instead:
//
//  * Each lane owns 16 consecutive columns of a 512-column slab and keeps two
//    256-entry fp32 tables in ITS OWN shared-memory bank: T_lo[e] (columns
//    0..7 of its unit) and T_hi[e] (columns 8..15), T[e] = sum_i (e_i ? x : -x).
//    Entry e of lane L sits at byte e*256 + 128*h + 4L, so every lookup of a
//    warp touches 32 distinct banks: one wavefront per 8 weight bits.  The
//    address of a lookup is one byte permute: (byte << 8) | 4L.
//  * Each warp streams its own row octets (octet o_begin + warp + 16t) from
//    HBM into a private 4-deep shared-memory ring with 16-byte cp.async
//    copies: per (octet, kernel) one copy per lane (512 contiguous bytes per
//    warp), plus the octet's 4 groups x K scale vectors.  The main loop has
//    no block-wide barrier.  Launches use programmatic dependent launch:
//    before waiting on the previous grid, a launch of up to 16 MB of packed
//    bits prefetches its first octets into L2 and (unless turned off,
//    because a kernel that lets this grid start early might write the
//    weights) starts the octets' shared-memory copies; every launch
//    prefetches its slice of x into L2; the read of x and every write happen
//    after the wait.  A chain of small layers thus overlaps one launch's tail
//    with the next launch's weights.
//  * Per (row pair, kernel) a lane does four lookups, one packed fp32x2 add
//    and one packed fp32x2 FMA with the two rows' fp16 group scales.
//  * The 32 lanes' partial sums of an octet's 8 rows are combined by a
//    transposing shuffle butterfly.
//  * A CTA covers one slab and a contiguous range of row octets and stores
//    its per-row partial sums; a second small grid (gemv_combine_kernel) adds
//    the slabs' partials in slab order, deterministically.  Measured faster
//    than combining inside this grid (a release/acquire counter and a reload
//    by the last CTA of a row range) and than a thread-block-cluster
//    reduction through distributed shared memory.
// Tables are built exactly sign-symmetric (T[~e] == -T[e]), so flipping every
// bit of a kernel and negating its scales reproduces y bit for bit.
#include "lut_common.cuh"

#ifdef MBOK_PHASE_STAMPS
#include <atomic>
#endif

namespace mbok {

// Phase stamps, compiled only into the profiling build (MBOK_PHASE_STAMPS):
// per CTA, globaltimer readings at the phase boundaries of a decode layer --
// main kernel: start, dependency wait returned, tables built, last warp out
// of the streaming loop, last warp's copies drained; combine kernel: start,
// dependency wait returned, end -- in one of kStampSlots slots per launch.
// They only record time: the kernels do the same work as without them.
#ifdef MBOK_PHASE_STAMPS
constexpr int kStampSlots = 64, kStampCtas = 1024;
__device__ unsigned long long g_main_stamps[kStampSlots][kStampCtas][5];
__device__ unsigned long long g_combine_stamps[kStampSlots][kStampCtas][3];
__device__ __forceinline__ unsigned long long stamp_now() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
#define MBOK_MAIN_STAMP(slot, pt) \
  do { if (blockIdx.x < kStampCtas) g_main_stamps[(slot) % kStampSlots][blockIdx.x][pt] = stamp_now(); } while (0)
#define MBOK_MAIN_STAMP_LAST(slot, pt) \
  do { if (blockIdx.x < kStampCtas) atomicMax(&g_main_stamps[(slot) % kStampSlots][blockIdx.x][pt], stamp_now()); } while (0)
#define MBOK_COMBINE_STAMP(slot, pt) \
  do { if (blockIdx.x < kStampCtas) g_combine_stamps[(slot) % kStampSlots][blockIdx.x][pt] = stamp_now(); } while (0)
#else
#define MBOK_MAIN_STAMP(slot, pt) ((void)0)
#define MBOK_MAIN_STAMP_LAST(slot, pt) ((void)0)
#define MBOK_COMBINE_STAMP(slot, pt) ((void)0)
#endif

constexpr int kSlabCols = 512;                  // columns per slab (32 lanes x 16)
constexpr int kUnitsPerSlab = kSlabCols / kUnit;
constexpr int kGroupsPerSlab = kSlabCols / kGroup;
constexpr int kGemvThreads = 512;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kLutBytes = 256 * 256;            // 256 entries x (32 lanes x 2 tables x 4 B)
constexpr int kDepth = 4;                       // octets in flight per warp (4 measured 1-4 % faster than 3)
constexpr int kPrefetchOctets = 16;             // L2 prefetch ahead of the dependency wait, per warp (launches <= 16 MB)

template <int K>
struct StageGeom {
  static constexpr int kBits = K * kUnitsPerSlab * 16;        // [k][lane][16 B]
  static constexpr int kAlpha = kGroupsPerSlab * K * 16;      // [group][k][8 x fp16]
  static constexpr int kBytes = kBits + kAlpha;               // one octet of one warp
  static constexpr int kRing = kGemvWarps * kDepth * kBytes;
  static constexpr int kSmem = kLutBytes + kRing;
};

struct GemvParams {
  const uint8_t* packed;
  const uint16_t* alpha;   // grouped scales (grouped form)
  const uint16_t* s_in;    // rank-1 form: fp16 [K][N]
  const uint16_t* s_out;   // rank-1 form: fp16 [K][M]
  const void* x;
  float* y;
  float* partial;      // [nslab * nk][O*8]
  Shape s;
  int nslab, cps;
  int nk;              // kernels handled by separate CTAs: 1 (grouped form) or K (rank-1 form)
  int weights_static;  // bits and scales may be read before the grid dependency wait
  int stamp_slot;      // profiling build only: this launch's phase-stamp slot
  int prefetch_octets; // octets per warp prefetched into L2 before the dependency wait
  int sv_scales_staged; // rank-1 form: each octet's 8 output scales are copied with its bits
                        // (M % 8 == 0 and s_out 16-byte aligned), not loaded after its lookups
};

// ---------------------------------------------------------------------------
// Lookup tables
// ---------------------------------------------------------------------------

// sum_{i<4} (n_i ? v_i : -v_i), associated as ((v0 + v1) + v2) + v3 so that
// complementing n negates the result exactly.
__device__ __forceinline__ float signed_sum4(const float v[4], uint32_t n) {
  float t = ((n & 1) ? v[0] : -v[0]) + ((n & 2) ? v[1] : -v[1]);
  t = t + ((n & 4) ? v[2] : -v[2]);
  return t + ((n & 8) ? v[3] : -v[3]);
}

// The 8 activations x[col0 .. col0+7] as fp32 (0 when !ok).
template <bool XF32>
__device__ __forceinline__ void load_x8(const void* x, int col0, bool ok, float v[8]) {
  if (!ok) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
    return;
  }
  if (XF32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + col0);
    const float4 t0 = p[0], t1 = p[1];
    v[0] = t0.x; v[1] = t0.y; v[2] = t0.z; v[3] = t0.w;
    v[4] = t1.x; v[5] = t1.y; v[6] = t1.z; v[7] = t1.w;
  } else {
    const uint4 t = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + col0);
    const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] = bf16_bits_to_float(w[e] & 0xFFFFu);
      v[2 * e + 1] = bf16_bits_to_float(w[e] >> 16);
    }
  }
}

// Warp w fills entries [32*(w&7), 32*(w&7)+32) of table h = w>>3 for all 32
// lanes from that table's 8 activations c[]: T[e] = A[e & 15] + B[e >> 4],
// A/B the signed sums of the table's low and high four columns.
__device__ __forceinline__ void build_tables(unsigned char* tab, const float c[8], int warp, int lane) {
  static_assert(kGemvWarps == 16, "the table build assigns 16 warps to (table, 32-entry block)");
  const int h = warp >> 3, blk = warp & 7;
  float A[16];
#pragma unroll
  for (int n = 0; n < 16; ++n) A[n] = signed_sum4(c, uint32_t(n));
  unsigned char* dst = tab + 128 * h + 4 * lane;
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const float B = signed_sum4(c + 4, uint32_t(2 * blk + m));
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      const int e = 32 * blk + 16 * m + n;
      *reinterpret_cast<float*>(dst + size_t(e) * 256) = A[n] + B;
    }
  }
}

// One octet (8 rows x this lane's 16 columns) of K kernels from a stage.
template <int K>
__device__ __forceinline__ void octet_dot(const unsigned char* tab, uint32_t lane4,
                                          const uint4* bits, const uint4* alpha, float2 acc[4]) {
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const uint4 wv = bits[k * kUnitsPerSlab];
    const uint4 av = alpha[k];
    const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
    const uint32_t a[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // word i holds row 2i (bytes 0,1) and row 2i+1 (bytes 2,3); byte b of the
      // word indexes the table for its 8 columns at offset (byte << 8) | 4L.
      const float t0 = lut(tab, __byte_perm(w[i], lane4, 0x5504));         // row 2i,   cols 0..7
      const float t1 = lut(tab + 128, __byte_perm(w[i], lane4, 0x5514));   // row 2i,   cols 8..15
      const float t2 = lut(tab, __byte_perm(w[i], lane4, 0x5524));         // row 2i+1, cols 0..7
      const float t3 = lut(tab + 128, __byte_perm(w[i], lane4, 0x5534));   // row 2i+1, cols 8..15
      const float2 s = __fadd2_rn(make_float2(t0, t2), make_float2(t1, t3));
      acc[i] = __ffma2_rn(half2_bits_to_float2(a[i]), s, acc[i]);
    }
  }
}

// One octet of K unscaled kernels (rank-1 form: the row scale comes later).
template <int K>
__device__ __forceinline__ void octet_sum(const unsigned char* tab, uint32_t lane4, const uint4* bits, float2 acc[4]) {
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const uint4 wv = bits[k * kUnitsPerSlab];
    const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float t0 = lut(tab, __byte_perm(w[i], lane4, 0x5504));
      const float t1 = lut(tab + 128, __byte_perm(w[i], lane4, 0x5514));
      const float t2 = lut(tab, __byte_perm(w[i], lane4, 0x5524));
      const float t3 = lut(tab + 128, __byte_perm(w[i], lane4, 0x5534));
      acc[i] = __fadd2_rn(acc[i], __fadd2_rn(make_float2(t0, t2), make_float2(t1, t3)));
    }
  }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------

// Copy octet o (this warp's K x 512 columns of bits of kernels kb..kb+K-1
// and, in the grouped form, its 4 groups x K scale vectors) into stage `st`;
// one commit group per octet.
template <int K, bool SV>
__device__ __forceinline__ void issue_octet(const GemvParams& p, int slab, int units, int groups, int o, int kb,
                                            unsigned char* st, int lane) {
  using G = StageGeom<K>;
  if (lane < units) {
#pragma unroll
    for (int k = 0; k < K; ++k)
      cp_async16(st + k * kUnitsPerSlab * 16 + lane * 16,
                 p.packed + unit_offset(p.s, o, kb + k, slab * kUnitsPerSlab + lane));
  }
  if (!SV && lane < groups * K)
    cp_async16(st + G::kBits + lane * 16, p.alpha + alpha_offset(p.s, o, slab * kGroupsPerSlab, 0) + lane * 8);
  // rank-1 form: rows 8o .. 8o+7 of s_out^kb into the stage's scale slot
  if (SV && p.sv_scales_staged && lane == 0)
    cp_async16(st + G::kBits, p.s_out + size_t(kb) * p.s.M + size_t(o) * kOctet);
  cp_async_commit();
}

template <int K, bool SV>
__device__ __forceinline__ void prefetch_octet(const GemvParams& p, int slab, int units, int groups, int o, int kb,
                                               int lane) {
  // 128-byte lines: units*16 bytes per kernel, groups*K*16 bytes of scales
  const int lines = (units + 7) / 8;
  if (lane < lines * K) {
    const int k = lane / lines, l = lane % lines;
    prefetch_l2(p.packed + unit_offset(p.s, o, kb + k, slab * kUnitsPerSlab) + 128 * l);
  } else if (!SV && lane < lines * K + (groups * K * 16 + 127) / 128) {
    const int l = lane - lines * K;
    prefetch_l2(reinterpret_cast<const uint8_t*>(p.alpha + alpha_offset(p.s, o, slab * kGroupsPerSlab, 0)) + 128 * l);
  }
}

// SV = false: the grouped form, K kernels per CTA, scales per (kernel, row,
// 128-column group) applied per lookup pair.  SV = true: the rank-1 form,
// one kernel kk per CTA (K = 1 here; p.nk CTAs per slab), the tables built
// from s_in^kk (.) x and each row's total scaled by s_out^kk[row].
// The body of one CTA; `bid` is its index within the launch (or within its
// matrix, for gemv_lut8_multi_kernel).
template <int K, bool XF32, bool SV>
__device__ __forceinline__ void gemv_lut8_body(const GemvParams& p, int bid) {
  using G = StageGeom<K>;
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* tab = smem;
  if (threadIdx.x == 0) MBOK_MAIN_STAMP(p.stamp_slot, 0);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nvs = SV ? p.nslab * p.nk : p.nslab;   // (slab, kernel) CTAs per row range
  const int vs = bid % nvs, c = bid / nvs;
  const int slab = SV ? vs % p.nslab : vs;
  const int kk = SV ? vs / p.nslab : 0;
  const int o_begin = int((long long)c * p.s.O / p.cps);
  const int o_end = int((long long)(c + 1) * p.s.O / p.cps);
  const int units = min(kUnitsPerSlab, p.s.Q - slab * kUnitsPerSlab);
  const int groups = units / kUnitsPerGroup;
  const int q = slab * kUnitsPerSlab + lane;
  const bool lane_ok = lane < units;
  const uint32_t lane4 = 4u * lane;
  const int Mpad = p.s.O * kOctet;
  unsigned char* ring = smem + kLutBytes + warp * kDepth * G::kBytes;
  // this warp's octets: o_begin + warp + 16t, t = 0 .. n_mine-1
  const int first = o_begin + warp;
  const int n_mine = first < o_end ? (o_end - first + kGemvWarps - 1) / kGemvWarps : 0;

  // Before the dependency wait (launches of up to 16 MB): L2 prefetches of
  // this warp's first octets, and unless the caller turned it off
  // (mbok_gemv_set_static_weights) the first octets' copies into shared
  // memory as well -- weights are not written by kernels that let this grid
  // start early.
  for (int t = 0; t < p.prefetch_octets && t < n_mine; ++t)
    prefetch_octet<K, SV>(p, slab, units, groups, first + t * kGemvWarps, kk, lane);
  if (p.weights_static) {
#pragma unroll
    for (int t = 0; t < kDepth; ++t) {
      if (t < n_mine) issue_octet<K, SV>(p, slab, units, groups, first + t * kGemvWarps, kk, ring + t * G::kBytes, lane);
      else cp_async_commit();   // keep one group per slot
    }
  }
  // The slab's activations (and input scales) into L2 as well.  This is safe
  // even when the previous grid writes x: L2 is the device's point of
  // coherence, so a line fetched early is updated in place by that write, and
  // the L1-cached read of x below still comes after the wait.
  const int col0 = q * kUnit + 8 * (warp >> 3);
  if (warp == 0 && lane_ok) {
    prefetch_l2(static_cast<const unsigned char*>(p.x) + size_t(q) * kUnit * (XF32 ? 4 : 2));
    if (SV) prefetch_l2(p.s_in + size_t(kk) * p.s.N + size_t(q) * kUnit);
  }
  // rank-1 form: the kernel's input scales for this lane's 8 columns -- a
  // weight, so read before the wait when weights are static
  uint4 sv = make_uint4(0u, 0u, 0u, 0u);
  if (SV && lane_ok && p.weights_static) sv = *reinterpret_cast<const uint4*>(p.s_in + size_t(kk) * p.s.N + col0);
  allow_dependents();
  // x, the workspace and (unless static) the weights may be written by the
  // previous grid: wait for it.
  grid_dependency_wait();
  if (threadIdx.x == 0) MBOK_MAIN_STAMP(p.stamp_slot, 1);

  // x first: its load must not queue behind this warp's weight copies.
  float xv[8];
  load_x8<XF32>(p.x, col0, lane_ok, xv);
  if (SV && lane_ok) {
    // rank-1 form: the kernel's input scale, applied before the tables
    if (!p.weights_static) sv = *reinterpret_cast<const uint4*>(p.s_in + size_t(kk) * p.s.N + col0);
    const uint32_t w[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = half2_bits_to_float2(w[e]);
      xv[2 * e] *= f.x;
      xv[2 * e + 1] *= f.y;
    }
  }
  if (!p.weights_static) {
#pragma unroll
    for (int t = 0; t < kDepth; ++t) {
      if (t < n_mine) issue_octet<K, SV>(p, slab, units, groups, first + t * kGemvWarps, kk, ring + t * G::kBytes, lane);
      else cp_async_commit();   // keep one group per slot
    }
  }
  build_tables(tab, xv, warp, lane);
  __syncthreads();
  if (threadIdx.x == 0) MBOK_MAIN_STAMP(p.stamp_slot, 2);

  for (int t = 0; t < n_mine; ++t) {
    unsigned char* st = ring + (t % kDepth) * G::kBytes;
    cp_async_wait<kDepth - 1>();   // octet t has landed (this lane's copies)
    __syncwarp();                  // ... and every lane's copies
    float2 acc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
    if (lane_ok) {
      const uint4* bits = reinterpret_cast<const uint4*>(st) + lane;
      if (SV) {
        octet_sum<K>(tab, lane4, bits, acc);
      } else {
        const uint4* al = reinterpret_cast<const uint4*>(st + G::kBits) + (lane / kUnitsPerGroup) * K;
        octet_dot<K>(tab, lane4, bits, al, acc);
      }
    }
    // rank-1 form: this lane's row scale, read before the slot is refilled
    float so = 0.f;
    if (SV && p.sv_scales_staged)
      so = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(st + G::kBits)[(lane >> 2) & 7]));
    __syncwarp();                  // all lanes are done reading the slot
    if (t + kDepth < n_mine)
      issue_octet<K, SV>(p, slab, units, groups, first + (t + kDepth) * kGemvWarps, kk, st, lane);
    else
      cp_async_commit();
    float total = octet_reduce(acc, lane);
    const int o = first + t * kGemvWarps;
    const int row = o * kOctet + ((lane >> 2) & 7);
    if ((lane & 3) == 0) {
      if (SV) {
        // A scale loaded here would hold the warp for a memory round trip
        // per octet: the rank-1 loop took 5.25 us on q_proj (K = 3, 4096 x
        // 4096) against 1.70 us for the grouped form's.
        if (!p.sv_scales_staged && row < p.s.M)
          so = __half2float(__ushort_as_half(p.s_out[size_t(kk) * p.s.M + row]));
        total = row < p.s.M ? total * so : 0.f;
      }
      if (nvs == 1) {
        if (row < p.s.M) p.y[row] = total;
      } else {
        __stcg(p.partial + size_t(vs) * Mpad + row, total);
      }
    }
  }
  if (lane == 0) MBOK_MAIN_STAMP_LAST(p.stamp_slot, 3);
  cp_async_wait<0>();
  if (lane == 0) MBOK_MAIN_STAMP_LAST(p.stamp_slot, 4);
  // With several CTAs per row range the partials are combined by
  // gemv_combine_kernel, launched right behind this grid.
}

template <int K, bool XF32, bool SV>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_lut8_kernel(GemvParams p) {
  gemv_lut8_body<K, XF32, SV>(p, int(blockIdx.x));
}

// Several matrices that share x (q/k/v, gate/up), each with its own K and
// row count, in one launch: CTAs [cta0[s], cta0[s+1]) run matrix s with that
// matrix's parameters (its own packed bits, scales, shape, output rows and
// partial sums); K is a runtime switch per CTA.
constexpr int kMaxSegments = 8;

struct GemvMultiParams {
  GemvParams seg[kMaxSegments];
  int cta0[kMaxSegments + 1];
  int nseg;
};

template <bool XF32>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_lut8_multi_kernel(const __grid_constant__ GemvMultiParams mp) {
  int sg = 0;
  while (sg + 1 < mp.nseg && int(blockIdx.x) >= mp.cta0[sg + 1]) ++sg;
  const GemvParams& p = mp.seg[sg];
  const int bid = int(blockIdx.x) - mp.cta0[sg];
  switch (p.s.K) {
    case 1: gemv_lut8_body<1, XF32, false>(p, bid); break;
    case 2: gemv_lut8_body<2, XF32, false>(p, bid); break;
    case 3: gemv_lut8_body<3, XF32, false>(p, bid); break;
    default: gemv_lut8_body<4, XF32, false>(p, bid); break;
  }
}

struct CombineMultiParams {
  const float* partial[kMaxSegments];   // matrix s: [nslab][O_s * 8]
  int row0[kMaxSegments + 1];           // first output row of matrix s; row0[nseg] = total rows
  int mpad[kMaxSegments];               // O_s * 8
  int nseg, nvs;
};

// y[R] for the concatenated outputs: the matrix s that row R falls in, then
// its slabs' partials in slab order (as gemv_combine_kernel).
__global__ void __launch_bounds__(256) gemv_combine_multi_kernel(const __grid_constant__ CombineMultiParams cm,
                                                                 float* __restrict__ y) {
  allow_dependents();
  grid_dependency_wait();
  const int R = blockIdx.x * blockDim.x + threadIdx.x;
  if (R >= cm.row0[cm.nseg]) return;
  int sg = 0;
  while (sg + 1 < cm.nseg && R >= cm.row0[sg + 1]) ++sg;
  const int r = R - cm.row0[sg];
  const float* part = cm.partial[sg] + r;
  const size_t stride = size_t(cm.mpad[sg]);
  const int nvs = cm.nvs;
  float sum = 0.f;
  // As gemv_combine_kernel, but with up to 8 slabs the plain loop: batching
  // those measured slower here (mixed-K LLaMA-13B sweep 454 -> 437 tokens/s);
  // 16 at once above 8 slabs took it 454 -> 472.
  if (nvs <= 8) {
    for (int t = 0; t < nvs; ++t) sum += __ldcg(part + size_t(t) * stride);
  } else {
    float v[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) v[t] = t < nvs ? __ldcg(part + size_t(t) * stride) : 0.f;
#pragma unroll
    for (int t = 0; t < 16; ++t)
      if (t < nvs) sum += v[t];
    for (int t = 16; t < nvs; ++t) sum += __ldcg(part + size_t(t) * stride);
  }
  y[R] = sum;
}

// y[r] = sum over the nvs partials of row r, in (kernel, slab) order.  A
// separate grid, so that no CTA of the main kernel waits on another: its
// dependency wait returns once every partial of the previous grid is written.
__global__ void __launch_bounds__(256) gemv_combine_kernel(const float* __restrict__ partial, float* __restrict__ y,
                                                           int M, int Mpad, int nvs, int stamp_slot) {
  if (threadIdx.x == 0) MBOK_COMBINE_STAMP(stamp_slot, 0);
  allow_dependents();
  grid_dependency_wait();
  if (threadIdx.x == 0) MBOK_COMBINE_STAMP(stamp_slot, 1);
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= M) return;
  // The first partials (8 with up to 8 slabs, else 16) are loaded before any
  // is added, so they cost one L2 round trip; the sum is the same slab-order
  // sum.  Measured (bench, same box): 8 wide, q_proj (8 slabs) 4.88 -> 4.68 us
  // per layer; 16 wide, 7B down (22 slabs) 8.06 -> 7.73 us and the fused
  // LLaMA-13B sweep (10 and 27 slabs) 455 -> 464 tokens/s, but 5.32 us on
  // q_proj.  The multi-matrix combine batches only above 8 slabs.
  float sum = 0.f;
  if (nvs <= 8) {
    float v[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) v[t] = t < nvs ? __ldcg(partial + size_t(t) * Mpad + r) : 0.f;
#pragma unroll
    for (int t = 0; t < 8; ++t)
      if (t < nvs) sum += v[t];
  } else {
    float v[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) v[t] = t < nvs ? __ldcg(partial + size_t(t) * Mpad + r) : 0.f;
#pragma unroll
    for (int t = 0; t < 16; ++t)
      if (t < nvs) sum += v[t];
    for (int t = 16; t < nvs; ++t) sum += __ldcg(partial + size_t(t) * Mpad + r);
  }
  y[r] = sum;
  if (threadIdx.x == 0) MBOK_COMBINE_STAMP(stamp_slot, 2);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

struct GemvPlan {
  int nslab, cps;
};

// nk = kernels given their own CTAs (1 in the grouped form, K in the rank-1
// form): nslab * nk CTAs per row range.
inline GemvPlan gemv_plan(const Shape& s, int sm_count, int nk) {
  GemvPlan pl;
  pl.nslab = (s.N + kSlabCols - 1) / kSlabCols;
  int cps = sm_count / (pl.nslab * nk);
  if (cps < 1) cps = 1;
  if (cps > s.O) cps = s.O;
  pl.cps = cps;
  return pl;
}

// Workspace: the per-CTA partial sums [nslab * nk][O * 8] (fp32), written and
// read by every call; nothing in it survives a call, so it needs no
// initialisation and any call may reuse it.
static size_t workspace_bytes_for(const Shape& s, int nk) {
  const size_t nvs = size_t((s.N + kSlabCols - 1) / kSlabCols) * nk;
  if (nvs <= 1) return 0;
  return nvs * size_t(s.O) * kOctet * sizeof(float);
}
size_t gemv_lut_workspace_bytes(const Shape& s) { return workspace_bytes_for(s, 1); }
size_t gemv_svid_workspace_bytes(const Shape& s) { return workspace_bytes_for(s, s.K); }

#ifdef MBOK_PHASE_STAMPS
static std::atomic<int> g_stamp_next{0};   // slot of the next single-matrix launch
#endif

template <int K, bool XF32, bool SV>
static cudaError_t launch_k(const GemvParams& p_in, int grid, cudaStream_t stream) {
  using G = StageGeom<K>;
  GemvParams p = p_in;
#ifdef MBOK_PHASE_STAMPS
  p.stamp_slot = g_stamp_next.fetch_add(1) % kStampSlots;
#else
  p.stamp_slot = 0;
#endif
  auto fn = gemv_lut8_kernel<K, XF32, SV>;
  static PerDeviceOnce attr_once;   // the attributes are per device context
  const cudaError_t ae = set_smem_attr_once(attr_once, reinterpret_cast<const void*>(fn), G::kSmem, true);
  if (ae != cudaSuccess) return ae;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = G::kSmem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, fn, p);
  if (e != cudaSuccess) return e;
  const int nvs = p.nslab * (SV ? p.nk : 1);
  if (nvs > 1) {
    cudaLaunchConfig_t c2 = {};
    c2.gridDim = dim3((p.s.M + 255) / 256);
    c2.blockDim = dim3(256);
    c2.stream = stream;
    c2.attrs = attr;
    c2.numAttrs = 1;
    e = cudaLaunchKernelEx(&c2, gemv_combine_kernel, static_cast<const float*>(p.partial), p.y, p.s.M,
                           p.s.O * kOctet, nvs, p.stamp_slot);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

// What a launch reads before the grid dependency wait.  Launches of up to
// 16 MB of packed bits prefetch each warp's first kPrefetchOctets octets into
// L2 and, with static weights, copy the first tiles into shared memory:
// measured in a chain of layers, that hides their DRAM latency behind the
// previous layer's tail (q_proj 4.82 vs 5.26 us/layer without the prefetch,
// 4.86 vs 5.32 us without the copies).  Larger launches read nothing ahead of
// the wait: there the early traffic competes with the previous layer's own
// streaming (7B gate 8.74 -> 8.25 us/layer; fused LLaMA-13B sweep 402 ->
// 413 tokens/s without the early copies and 413 -> 453 without the prefetch).
constexpr size_t kEarlyStageMaxBytes = size_t(16) << 20;
inline bool stage_early(bool weights_static, size_t packed_bytes) {
  return weights_static && packed_bytes <= kEarlyStageMaxBytes;
}
inline int prefetch_depth(size_t packed_bytes) { return packed_bytes <= kEarlyStageMaxBytes ? kPrefetchOctets : 0; }

static GemvParams make_params(const uint8_t* packed, const Shape& s, const void* x, float* y, void* workspace,
                              bool weights_static, int nk, int ctas_per_sm = 1) {
  const GemvPlan pl = gemv_plan(s, device_sm_count() * ctas_per_sm, nk);
  GemvParams p;
  p.packed = packed;
  p.alpha = nullptr;
  p.s_in = nullptr;
  p.s_out = nullptr;
  p.x = x;
  p.y = y;
  p.s = s;
  p.nslab = pl.nslab;
  p.cps = pl.cps;
  p.nk = nk;
  p.weights_static = stage_early(weights_static, size_t(s.O) * kOctet * s.K * (s.N / 8)) ? 1 : 0;
  p.stamp_slot = 0;
  p.prefetch_octets = prefetch_depth(size_t(s.O) * kOctet * s.K * (s.N / 8));
  p.sv_scales_staged = 0;
  p.partial = pl.nslab * nk > 1 ? static_cast<float*>(workspace) : nullptr;
  return p;
}

// y = W x for one vector; workspace as sized by gemv_lut_workspace_bytes.
cudaError_t launch_gemv_lut(const uint8_t* packed, const uint16_t* alpha, const Shape& s,
                            const void* x, bool x_f32, float* y, void* workspace,
                            cudaStream_t stream, bool weights_static) {
  GemvParams p = make_params(packed, s, x, y, workspace, weights_static, 1);
  p.alpha = alpha;
  const int grid = p.nslab * p.cps;
  switch (s.K * 2 + (x_f32 ? 1 : 0)) {
    case 2: return launch_k<1, false, false>(p, grid, stream);
    case 3: return launch_k<1, true, false>(p, grid, stream);
    case 4: return launch_k<2, false, false>(p, grid, stream);
    case 5: return launch_k<2, true, false>(p, grid, stream);
    case 6: return launch_k<3, false, false>(p, grid, stream);
    case 7: return launch_k<3, true, false>(p, grid, stream);
    case 8: return launch_k<4, false, false>(p, grid, stream);
    default: return launch_k<4, true, false>(p, grid, stream);
  }
}

// ---- several matrices sharing x in one launch ------------------------------

// Partial sums of every matrix, one region per matrix: [nslab][O_s * 8].
size_t gemv_multi_workspace_bytes(int nseg, const int* K, const int* M, int N) {
  const size_t nslab = size_t((N + kSlabCols - 1) / kSlabCols);
  if (nslab <= 1) return 0;
  size_t total = 0;
  for (int i = 0; i < nseg; ++i) total += nslab * size_t(make_shape(K[i], M[i], N).O) * kOctet * sizeof(float);
  return total;
}

// y[0 .. sum M) = the matrices' outputs one after another, for one vector.
// The row ranges per slab (cps) are shared out over the matrices by their
// packed bytes (M_s * K_s), so one launch fills the SMs about as a single
// matrix of the summed size would.
cudaError_t launch_gemv_lut_multi(int nseg, const uint8_t* const* packed, const uint16_t* const* alpha, const int* K,
                                  const int* M, int N, const void* x, bool x_f32, float* y, void* workspace,
                                  cudaStream_t stream, bool weights_static) {
  if (nseg < 1 || nseg > kMaxSegments) return cudaErrorInvalidValue;
  const int sm = device_sm_count();
  const int nslab = (N + kSlabCols - 1) / kSlabCols;
  double wsum = 0.0;
  for (int i = 0; i < nseg; ++i) wsum += double(M[i]) * K[i];
  const int budget = sm / nslab > nseg ? sm / nslab : nseg;   // row ranges per slab, all matrices together
  GemvMultiParams mp;
  CombineMultiParams cm;
  mp.nseg = cm.nseg = nseg;
  cm.nvs = nslab;
  int cta = 0, row = 0, max_k = 1;
  size_t poff = 0;
  size_t launch_bytes = 0;
  for (int i = 0; i < nseg; ++i) launch_bytes += size_t(make_shape(K[i], M[i], N).O) * kOctet * K[i] * (N / 8);
  const bool early = stage_early(weights_static, launch_bytes);
  for (int i = 0; i < nseg; ++i) {
    const Shape s = make_shape(K[i], M[i], N);
    GemvParams& p = mp.seg[i];
    p.packed = packed[i];
    p.alpha = alpha[i];
    p.s_in = nullptr;
    p.s_out = nullptr;
    p.x = x;
    p.y = y + row;
    p.s = s;
    p.nslab = nslab;
    int cps = int(double(budget) * double(M[i]) * K[i] / wsum);
    if (cps < 1) cps = 1;
    if (cps > s.O) cps = s.O;
    p.cps = cps;
    p.nk = 1;
    p.weights_static = early ? 1 : 0;
    p.stamp_slot = 0;
    p.prefetch_octets = prefetch_depth(launch_bytes);
    p.sv_scales_staged = 0;
    p.partial = nslab > 1 ? static_cast<float*>(workspace) + poff : nullptr;
    mp.cta0[i] = cta;
    cm.partial[i] = p.partial;
    cm.row0[i] = row;
    cm.mpad[i] = s.O * kOctet;
    cta += nslab * cps;
    row += M[i];
    if (nslab > 1) poff += size_t(nslab) * s.O * kOctet;
    if (K[i] > max_k) max_k = K[i];
  }
  mp.cta0[nseg] = cta;
  cm.row0[nseg] = row;

  auto fn = x_f32 ? gemv_lut8_multi_kernel<true> : gemv_lut8_multi_kernel<false>;
  static PerDeviceOnce attr_once[2];   // per variant; the attributes are per device context
  const cudaError_t ae = set_smem_attr_once(attr_once[x_f32 ? 1 : 0], reinterpret_cast<const void*>(fn),
                                            StageGeom<4>::kSmem, true);
  if (ae != cudaSuccess) return ae;
  const int smem = max_k == 1 ? StageGeom<1>::kSmem
                   : max_k == 2 ? StageGeom<2>::kSmem
                   : max_k == 3 ? StageGeom<3>::kSmem
                                : StageGeom<4>::kSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cta);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, fn, mp);
  if (e != cudaSuccess) return e;
  if (nslab > 1) {
    cudaLaunchConfig_t c2 = {};
    c2.gridDim = dim3((row + 255) / 256);
    c2.blockDim = dim3(256);
    c2.stream = stream;
    c2.attrs = attr;
    c2.numAttrs = 1;
    e = cudaLaunchKernelEx(&c2, gemv_combine_multi_kernel, cm, y);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

// CTAs of the rank-1 kernel that one SM holds at once (queried once per
// device).  Its one-kernel stages leave room for two 512-thread CTAs per SM,
// and its row ranges are sized for all of them.
template <bool XF32>
static int svid_ctas_per_sm() {
  const void* fn = reinterpret_cast<const void*>(gemv_lut8_kernel<1, XF32, true>);
  static PerDeviceOnce attr_once;   // the occupancy depends on the shared-memory attributes
  if (set_smem_attr_once(attr_once, fn, StageGeom<1>::kSmem, true) != cudaSuccess) return 1;
  static PerDeviceValue<int> cache;
  const int n = cache.get(current_device(), [fn]() -> int {
    int v = 0;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, fn, kGemvThreads, StageGeom<1>::kSmem) == cudaSuccess
               ? v
               : 0;
  });
  return n >= 1 ? n : 1;
}

// Rank-1 form: y = sum_k s_out^k (.) (B_k (s_in^k (.) x)) for one vector;
// workspace as sized by gemv_svid_workspace_bytes.
cudaError_t launch_gemv_svid(const uint8_t* packed, const uint16_t* s_in, const uint16_t* s_out, const Shape& s,
                             const void* x, bool x_f32, float* y, void* workspace, cudaStream_t stream,
                             bool weights_static) {
  const int per_sm = x_f32 ? svid_ctas_per_sm<true>() : svid_ctas_per_sm<false>();
  GemvParams p = make_params(packed, s, x, y, workspace, weights_static, s.K, per_sm);
  p.s_in = s_in;
  p.s_out = s_out;
  // each octet's scales are one aligned 16-byte copy when M % 8 == 0
  p.sv_scales_staged = (s.M % kOctet == 0 && (reinterpret_cast<uintptr_t>(s_out) & 15) == 0) ? 1 : 0;
  const int grid = p.nslab * p.nk * p.cps;
  return x_f32 ? launch_k<1, true, true>(p, grid, stream) : launch_k<1, false, true>(p, grid, stream);
}

}  // namespace mbok

#ifdef MBOK_PHASE_STAMPS
// Profiling build only (not part of the C ABI in mbok.h).
// Copies the stamp arrays out: main [64][1024][5], combine [64][1024][3]
// unsigned 64-bit nanoseconds; returns a cudaError_t code.
extern "C" int mbok_debug_phase_stamps(void* main_host, size_t main_bytes, void* combine_host,
                                       size_t combine_bytes) {
  cudaError_t e = cudaMemcpyFromSymbol(main_host, mbok::g_main_stamps, main_bytes);
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(combine_host, mbok::g_combine_stamps, combine_bytes);
  return int(e);
}

// Zeroes both arrays; with reset_slots != 0 the next launch takes slot 0.
extern "C" int mbok_debug_phase_reset(int reset_slots) {
  void* a = nullptr;
  void* b = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&a, mbok::g_main_stamps);
  if (e == cudaSuccess) e = cudaMemset(a, 0, sizeof(mbok::g_main_stamps));
  if (e == cudaSuccess) e = cudaGetSymbolAddress(&b, mbok::g_combine_stamps);
  if (e == cudaSuccess) e = cudaMemset(b, 0, sizeof(mbok::g_combine_stamps));
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (reset_slots) mbok::g_stamp_next.store(0);
  return int(e);
}
#endif
