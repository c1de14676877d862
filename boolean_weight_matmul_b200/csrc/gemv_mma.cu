// Small-batch GEMV Y = W X for 1..16 activation vectors on tensor cores, sm_100a.
//
// The layer is y_r = sum_g sum_k alpha_{k,r,g} * s_{k,r,g} with
// s_{k,r,g} = sum_{j in g} b_{k,r,j} x_j, b in {-1,+1} (Paper-Notes page,
// 方法详解 / 关键设计: W x as K Boolean products, one scale per group).  For
// more than one vector the per-bit work of a lookup table grows with the
// batch, so this kernel computes the K Boolean products s_{k,.,g} as exact
// tensor-core products instead:
//
//  * A = the +-1 signs of one kernel for 16 rows x 16 columns, built in
//    registers as bf16 pairs (0x3F80 = +1, 0xBF80 = -1): each pair is one
//    shift and one three-input logic op on the bit pattern.  Signs are exact
//    in bf16, bf16 activations are exact, and products are exact in the fp32
//    accumulator, so every s_{k,r,g} is an fp32 sum of exact terms.
//  * B = the activations: column n of the 8-wide MMA tile is vector n.  fp32
//    activations are split exactly into three bf16 parts (hi + mid + lo) that
//    take three columns; their results are added back at the end.
//  * One m16n8k16 MMA per (kernel, 16 columns, 8 columns of B); after each
//    128-column group the fp32 result is scaled by the group's fp16 scales
//    and added into the output accumulators (fp32 FMA), so the scales are
//    applied exactly as the method's grouped sum states.
//  * A CTA owns one 16-row tile (two storage octets) and all N columns.  The
//    tile's bits and scales stream through a ring of up to 8 stages in
//    1024-column slices: per slice, one bulk asynchronous copy per (octet,
//    kernel) (the slice is contiguous in storage format 1) and one per octet
//    for the scales, completing on the stage's mbarrier.  The 8 warps split
//    a slice's 64-column chunks; their partial sums meet in shared memory,
//    summed in warp order: no cross-CTA combine, no workspace,
//    deterministic.  Activations are shared by all CTAs, so they are read
//    from global memory (L1/L2-resident), one chunk ahead of their use.
//  * The k-index of an MMA is a permutation of the 16 columns it covers:
//    thread (g, t) of a warp reads the halfword of row g for unit 4c + t of
//    chunk c, and MMA j of the chunk takes bits 4j..4j+3 of it (columns
//    16(4c+t) + 4j .. +3).  B uses the same permutation, which is simply 16
//    consecutive activations of that unit per thread.
//  * Launches use programmatic dependent launch: before waiting on the
//    previous grid a CTA asks L2 to prefetch its tile's bits and scales and,
//    unless told that an earlier kernel on the stream may write the weights,
//    issues the copies of its first slices.
//  * Every mbarrier wait is bounded (1 s); on timeout the CTA records an
//    error flag (bit 2 of mbok_read_device_errors), skips the rest of its
//    work, waits (bounded) for its copies in flight and exits without
//    storing.
#include "mbok_common.cuh"

namespace mbok {

constexpr int kMmaWarps = 8;
constexpr int kMmaThreads = kMmaWarps * 32;
constexpr int kChunkCols = 64;                      // 4 units, 4 MMAs per kernel
// Ring stages: 4, or for rows of 8 or more slices (N > 7168) 8 where they
// leave room for three CTAs per SM (228 KB / 3, less each CTA's 1 KB
// reservation and its static shared memory).  Measured: 7B down (11 slices)
// b4 17.4 -> 16.4 us, b16 21.0 -> 20.0 us with the deep ring; with 5 slices
// (LLaMA-13B gate, N = 5120) the extra stages only took L1 room from the
// activations (b4 31.1 -> 33.2 us), so short rows keep 4.
constexpr int kMmaShortStages = 4;
constexpr int kMmaMaxStages = 8;
constexpr int kMmaDeepMinSlices = 8;
constexpr int kMmaCtaSmemBudget = 74 * 1024;
constexpr int kMaxNT = 2;                           // up to 16 columns of B per launch
constexpr unsigned long long kMmaWaitNs = 1000000000ull;
constexpr unsigned long long kMmaDrainNs = 200000000ull;

// One ring stage: a slice of kCols columns of the tile's two octets (bits of
// every kernel, scales).  Activations are read from global memory (they are
// shared by every CTA and stay in L1/L2), one chunk ahead of their use.
template <int K, int NT, bool XF32, bool DEEP = false>
struct MmaGeom {
  static constexpr int kCols = 1024;
  static constexpr int kUnits = kCols / kUnit;
  static constexpr int kGroups = kCols / kGroup;
  static constexpr int kChunks = kCols / kChunkCols;
  static constexpr int kMaxVec = XF32 ? (8 * NT) / 3 : 8 * NT;
  static constexpr int kBits = 2 * K * kUnits * 16;             // [octet][k][unit][8 rows][2 B]
  static constexpr int kAlpha = 2 * kGroups * K * 16;           // [octet][group][k][8 rows][2 B]
  static constexpr int kStage = kBits + kAlpha;
  static constexpr int kRed = kMmaWarps * NT * 8 * 16 * 4;
  // a power of two (stage index and phase are a mask and a shift): 8 where
  // it fits the budget (K <= 3), else 4
  static constexpr int kDeepStages = (kMmaCtaSmemBudget - kRed) / kStage >= kMmaMaxStages ? kMmaMaxStages
                                                                                          : kMmaShortStages;
  static constexpr int kStages = DEEP ? kDeepStages : kMmaShortStages;
  static constexpr int kSmem = kStages * kStage + kRed;
};

__device__ unsigned int g_gemv_mma_error;

struct GemvMmaParams {
  const uint8_t* packed;
  const uint16_t* alpha;
  const void* x;        // [nb][N] bf16 or fp32
  float* y;             // [nb][M]
  Shape s;
  int nb;               // vectors in this launch
  int weights_static;   // bits and scales may be read before the grid dependency wait
  uint32_t mul[8];      // 2^(15 - 2i): sign_pair factors
};

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t mm_smem(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long mm_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;\n" : "=l"(t));
  return t;
}

__device__ __forceinline__ void grid_dependency_wait_mma() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void allow_dependents_mma() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mm_bar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(mm_smem(bar)), "r"(count));
}

__device__ __forceinline__ void mm_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(mm_smem(bar)) : "memory");
}

__device__ __forceinline__ void mm_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(mm_smem(bar)), "r"(bytes)
               : "memory");
}

// Bounded wait for phase `parity` of an mbarrier; false on timeout.
__device__ __forceinline__ bool mm_wait(uint64_t* bar, unsigned parity, unsigned long long limit) {
  const uint32_t a = mm_smem(bar);
  unsigned long long t0 = 0;
  for (unsigned it = 0;; ++it) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
    if ((it & 255u) == 0) {
      const unsigned long long t = mm_ns();
      if (t0 == 0) t0 = t;
      else if (t - t0 > limit) return false;
    }
  }
}

// Bulk copy global -> this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          mm_smem(dst)),
      "l"(src), "r"(bytes), "r"(mm_smem(bar))
      : "memory");
}

__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// Operands
// ---------------------------------------------------------------------------

// Bits p and p+1 of the halfword h as a bf16 pair of signs (+1 for a set
// bit).  u = h | h << 15 holds bit p at p and bit p+1 at p+16.  The pair is
// (~u & (0x80008000 >> s)) * 2^s + 0x3F803F80 with s = 15 - p: the two
// isolated (inverted) bits land on the sign positions of 1.0 / 1.0 without
// carries.  One logic op (ALU pipe) and one integer multiply-add; the factor
// 2^s comes from the kernel parameters (mul[p/2]) so that the multiply-add
// stays an IMAD on the FMA pipe instead of becoming a shift on the ALU pipe.
template <int P>
__device__ __forceinline__ uint32_t sign_pair(uint32_t u, const uint32_t* mul) {
  static_assert(P % 2 == 0 && P < 15, "pairs start at an even bit below 15");
  constexpr uint32_t kMask = 0x80008000u >> (15 - P);
  return (~u & kMask) * mul[P / 2] + 0x3F803F80u;
}

__device__ __forceinline__ uint32_t spread(uint32_t h) { return h | (h << 15); }

__device__ __forceinline__ uint32_t f32_to_bf16_rn(float v) {
  return uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(v)));
}

// Part `part` (0 = hi, 1 = mid, 2 = lo) of the exact three-way bf16 split of v.
__device__ __forceinline__ uint32_t bf16_part(float v, int part) {
  const uint32_t h = f32_to_bf16_rn(v);
  if (part == 0) return h;
  const float r = __fsub_rn(v, __uint_as_float(h << 16));
  const uint32_t m = f32_to_bf16_rn(r);
  if (part == 1) return m;
  return f32_to_bf16_rn(__fsub_rn(r, __uint_as_float(m << 16)));
}

// The B fragment words of one chunk for column n of B: the 16 activations of
// unit q of vector n (or n/3, part n%3, for fp32) as 8 bf16 pairs; zeros for
// unused columns.
template <bool XF32>
__device__ __forceinline__ void load_b(const GemvMmaParams& p, int n, int q, uint32_t b[8]) {
  const int vec = XF32 ? n / 3 : n;
  if (vec >= p.nb) {
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = 0u;
    return;
  }
  if (!XF32) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.x) + size_t(vec) * p.s.N + q * kUnit);
    const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
    b[0] = v0.x; b[1] = v0.y; b[2] = v0.z; b[3] = v0.w;
    b[4] = v1.x; b[5] = v1.y; b[6] = v1.z; b[7] = v1.w;
  } else {
    const int part = n - 3 * vec;
    const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(p.x) + size_t(vec) * p.s.N + q * kUnit);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldg(src + i);
      b[2 * i] = bf16_part(v.x, part) | (bf16_part(v.y, part) << 16);
      b[2 * i + 1] = bf16_part(v.z, part) | (bf16_part(v.w, part) << 16);
    }
  }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------

// Thread 0: copy slice `sl` of the tile (octets o0, o0+1) into a ring stage.
template <int K, int NT, bool XF32>
__device__ __forceinline__ void issue_slice(const GemvMmaParams& p, int o0, int n_oct, int sl, unsigned char* stage,
                                            uint64_t* full) {
  using G = MmaGeom<K, NT, XF32>;
  const Shape& s = p.s;
  const int u0 = sl * G::kUnits;
  const int nu = min(G::kUnits, s.Q - u0);
  const int ng = nu / kUnitsPerGroup;
  const uint32_t bits_bytes = uint32_t(nu) * 16;
  const uint32_t alpha_bytes = uint32_t(ng) * K * 16;
  mm_arrive_expect_tx(full, uint32_t(n_oct) * (K * bits_bytes + alpha_bytes));
  for (int oi = 0; oi < n_oct; ++oi) {
#pragma unroll
    for (int k = 0; k < K; ++k)
      bulk_copy(stage + (oi * K + k) * G::kUnits * 16, p.packed + unit_offset(s, o0 + oi, k, u0), bits_bytes, full);
    bulk_copy(stage + G::kBits + oi * G::kGroups * K * 16, p.alpha + alpha_offset(s, o0 + oi, u0 / kUnitsPerGroup, 0),
              alpha_bytes, full);
  }
}

// Whether a group's scaling is deferred by one slice (two accumulator sets)
// or done right after its MMAs (one set, for the register-heavy variants).
template <int K, int NT>
struct MmaDefer {
  static constexpr bool value = !(NT == 2 && K >= 3);
  static constexpr int kSets = value ? 2 : 1;
};

// Per-warp accumulators.  Warp w owns group w of every 1024-column slice
// (chunks 2w and 2w+1).  With deferral a group's MMAs accumulate into d[P]
// (P = slice parity) and are scaled into the output accumulators one slice
// later, so the next group's MMAs hide the latency of the MMA chain.
template <int K, int NT>
struct MmaAcc {
  static constexpr int kSets = MmaDefer<K, NT>::kSets;
  float d[kSets][K][NT][4];
  bool have[kSets];
  float y[NT][4];

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int q = 0; q < kSets; ++q) {
      have[q] = false;
#pragma unroll
      for (int k = 0; k < K; ++k)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) d[q][k][nt][i] = 0.f;
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) y[nt][i] = 0.f;
  }

  // y += alpha * d[P] with the group's scales at `alph` (group w of a stage).
  template <int P>
  __device__ __forceinline__ void flush(const unsigned char* alph, int w, int g, int n_oct, int groups_per_stage) {
    if (!have[P]) return;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const float a0 = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(alph + (w * K + k) * 16 + 2 * g)));
      const float a1 = n_oct > 1 ? __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(
                                       alph + ((groups_per_stage + w) * K + k) * 16 + 2 * g)))
                                 : 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        y[nt][0] = __fmaf_rn(a0, d[P][k][nt][0], y[nt][0]);
        y[nt][1] = __fmaf_rn(a0, d[P][k][nt][1], y[nt][1]);
        y[nt][2] = __fmaf_rn(a1, d[P][k][nt][2], y[nt][2]);
        y[nt][3] = __fmaf_rn(a1, d[P][k][nt][3], y[nt][3]);
#pragma unroll
        for (int i = 0; i < 4; ++i) d[P][k][nt][i] = 0.f;
      }
    }
    have[P] = false;
  }
};

// Everything a slice step needs besides the accumulators.
struct MmaCtx {
  unsigned char* smem;
  uint64_t* full;
  uint64_t* empty;
  int* s_abort;
  int issued;          // thread 0: slices whose copies were issued
  int o0, n_oct, n_slices, lane, warp, g, t;
};

// The activations of chunk `half` (0 or 1) of this warp's group in slice sl.
template <int K, int NT, bool XF32>
__device__ __forceinline__ void load_group_b(const GemvMmaParams& p, const MmaCtx& c, int sl, int half,
                                             uint32_t b[NT][8]) {
  using G = MmaGeom<K, NT, XF32>;
  const int q = sl * G::kUnits + 8 * c.warp + 4 * half + c.t;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) load_b<XF32>(p, c.g + 8 * nt, q, b[nt]);
}

// Groups of slice sl (8, fewer in a ragged last slice).
template <int K, int NT, bool XF32>
__device__ __forceinline__ int slice_groups(const Shape& s, int sl) {
  using G = MmaGeom<K, NT, XF32>;
  return min(G::kGroups, s.G - sl * G::kGroups);
}

// MMAs of one chunk (16 rows x 64 columns, K kernels) into d[P].  With one
// 8-column tile of B and K <= 3, all K kernels' sign fragments are built
// first and the MMAs issued kernel-inner, so the K accumulator chains
// interleave instead of each stalling the warp (measured: down K=2 batch 4
// 22.0 -> 17.9 us; with two tiles or K = 4 the extra live fragments cost more
// registers than the interleave saves, so those keep one kernel at a time).
template <int P, int K, int NT, bool XF32>
__device__ __forceinline__ void chunk_mmas(const GemvMmaParams& p, const unsigned char* bits, int uq, int g, int n_oct,
                                           const uint32_t b[NT][8], MmaAcc<K, NT>& acc) {
  using G = MmaGeom<K, NT, XF32>;
  if constexpr (NT > 1 || K > 3) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const uint32_t h0 = *reinterpret_cast<const uint16_t*>(bits + (k * G::kUnits + uq) * 16 + 2 * g);
      const uint32_t h1 =
          n_oct > 1 ? *reinterpret_cast<const uint16_t*>(bits + ((K + k) * G::kUnits + uq) * 16 + 2 * g) : 0u;
      const uint32_t v0 = spread(h0), v1 = spread(h1);
      uint32_t a[4][4];
      a[0][0] = sign_pair<0>(v0, p.mul);  a[0][1] = sign_pair<0>(v1, p.mul);  a[0][2] = sign_pair<2>(v0, p.mul);  a[0][3] = sign_pair<2>(v1, p.mul);
      a[1][0] = sign_pair<4>(v0, p.mul);  a[1][1] = sign_pair<4>(v1, p.mul);  a[1][2] = sign_pair<6>(v0, p.mul);  a[1][3] = sign_pair<6>(v1, p.mul);
      a[2][0] = sign_pair<8>(v0, p.mul);  a[2][1] = sign_pair<8>(v1, p.mul);  a[2][2] = sign_pair<10>(v0, p.mul); a[2][3] = sign_pair<10>(v1, p.mul);
      a[3][0] = sign_pair<12>(v0, p.mul); a[3][1] = sign_pair<12>(v1, p.mul); a[3][2] = sign_pair<14>(v0, p.mul); a[3][3] = sign_pair<14>(v1, p.mul);
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc.d[P][k][nt], a[j], b[nt][2 * j], b[nt][2 * j + 1]);
    }
  } else {
    uint32_t a[K][4][4];
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const uint32_t h0 = *reinterpret_cast<const uint16_t*>(bits + (k * G::kUnits + uq) * 16 + 2 * g);
      const uint32_t h1 =
          n_oct > 1 ? *reinterpret_cast<const uint16_t*>(bits + ((K + k) * G::kUnits + uq) * 16 + 2 * g) : 0u;
      const uint32_t v0 = spread(h0), v1 = spread(h1);
      a[k][0][0] = sign_pair<0>(v0, p.mul);  a[k][0][1] = sign_pair<0>(v1, p.mul);  a[k][0][2] = sign_pair<2>(v0, p.mul);  a[k][0][3] = sign_pair<2>(v1, p.mul);
      a[k][1][0] = sign_pair<4>(v0, p.mul);  a[k][1][1] = sign_pair<4>(v1, p.mul);  a[k][1][2] = sign_pair<6>(v0, p.mul);  a[k][1][3] = sign_pair<6>(v1, p.mul);
      a[k][2][0] = sign_pair<8>(v0, p.mul);  a[k][2][1] = sign_pair<8>(v1, p.mul);  a[k][2][2] = sign_pair<10>(v0, p.mul); a[k][2][3] = sign_pair<10>(v1, p.mul);
      a[k][3][0] = sign_pair<12>(v0, p.mul); a[k][3][1] = sign_pair<12>(v1, p.mul); a[k][3][2] = sign_pair<14>(v0, p.mul); a[k][3][3] = sign_pair<14>(v1, p.mul);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int k = 0; k < K; ++k)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc.d[P][k][nt], a[k][j], b[nt][2 * j], b[nt][2 * j + 1]);
  }
}

// One slice: wait for its copies, run this warp's group into d[P]; with
// deferral, scale the previous slice's group from that slice's (still held)
// stage and release it, else scale this group and release this stage.  The
// stage refilled at slice sl is that of slice sl - 2 (sl - 1 without
// deferral), released by every warp one step earlier.  False if a wait gave
// up.  b0 holds the activations of this warp's chunk 0 in slice sl; b1 is
// filled with those of chunk 1, and b0 with the next slice's chunk 0.
template <int P, int K, int NT, bool XF32, bool DEEP>
__device__ __forceinline__ bool mma_slice(const GemvMmaParams& p, MmaCtx& c, MmaAcc<K, NT>& acc, int sl,
                                          uint32_t b0[NT][8], uint32_t b1[NT][8]) {
  using G = MmaGeom<K, NT, XF32, DEEP>;
  constexpr bool kDefer = MmaDefer<K, NT>::value;
  constexpr int kLag = kDefer ? 2 : 1;
  constexpr int stage_bytes = G::kStage;
  const int st = sl % G::kStages;
  const unsigned phase = unsigned(sl / G::kStages) & 1u;
  // Every decision below is made warp-uniform (the MMAs are warp-wide).
  bool good = true;
  if (c.warp == 0) {
    if (c.lane == 0 && sl >= kLag && c.issued < c.n_slices) {
      const int pst = (sl - kLag) % G::kStages;
      good = mm_wait(&c.empty[pst], unsigned((sl - kLag) / G::kStages) & 1u, kMmaWaitNs);
      if (good) {
        issue_slice<K, NT, XF32>(p, c.o0, c.n_oct, c.issued, c.smem + pst * stage_bytes, &c.full[pst]);
        ++c.issued;
      }
    }
    good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
  }
  if (good) good = *reinterpret_cast<volatile int*>(c.s_abort) == 0;
  if (good) good = mm_wait(&c.full[st], phase, kMmaWaitNs);
  good = __all_sync(0xffffffffu, good);
  if (!good) {
    if (c.lane == 0) {
      atomicOr(&g_gemv_mma_error, 1u);
      *reinterpret_cast<volatile int*>(c.s_abort) = 1;
    }
    return false;
  }

  const unsigned char* bits = c.smem + st * stage_bytes;
  const int w = c.warp;
  if (w < slice_groups<K, NT, XF32>(p.s, sl)) {
    load_group_b<K, NT, XF32>(p, c, sl, 1, b1);
    chunk_mmas<P, K, NT, XF32>(p, bits, 8 * w + c.t, c.g, c.n_oct, b0, acc);
    if (sl + 1 < c.n_slices && w < slice_groups<K, NT, XF32>(p.s, sl + 1)) load_group_b<K, NT, XF32>(p, c, sl + 1, 0, b0);
    chunk_mmas<P, K, NT, XF32>(p, bits, 8 * w + 4 + c.t, c.g, c.n_oct, b1, acc);
    acc.have[P] = true;
  }
  if (kDefer) {
    if (sl >= 1) {
      const int pst = (sl - 1) % G::kStages;
      acc.template flush<MmaDefer<K, NT>::kSets - 1 - P>(c.smem + pst * stage_bytes + G::kBits, w, c.g, c.n_oct,
                                                          G::kGroups);
      __syncwarp();
      if (c.lane == 0) mm_arrive(&c.empty[pst]);
    }
  } else {
    acc.template flush<0>(bits + G::kBits, w, c.g, c.n_oct, G::kGroups);
    __syncwarp();
    if (c.lane == 0) mm_arrive(&c.empty[st]);
  }
  return true;
}

// MINB: CTAs per SM the register budget is cut for -- 3 for grids large
// enough to fill three per SM (more warps to hide latency), else 2 (the
// scheduler would otherwise crowd a small grid onto fewer SMs); 1 for the
// register-heavy variants with two 8-column tiles and K >= 3.
template <int K, int NT, bool XF32, int MINB, bool DEEP>
__global__ void __launch_bounds__(kMmaThreads, MINB) gemv_mma_kernel(GemvMmaParams p) {
  using G = MmaGeom<K, NT, XF32, DEEP>;
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int stage_bytes = G::kStage;
  float (*red)[NT * 8][16] = reinterpret_cast<float (*)[NT * 8][16]>(smem + G::kStages * stage_bytes);
  __shared__ __align__(8) uint64_t full[G::kStages], empty[G::kStages];
  __shared__ int s_abort;

  MmaCtx c;
  c.smem = smem;
  c.full = full;
  c.empty = empty;
  c.s_abort = &s_abort;
  c.issued = 0;
  c.lane = threadIdx.x & 31;
  c.warp = threadIdx.x >> 5;
  c.g = c.lane >> 2;
  c.t = c.lane & 3;
  const Shape& s = p.s;
  c.o0 = 2 * blockIdx.x;
  c.n_oct = (c.o0 + 1 < s.O) ? 2 : 1;
  c.n_slices = (s.N + G::kCols - 1) / G::kCols;

  if (threadIdx.x == 0) {
    for (int i = 0; i < G::kStages; ++i) {
      mm_bar_init(&full[i], 1);
      mm_bar_init(&empty[i], kMmaWarps);
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    // Weights that no earlier kernel on the stream writes: the ring's first
    // slices are copied before the dependency wait.
    if (p.weights_static) {
      for (; c.issued < G::kStages && c.issued < c.n_slices; ++c.issued)
        issue_slice<K, NT, XF32>(p, c.o0, c.n_oct, c.issued, smem + c.issued * stage_bytes, &full[c.issued]);
    }
  }
  // Before the dependency wait: L2 prefetch of this tile's bits and scales.
  if (c.warp == 1) {
    const size_t bits_bytes = size_t(c.n_oct) * s.K * s.N;
    const size_t alpha_bytes = size_t(c.n_oct) * s.G * s.K * kOctet * 2;
    const uint8_t* bsrc = p.packed + unit_offset(s, c.o0, 0, 0);
    const uint8_t* asrc = reinterpret_cast<const uint8_t*>(p.alpha + alpha_offset(s, c.o0, 0, 0));
    constexpr size_t kPiece = 16384;
    for (size_t off = size_t(c.lane) * kPiece; off < bits_bytes; off += 32 * kPiece)
      bulk_prefetch_l2(bsrc + off, uint32_t(min(kPiece, bits_bytes - off)));
    if (c.lane == 31) {
      for (size_t off = 0; off < alpha_bytes; off += kPiece)
        bulk_prefetch_l2(asrc + off, uint32_t(min(kPiece, alpha_bytes - off)));
    }
  }
  allow_dependents_mma();
  grid_dependency_wait_mma();
  __syncthreads();   // barrier initialisation visible to all threads

  if (threadIdx.x == 0) {
    for (; c.issued < G::kStages && c.issued < c.n_slices; ++c.issued)
      issue_slice<K, NT, XF32>(p, c.o0, c.n_oct, c.issued, smem + c.issued * stage_bytes, &full[c.issued]);
  }

  MmaAcc<K, NT> acc;
  acc.init();
  uint32_t b0[NT][8], b1[NT][8];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 8; ++i) b0[nt][i] = 0u;
  if (c.warp < slice_groups<K, NT, XF32>(s, 0)) load_group_b<K, NT, XF32>(p, c, 0, 0, b0);

  constexpr bool kDefer = MmaDefer<K, NT>::value;
  int done = 0;   // slices completed
  if (kDefer) {
    for (int sl = 0; sl < c.n_slices; sl += 2) {
      if (!mma_slice<0, K, NT, XF32, DEEP>(p, c, acc, sl, b0, b1)) break;
      ++done;
      if (sl + 1 < c.n_slices) {
        if (!mma_slice<MmaDefer<K, NT>::kSets - 1, K, NT, XF32, DEEP>(p, c, acc, sl + 1, b0, b1)) break;
        ++done;
      }
    }
    // The last slice's group is still pending; its stage is still held.
    if (done == c.n_slices && c.n_slices >= 1) {
      const int last = c.n_slices - 1;
      const unsigned char* alph = smem + (last % G::kStages) * stage_bytes + G::kBits;
      if (last & 1) acc.template flush<MmaDefer<K, NT>::kSets - 1>(alph, c.warp, c.g, c.n_oct, G::kGroups);
      else acc.template flush<0>(alph, c.warp, c.g, c.n_oct, G::kGroups);
    }
  } else {
    for (int sl = 0; sl < c.n_slices; ++sl) {
      if (!mma_slice<0, K, NT, XF32, DEEP>(p, c, acc, sl, b0, b1)) break;
      ++done;
    }
  }

  // Partial sums of this warp: rows g, g+8, columns 8nt + 2t, 8nt + 2t + 1.
  const int warp = c.warp, g = c.g, t = c.t;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    red[warp][8 * nt + 2 * t][g] = acc.y[nt][0];
    red[warp][8 * nt + 2 * t + 1][g] = acc.y[nt][1];
    red[warp][8 * nt + 2 * t][g + 8] = acc.y[nt][2];
    red[warp][8 * nt + 2 * t + 1][g + 8] = acc.y[nt][3];
  }
  __syncthreads();
  const bool aborted = *reinterpret_cast<volatile int*>(&s_abort) != 0;
  if (aborted) {
    // Wait (bounded) for every copy this CTA issued, then leave without storing.
    if (threadIdx.x == 0) {
      for (int sl = 0; sl < c.issued; ++sl)
        mm_wait(&full[sl % G::kStages], unsigned(sl / G::kStages) & 1u, kMmaDrainNs);
    }
    return;
  }
  // Thread (vector, row): sum over warps in order (and over the three parts
  // of an fp32 vector, hi + mid first).
  const int vec = threadIdx.x >> 4, r = threadIdx.x & 15;
  const int row = 16 * blockIdx.x + r;
  if (vec < p.nb && row < s.M) {
    float total;
    if (!XF32) {
      total = 0.f;
#pragma unroll
      for (int w = 0; w < kMmaWarps; ++w) total += red[w][vec][r];
    } else {
      float part[3];
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        part[q] = 0.f;
#pragma unroll
        for (int w = 0; w < kMmaWarps; ++w) part[q] += red[w][3 * vec + q][r];
      }
      total = (part[0] + part[1]) + part[2];
    }
    p.y[size_t(vec) * s.M + row] = total;
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

template <int K, int NT, bool XF32, int MINB, bool DEEP>
static cudaError_t launch_mma_k(const GemvMmaParams& p, cudaStream_t stream) {
  auto fn = gemv_mma_kernel<K, NT, XF32, MINB, DEEP>;
  using G = MmaGeom<K, NT, XF32, DEEP>;
  static PerDeviceOnce attr_once;   // the attribute is per device context
  const cudaError_t ae = set_smem_attr_once(attr_once, reinterpret_cast<const void*>(fn), G::kSmem);
  if (ae != cudaSuccess) return ae;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.s.O + 1) / 2);
  cfg.blockDim = dim3(kMmaThreads);
  cfg.dynamicSmemBytes = G::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, fn, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int K, bool DEEP>
static cudaError_t launch_mma_nt_d(const GemvMmaParams& p, bool x_f32, cudaStream_t stream) {
  const int cols = x_f32 ? 3 * p.nb : p.nb;
  const bool big_grid = (p.s.O + 1) / 2 >= 3 * device_sm_count();
  if (cols <= 8) {
    if (big_grid)
      return x_f32 ? launch_mma_k<K, 1, true, 3, DEEP>(p, stream) : launch_mma_k<K, 1, false, 3, DEEP>(p, stream);
    return x_f32 ? launch_mma_k<K, 1, true, 2, DEEP>(p, stream) : launch_mma_k<K, 1, false, 2, DEEP>(p, stream);
  }
  constexpr int kMinB2 = K >= 3 ? 1 : 2;
  return x_f32 ? launch_mma_k<K, 2, true, kMinB2, DEEP>(p, stream)
               : launch_mma_k<K, 2, false, kMinB2, DEEP>(p, stream);
}

template <int K>
static cudaError_t launch_mma_nt(const GemvMmaParams& p, bool x_f32, cudaStream_t stream) {
  const int slices = (p.s.N + MmaGeom<K, 1, false>::kCols - 1) / MmaGeom<K, 1, false>::kCols;
  return slices >= kMmaDeepMinSlices ? launch_mma_nt_d<K, true>(p, x_f32, stream)
                                     : launch_mma_nt_d<K, false>(p, x_f32, stream);
}

// Self-check of the bounded waits: one warp waits, with the kernels' own wait
// helper, on an mbarrier that nothing completes; when the wait gives up it
// records the same flag a stuck copy would.
__global__ void wait_timeout_probe_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) mm_bar_init(&bar, 1);
  __syncwarp();
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  __syncwarp();
  const bool done = __all_sync(0xffffffffu, mm_wait(&bar, 0u, limit_ns));
  if (!done && threadIdx.x == 0) atomicOr(&g_gemv_mma_error, 1u);
}

cudaError_t launch_wait_timeout_probe(unsigned timeout_us, cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(1000ull * timeout_us);
  return cudaGetLastError();
}

// Reads and clears the kernel's error flag; ~0u if the read itself failed.
unsigned gemv_mma_error_flags() {
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_gemv_mma_error, sizeof(v)) != cudaSuccess) return ~0u;
  const unsigned z = 0;
  if (v != 0 && cudaMemcpyToSymbol(g_gemv_mma_error, &z, sizeof(z)) != cudaSuccess) return ~0u;
  return v;
}

// Y[b] = W X[b] for b < batch (x: [batch][N], y: [batch][M]); launches cover
// up to 16 bf16 or 5 fp32 vectors each.
cudaError_t launch_gemv_mma(const uint8_t* packed, const uint16_t* alpha, const Shape& s,
                            const void* x, bool x_f32, int batch, float* y, cudaStream_t stream,
                            bool weights_static) {
  const int per_launch = x_f32 ? (8 * kMaxNT) / 3 : 8 * kMaxNT;
  const size_t x_elem = x_f32 ? 4 : 2;
  for (int b0 = 0; b0 < batch; b0 += per_launch) {
    GemvMmaParams p;
    p.packed = packed;
    p.alpha = alpha;
    p.x = static_cast<const char*>(x) + size_t(b0) * s.N * x_elem;
    p.y = y + size_t(b0) * s.M;
    p.s = s;
    p.nb = batch - b0 < per_launch ? batch - b0 : per_launch;
    p.weights_static = weights_static ? 1 : 0;
    for (int i = 0; i < 8; ++i) p.mul[i] = 1u << (15 - 2 * i);
    cudaError_t e;
    switch (s.K) {
      case 1: e = launch_mma_nt<1>(p, x_f32, stream); break;
      case 2: e = launch_mma_nt<2>(p, x_f32, stream); break;
      case 3: e = launch_mma_nt<3>(p, x_f32, stream); break;
      default: e = launch_mma_nt<4>(p, x_f32, stream); break;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace mbok
