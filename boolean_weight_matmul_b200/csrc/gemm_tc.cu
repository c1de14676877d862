// Prefill GEMM  Y[t][r] = sum_j Wt[r][j] X[t][j]  on the sm_100a tensor cores
// (tcgen05.mma, accumulator in tensor memory).
//
// W = sum_k alpha_k B_k (Paper-Notes page, 方法详解 / 关键设计: multi-kernel
// Boolean weights with group-wise scales) is never stored densely: each CTA
// unpacks the bf16 weight tile it needs into shared memory right before the
// tensor cores read it.  Once decoded the product is a dense contraction, so
// it runs as bf16 x bf16 -> fp32 MMAs.
//
// Persistent CTAs (one per SM) walk the tiles of 256 weight rows x n tokens
// (n <= 256, chosen on the host against wave quantisation) in K-steps of 64
// columns through a 3-stage shared-memory ring.  The 256 rows are two M=128
// MMAs that share each X tile, which halves the X traffic through L2 per
// flop (measured: with 128-row tiles the X re-reads, not the tensor cores or
// the unpack, bounded the kernel).  Per stage:
//   * X tile, 256 tokens x 64 columns bf16 (32 KB): one TMA tensor load with
//     128-byte swizzle; the tile's packed bits (16 octets x K x 64 bytes) and
//     scales (16 octets x K x 8 fp16) come with two more TMA loads (warp 0);
//   * W tile, 256 rows x 64 columns bf16 (32 KB): written by 16 unpack warps
//     (two rows x 16 columns per thread) in the same swizzled K-major layout;
//     each element is its weight level rounded once to bf16, selected from
//     the 2^K levels of its (row, group) by its K bits (see the unpack
//     section below);
//   * one thread (warp 1) issues 2 x 4 tcgen05.mma (M=128, N=n, K=16), one
//     set per row half, into the tensor-memory accumulators and commits them
//     to the stage's "empty" barrier.
// The two row halves accumulate in tensor-memory columns 0.. and 256..; 4
// dedicated epilogue warps (one per 32-lane quarter) drain them.  TMEM lane =
// weight row, column = token, so a warp's 32 lanes store 32 consecutive
// elements of one output row of Y.
// Every mbarrier wait is bounded (1 s); on timeout the CTA records an error
// flag, drains what it issued (bounded), frees its tensor memory and exits.
#include "tc_common.cuh"

namespace mbok {

constexpr int kTcRows = 256;      // weight rows per CTA: two M=128 MMAs share each X tile
constexpr int kTcHalf = 128;      // MMA M
constexpr int kTcTokens = 256;    // largest token tile per CTA (MMA N); the host picks <= this
constexpr int kTcBK = 64;         // columns per stage (one 128-byte swizzle row)
constexpr int kTcXBytes = kTcTokens * kTcBK * 2;   // 32 KB
constexpr int kTcWBytes = kTcRows * kTcBK * 2;     // 32 KB (two 16 KB halves)
constexpr int kTcOctets = kTcRows / kOctet;        // 32 row octets per tile
constexpr int kTcBitsRow = kTcBK / 8;              // 64 columns = 8 bytes per row = 64 bytes per octet
constexpr int kTcBitsBytes = kTcOctets * MBOK_MAX_K * kTcBitsRow * kOctet;   // 8 KB (K = 4)
constexpr int kTcAlphaBytes = kTcOctets * MBOK_MAX_K * 16;                 // 2 KB (K = 4)
// One stage: X tile, the W tile (two tiles, hi and lo, when each weight is
// split into two bf16 terms), the packed bits and the scales.  Three stages,
// or two with the split.
template <bool SPLIT>
struct TcGeom {
  static constexpr int kStages = SPLIT ? 2 : 3;
  static constexpr int kWTiles = SPLIT ? 2 : 1;
  static constexpr int kBitsOff = kTcXBytes + kWTiles * kTcWBytes;
  static constexpr int kAlphaOff = kBitsOff + kTcBitsBytes;
  static constexpr int kStageBytes = kAlphaOff + kTcAlphaBytes;
  static constexpr int kSmem = kStages * kStageBytes + 1024 + 256;   // + alignment + barriers
};
constexpr int kTcUnpackWarps = 16;
constexpr int kTcEpiWarp0 = 2 + kTcUnpackWarps;                 // 4 epilogue warps follow the unpack warps
constexpr int kTcThreads = (2 + kTcUnpackWarps + 4) * 32;       // TMA, MMA, 16 unpack, 4 epilogue
constexpr unsigned kTcTmemCols = 512;      // row halves 0 and 1: columns 0.. and 256..

// Instruction descriptor: D f32, A bf16, B bf16, both K-major, M=128, N=n.
inline uint32_t tc_idesc(int n) { return tc_idesc_bf16(kTcHalf, n); }

__device__ unsigned int g_gemm_error;

struct TcParams {
  const uint8_t* packed;
  const uint16_t* alpha;
  uint16_t* Y;
  Shape s;
  int T;
  int n_tile;       // tokens per CTA tile (multiple of 16, <= kTcTokens)
  uint32_t idesc;   // instruction descriptor for N = n_tile
};

// ---------------------------------------------------------------------------
// Unpack: one row x 16 columns of W (all K kernels) -> bf16 in the swizzled tile
// ---------------------------------------------------------------------------
//
// An element of the tile is the weight level its K bits select, rounded once:
//     Wt[r][j] = RN_bf16( s_0 a_0 + s_1 a_1 + ... + s_{K-1} a_{K-1} ),
// s_k = +1 for a set bit and -1 for a clear one, a_k the fp16 group scales,
// the sum taken in fp32 in kernel order.  K kernels give at most 2^K levels
// per (row, group) (Paper-Notes page, 关键设计: K Boolean kernels represent
// 2^K weight values), so each level is formed once per (row, group) and the
// per-element work is a selection:
//  * K = 1: the level is +-a_0; one LOP3 applies the sign bit pair.
//  * K = 2: the four levels sit in two registers as bf16; a byte permute
//    (PRMT) whose selector is built from the two bits of each element picks
//    an element pair's levels at once.
//  * K = 3, 4: the levels are sign-symmetric (the level of the complemented
//    bits is the negated level, exactly, since rounding to nearest is
//    symmetric), so only the 2^(K-1) levels with s_0 = +1 are kept: the other
//    bits are replaced by t_k = XNOR(b_k, b_0), a PRMT (two and a select for
//    K = 4) picks M[t], and the sign of b_0 is applied with one LOP3.
// The PRMT selector of columns (2p, 2p+1) needs 2*index in both nibbles of
// each output halfword; index bits sit in a precomputed word Z at 2p+1,
// 2p+2 (column 2p) and 2p+9, 2p+10 (column 2p+1), so the selector is
// ((Z >> 2p) & 0x0606) * 0x11 + 0x1010.

// bf16 pair (lo, hi), each rounded to nearest even from fp32.
__device__ __forceinline__ uint32_t tc_pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Sign-applied level pair for columns (2i, 2i+1): the level's sign flips
// where the bit of kernel 0 is 0.  u = h | (h << 15) holds bit b at b and at
// 15 + b, so one left shift by 15 - 2i puts bit 2i at 15 and bit 2i+1 at 31.
template <int I>
__device__ __forceinline__ uint32_t tc_signed_pair(uint32_t u, uint32_t lev) {
  const uint32_t s = u << (15 - 2 * I);
  uint32_t r;
  // r = (~s & 0x80008000) ^ lev
  asm("lop3.b32 %0, %1, %2, %3, 0xA6;\n" : "=r"(r) : "r"(s), "r"(0x80008000u), "r"(lev));
  return r;
}

// Index words of 16 columns from two 16-bit planes (A: index bit 0, B:
// index bit 1): z[0] covers columns 0..7, z[1] columns 8..15 (layout above).
__device__ __forceinline__ void tc_index_words(uint32_t A, uint32_t B, uint32_t z[2]) {
  z[0] = ((A & 0x55u) << 1) | ((A & 0xAAu) << 8) | ((B & 0x55u) << 2) | ((B & 0xAAu) << 9);
  z[1] = ((A & 0x5500u) >> 7) | (A & 0xAA00u) | ((B & 0x5500u) >> 6) | ((B & 0xAA00u) << 1);
}

// prmt.b32 in its default mode, where bit 3 of a selector nibble replicates
// the sign (bit 7) of the selected byte (the __byte_perm intrinsic only
// honours the low three bits of each nibble).
__device__ __forceinline__ uint32_t tc_prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// PRMT selector for column pair I from the index words.
template <int I>
__device__ __forceinline__ uint32_t tc_selector(const uint32_t z[2]) {
  const uint32_t v = (z[I >> 2] >> (2 * (I & 3))) & 0x0606u;
  return v * 0x11u + 0x1010u;
}

// Levels of one (row, group) from its K fp16 scales (kernel order), as fp32:
//   K = 1: v = {a0};
//   K = 2: v = {V0, V1, V2, V3}, V[b0 + 2 b1] = s0 a0 + s1 a1;
//   K = 3: v = {M0 .. M3}, M[t1 + 2 t2] = (a0 + s1 a1) + s2 a2;
//   K = 4: v = {M0 .. M7}, M[t1 + 2 t2 + 4 t3] = ((a0 + s1 a1) + s2 a2) + s3 a3.
template <int K>
__device__ __forceinline__ void tc_level_values(const unsigned char* alpha, int o, int i, float v[8]) {
  float a[K];
#pragma unroll
  for (int k = 0; k < K; ++k)
    a[k] = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(alpha + (o * K + k) * 16 + 2 * i)));
  if (K == 1) {
    v[0] = a[0];
  } else if (K == 2) {
    const float d = a[0] - a[1], e = a[0] + a[1];
    v[0] = -e; v[1] = d; v[2] = -d; v[3] = e;
  } else {
    const float x = a[0] - a[1], y = a[0] + a[1];
    const float a2 = a[K > 2 ? 2 : 0];
    const float c0 = x - a2, c1 = y - a2, c2 = x + a2, c3 = y + a2;
    if (K == 3) {
      v[0] = c0; v[1] = c1; v[2] = c2; v[3] = c3;
    } else {
      const float a3 = a[K > 3 ? 3 : 0];
      v[0] = c0 - a3; v[1] = c1 - a3; v[2] = c2 - a3; v[3] = c3 - a3;
      v[4] = c0 + a3; v[5] = c1 + a3; v[6] = c2 + a3; v[7] = c3 + a3;
    }
  }
}

// The level registers of one (row, group): P holds the levels rounded once
// to bf16 (low half first; K = 1: (a0, a0)), and, for the split, L holds
// what that rounding left, v - RN_bf16(v) (exact in fp32), rounded to bf16.
// Rounding to nearest is sign-symmetric, so both stay exact negations of the
// complemented levels.
template <int K, bool SPLIT>
__device__ __forceinline__ void tc_levels(const unsigned char* alpha, int o, int i, uint32_t P[4], uint32_t L[4]) {
  float v[8];
  tc_level_values<K>(alpha, o, i, v);
  constexpr int kN = K == 1 ? 1 : (K == 4 ? 8 : 4);
  float hi[8], lo[8];
#pragma unroll
  for (int n = 0; n < kN; ++n) {
    hi[n] = __bfloat162float(__float2bfloat16_rn(v[n]));
    lo[n] = v[n] - hi[n];
  }
  if (K == 1) {
    P[0] = tc_pack_bf16x2(hi[0], hi[0]);
    if (SPLIT) L[0] = tc_pack_bf16x2(lo[0], lo[0]);
  } else {
#pragma unroll
    for (int n = 0; n < kN / 2; ++n) {
      P[n] = tc_pack_bf16x2(hi[2 * n], hi[2 * n + 1]);
      if (SPLIT) L[n] = tc_pack_bf16x2(lo[2 * n], lo[2 * n + 1]);
    }
  }
}

// One row x 16 columns: h[k] = the row's 16 bits of kernel k (column b in
// bit b), P = its levels; out[I] = bf16 pair of columns (2I, 2I+1).
template <int K>
__device__ __forceinline__ void tc_unpack_row(const uint32_t h[K], const uint32_t P[4], uint32_t out[8]) {
  const uint32_t u0 = h[0] | (h[0] << 15);
  if (K == 1) {
#define MBOK_PAIR(I) out[I] = tc_signed_pair<I>(u0, P[0]);
    MBOK_PAIR(0) MBOK_PAIR(1) MBOK_PAIR(2) MBOK_PAIR(3) MBOK_PAIR(4) MBOK_PAIR(5) MBOK_PAIR(6) MBOK_PAIR(7)
#undef MBOK_PAIR
  } else if (K == 2) {
    uint32_t z[2];
    tc_index_words(h[0], h[1], z);
#define MBOK_PAIR(I) out[I] = __byte_perm(P[0], P[1], tc_selector<I>(z));
    MBOK_PAIR(0) MBOK_PAIR(1) MBOK_PAIR(2) MBOK_PAIR(3) MBOK_PAIR(4) MBOK_PAIR(5) MBOK_PAIR(6) MBOK_PAIR(7)
#undef MBOK_PAIR
  } else {
    // t_k = XNOR(b_k, b_0): the bits relative to kernel 0 (only bits 0..15 are read)
    const uint32_t t1 = ~(h[1] ^ h[0]), t2 = ~(h[2 % K] ^ h[0]);
    uint32_t z[2];
    tc_index_words(t1, t2, z);
    if (K == 3) {
#define MBOK_PAIR(I) out[I] = tc_signed_pair<I>(u0, __byte_perm(P[0], P[1], tc_selector<I>(z)));
      MBOK_PAIR(0) MBOK_PAIR(1) MBOK_PAIR(2) MBOK_PAIR(3) MBOK_PAIR(4) MBOK_PAIR(5) MBOK_PAIR(6) MBOK_PAIR(7)
#undef MBOK_PAIR
    } else {
      const uint32_t t3 = ~(h[3 % K] ^ h[0]) & 0xFFFFu;
      const uint32_t u3 = t3 | (t3 << 15);
      // 16-bit masks from bit 15 / bit 31 of the shifted t3 word (sign-replicating permute)
#define MBOK_PAIR(I)                                                           \
  {                                                                            \
    const uint32_t sel = tc_selector<I>(z);                                    \
    const uint32_t lo = __byte_perm(P[0], P[1], sel);                          \
    const uint32_t hi = __byte_perm(P[2], P[3], sel);                          \
    const uint32_t m = tc_prmt(u3 << (15 - 2 * I), 0u, 0xBB99u);               \
    out[I] = tc_signed_pair<I>(u0, (hi & m) | (lo & ~m));                      \
  }
      MBOK_PAIR(0) MBOK_PAIR(1) MBOK_PAIR(2) MBOK_PAIR(3) MBOK_PAIR(4) MBOK_PAIR(5) MBOK_PAIR(6) MBOK_PAIR(7)
#undef MBOK_PAIR
    }
  }
}

// Unpack one row x 16 columns: thread tid -> row r = tid >> 2, unit u = tid & 3
// of the 256 x 64 tile, with the row's levels P for the stage's group.  Bits
// come from the stage's TMA-loaded copy, [octet][k][unit][row] halfwords.
template <int K, bool SPLIT>
__device__ __forceinline__ void tc_unpack_from_smem(const unsigned char* bits, const uint32_t P[4],
                                                    const uint32_t L[4], unsigned char* wtile, int tid) {
  const int r = tid >> 2, u = tid & 3;
  const int o = r >> 3, i = r & 7;
  uint32_t h[K], out[8];
#pragma unroll
  for (int k = 0; k < K; ++k)
    h[k] = *reinterpret_cast<const uint16_t*>(bits + ((o * K + k) * 4 + u) * 16 + 2 * i);
  // 16 columns = chunks 2u and 2u+1 of the row's 128-byte line, swizzled; the
  // 8 threads of a store phase hold 2 rows of opposite parity x 4 units, i.e.
  // 8 distinct chunks.
  const int c0 = (2 * u) ^ (r & 7), c1 = (2 * u + 1) ^ (r & 7);
  tc_unpack_row<K>(h, P, out);
  unsigned char* line = wtile + r * 128;
  *reinterpret_cast<uint4*>(line + c0 * 16) = make_uint4(out[0], out[1], out[2], out[3]);
  *reinterpret_cast<uint4*>(line + c1 * 16) = make_uint4(out[4], out[5], out[6], out[7]);
  if (SPLIT) {
    // the same selection from the residual levels, into the second tile
    tc_unpack_row<K>(h, L, out);
    line += kTcWBytes;
    *reinterpret_cast<uint4*>(line + c0 * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    *reinterpret_cast<uint4*>(line + c1 * 16) = make_uint4(out[4], out[5], out[6], out[7]);
  }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------

// Drain part of one accumulator tile to Y: this warp's TMEM lane quarter q
// (rows 32q .. 32q+31 of each 128-row half) and the tile's 16-column chunks
// first, first + stride, ... (chunk j: half j / cph, columns 16 (j % cph)),
// loaded kTcDrainBatch at a time per tcgen05.wait::ld.
constexpr int kTcDrainBatch = 1;   // 2 or 3 chunks per wait spilled at the 80-register budget and measured slower
__device__ __forceinline__ void tc_drain(const TcParams& p, uint32_t tmem, int tile, int row_tiles, int q, int lane,
                                         int first, int stride) {
  const int cph = p.n_tile / 16;   // n_tile is a multiple of 16 (the MMA's N)
  const int nch = 2 * cph;
  const int t0 = (tile / row_tiles) * p.n_tile;
  const int rbase = (tile % row_tiles) * kTcRows + 32 * q + lane;
  // Row pairs stored as one 4-byte bf16 pair: needs an even row count (every
  // pair then lies inside Y's rows and stays 4-byte aligned) and an aligned Y.
  const bool pairs = (p.s.M % 2) == 0 && (reinterpret_cast<uintptr_t>(p.Y) % 4) == 0;
  for (int j0 = first; j0 < nch; j0 += kTcDrainBatch * stride) {
    uint32_t v[kTcDrainBatch][16];
#pragma unroll
    for (int u = 0; u < kTcDrainBatch; ++u) {
      const int j = j0 + u * stride;
      if (j < nch) {
        const uint32_t taddr = tmem + (uint32_t(32 * q) << 16) + uint32_t((j / cph) * 256 + (j % cph) * 16);
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
            : "=r"(v[u][0]), "=r"(v[u][1]), "=r"(v[u][2]), "=r"(v[u][3]), "=r"(v[u][4]), "=r"(v[u][5]),
              "=r"(v[u][6]), "=r"(v[u][7]), "=r"(v[u][8]), "=r"(v[u][9]), "=r"(v[u][10]), "=r"(v[u][11]),
              "=r"(v[u][12]), "=r"(v[u][13]), "=r"(v[u][14]), "=r"(v[u][15])
            : "r"(taddr));
      }
    }
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
    for (int u = 0; u < kTcDrainBatch; ++u) {
      const int j = j0 + u * stride;
      if (j >= nch) continue;
      const int r = rbase + (j / cph) * kTcHalf;
      const int c = t0 + (j % cph) * 16;
      if (pairs) {
        // Lanes 2i and 2i+1 hold rows r, r+1: after one exchange per token the
        // even lane has both rows of tokens 0..7 and the odd lane both rows of
        // tokens 8..15, each stored as one bf16 pair (r0 = the even row).
        const bool odd = lane & 1;
        const int r0 = r & ~1;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t mine = odd ? v[u][i] : v[u][8 + i];
          const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
          const float lo = __uint_as_float(odd ? other : v[u][i]);        // row r0
          const float hi = __uint_as_float(odd ? v[u][8 + i] : other);    // row r0 + 1
          const int t = c + (odd ? 8 + i : i);
          if (r0 < p.s.M && t < p.T)
            *reinterpret_cast<uint32_t*>(p.Y + size_t(t) * p.s.M + r0) = tc_pack_bf16x2(lo, hi);
        }
      } else if (r < p.s.M) {
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          if (c + jj < p.T)
            p.Y[size_t(c + jj) * p.s.M + r] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[u][jj])));
        }
      }
    }
  }
}

// Warps that drain the CTA's last tile: the 16 unpack warps, idle by then,
// join the 4 epilogue warps (five per TMEM lane quarter).
constexpr int kTcLastDrainWarps = kTcUnpackWarps + 4;

template <int K, bool SPLIT>
__global__ void __launch_bounds__(kTcThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap bmap,
               const __grid_constant__ CUtensorMap amap, TcParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using G = TcGeom<SPLIT>;
  constexpr int kTcStages = G::kStages;
  constexpr int kTcStageBytes = G::kStageBytes;
  uint64_t* full_x = reinterpret_cast<uint64_t*>(smem + kTcStages * kTcStageBytes);   // stage's X tile landed
  uint64_t* full_w = full_x + kTcStages;   // stage's W tile unpacked (split: its rows 0..127)
  uint64_t* empty = full_w + kTcStages;    // stage's MMAs done
  uint64_t* tfull = empty + kTcStages;     // accumulator b holds a finished tile
  uint64_t* tempty = tfull + 2;            // accumulator b drained by the epilogue
  uint64_t* full_b = tempty + 2;           // stage's bits and scales landed (issued first: the unpack needs only them)
  uint64_t* full_w1 = full_b + kTcStages;  // split only: stage's W rows 128..255 unpacked
  uint64_t* last_full = full_w1 + kTcStages;   // the CTA's last tile is in the accumulator (completes once)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(last_full + 1);
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = p.s.N / kTcBK;
  const int row_tiles = (p.s.M + kTcRows - 1) / kTcRows;
  const int ntiles = row_tiles * ((p.T + p.n_tile - 1) / p.n_tile);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      tc_mbar_init(&full_x[s], 1);
      tc_mbar_init(&full_b[s], 1);
      tc_mbar_init(&full_w[s], kTcUnpackWarps * 32);
      tc_mbar_init(&full_w1[s], kTcUnpackWarps * 32);
      tc_mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc_mbar_init(&tfull[b], 1);
      tc_mbar_init(&tempty[b], 4 * 32);
    }
    tc_mbar_init(last_full, 1);
    s_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(tc_smem(tmem_slot)),
                 "r"(kTcTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  // Tile i of this CTA is tile blockIdx.x + i * gridDim.x; row tiles vary
  // fastest, so CTAs that run together share their X tile through L2.
  if (warp == 0) {
    // ---- TMA producer ----
    if (lane == 0) {
      int g = 0;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int r0 = (tile % row_tiles) * kTcRows, t0 = (tile / row_tiles) * p.n_tile;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % kTcStages;
          if (g >= kTcStages && !tc_wait(&empty[s], unsigned((g / kTcStages) - 1) & 1u)) { ok = false; break; }
          unsigned char* st = smem + s * kTcStageBytes;
          tc_arrive_expect_tx(&full_b[s], kTcOctets * K * (kTcBitsRow * kOctet + 16));
          tc_tma_load_2d(st + G::kBitsOff, &bmap, kb * kTcBitsRow * kOctet, (r0 / kOctet) * K, &full_b[s]);
          tc_tma_load_2d(st + G::kAlphaOff, &amap, ((kb * kTcBK) / kGroup) * K * kOctet,
                         r0 / kOctet, &full_b[s]);
          tc_arrive_expect_tx(&full_x[s], unsigned(p.n_tile) * kTcBK * 2);
          tc_tma_load_2d(st, &xmap, kb * kTcBK, t0, &full_x[s]);
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      int g = 0, i = 0;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++i) {
        if (i > 0 && !tc_wait(&tempty[0], unsigned(i - 1) & 1u)) { ok = false; break; }
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % kTcStages;
          const unsigned ph = unsigned(g / kTcStages) & 1u;
          if (!tc_wait(&full_x[s], ph)) { ok = false; break; }
          const uint32_t xs = tc_smem(smem + s * kTcStageBytes);
          const uint32_t ws = xs + kTcXBytes;
          if constexpr (SPLIT) {
            // Each 128-row half of W (both its tiles) is issued as soon as it
            // is unpacked: measured faster for the split (106.0 -> 101.8 us).
            // The single tile keeps the k-outer order over both halves.
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (!tc_wait(h == 0 ? &full_w[s] : &full_w1[s], ph)) { ok = false; break; }
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < kTcBK / 16; ++kk) {
                const uint64_t bdesc = tc_desc_sw128(xs + kk * 32);
                tc_mma(tmem + uint32_t(h * 256), tc_desc_sw128(ws + h * (kTcHalf * 128) + kk * 32), bdesc, p.idesc,
                       (kb > 0 || kk > 0) ? 1u : 0u);
                // the residual tile into the same accumulator
                tc_mma(tmem + uint32_t(h * 256), tc_desc_sw128(ws + kTcWBytes + h * (kTcHalf * 128) + kk * 32), bdesc,
                       p.idesc, 1u);
              }
            }
            if (!ok) break;
          } else {
            if (!tc_wait(&full_w[s], ph)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kTcBK / 16; ++kk) {
              const uint64_t bdesc = tc_desc_sw128(xs + kk * 32);
#pragma unroll
              for (int h = 0; h < 2; ++h)
                tc_mma(tmem + uint32_t(h * 256), tc_desc_sw128(ws + h * (kTcHalf * 128) + kk * 32), bdesc, p.idesc,
                       (kb > 0 || kk > 0) ? 1u : 0u);
            }
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&tfull[0]);
        if (tile + int(gridDim.x) >= ntiles) tc_commit(last_full);   // the unpack warps may join its drain
      }
    }
  } else if (warp < kTcEpiWarp0) {
    // ---- unpack warps ----
    const int tid = threadIdx.x - 64;
    uint32_t lev[2][4] = {}, res[2][4] = {};   // this thread's two rows' levels for the current group
    int g = 0;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < nkb; ++kb, ++g) {
        const int s = g % kTcStages;
        // the stage's bits landing also means its previous MMAs are done (the
        // slot is refilled only after them), so its W tile may be written
        if (!tc_wait(&full_b[s], unsigned(g / kTcStages) & 1u)) { ok = false; break; }
        unsigned char* st = smem + s * kTcStageBytes;
        // Pass j unpacks rows 128 j .. 128 j + 127.  A 128-column group spans
        // two 64-column stages: its levels are formed on the first and kept
        // for the second.  The split releases each half to the MMA thread as
        // soon as it is written (full_w, full_w1); the single tile releases
        // the whole tile at the end on full_w (a second 512-thread arrival
        // per stage measured 2 us slower over the GEMM).
        if constexpr (SPLIT) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if ((kb & 1) == 0) {
              const int r = (tid + j * kTcUnpackWarps * 32) >> 2;
              tc_levels<K, SPLIT>(st + G::kAlphaOff, r >> 3, r & 7, lev[j], res[j]);
            }
            tc_unpack_from_smem<K, SPLIT>(st + G::kBitsOff, lev[j], res[j], st + kTcXBytes,
                                          tid + j * kTcUnpackWarps * 32);
            asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // generic writes -> tensor core reads
            tc_arrive(j == 0 ? &full_w[s] : &full_w1[s]);
          }
        } else {
          if ((kb & 1) == 0) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int r = (tid + j * kTcUnpackWarps * 32) >> 2;
              tc_levels<K, SPLIT>(st + G::kAlphaOff, r >> 3, r & 7, lev[j], res[j]);
            }
          }
#pragma unroll
          for (int j = 0; j < 2; ++j)
            tc_unpack_from_smem<K, SPLIT>(st + G::kBitsOff, lev[j], res[j], st + kTcXBytes,
                                          tid + j * kTcUnpackWarps * 32);
          asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");   // generic writes -> tensor core reads
          tc_arrive(&full_w[s]);
        }
      }
    }
    // The CTA's last tile: help the epilogue warps drain it.  The MMA thread
    // commits that tile to last_full as well as to tfull; last_full completes
    // once, whereas a parity wait on tfull from here could pass on an earlier
    // phase of it.
    const int n_mine = blockIdx.x < ntiles ? (ntiles - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
    if (ok && n_mine > 0) {
      if (!tc_wait(last_full, 0u)) {
        ok = false;
      } else {
        tc_fence_after();
        tc_drain(p, tmem, int(blockIdx.x) + (n_mine - 1) * int(gridDim.x), row_tiles, warp & 3, lane,
                 (warp - 2) >> 2, kTcLastDrainWarps / 4);
      }
    }
  } else {
    // ---- epilogue warps: TMEM quarter (warp & 3) of both row halves ----
    const int quarter = warp & 3;
    int i = 0;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++i) {
      if (!tc_wait(&tfull[0], unsigned(i) & 1u)) { ok = false; break; }
      tc_fence_after();
      const bool last = tile + int(gridDim.x) >= ntiles;
      if (last)   // shared with the unpack warps: every fifth chunk of this quarter
        tc_drain(p, tmem, tile, row_tiles, quarter, lane, (warp - 2) >> 2, kTcLastDrainWarps / 4);
      else
        tc_drain(p, tmem, tile, row_tiles, quarter, lane, 0, 1);
      tc_fence_before();
      tc_arrive(&tempty[0]);
    }
  }

  if (!ok) atomicOr(&s_fail, 1);
  tc_fence_before();
  __syncthreads();
  if (s_fail != 0 && threadIdx.x == 0) {
    // Record the failure and let every copy and MMA this CTA issued complete
    // (bounded) before its shared memory and tensor memory are released.
    atomicOr(&g_gemm_error, 1u);
    for (int s = 0; s < kTcStages; ++s) {
      (void)tc_wait(&full_x[s], 0u, kTcDrainNs);
      (void)tc_wait(&full_x[s], 1u, kTcDrainNs);
      (void)tc_wait(&full_b[s], 0u, kTcDrainNs);
      (void)tc_wait(&full_b[s], 1u, kTcDrainNs);
      (void)tc_wait(&empty[s], 0u, kTcDrainNs);
      (void)tc_wait(&empty[s], 1u, kTcDrainNs);
    }
    for (int b = 0; b < 2; ++b) {
      (void)tc_wait(&tfull[b], 0u, kTcDrainNs);
      (void)tc_wait(&tfull[b], 1u, kTcDrainNs);
    }
    (void)tc_wait(last_full, 0u, kTcDrainNs);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTcTmemCols));
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

EncodeTiledFn tensor_map_encoder() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

unsigned gemm_error_flags() {
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_gemm_error, sizeof(v)) != cudaSuccess) return ~0u;
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(g_gemm_error, &zero, sizeof(zero)) != cudaSuccess) return ~0u;
  return v;
}

template <int K, bool SPLIT>
static cudaError_t launch_tc_k(const CUtensorMap& xm, const CUtensorMap& bm, const CUtensorMap& am,
                               const TcParams& p, cudaStream_t stream) {
  auto fn = gemm_tc_kernel<K, SPLIT>;
  constexpr int kTcSmem = TcGeom<SPLIT>::kSmem;
  static PerDeviceOnce attr_once;   // the attribute is per device context
  const cudaError_t ae = set_smem_attr_once(attr_once, reinterpret_cast<const void*>(fn), kTcSmem);
  if (ae != cudaSuccess) return ae;
  const int tiles = ((p.s.M + kTcRows - 1) / kTcRows) * ((p.T + p.n_tile - 1) / p.n_tile);
  const int grid = tiles < device_sm_count() ? tiles : device_sm_count();
  fn<<<grid, kTcThreads, kTcSmem, stream>>>(xm, bm, am, p);
  return cudaGetLastError();
}

// Token tile (MMA N, a multiple of 16 up to 256) that minimises the time of
// the wave-quantised grid, waves x tile width, for a 128-row tile and one CTA
// per SM; ties go to the wider tile.
int tc_token_tile(int M, int T, int sms) {
  const long long row_tiles = (M + kTcRows - 1) / kTcRows;
  int best = kTcTokens;
  long long best_cost = -1;
  for (int n = kTcTokens; n >= 128; n -= 16) {
    const long long tiles = row_tiles * ((T + n - 1) / n);
    const long long waves = (tiles + sms - 1) / sms;
    const long long cost = waves * n;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = n;
    }
  }
  return best;
}

// split: each weight as two bf16 terms (see the header).  Returns
// cudaErrorNotSupported when the tensor-map encoder is unavailable.
cudaError_t launch_gemm_tc(const uint8_t* packed, const uint16_t* alpha, const Shape& s, const uint16_t* X,
                           int T, uint16_t* Y, bool split, cudaStream_t stream) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  const int n_tile = tc_token_tile(s.M, T, device_sm_count());
  const cuuint32_t ones[2] = {1, 1};
  CUtensorMap xm, bm, am;
  {  // X: bf16 [T][N], box 64 columns x 256 tokens, 128-byte swizzle
    const cuuint64_t dims[2] = {cuuint64_t(s.N), cuuint64_t(T)};
    const cuuint64_t strides[1] = {cuuint64_t(s.N) * 2};
    const cuuint32_t box[2] = {cuuint32_t(kTcBK), cuuint32_t(n_tile)};
    if (enc(&xm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, ones,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {  // bits: bytes [O*K][N] (one row = one (octet, kernel)), box 64 bytes x 16K rows
    const cuuint64_t dims[2] = {cuuint64_t(s.N), cuuint64_t(s.O) * s.K};
    const cuuint64_t strides[1] = {cuuint64_t(s.N)};
    const cuuint32_t box[2] = {cuuint32_t(kTcBitsRow * kOctet), cuuint32_t(kTcOctets * s.K)};
    if (enc(&bm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed), dims, strides, box, ones,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {  // scales: fp16 [O][G*K*8], box K*8 values x 16 octets
    const cuuint64_t dims[2] = {cuuint64_t(s.G) * s.K * kOctet, cuuint64_t(s.O)};
    const cuuint64_t strides[1] = {cuuint64_t(s.G) * s.K * kOctet * 2};
    const cuuint32_t box[2] = {cuuint32_t(s.K * kOctet), cuuint32_t(kTcOctets)};
    if (enc(&am, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(alpha), dims, strides, box, ones,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  TcParams p;
  p.packed = packed;
  p.alpha = alpha;
  p.Y = Y;
  p.s = s;
  p.T = T;
  p.n_tile = n_tile;
  p.idesc = tc_idesc(n_tile);
  switch (s.K) {
    case 1: return split ? launch_tc_k<1, true>(xm, bm, am, p, stream) : launch_tc_k<1, false>(xm, bm, am, p, stream);
    case 2: return split ? launch_tc_k<2, true>(xm, bm, am, p, stream) : launch_tc_k<2, false>(xm, bm, am, p, stream);
    case 3: return split ? launch_tc_k<3, true>(xm, bm, am, p, stream) : launch_tc_k<3, false>(xm, bm, am, p, stream);
    default: return split ? launch_tc_k<4, true>(xm, bm, am, p, stream) : launch_tc_k<4, false>(xm, bm, am, p, stream);
  }
}

}  // namespace mbok
