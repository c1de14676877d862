// Decode GEMV y = W x for one activation vector (batch 1) with 4-bit lookup
// tables over whole rows, sm_100a.
//
// The method evaluates W x as K Boolean matrix-vector products scaled by the
// group scales (Paper-Notes page, 方法详解 / 关键设计):
//     y_r = sum_g sum_k alpha_{k,r,g} * s_{k,r,g},   s_{k,r,g} = sum_{j in g} b_{k,r,j} x_j.
// Each CTA owns whole rows, so one launch produces y with no partial sums in
// memory and no second launch: in a chain of dependent launches every extra
// grid (or a grid-wide fence and counter) costs about a microsecond, more than
// a decode layer's own HBM time.  Whole rows need tables for every column, so
// the tables are 4-bit: a lane owning 16 columns keeps, in its own shared
// memory bank, four 16-entry fp32 tables T_n[e] = sum_{i<4} (e_i ? x : -x)
// over columns 4n..4n+3 of its unit (N/8 KB per CTA: 64 KB at N = 4096).
// Entry e of table n of lane L sits at byte (n&1)*4096 + (n>>1)*128 + 256e + 4L
// of its block's 8 KB, so a warp's lookups touch 32 distinct banks, and the
// address of a nibble is one byte permute of a nibble-spread word.
//
//  * Warps: one per block of 32 units (512 columns), lane = unit, plus one
//    producer warp.  A warp builds its block's tables from x and then reads
//    only those: no block-wide barrier before the main loop.
//  * Weights: one ring stage per row octet (its K*N bytes of bits and its
//    16*G*K bytes of scales, two bulk asynchronous copies completing on an
//    mbarrier).  Before waiting on the preceding launch (weights are not
//    written by kernels that let this grid start early) the producer fills
//    the ring and prefetches the rest of the CTA's octets into L2, so HBM
//    streams the layer while the preceding kernel finishes; x and y are
//    touched only after the wait.
//  * Per (row pair, kernel) a lane does eight lookups, three packed fp32x2
//    adds and one packed fp32x2 FMA with the two rows' fp16 group scales.
//  * Per octet the 32 lanes' partials are summed by a transposing shuffle
//    butterfly; the blocks' row sums meet in shared memory and are added in
//    block order, so the result is deterministic.
// Tables are exactly sign-symmetric (T[~e] == -T[e]), so flipping every bit
// of a kernel and negating its scales reproduces y bit for bit.
// Every mbarrier wait is bounded (1 s); on timeout the CTA records an error
// flag (bit 0 of mbok_read_device_errors), drains its copies (bounded),
// leaves its rows of y unwritten and exits.
#include "lut_common.cuh"
#include "tc_common.cuh"

namespace mbok {

constexpr int kL4TableBytes = 8192;   // one block: 4 nibble tables x 16 entries x 32 lanes x 4 B
constexpr int kL4MaxBlocks = 20;      // N <= 10240
constexpr int kL4MaxStages = 16;
constexpr int kL4MaxPairsPerCta = 128;
// Largest dynamic shared memory of one CTA: the 227 KB opt-in limit less room
// for the kernel's static shared variables.
constexpr int kL4SmemLimit = 232448 - 512;

__device__ unsigned int g_lut4_error;

struct Lut4Params {
  const uint8_t* packed;
  const uint16_t* alpha;
  const void* x;
  float* y;
  Shape s;
  int nblk;          // unit blocks = consumer warps
  int pairs;         // row pairs ceil(M/2)
  int ncta;          // CTAs
  int stages;        // ring depth
  int stage_bytes;   // K*N + 16*G*K
  int red_rows;      // row slots per block in the reduction buffer
  int weights_static;
};

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(tc_smem(dst)),
      "l"(src), "r"(bytes), "r"(tc_smem(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_prefetch_l2(const void* src, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(src), "r"(bytes) : "memory");
}

// x[col0 .. col0+15] as fp32 (0 when !ok).
template <bool XF32>
__device__ __forceinline__ void load_x16(const void* x, int col0, bool ok, float v[16]) {
  if (!ok) {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = 0.f;
    return;
  }
  if (XF32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + col0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 t = p[i];
      v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + col0);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 t = p[h];
      const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[8 * h + 2 * e] = bf16_bits_to_float(w[e] & 0xFFFFu);
        v[8 * h + 2 * e + 1] = bf16_bits_to_float(w[e] >> 16);
      }
    }
  }
}

// This lane's four nibble tables from its 16 activations:
// T_n[e] = A[e & 3] + B[e >> 2], A[m] = (+-x_{4n}) + (+-x_{4n+1}), B[m] = (+-x_{4n+2}) + (+-x_{4n+3}),
// a set bit of e meaning +x.  Both halves flip sign exactly with their bits.
__device__ __forceinline__ void build_tables4(unsigned char* tb, const float v[16], int lane) {
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    const float* c = v + 4 * n;
    float A[4], B[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      A[m] = ((m & 1) ? c[0] : -c[0]) + ((m & 2) ? c[1] : -c[1]);
      B[m] = ((m & 1) ? c[2] : -c[2]) + ((m & 2) ? c[3] : -c[3]);
    }
    unsigned char* dst = tb + (n & 1) * 4096 + (n >> 1) * 128 + 4 * lane;
#pragma unroll
    for (int e = 0; e < 16; ++e) *reinterpret_cast<float*>(dst + e * 256) = A[e & 3] + B[e >> 2];
  }
}

// The two rows' sums of one 32-bit word w (row 2p in bits 0..15, row 2p+1 in
// bits 16..31) of this lane's unit: eight lookups, fixed association.  The
// table address of a nibble comes from one byte permute: byte 0 = 4L (this
// lane's bank), byte 1 = the nibble plus the low four bits of the table
// region in its high half (rlo), byte 2 = the region's higher bits (from
// lane4h), so address = 4096 * region + 256 * nibble + 4L, where region
// 2b holds block b's tables of nibbles 0 and 2 and region 2b + 1 those of
// nibbles 1 and 3 (the second table of a region 128 bytes on).
__device__ __forceinline__ float2 pair_sum4(const unsigned char* tab, uint32_t rlo_e, uint32_t rlo_d,
                                            uint32_t lane4h, uint32_t w) {
  const uint32_t E = (w & 0x0F0F0F0Fu) | rlo_e;          // nibbles 0 and 2 of both rows
  const uint32_t D = ((w >> 4) & 0x0F0F0F0Fu) | rlo_d;   // nibbles 1 and 3
  const float a0 = lut(tab, __byte_perm(E, lane4h, 0x5604));
  const float a2 = lut(tab + 128, __byte_perm(E, lane4h, 0x5614));
  const float b0 = lut(tab, __byte_perm(E, lane4h, 0x5624));
  const float b2 = lut(tab + 128, __byte_perm(E, lane4h, 0x5634));
  const float a1 = lut(tab, __byte_perm(D, lane4h, 0x5604));
  const float a3 = lut(tab + 128, __byte_perm(D, lane4h, 0x5614));
  const float b1 = lut(tab, __byte_perm(D, lane4h, 0x5624));
  const float b3 = lut(tab + 128, __byte_perm(D, lane4h, 0x5634));
  return __fadd2_rn(__fadd2_rn(make_float2(a0, b0), make_float2(a1, b1)),
                    __fadd2_rn(make_float2(a2, b2), make_float2(a3, b3)));
}

template <int K, bool XF32>
__global__ void __launch_bounds__((kL4MaxBlocks + 1) * 32, 1) gemv_lut4_kernel(const Lut4Params p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int NB = p.nblk, S = p.stages, SB = p.stage_bytes;
  unsigned char* tab = smem;
  unsigned char* ring = smem + NB * kL4TableBytes;
  float* red = reinterpret_cast<float*>(ring + size_t(S) * SB);
  uint64_t* full = reinterpret_cast<uint64_t*>(red + NB * p.red_rows);
  uint64_t* empty = full + S;
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int p0 = int((long long)c * p.pairs / p.ncta), p1 = int((long long)(c + 1) * p.pairs / p.ncta);
  const int r0 = 2 * p0, r1 = min(2 * p1, p.s.M);
  const int o_first = r0 >> 3;
  const int n_oct = ((r1 - 1) >> 3) - o_first + 1;
  const int KN = K * p.s.N;
  const int AB = 16 * p.s.G * K;   // scale bytes of one octet

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      tc_mbar_init(&full[i], 1);
      tc_mbar_init(&empty[i], NB);
    }
    s_fail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();

  const bool producer = warp == NB && lane == 0;
  const int n_first = min(S, n_oct);
  int issued = 0;   // producer: stages issued so far
  auto issue = [&](int t) {
    ++issued;
    const int o = o_first + t;
    unsigned char* st = ring + size_t(t % S) * SB;
    tc_arrive_expect_tx(&full[t % S], unsigned(KN + AB));
    bulk_g2s(st, p.packed + size_t(o) * KN, unsigned(KN), &full[t % S]);
    bulk_g2s(st + KN, reinterpret_cast<const unsigned char*>(p.alpha) + size_t(o) * AB, unsigned(AB), &full[t % S]);
  };
  auto issue_first = [&]() {
    for (int t = 0; t < n_first; ++t) issue(t);
    // the rest of this CTA's octets into L2: HBM streams them from now on
    for (int t = n_first; t < n_oct; ++t) {
      const int o = o_first + t;
      bulk_prefetch_l2(p.packed + size_t(o) * KN, unsigned(KN));
      bulk_prefetch_l2(reinterpret_cast<const unsigned char*>(p.alpha) + size_t(o) * AB, unsigned(AB));
    }
  };
  if (producer && p.weights_static) issue_first();
  allow_dependents();
  // x and y (and, unless static, the weights) may be touched by the
  // preceding grid: wait for it.
  grid_dependency_wait();
  if (producer && !p.weights_static) issue_first();

  bool ok = true;
  if (warp < NB) {
    const int q = warp * 32 + lane;   // this lane's 16-column unit
    const bool qok = q < p.s.Q;
    unsigned char* tb = tab + warp * kL4TableBytes;   // this block's tables (regions 2b, 2b + 1)
    {
      float v[16];
      load_x16<XF32>(p.x, 16 * q, qok, v);
      build_tables4(tb, v, lane);
    }
    __syncwarp();
    const uint32_t rlo_e = uint32_t((2 * warp) & 15) * 0x10101010u;
    const uint32_t rlo_d = uint32_t((2 * warp + 1) & 15) * 0x10101010u;
    const uint32_t lane4h = 4u * lane | (uint32_t((2 * warp) >> 4) << 16);
    const int g = q >> 3;
    for (int t = 0; t < n_oct; ++t) {
      const int sl = t % S;
      if (!tc_wait(&full[sl], unsigned(t / S) & 1u)) {
        ok = false;
        break;
      }
      const unsigned char* st = ring + size_t(sl) * SB;
      const int o = o_first + t;
      const int pa = max(0, (r0 - 8 * o) >> 1);
      const int pb = min(4, (r1 - 8 * o + 1) >> 1);   // pairs [pa, pb) of this octet are this CTA's
      float2 acc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
      if (qok) {
        uint32_t w[K][4], a[K][4];
#pragma unroll
        for (int k = 0; k < K; ++k) {
          const uint4 wv = *reinterpret_cast<const uint4*>(st + (size_t(k) * p.s.Q + q) * 16);
          const uint4 av = *reinterpret_cast<const uint4*>(st + KN + (g * K + k) * 16);
          w[k][0] = wv.x; w[k][1] = wv.y; w[k][2] = wv.z; w[k][3] = wv.w;
          a[k][0] = av.x; a[k][1] = av.y; a[k][2] = av.z; a[k][3] = av.w;
        }
        // a pair's K kernels: 8K independent lookups (the guard is warp-uniform)
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          if (pp >= pa && pp < pb) {
#pragma unroll
            for (int k = 0; k < K; ++k)
              acc[pp] = __ffma2_rn(half2_bits_to_float2(a[k][pp]), pair_sum4(tab, rlo_e, rlo_d, lane4h, w[k][pp]),
                                   acc[pp]);
          }
        }
      }
      __syncwarp();   // every lane is done with the stage
      if (lane == 0) tc_arrive(&empty[sl]);
      const float total = octet_reduce(acc, lane);
      if ((lane & 3) == 0) red[warp * p.red_rows + 8 * t + ((lane >> 2) & 7)] = total;
    }
  } else if (producer) {
    for (int t = S; t < n_oct; ++t) {
      const int sl = t % S;
      if (!tc_wait(&empty[sl], unsigned(t / S - 1) & 1u)) {
        ok = false;
        break;
      }
      issue(t);
    }
  }
  if (!ok) atomicOr(&s_fail, 1);
  __syncthreads();
  if (s_fail != 0) {
    if (producer) {
      // Let the copies still in flight land before the shared memory goes
      // away: only the last phase issued into each slot can be outstanding.
      for (int sl = 0; sl < S && sl < issued; ++sl) {
        int t_last = sl;
        while (t_last + S < issued) t_last += S;
        (void)tc_wait(&full[sl], unsigned(t_last / S) & 1u, kTcDrainNs);
      }
    }
    if (threadIdx.x == 0) atomicOr(&g_lut4_error, 1u);
    return;
  }
  // y: rows [r0, r1), the blocks' sums added in block order
  for (int i = threadIdx.x; i < r1 - r0; i += blockDim.x) {
    const int ri = r0 + i - 8 * o_first;
    float sum = 0.f;
    for (int b = 0; b < NB; ++b) sum += red[b * p.red_rows + ri];
    p.y[r0 + i] = sum;
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

struct Lut4Plan {
  bool ok;
  Lut4Params p;
  int smem, threads;
};

// Launch geometry for shape s on `sm` SMs; ok = false when the tables and a
// ring of at least two octets do not fit one CTA's shared memory.
static Lut4Plan lut4_plan(const Shape& s, int sm) {
  Lut4Plan pl = {};
  pl.ok = false;
  const int nb = (s.Q + 31) / 32;
  if (nb > kL4MaxBlocks) return pl;
  const int pairs = (s.M + 1) / 2;
  int ncta = pairs < sm ? pairs : sm;
  if ((pairs + ncta - 1) / ncta > kL4MaxPairsPerCta) ncta = (pairs + kL4MaxPairsPerCta - 1) / kL4MaxPairsPerCta;
  const int ppc = (pairs + ncta - 1) / ncta;
  const int max_oct = (2 * ppc + 7) / 8 + 1;   // octets one CTA's rows can touch
  const int red_rows = 8 * max_oct;
  const int sb = s.K * s.N + 16 * s.G * s.K;
  const int fixed = nb * kL4TableBytes + nb * red_rows * 4;
  int stages = (kL4SmemLimit - fixed) / (sb + 16);
  if (stages > max_oct) stages = max_oct;
  if (stages > kL4MaxStages) stages = kL4MaxStages;
  if (stages < 2 && stages < max_oct) return pl;
  if (stages < 1) return pl;
  pl.p.s = s;
  pl.p.nblk = nb;
  pl.p.pairs = pairs;
  pl.p.ncta = ncta;
  pl.p.stages = stages;
  pl.p.stage_bytes = sb;
  pl.p.red_rows = red_rows;
  pl.smem = fixed + stages * sb + 16 * stages;
  pl.threads = (nb + 1) * 32;
  pl.ok = pl.smem <= kL4SmemLimit;
  return pl;
}

bool gemv_lut4_supported(const Shape& s) { return lut4_plan(s, device_sm_count()).ok; }

unsigned gemv_lut4_error_flags() {
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_lut4_error, sizeof(v)) != cudaSuccess) return ~0u;
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(g_lut4_error, &zero, sizeof(zero)) != cudaSuccess) return ~0u;
  return v;
}

template <int K, bool XF32>
static cudaError_t launch_lut4_k(const Lut4Plan& pl, cudaStream_t stream) {
  auto fn = gemv_lut4_kernel<K, XF32>;
  static PerDeviceOnce attr_once;   // the attribute is per device context
  const cudaError_t ae = set_smem_attr_once(attr_once, reinterpret_cast<const void*>(fn), kL4SmemLimit, true);
  if (ae != cudaSuccess) return ae;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.p.ncta);
  cfg.blockDim = dim3(pl.threads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, fn, pl.p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// y = W x for one vector, one launch, no workspace.  Returns
// cudaErrorNotSupported when the shape's tables do not fit (N > 10240).
cudaError_t launch_gemv_lut4(const uint8_t* packed, const uint16_t* alpha, const Shape& s, const void* x,
                             bool x_f32, float* y, cudaStream_t stream, bool weights_static) {
  Lut4Plan pl = lut4_plan(s, device_sm_count());
  if (!pl.ok) return cudaErrorNotSupported;
  pl.p.packed = packed;
  pl.p.alpha = alpha;
  pl.p.x = x;
  pl.p.y = y;
  pl.p.weights_static = weights_static ? 1 : 0;
  switch (s.K * 2 + (x_f32 ? 1 : 0)) {
    case 2: return launch_lut4_k<1, false>(pl, stream);
    case 3: return launch_lut4_k<1, true>(pl, stream);
    case 4: return launch_lut4_k<2, false>(pl, stream);
    case 5: return launch_lut4_k<2, true>(pl, stream);
    case 6: return launch_lut4_k<3, false>(pl, stream);
    case 7: return launch_lut4_k<3, true>(pl, stream);
    case 8: return launch_lut4_k<4, false>(pl, stream);
    default: return launch_lut4_k<4, true>(pl, stream);
  }
}

}  // namespace mbok
