// Decode GEMV y = W x for one activation vector (batch 1), sm_100a.
//
// The method evaluates W x as K Boolean matrix-vector products scaled by the
// group scales (Paper-Notes page, 方法详解 / 关键设计).  With b in {-1,+1},
//     y_r = sum_g sum_k alpha_{k,r,g} * s_{k,r,g},   s_{k,r,g} = sum_{j in g} b_{k,r,j} x_j.
// The prior-art operator on the FluxBin page (算子创新: LUT-based GEMV that
// streams uint32 weight words, extracts pattern indices with bit operations
// and fetches precomputed partial sums) motivates a lookup table; this kernel
// is designed for the B200 shared-memory pipe instead:
//
//  * Each lane owns 16 consecutive columns of a 512-column slab and keeps two
//    256-entry fp32 tables in ITS OWN shared-memory bank: T_lo[e] (columns
//    0..7 of its unit) and T_hi[e] (columns 8..15), T[e] = sum_i (e_i ? x : -x).
//    Entry e of lane L sits at byte e*256 + 128*h + 4L, so every lookup of a
//    warp touches 32 distinct banks: one wavefront per 8 weight bits.
//  * One 16-byte load per lane brings 8 rows x 16 columns of one kernel
//    (storage format 1), i.e. each warp load is 512 contiguous bytes.
//  * Per (row, kernel) the lane adds two lookups and applies its group scale
//    with one FMA (the lane's 16 columns lie in one group).
//  * The 32 lanes' partial sums of an octet's 8 rows are combined by a
//    transposing butterfly (9 shuffles per lane per octet).
//  * A CTA covers one slab and a contiguous range of row octets; slabs are
//    combined deterministically: the last CTA of a row range to finish sums
//    the per-slab partials in slab order.
// Tables are built exactly sign-symmetric (T[~e] == -T[e]), so flipping every
// bit of a kernel and negating its scales reproduces y bit for bit.
#include "mbok_common.cuh"

namespace mbok {

constexpr int kSlabCols = 512;                    // columns per slab (32 lanes x 16)
constexpr int kGemvThreads = 512;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kLutBytes = 256 * 256;              // 256 entries x (32 lanes x 2 tables x 4 B)
constexpr size_t kMaxCps = 1024;                  // max row ranges (counters) per call
constexpr size_t kCounterBytes = kMaxCps * sizeof(unsigned);
static_assert(kGemvWarps == 16, "table build assigns 16 warps to (table, 32-entry block)");

struct GemvParams {
  const uint8_t* packed;
  const uint16_t* alpha;
  const void* x;
  float* y;
  float* partial;      // [nslab][O*8]
  unsigned* counter;   // [cps]
  Shape s;
  int nslab, cps;
};

template <int K>
struct OctetRegs {
  uint4 bits[K];
  uint4 alpha[K];
};

template <int K>
__device__ __forceinline__ void load_octet(const GemvParams& p, int o, int q, bool lane_ok,
                                           OctetRegs<K>& r) {
  const int g = q / kUnitsPerGroup;
#pragma unroll
  for (int k = 0; k < K; ++k) {
    if (lane_ok) {
      r.bits[k] = __ldg(reinterpret_cast<const uint4*>(p.packed + unit_offset(p.s, o, k, q)));
      r.alpha[k] = __ldg(reinterpret_cast<const uint4*>(p.alpha + alpha_offset(p.s, o, g, k)));
    } else {
      r.bits[k] = make_uint4(0, 0, 0, 0);
      r.alpha[k] = make_uint4(0, 0, 0, 0);
    }
  }
}

__device__ __forceinline__ float lut(const unsigned char* base, uint32_t off) {
  return *reinterpret_cast<const float*>(base + off);
}

template <int K>
__device__ __forceinline__ void octet_dot(const unsigned char* tab, uint32_t lane4,
                                          const OctetRegs<K>& r, float acc[8]) {
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const uint32_t w[4] = {r.bits[k].x, r.bits[k].y, r.bits[k].z, r.bits[k].w};
    const uint32_t a[4] = {r.alpha[k].x, r.alpha[k].y, r.alpha[k].z, r.alpha[k].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // word i holds row 2i (low halfword) and row 2i+1 (high halfword)
      const float t0 = lut(tab, ((w[i] << 8) & 0xFF00u) | lane4);          // row 2i,   cols 0..7
      const float t1 = lut(tab + 128, (w[i] & 0xFF00u) | lane4);           // row 2i,   cols 8..15
      const float t2 = lut(tab, ((w[i] >> 8) & 0xFF00u) | lane4);          // row 2i+1, cols 0..7
      const float t3 = lut(tab + 128, ((w[i] >> 16) & 0xFF00u) | lane4);   // row 2i+1, cols 8..15
      const float2 al = half2_bits_to_float2(a[i]);                       // scales of rows 2i, 2i+1
      acc[2 * i] = fmaf(al.x, t0 + t1, acc[2 * i]);
      acc[2 * i + 1] = fmaf(al.y, t2 + t3, acc[2 * i + 1]);
    }
  }
}

// Sum acc[0..7] over the 32 lanes; returns, in every lane, the total of row
// ((lane >> 2) & 7).  Fixed order, hence deterministic.
__device__ __forceinline__ float octet_reduce(const float acc[8], int lane) {
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
    const float4 t0 = __ldg(p), t1 = __ldg(p + 1);
    v[0] = t0.x; v[1] = t0.y; v[2] = t0.z; v[3] = t0.w;
    v[4] = t1.x; v[5] = t1.y; v[6] = t1.z; v[7] = t1.w;
  } else {
    const uint4 t = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + col0));
    const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] = bf16_bits_to_float(w[e] & 0xFFFFu);
      v[2 * e + 1] = bf16_bits_to_float(w[e] >> 16);
    }
  }
}

// Warp w fills entries [32*(w&7), 32*(w&7)+32) of table h = w>>3 for all 32
// lanes: T[e] = A[e & 15] + B[e >> 4], A/B the signed sums of the table's low
// and high four columns.
template <bool XF32>
__device__ __forceinline__ void build_tables(unsigned char* tab, const void* x, int col0, bool ok,
                                             int warp, int lane) {
  const int h = warp >> 3, blk = warp & 7;
  float c[8];
  load_x8<XF32>(x, col0 + 8 * h, ok, c);
  float A[16];
#pragma unroll
  for (int n = 0; n < 16; ++n) A[n] = signed_sum4(c, uint32_t(n));
  const float B0 = signed_sum4(c + 4, uint32_t(2 * blk));
  const float B1 = signed_sum4(c + 4, uint32_t(2 * blk + 1));
  unsigned char* dst = tab + 128 * h + 4 * lane;
#pragma unroll
  for (int n = 0; n < 32; ++n) {
    const int e = 32 * blk + n;
    *reinterpret_cast<float*>(dst + size_t(e) * 256) = A[n & 15] + ((n < 16) ? B0 : B1);
  }
}

template <int K, bool XF32>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_lut8_kernel(GemvParams p) {
  extern __shared__ __align__(1024) unsigned char tab[];
  __shared__ int s_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int slab = blockIdx.x % p.nslab, c = blockIdx.x / p.nslab;
  const int o_begin = int((long long)c * p.s.O / p.cps);
  const int o_end = int((long long)(c + 1) * p.s.O / p.cps);
  const int q = slab * 32 + lane;
  const bool lane_ok = q < p.s.Q;
  const uint32_t lane4 = 4u * lane;
  const int Mpad = p.s.O * kOctet;

  // Issue the first octet's loads before building the tables.
  int o = o_begin + warp;
  OctetRegs<K> cur;
  if (o < o_end) load_octet<K>(p, o, q, lane_ok, cur);

  build_tables<XF32>(tab, p.x, q * kUnit, lane_ok, warp, lane);
  __syncthreads();

  for (; o < o_end; o += kGemvWarps) {
    OctetRegs<K> nxt;
    const int on = o + kGemvWarps;
    if (on < o_end) load_octet<K>(p, on, q, lane_ok, nxt);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    octet_dot<K>(tab, lane4, cur, acc);
    const float total = octet_reduce(acc, lane);
    const int row = o * kOctet + ((lane >> 2) & 7);
    if ((lane & 3) == 0) {
      if (p.nslab == 1) {
        if (row < p.s.M) p.y[row] = total;
      } else {
        p.partial[size_t(slab) * Mpad + row] = total;
      }
    }
    cur = nxt;
  }

  if (p.nslab == 1) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(&p.counter[c], 1u);
    s_last = (prev == unsigned(p.nslab - 1));
    if (s_last) p.counter[c] = 0u;  // every slab of this row range has arrived
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int r_end = min(o_end * kOctet, p.s.M);
  for (int r = o_begin * kOctet + threadIdx.x; r < r_end; r += blockDim.x) {
    float sum = 0.f;
    for (int t = 0; t < p.nslab; ++t) sum += __ldcg(p.partial + size_t(t) * Mpad + r);
    p.y[r] = sum;
  }
}

struct GemvPlan {
  int nslab, cps;
};

inline GemvPlan gemv_plan(const Shape& s, int sm_count) {
  GemvPlan pl;
  pl.nslab = (s.N + kSlabCols - 1) / kSlabCols;
  int cps = sm_count / pl.nslab;
  if (cps < 1) cps = 1;
  if (cps > s.O) cps = s.O;
  if (cps > int(kMaxCps)) cps = int(kMaxCps);
  pl.cps = cps;
  return pl;
}

// Workspace: the first kCounterBytes hold one arrival counter per row range
// (at most kMaxCps ranges); calls leave them at zero.  Per-slab partial sums
// follow.  The counter block has a fixed size so that calls of any shape can
// share one workspace.

size_t gemv_lut_workspace_bytes(const Shape& s) {
  const size_t nslab = (s.N + kSlabCols - 1) / kSlabCols;
  if (nslab <= 1) return 0;
  return kCounterBytes + nslab * size_t(s.O) * kOctet * sizeof(float);
}

template <int K, bool XF32>
static cudaError_t launch_k(const GemvParams& p, int grid, cudaStream_t stream) {
  auto fn = gemv_lut8_kernel<K, XF32>;
  static bool attr_set = false;   // set once, outside any stream capture
  if (!attr_set) {
    const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  fn<<<grid, kGemvThreads, kLutBytes, stream>>>(p);
  return cudaGetLastError();
}

// y = W x for one vector; workspace as sized by gemv_lut_workspace_bytes.
cudaError_t launch_gemv_lut(const uint8_t* packed, const uint16_t* alpha, const Shape& s,
                            const void* x, bool x_f32, float* y, void* workspace,
                            cudaStream_t stream) {
  const GemvPlan pl = gemv_plan(s, device_sm_count());
  GemvParams p;
  p.packed = packed;
  p.alpha = alpha;
  p.x = x;
  p.y = y;
  p.s = s;
  p.nslab = pl.nslab;
  p.cps = pl.cps;
  p.partial = nullptr;
  p.counter = nullptr;
  if (pl.nslab > 1) {
    p.counter = static_cast<unsigned*>(workspace);
    p.partial = reinterpret_cast<float*>(static_cast<char*>(workspace) + kCounterBytes);
  }
  const int grid = pl.nslab * pl.cps;
  switch (s.K * 2 + (x_f32 ? 1 : 0)) {
    case 2: return launch_k<1, false>(p, grid, stream);
    case 3: return launch_k<1, true>(p, grid, stream);
    case 4: return launch_k<2, false>(p, grid, stream);
    case 5: return launch_k<2, true>(p, grid, stream);
    case 6: return launch_k<3, false>(p, grid, stream);
    case 7: return launch_k<3, true>(p, grid, stream);
    case 8: return launch_k<4, false>(p, grid, stream);
    default: return launch_k<4, true>(p, grid, stream);
  }
}

}  // namespace mbok
