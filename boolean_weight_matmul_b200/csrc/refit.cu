// Closed-form least-squares scales for fixed Boolean kernels.
//
// Once the Boolean matrices are fixed the group scales have a closed-form
// least-squares solution, and the method alternates between updating B for
// fixed scales and the scales for fixed B (Paper-Notes page, 关键设计,
// 缩放因子的高效优化).  Per (row r, group g), with b_k the +-1 signs of
// kernel k on the group's 128 columns and w the dense weights there,
//     minimise ||w - sum_k alpha_k b_k||^2   <=>   G alpha = c,
//     G_kl = sum_j b_kj b_lj = 128 - 2 popcount(b_k xor b_l)   (exact integers),
//     c_k  = sum_j b_kj w_j   (fp64, column order j = 0..127),
//     alpha = adj(G) c / det(G)   (adjugate and determinant in exact integers;
//             numerator summed in fp64 in kernel order; one division; one
//             rounding fp64 -> fp16, nearest even).
// A kernel whose signs on the group depend linearly on earlier ones (an exact
// zero determinant) is left out, in kernel order, and gets scale 0.  Every
// floating-point step is an explicit IEEE operation (no contraction), so the
// result is bit-for-bit deterministic.  One thread owns one (row, group).
#include "mbok_common.cuh"

namespace mbok {

constexpr int kRefitThreads = 256;              // 32 groups x 8 rows
constexpr int kRefitGroupsPerBlock = kRefitThreads / kOctet;

// Determinant of the n x n submatrix of G on rows/columns idx[0..n).
__device__ __forceinline__ long long sub_det(const long long G[4][4], const int* idx, int n) {
  if (n == 0) return 1;
  if (n == 1) return G[idx[0]][idx[0]];
  if (n == 2) return G[idx[0]][idx[0]] * G[idx[1]][idx[1]] - G[idx[0]][idx[1]] * G[idx[1]][idx[0]];
  // Laplace expansion along the first row
  long long total = 0;
  for (int col = 0; col < n; ++col) {
    int rest[3];
    int m = 0;
    for (int c = 0; c < n; ++c)
      if (c != col) rest[m++] = idx[c];
    // minor: rows idx[1..n), columns rest[0..n-1)
    long long minor;
    if (n == 3) {
      minor = G[idx[1]][rest[0]] * G[idx[2]][rest[1]] - G[idx[1]][rest[1]] * G[idx[2]][rest[0]];
    } else {   // n == 4: 3 x 3 minor
      const int r0 = idx[1], r1 = idx[2], r2 = idx[3];
      minor = G[r0][rest[0]] * (G[r1][rest[1]] * G[r2][rest[2]] - G[r1][rest[2]] * G[r2][rest[1]]) -
              G[r0][rest[1]] * (G[r1][rest[0]] * G[r2][rest[2]] - G[r1][rest[2]] * G[r2][rest[0]]) +
              G[r0][rest[2]] * (G[r1][rest[0]] * G[r2][rest[1]] - G[r1][rest[1]] * G[r2][rest[0]]);
    }
    total += ((col & 1) ? -1 : 1) * G[idx[0]][idx[col]] * minor;
  }
  return total;
}

// Cofactor (i, j) of the n x n submatrix on idx: (-1)^(i+j) det(minor without row i, column j).
__device__ __forceinline__ long long sub_cofactor(const long long G[4][4], const int* idx, int n, int i, int j) {
  // The minor as its own index lists (rows and columns differ), determinant by
  // explicit formulas for size <= 3.
  int rr[3], cc[3];
  int mr = 0, mc = 0;
  for (int a = 0; a < n; ++a) {
    if (a != i) rr[mr++] = idx[a];
    if (a != j) cc[mc++] = idx[a];
  }
  const int m = n - 1;
  long long d;
  if (m == 0) d = 1;
  else if (m == 1) d = G[rr[0]][cc[0]];
  else if (m == 2) d = G[rr[0]][cc[0]] * G[rr[1]][cc[1]] - G[rr[0]][cc[1]] * G[rr[1]][cc[0]];
  else
    d = G[rr[0]][cc[0]] * (G[rr[1]][cc[1]] * G[rr[2]][cc[2]] - G[rr[1]][cc[2]] * G[rr[2]][cc[1]]) -
        G[rr[0]][cc[1]] * (G[rr[1]][cc[0]] * G[rr[2]][cc[2]] - G[rr[1]][cc[2]] * G[rr[2]][cc[0]]) +
        G[rr[0]][cc[2]] * (G[rr[1]][cc[0]] * G[rr[2]][cc[1]] - G[rr[1]][cc[1]] * G[rr[2]][cc[0]]);
  return ((i + j) & 1) ? -d : d;
}

template <int K>
__global__ void __launch_bounds__(kRefitThreads)
refit_alpha_kernel(const float* __restrict__ W, const uint8_t* __restrict__ packed, Shape s,
                   __half* __restrict__ alpha) {
  const int i = threadIdx.x % kOctet;                                  // row in octet
  const int g = blockIdx.x * kRefitGroupsPerBlock + threadIdx.x / kOctet;
  const int o = blockIdx.y;
  if (g >= s.G) return;
  const int r = o * kOctet + i;
  if (r >= s.M) {
#pragma unroll
    for (int k = 0; k < K; ++k) alpha[alpha_offset(s, o, g, k) + i] = __float2half(0.f);
    return;
  }

  // The group's sign bits of every kernel: 8 halfwords = 4 words per kernel.
  uint32_t bits[K][4];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const uint8_t* unit0 = packed + unit_offset(s, o, k, g * kUnitsPerGroup) + 2 * i;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t lo = *reinterpret_cast<const uint16_t*>(unit0 + size_t(2 * u) * 16);
      const uint32_t hi = *reinterpret_cast<const uint16_t*>(unit0 + size_t(2 * u + 1) * 16);
      bits[k][u] = lo | (hi << 16);
    }
  }

  // c_k = sum_j b_kj w_j in fp64, column order.
  double c[K];
#pragma unroll
  for (int k = 0; k < K; ++k) c[k] = 0.0;
  const float4* src = reinterpret_cast<const float4*>(W + size_t(r) * s.N + size_t(g) * kGroup);
#pragma unroll 4
  for (int v = 0; v < kGroup / 4; ++v) {
    const float4 t = src[v];
    const float wv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * v + e;
      const double wj = double(wv[e]);
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const bool pos = (bits[k][j >> 5] >> (j & 31)) & 1u;
        c[k] = __dadd_rn(c[k], pos ? wj : -wj);
      }
    }
  }

  // Gram matrix: exact integers.
  long long G[4][4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int l = 0; l < 4; ++l) G[k][l] = 0;
#pragma unroll
  for (int k = 0; k < K; ++k)
#pragma unroll
    for (int l = 0; l < K; ++l) {
      int dis = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) dis += __popc(bits[k][u] ^ bits[l][u]);
      G[k][l] = kGroup - 2 * dis;
    }

  // Independent kernels, in kernel order.
  int act[4];
  int na = 0;
  for (int k = 0; k < K; ++k) {
    act[na] = k;
    if (sub_det(G, act, na + 1) != 0) ++na;
  }

  double a[K];
#pragma unroll
  for (int k = 0; k < K; ++k) a[k] = 0.0;
  if (na > 0) {
    const double det = double(sub_det(G, act, na));
    for (int p = 0; p < na; ++p) {
      // adj(G)[p][q] = cofactor(q, p)
      double num = 0.0;
      for (int q = 0; q < na; ++q)
        num = __dadd_rn(num, __dmul_rn(double(sub_cofactor(G, act, na, q, p)), c[act[q]]));
      const double v = __ddiv_rn(num, det);
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (k == act[p]) a[k] = v;
    }
  }
#pragma unroll
  for (int k = 0; k < K; ++k) alpha[alpha_offset(s, o, g, k) + i] = __double2half(a[k]);
}

cudaError_t launch_refit_alpha(const float* W, const uint8_t* packed, const Shape& s, __half* alpha,
                               cudaStream_t stream) {
  dim3 grid((s.G + kRefitGroupsPerBlock - 1) / kRefitGroupsPerBlock, s.O);
  switch (s.K) {
    case 1: refit_alpha_kernel<1><<<grid, kRefitThreads, 0, stream>>>(W, packed, s, alpha); break;
    case 2: refit_alpha_kernel<2><<<grid, kRefitThreads, 0, stream>>>(W, packed, s, alpha); break;
    case 3: refit_alpha_kernel<3><<<grid, kRefitThreads, 0, stream>>>(W, packed, s, alpha); break;
    default: refit_alpha_kernel<4><<<grid, kRefitThreads, 0, stream>>>(W, packed, s, alpha); break;
  }
  return cudaGetLastError();
}

}  // namespace mbok
