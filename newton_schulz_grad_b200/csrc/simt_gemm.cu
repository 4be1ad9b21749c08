// FFMA (CUDA-core) kernels of the Gram Newton-Schulz chain.
//
// Used for the fp32 dtype (the tensor cores have no fp32-exact product; tf32
// would lose the 1e-4 budget) and for thin bf16 matrices (min side <= 64),
// whose Gram matrices stay in fp32 because bf16 rounding of G and p(G) alone
// exceeds the error budget there.  The three kernels are the three products
// of one iteration (Gram Newton-Schulz, as the DMuon FAQ's related-work
// entry names the default "gram" backend):
//   gram:  G = alpha * X X^T           (one triangle of 64x64 tiles, mirrored)
//   poly:  P = b G + c G G             (G symmetric, so G G = G G^T)
//   apply: Y = alpha * (a X + P X)
// 64x64 output tiles, k-slices of 16 staged in shared memory, 256 threads
// with a 4x4 register tile each; fp32 accumulation in a fixed order, blocked:
// each run of 256 k is summed on its own and then added to the total, so the
// rounding error grows with 256 + k / 256 rather than k (a 1 x 2^20 fp32
// vector: 6e-4 relative error unblocked, well inside 1e-4 blocked).  For
// k <= 256 the result is the plain running sum.
#include "common.cuh"
#include "internal.h"

namespace dmuon {
namespace {

constexpr int SB = 64;
constexpr int SK = 16;
constexpr int kBlockSlices = 16;  // k-slices per accumulation block (256 k)
constexpr int kThreads = 256;

enum { kGram = 0, kPoly = 1, kApply = 2 };

struct SimtArgs {
  const void* A;    // left operand rows (X for gram, G for poly, P for apply)
  const void* B;    // right operand (X for gram, G for poly, X for apply)
  const void* E;    // epilogue operand (G for poly, X for apply)
  void* C;          // output
  int64_t sA, sB, sE, sC;  // batch strides (elements)
  int64_t lda, ldb, lde, ldc;
  int m, n, k;      // output m x n, reduction length k
  float p0, p1;     // gram: alpha; poly: b, c; apply: a, alpha
  const float* scale;
  int tiles_n, tiles_per_mat;
  int batch;
  int* status;      // device status word (bounds errors of debug builds)
};

template <typename T>
__device__ __forceinline__ float ld(const T* p, int64_t i) {
  return Elt<T>::to_f(p[i]);
}

// linear triangle index l -> (ti, tj) with tj <= ti
__device__ __forceinline__ void tri_decode(int l, int& ti, int& tj) {
  int t = (int)((sqrtf(8.f * (float)l + 1.f) - 1.f) * 0.5f);
  while ((t + 1) * (t + 2) / 2 <= l) ++t;
  while (t * (t + 1) / 2 > l) --t;
  ti = t;
  tj = l - t * (t + 1) / 2;
}

template <typename TA, typename TB, typename TE, typename TC, int MODE>
__global__ void __launch_bounds__(kThreads) k_simt(const SimtArgs a) {
  __shared__ float As[SK][SB + 4];
  __shared__ float Bs[SK][SB + 4];
  const int tile = blockIdx.x;
  const int b = blockIdx.y;
  int ti, tj;
  if (MODE == kApply) {
    ti = tile / a.tiles_n;
    tj = tile % a.tiles_n;
  } else {
    tri_decode(tile, ti, tj);
  }
  const int i0 = ti * SB, j0 = tj * SB;
  const TA* A = static_cast<const TA*>(a.A) + (int64_t)b * a.sA;
  const TB* B = static_cast<const TB*>(a.B) + (int64_t)b * a.sB;
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  float acc[4][4], part[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = part[i][j] = 0.f;

  int slices = 0;
  for (int k0 = 0; k0 < a.k; k0 += SK) {
    {  // A tile: rows i0..i0+63, k0..k0+15 -> As[k][row]
      const int row = tid / 4, kq = (tid % 4) * 4;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int gr = i0 + row, gk = k0 + kq + e;
        As[kq + e][row] = (gr < a.m && gk < a.k &&
                           DMUON_IN(a.status, (int64_t)b * a.sA + (int64_t)gr * a.lda + gk, 1, a.batch * a.sA) &&
                           DMUON_IN(a.status, gk, 1, a.lda))
                              ? ld(A, (int64_t)gr * a.lda + gk)
                              : 0.f;
      }
    }
    if (MODE == kApply) {  // B is k x n row-major: Bs[k][j]
      const int kk = tid / 16, jq = (tid % 16) * 4;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int gk = k0 + kk, gj = j0 + jq + e;
        Bs[kk][jq + e] = (gk < a.k && gj < a.n &&
                          DMUON_IN(a.status, (int64_t)b * a.sB + (int64_t)gk * a.ldb + gj, 1, a.batch * a.sB) &&
                          DMUON_IN(a.status, gj, 1, a.ldb))
                             ? ld(B, (int64_t)gk * a.ldb + gj)
                             : 0.f;
      }
    } else {  // B rows j0.. (k-major, like A)
      const int row = tid / 4, kq = (tid % 4) * 4;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int gr = j0 + row, gk = k0 + kq + e;
        Bs[kq + e][row] = (gr < a.n && gk < a.k &&
                           DMUON_IN(a.status, (int64_t)b * a.sB + (int64_t)gr * a.ldb + gk, 1, a.batch * a.sB) &&
                           DMUON_IN(a.status, gk, 1, a.ldb))
                              ? ld(B, (int64_t)gr * a.ldb + gk)
                              : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = fmaf(av[i], bv[j], part[i][j]);
    }
    __syncthreads();
    if (++slices == kBlockSlices || k0 + SK >= a.k) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] += part[i][j];
          part[i][j] = 0.f;
        }
      slices = 0;
    }
  }

  TC* Cm = static_cast<TC*>(a.C) + (int64_t)b * a.sC;
  const TE* Em = static_cast<const TE*>(a.E) + (int64_t)b * a.sE;
  float alpha;
  if (MODE == kGram) {
    const float s = a.scale ? a.scale[b] : 1.f;
    alpha = a.p0 * (s * s);
  } else if (MODE == kApply) {
    alpha = a.p1 * (a.scale ? a.scale[b] : 1.f);
  } else {
    alpha = 1.f;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i0 + ty * 4 + i;
    if (r >= a.m) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = j0 + tx * 4 + j;
      if (c >= a.n) continue;
      if (MODE != kGram && (!DMUON_IN(a.status, (int64_t)b * a.sE + (int64_t)r * a.lde + c, 1, a.batch * a.sE) ||
                            !DMUON_IN(a.status, c, 1, a.lde)))
        continue;
      float v;
      if (MODE == kGram) {
        v = alpha * acc[i][j];
      } else if (MODE == kPoly) {
        v = fmaf(a.p1, acc[i][j], a.p0 * ld(Em, (int64_t)r * a.lde + c));
      } else {
        v = alpha * fmaf(a.p0, ld(Em, (int64_t)r * a.lde + c), acc[i][j]);
      }
      const bool here = DMUON_IN(a.status, (int64_t)b * a.sC + (int64_t)r * a.ldc + c, 1, a.batch * a.sC) &&
                        DMUON_IN(a.status, c, 1, a.ldc);
      if (MODE == kApply) {
        if (here) Cm[(int64_t)r * a.ldc + c] = Elt<TC>::from_f(v);
      } else {
        if (r >= c && here) Cm[(int64_t)r * a.ldc + c] = Elt<TC>::from_f(v);
        if (r > c && DMUON_IN(a.status, (int64_t)b * a.sC + (int64_t)c * a.ldc + r, 1, a.batch * a.sC) &&
            DMUON_IN(a.status, r, 1, a.ldc))
          Cm[(int64_t)c * a.ldc + r] = Elt<TC>::from_f(v);
      }
    }
  }
}

int tri_tiles(int m) {
  const int t = (m + SB - 1) / SB;
  return t * (t + 1) / 2;
}

}  // namespace

cudaError_t simt_gram(const void* X, void* G, int batch, int m, int n, int64_t ldx, int64_t ldg,
                      float alpha, const float* scale, bool xbf16, cudaStream_t st, int* status) {
  if (batch == 0) return cudaSuccess;
  SimtArgs a{};
  a.batch = batch; a.status = status;
  a.A = X; a.B = X; a.E = nullptr; a.C = G;
  a.sA = a.sB = (int64_t)m * ldx; a.sC = (int64_t)m * ldg;
  a.lda = a.ldb = ldx; a.ldc = ldg;
  a.m = m; a.n = m; a.k = n;
  a.p0 = alpha; a.scale = scale;
  a.tiles_per_mat = tri_tiles(m);
  dim3 grid(a.tiles_per_mat, batch);
  if (xbf16)
    k_simt<__nv_bfloat16, __nv_bfloat16, float, float, kGram><<<grid, kThreads, 0, st>>>(a);
  else
    k_simt<float, float, float, float, kGram><<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t simt_poly(const void* G, void* P, int batch, int m, int64_t ldg, int64_t ldp, float b,
                      float c, cudaStream_t st, int* status) {
  if (batch == 0) return cudaSuccess;
  SimtArgs a{};
  a.batch = batch; a.status = status;
  a.A = G; a.B = G; a.E = G; a.C = P;
  a.sA = a.sB = a.sE = (int64_t)m * ldg; a.sC = (int64_t)m * ldp;
  a.lda = a.ldb = a.lde = ldg; a.ldc = ldp;
  a.m = m; a.n = m; a.k = m;
  a.p0 = b; a.p1 = c;
  a.tiles_per_mat = tri_tiles(m);
  dim3 grid(a.tiles_per_mat, batch);
  k_simt<float, float, float, float, kPoly><<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t simt_apply(const void* P, const void* X, void* Y, int batch, int m, int n, int64_t ldp,
                       int64_t ldx, int64_t ldy, float a_coef, float alpha, const float* scale,
                       bool xbf16, cudaStream_t st, int* status) {
  if (batch == 0) return cudaSuccess;
  SimtArgs a{};
  a.batch = batch; a.status = status;
  a.A = P; a.B = X; a.E = X; a.C = Y;
  a.sA = (int64_t)m * ldp; a.sB = a.sE = (int64_t)m * ldx; a.sC = (int64_t)m * ldy;
  a.lda = ldp; a.ldb = a.lde = ldx; a.ldc = ldy;
  a.m = m; a.n = n; a.k = m;
  a.p0 = a_coef; a.p1 = alpha; a.scale = scale;
  a.tiles_n = (n + SB - 1) / SB;
  a.tiles_per_mat = ((m + SB - 1) / SB) * a.tiles_n;
  dim3 grid(a.tiles_per_mat, batch);
  if (xbf16)
    k_simt<float, __nv_bfloat16, __nv_bfloat16, __nv_bfloat16, kApply><<<grid, kThreads, 0, st>>>(a);
  else
    k_simt<float, float, float, float, kApply><<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace dmuon
