// Whole Newton-Schulz chain for thin matrices (m <= 64) in one launch.
//
// For m <= 64 the Gram matrix G = X X^T is at most 64 x 64 and stays in fp32
// (bf16 rounding of G and p(G) alone would exceed the error budget of such
// thin matrices).  One cluster of kCluster CTAs handles one matrix: CTA r
// keeps columns [r*w, (r+1)*w) of X in shared memory for all iterations, so
// X is read once and written once.  Each iteration (Gram Newton-Schulz, the
// DMuon FAQ's related-work entry for the default "gram" backend):
//   1. partial Gram matrix of the CTA's columns (lower triangle, fp32, 2 x 2
//      blocks per thread);
//   2. all-reduce over the cluster through distributed shared memory: every
//      CTA sums the kCluster partials in rank order, so all CTAs hold the
//      same G, bit for bit, whatever the launch;
//   3. P = b G + c G G in shared memory (each CTA, redundantly; m^3 <= 262144);
//   4. X <- a X + P X on the CTA's own columns (4 rows per thread and step),
//      rounded to the storage type.
// Step 0 folds the normalisation in: G0 = s^2 x0 x0^T and X1 = s (a x0 + P x0).
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace dmuon {
namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 256;
constexpr int kMaxM = kSmallM;  // 64

struct SmallArgs {
  void* X;           // batch x m x ld (in: x0, out: the result), storage T
  int64_t sX, ld;
  int m, n, w;       // w: columns per CTA (multiple of 8)
  int lw;            // shared row pitch (see pitch())
  int steps;
  const float* scale;  // per matrix 1/(||x0|| + eps)
  float coeffs[3 * 16];  // a, b, c per iteration (at most 16 here)
  int batch;
  int* status;         // device status word (bounds errors of debug builds)
};

// Two consecutive elements of a shared row as fp32 (c even).
template <typename T>
__device__ __forceinline__ float2 ld2(const T* p);
template <>
__device__ __forceinline__ float2 ld2<float>(const float* p) {
  return *reinterpret_cast<const float2*>(p);
}
template <>
__device__ __forceinline__ float2 ld2<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

template <typename T>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 1)
    k_small_ns(const __grid_constant__ SmallArgs a) {
  extern __shared__ __align__(16) uint8_t dyn[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int mat = blockIdx.x / kCluster;
  const int m = a.m, w = a.w, lw = a.lw;
  const int m2 = (m + 1) & ~1;                        // rows padded to pairs
  const int m4 = (m + 3) & ~3;                        // rows padded to quads
  float* Gp = reinterpret_cast<float*>(dyn);          // [64][64] partial (this CTA)
  float* G = Gp + kMaxM * kMaxM;                      // [64][64] reduced
  float* Pt = G + kMaxM * kMaxM;                      // [64][64] p(G) - a I, transposed
  T* Xs = reinterpret_cast<T*>(Pt + kMaxM * kMaxM);   // [m4][lw] this CTA's columns
  T* Xg = static_cast<T*>(a.X) + (int64_t)mat * a.sX;
  const int c0 = rank * w;
  const int cw = max(0, min(w, a.n - c0));            // valid columns of this CTA
  const int tid = threadIdx.x;

  // rows >= m and columns >= cw are zero, so they add nothing below
  for (int i = tid; i < m4 * w; i += kThreads) {
    const int r = i / w, c = i % w;
    Xs[r * lw + c] = (r < m && c < cw &&
                      DMUON_IN(a.status, (int64_t)mat * a.sX + (int64_t)r * a.ld + c0 + c, 1, a.batch * a.sX) &&
                      DMUON_IN(a.status, c0 + c, 1, a.ld))
                         ? Xg[(int64_t)r * a.ld + c0 + c]
                         : Elt<T>::from_f(0.f);
  }
  for (int i = tid; i < kMaxM * kMaxM; i += kThreads) Pt[i] = 0.f;
  const float s = a.scale[mat];
  const int hb = m2 / 2;                 // 2 x 2 blocks per side
  const int tri = hb * (hb + 1) / 2;     // lower-triangle blocks
  __syncthreads();

  for (int k = 0; k < a.steps; ++k) {
    const float ca = a.coeffs[3 * k], cb = a.coeffs[3 * k + 1], cc = a.coeffs[3 * k + 2];
    // 1. partial Gram matrix over this CTA's columns: each thread a 2 x 2
    //    block (rows 2p, 2p+1; columns 2q, 2q+1; p >= q), fixed order in c
    for (int t = tid; t < tri; t += kThreads) {
      int p = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
      while ((p + 1) * (p + 2) / 2 <= t) ++p;
      while (p * (p + 1) / 2 > t) --p;
      const int q = t - p * (p + 1) / 2;
      const T* x0 = Xs + (2 * p) * lw;
      const T* x1 = x0 + lw;
      const T* y0 = Xs + (2 * q) * lw;
      const T* y1 = y0 + lw;
      float s00 = 0.f, s01 = 0.f, s10 = 0.f, s11 = 0.f;
      for (int c = 0; c < w; c += 2) {
        const float2 a0 = ld2<T>(x0 + c), a1 = ld2<T>(x1 + c), b0 = ld2<T>(y0 + c), b1 = ld2<T>(y1 + c);
        s00 = fmaf(a0.y, b0.y, fmaf(a0.x, b0.x, s00));
        s01 = fmaf(a0.y, b1.y, fmaf(a0.x, b1.x, s01));
        s10 = fmaf(a1.y, b0.y, fmaf(a1.x, b0.x, s10));
        s11 = fmaf(a1.y, b1.y, fmaf(a1.x, b1.x, s11));
      }
      Gp[(2 * p) * kMaxM + 2 * q] = s00;
      Gp[(2 * p) * kMaxM + 2 * q + 1] = s01;
      Gp[(2 * p + 1) * kMaxM + 2 * q] = s10;
      Gp[(2 * p + 1) * kMaxM + 2 * q + 1] = s11;
    }
    cluster.sync();
    // 2. all-reduce in rank order (every CTA gets the same sums); step 0
    //    scales by s^2
    const float g2 = k == 0 ? s * s : 1.f;
    for (int t = tid; t < m * m; t += kThreads) {
      const int i = t / m, j = t % m;
      if (j > i) continue;
      float sum = 0.f;
#pragma unroll
      for (int r = 0; r < kCluster; ++r) sum += cluster.map_shared_rank(Gp, r)[i * kMaxM + j];
      sum *= g2;
      G[i * kMaxM + j] = sum;
      G[j * kMaxM + i] = sum;
    }
    cluster.sync();  // the partials are rewritten next round only after every CTA read them
    // 3. P = b G + c G G (G symmetric), stored transposed for step 4
    for (int t = tid; t < m * m; t += kThreads) {
      const int i = t / m, j = t % m;
      float acc = 0.f;
      for (int q = 0; q < m; ++q) acc = fmaf(G[i * kMaxM + q], G[q * kMaxM + j], acc);
      Pt[j * kMaxM + i] = fmaf(cc, acc, cb * G[i * kMaxM + j]);
    }
    __syncthreads();
    // 4. X <- alpha (a X + P X): a thread owns column c (alone, so row r still
    //    holds its old value when the a X term reads it back) and computes four
    //    rows at a time from one 16-byte read of P^T
    const float alpha = k == 0 ? s : 1.f;
    for (int c = tid; c < cw; c += kThreads) {
      float col[kMaxM];
#pragma unroll
      for (int r = 0; r < kMaxM; ++r) col[r] = r < m ? Elt<T>::to_f(Xs[r * lw + c]) : 0.f;
      for (int r = 0; r < m4; r += 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < kMaxM; ++q) {
          if (q < m) {
            const float4 p = *reinterpret_cast<const float4*>(Pt + q * kMaxM + r);
            acc.x = fmaf(p.x, col[q], acc.x);
            acc.y = fmaf(p.y, col[q], acc.y);
            acc.z = fmaf(p.z, col[q], acc.z);
            acc.w = fmaf(p.w, col[q], acc.w);
          }
        }
        const float o[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (r + u < m) {
            const float xr = Elt<T>::to_f(Xs[(r + u) * lw + c]);
            Xs[(r + u) * lw + c] = Elt<T>::from_f(alpha * fmaf(ca, xr, o[u]));
          }
        }
      }
    }
    __syncthreads();
  }
  for (int i = tid; i < m * w; i += kThreads) {
    const int r = i / w, c = i % w;
    if (c < cw && DMUON_IN(a.status, (int64_t)mat * a.sX + (int64_t)r * a.ld + c0 + c, 1, a.batch * a.sX) &&
        DMUON_IN(a.status, c0 + c, 1, a.ld))
      Xg[(int64_t)r * a.ld + c0 + c] = Xs[r * lw + c];
  }
}

// shared row pitch: w plus 8 bytes (keeps 8-byte pair loads aligned and moves
// consecutive rows to different banks)
int pitch(int w, size_t es) { return w + (int)(8 / es); }
size_t small_smem(int m, int w, size_t es) {
  return 3 * (size_t)kMaxM * kMaxM * sizeof(float) + (size_t)((m + 3) & ~3) * pitch(w, es) * es;
}

}  // namespace

int small_ns_max_n(int m, size_t es) {
  const size_t budget = 200 * 1024 - 3 * (size_t)kMaxM * kMaxM * sizeof(float);
  int w = (int)(budget / ((size_t)((m + 3) & ~3) * es)) - 8;
  w = w / 8 * 8;
  return w * kCluster;
}

cudaError_t small_ns(void* X, int batch, int m, int n, int64_t ld, int steps, const float* coeffs,
                     const float* scale, bool xbf16, cudaStream_t st, int* status) {
  if (batch == 0) return cudaSuccess;
  if (m > kMaxM || steps > 16) return cudaErrorInvalidValue;
  SmallArgs a{};
  a.batch = batch;
  a.status = status;
  a.X = X;
  a.ld = ld;
  a.sX = (int64_t)m * ld;
  a.m = m;
  a.n = n;
  a.w = ((n + kCluster - 1) / kCluster + 7) / 8 * 8;
  a.lw = pitch(a.w, xbf16 ? 2 : 4);
  a.steps = steps;
  a.scale = scale;
  for (int i = 0; i < 3 * steps; ++i) a.coeffs[i] = coeffs[i];
  const size_t es = xbf16 ? 2 : 4;
  if (a.w * kCluster < n || (size_t)n > (size_t)small_ns_max_n(m, es)) return cudaErrorInvalidValue;
  const size_t smem = small_smem(m, a.w, es);
  cudaError_t e;
  if (xbf16) {
    e = cudaFuncSetAttribute(k_small_ns<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_small_ns<__nv_bfloat16><<<batch * kCluster, kThreads, smem, st>>>(a);
  } else {
    e = cudaFuncSetAttribute(k_small_ns<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_small_ns<float><<<batch * kCluster, kThreads, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace dmuon
