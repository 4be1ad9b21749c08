// Global p-norm clipping of the Muon gradients (DMuon Training Guide,
// "Gradient Clipping": the Muon-only clip runs after the reduce and before
// momentum + Newton-Schulz; the default strategy is global p-norm clipping).
//
//   total = (sum over all matrices and elements of |g|^p)^(1/p)   (p = inf: max |g|)
//   coef  = min(1, max_norm / (total + 1e-6));   g <- fl(g * fl32(coef))
//
// Three launches, all on the caller's stream: per 64 x 64 tile partials of
// sum |g|^p (or max |g|) for every launch class of matrices; one block that
// reduces all partials in a fixed order in fp64 and computes the coefficient;
// an in-place scaling pass (a multiply by 1.0f when nothing is clipped, which
// leaves every value unchanged).  Deterministic: no atomics.
#include "common.cuh"
#include "internal.h"

namespace dmuon {
namespace {

constexpr int T64 = kElemTile;
constexpr int kThreads = 256;

__device__ __forceinline__ int clamp8(int64_t v) { return v < 8 ? (int)v : 8; }

// max that keeps a NaN (fmaxf drops it), so a NaN gradient makes the
// infinity norm NaN as it makes the sums NaN
template <typename F>
__device__ __forceinline__ F nan_max(F a, F b) {
  return (a > b || a != a) ? a : b;
}

// P = 1, 2: sum of |g|^P; P = 0: max |g| (the infinity norm)
template <int P>
__device__ __forceinline__ float accum(float acc, float v) {
  if (P == 0) return nan_max(acc, fabsf(v));
  if (P == 1) return acc + fabsf(v);
  return fmaf(v, v, acc);
}
template <int P>
__device__ __forceinline__ float combine(float a, float b) {
  return P == 0 ? nan_max(a, b) : a + b;
}

template <typename T, int P>
__global__ void __launch_bounds__(kThreads)
    k_clip_partials(const __grid_constant__ ElemTable tab, float* __restrict__ partials) {
  __shared__ float red[kThreads / 32];
  const int e = blockIdx.y;
  const MatEntry& me = tab.e[e];
  const int64_t R = tab.m, C = tab.n;  // source layout, no orientation here
  const int64_t tilesC = (C + T64 - 1) / T64;
  const int64_t r0 = (blockIdx.x / tilesC) * T64;
  const int64_t c0 = (blockIdx.x % tilesC) * T64;
  const int tid = threadIdx.x;
  const int cv = tid & 7, rr = tid >> 3;
  const bool vec = (me.pad & 1) != 0;
  const T* g = static_cast<const T*>(me.src);
  float acc = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t gr = r0 + rr + 32 * h, gc = c0 + cv * 8;
    if (gr >= R || gc >= C) continue;
    const int valid = clamp8(C - gc);
    float v[8];
    load8<T>(g + gr * C + gc, v, vec && valid == 8, valid);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i < valid) acc = accum<P>(acc, v[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc = combine<P>(acc, __shfl_xor_sync(0xffffffffu, acc, o));
  if ((tid & 31) == 0) red[tid >> 5] = acc;
  __syncthreads();
  if (tid == 0) {
    float t = red[0];
    for (int w = 1; w < kThreads / 32; ++w) t = combine<P>(t, red[w]);
    partials[(int64_t)e * tab.tiles_per_mat + blockIdx.x] = t;
  }
}

// One block: fixed-order fp64 reduction of all partials, then the coefficient.
__global__ void __launch_bounds__(kThreads)
    k_clip_coef(const float* __restrict__ partials, int64_t count, int p, float max_norm, float* coef,
                double* total_out) {
  __shared__ double red[kThreads];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < count; i += kThreads) {
    const double v = (double)partials[i];
    acc = p == 0 ? nan_max(acc, v) : acc + v;
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = kThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] = p == 0 ? nan_max(red[threadIdx.x], red[threadIdx.x + w])
                                                   : red[threadIdx.x] + red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double total = p == 0 ? red[0] : (p == 1 ? red[0] : sqrt(red[0]));
    // a NaN total gives coef 1 (nothing scaled; the NaN total is reported)
    const double c = (double)max_norm / (total + 1e-6);
    *coef = (float)(c < 1.0 ? c : 1.0);
    if (total_out) *total_out = total;
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
    k_clip_scale(const __grid_constant__ ElemTable tab, const float* __restrict__ coef) {
  const int e = blockIdx.y;
  const MatEntry& me = tab.e[e];
  const int64_t R = tab.m, C = tab.n;
  const int64_t tilesC = (C + T64 - 1) / T64;
  const int64_t r0 = (blockIdx.x / tilesC) * T64;
  const int64_t c0 = (blockIdx.x % tilesC) * T64;
  const int tid = threadIdx.x;
  const int cv = tid & 7, rr = tid >> 3;
  const bool vec = (me.pad & 1) != 0;
  T* g = static_cast<T*>(me.buf);
  const float k = *coef;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t gr = r0 + rr + 32 * h, gc = c0 + cv * 8;
    if (gr >= R || gc >= C) continue;
    const int valid = clamp8(C - gc);
    const bool v8 = vec && valid == 8;
    float v[8];
    load8<T>(g + gr * C + gc, v, v8, valid);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], k);
    store8<T>(g + gr * C + gc, v, v8, valid);
  }
}

}  // namespace

cudaError_t launch_clip_partials(const ElemTable& t, int dtype, int p, float* partials, cudaStream_t st) {
  if (t.count == 0) return cudaSuccess;
  dim3 grid((unsigned)t.tiles_per_mat, (unsigned)t.count);
  if (dtype == DMUON_BF16) {
    if (p == 0) k_clip_partials<__nv_bfloat16, 0><<<grid, kThreads, 0, st>>>(t, partials);
    else if (p == 1) k_clip_partials<__nv_bfloat16, 1><<<grid, kThreads, 0, st>>>(t, partials);
    else k_clip_partials<__nv_bfloat16, 2><<<grid, kThreads, 0, st>>>(t, partials);
  } else {
    if (p == 0) k_clip_partials<float, 0><<<grid, kThreads, 0, st>>>(t, partials);
    else if (p == 1) k_clip_partials<float, 1><<<grid, kThreads, 0, st>>>(t, partials);
    else k_clip_partials<float, 2><<<grid, kThreads, 0, st>>>(t, partials);
  }
  return cudaGetLastError();
}

cudaError_t launch_clip_coef(const float* partials, int64_t count, int p, float max_norm, float* coef,
                             double* total, cudaStream_t st) {
  k_clip_coef<<<1, kThreads, 0, st>>>(partials, count, p, max_norm, coef, total);
  return cudaGetLastError();
}

cudaError_t launch_clip_scale(const ElemTable& t, int dtype, const float* coef, cudaStream_t st) {
  if (t.count == 0) return cudaSuccess;
  dim3 grid((unsigned)t.tiles_per_mat, (unsigned)t.count);
  if (dtype == DMUON_BF16)
    k_clip_scale<__nv_bfloat16><<<grid, kThreads, 0, st>>>(t, coef);
  else
    k_clip_scale<float><<<grid, kThreads, 0, st>>>(t, coef);
  return cudaGetLastError();
}

}  // namespace dmuon
