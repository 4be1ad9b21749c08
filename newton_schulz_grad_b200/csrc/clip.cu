// Global p-norm clipping of the Muon gradients (DMuon Training Guide,
// "Gradient Clipping": the Muon-only clip runs after the reduce and before
// momentum + Newton-Schulz; the default strategy is global p-norm clipping).
//
//   total = (sum over all matrices and elements of |g|^p)^(1/p)   (p = inf: max |g|)
//   coef  = min(1, max_norm / (total + 1e-6)), NaN if total is NaN;
//   g <- fl(g * fl32(coef))
//
// Bucketed clipping (several independent clips at once) uses the same three
// kinds of launch: partials of every bucket's tables, one coefficient launch
// with one block per bucket, the scaling passes.
//
// Three launches, all on the caller's stream: per-chunk partials of sum |g|^p
// (or max |g|) for every launch class of matrices; one block that reduces all
// partials in a fixed order in fp64 and computes the coefficient; an in-place
// scaling pass (a multiply by 1.0f when nothing is clipped, which leaves every
// value unchanged).  Deterministic: no atomics.  The norm needs no 2D
// structure, so each matrix is read as one flat array: a block covers a
// contiguous chunk of 256 threads x 2 loads x 8 elements, and every warp load
// is 32 consecutive 8-element vectors.  Measured on 128 x 4096^2 bf16 (norm +
// scale, 3 passes): 2 loads per thread at 8 resident blocks per SM 5.79 TB/s;
// 4 loads at 6 blocks 5.22; 8 loads (80 registers, 3 blocks) 3.74.
#include "common.cuh"
#include "internal.h"

namespace dmuon {
namespace {

constexpr int kThreads = 256;
constexpr int kLoads = 2;  // per thread, 8 elements each
static_assert(kClipChunk == kThreads * kLoads * 8, "chunk size");

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
__global__ void __launch_bounds__(kThreads, 8)
    k_clip_partials(const __grid_constant__ ElemTable tab, float* __restrict__ partials) {
  __shared__ float red[kThreads / 32];
  const int e = blockIdx.y;
  const MatEntry& me = tab.e[e];
  const int64_t N = tab.m * tab.n;
  const int64_t base = (int64_t)blockIdx.x * kClipChunk;
  const int tid = threadIdx.x;
  const bool vec = (me.pad & 1) != 0;
  const T* g = static_cast<const T*>(me.src);
  float v[kLoads][8];
  int valid[kLoads];
#pragma unroll
  for (int h = 0; h < kLoads; ++h) {
    const int64_t i = base + ((int64_t)h * kThreads + tid) * 8;
    valid[h] = i < N ? clamp8(N - i) : 0;
    if (valid[h] > 0 && DMUON_IN(tab.status, i, valid[h], N)) {
      load8<T>(g + i, v[h], vec && valid[h] == 8, valid[h]);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[h][k] = 0.f;
    }
  }
  float acc = 0.f;
#pragma unroll
  for (int h = 0; h < kLoads; ++h)
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < valid[h]) acc = accum<P>(acc, v[h][k]);
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

// One block: fixed-order fp64 reduction of `count` partials, then the
// coefficient.  The single clip and every bucket of the bucketed one run this
// same code, so a bucket gets the bits of a separate clip of its gradients.
__device__ __forceinline__ void clip_coef_block(const float* __restrict__ partials, int64_t count, int p,
                                                float max_norm, float* coef, double* total_out) {
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
    // clamped to 1 by a comparison that keeps a NaN: a NaN total gives a NaN
    // coefficient, so every gradient becomes NaN (PyTorch's clip_grad_norm_)
    const double c = (double)max_norm / (total + 1e-6);
    *coef = (float)((c < 1.0 || c != c) ? c : 1.0);
    if (total_out) *total_out = total;
  }
}

__global__ void __launch_bounds__(kThreads)
    k_clip_coef(const float* __restrict__ partials, int64_t count, int p, float max_norm, float* coef,
                double* total_out) {
  clip_coef_block(partials, count, p, max_norm, coef, total_out);
}

// Block k: bucket k's partials [off[k], off[k + 1]).
__global__ void __launch_bounds__(kThreads)
    k_clip_coef_buckets(const float* __restrict__ partials, const __grid_constant__ ClipBuckets B, float* coefs) {
  const int k = blockIdx.x;
  clip_coef_block(partials + B.off[k], B.off[k + 1] - B.off[k], B.p[k], B.max_norm[k], coefs + k,
                  B.total ? B.total + k : nullptr);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 8)
    k_clip_scale(const __grid_constant__ ElemTable tab, const float* __restrict__ coef) {
  const int e = blockIdx.y;
  const MatEntry& me = tab.e[e];
  const int64_t N = tab.m * tab.n;
  const int64_t base = (int64_t)blockIdx.x * kClipChunk;
  const int tid = threadIdx.x;
  const bool vec = (me.pad & 1) != 0;
  T* g = static_cast<T*>(me.buf);
  const float k = *coef;
  float v[kLoads][8];
#pragma unroll
  for (int h = 0; h < kLoads; ++h) {
    const int64_t i = base + ((int64_t)h * kThreads + tid) * 8;
    if (i < N && DMUON_IN(tab.status, i, clamp8(N - i), N)) load8<T>(g + i, v[h], vec && N - i >= 8, clamp8(N - i));
  }
#pragma unroll
  for (int h = 0; h < kLoads; ++h) {
    const int64_t i = base + ((int64_t)h * kThreads + tid) * 8;
    if (i < N && DMUON_IN(tab.status, i, clamp8(N - i), N)) {
#pragma unroll
      for (int q = 0; q < 8; ++q) v[h][q] = __fmul_rn(v[h][q], k);
      store8<T>(g + i, v[h], vec && N - i >= 8, clamp8(N - i));
    }
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

cudaError_t launch_clip_coef_buckets(const float* partials, const ClipBuckets& b, int num_buckets, float* coefs,
                                     cudaStream_t st) {
  if (num_buckets <= 0 || num_buckets > kMaxClipBuckets) return cudaErrorInvalidValue;
  k_clip_coef_buckets<<<num_buckets, kThreads, 0, st>>>(partials, b, coefs);
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
