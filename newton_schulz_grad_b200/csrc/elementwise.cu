// Memory-bound stages of the Muon step.
//
//  * momentum + Nesterov input + Frobenius partial sums (one pass over g and
//    buf; DMuon Training Guide, Hyperparameter Guide, momentum and nesterov
//    rows), writing x0 into the oriented workspace layout: matrices with
//    rows > cols are transposed through a shared-memory tile so that the
//    Newton-Schulz chain always sees an m x n matrix with m <= n;
//  * fixed-order reduction of the partial sums into 1/(||x0||_F + eps);
//  * decoupled weight decay + shape-scaled update (Hyperparameter Guide, lr
//    row: lr scaled by 0.2 * sqrt(max(m, n))), reading the oriented result
//    back through the same tile transposition.
//
// Every block owns a 64 x 64 tile of the source matrix; 256 threads, each
// moving two 8-element (16-byte for bf16) vectors.  Arithmetic is fp32 with
// every operation rounded separately (__fmul_rn/__fadd_rn), so the stored
// results are fixed bit for bit.
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace dmuon {
namespace {

constexpr int T64 = kElemTile;
constexpr int kThreads = 256;

__device__ __forceinline__ int clamp8(int64_t v) { return v < 8 ? (int)v : 8; }

// 8 resident blocks per SM (<= 32 registers): the extra block keeps more
// loads in flight (measured +12 % bandwidth over the unbounded build).
// CLIP: the gradient is first scaled by the global clipping coefficient and
// rounded to the storage type, exactly the value a separate in-place clip
// would have stored, so a fused clipped step equals clip-then-step bit for bit.
// XT: element type of X in the workspace (T, or fp32 for bf16 matrices whose
// chain keeps X in fp32; x0 is rounded to T first either way).
template <typename T, typename XT, int MODE, bool CLIP>
__global__ void __launch_bounds__(kThreads, CLIP ? 6 : 8)
    k_momentum(const __grid_constant__ ElemTable tab, XT* __restrict__ X, float* __restrict__ partials,
               float mu, int nesterov, int dst_vec, const float* __restrict__ clip_coef) {
  __shared__ float s[T64][T64 + 1];
  __shared__ float red[kThreads / 32];
  const int e = blockIdx.y;
  const MatEntry& me = tab.e[e];
  const bool tr = me.transposed != 0;
  const bool src_vec = (me.pad & 1) != 0;
  const int64_t R = tr ? tab.n : tab.m;
  const int64_t C = tr ? tab.m : tab.n;
  const int64_t tilesC = (C + T64 - 1) / T64;
  const int64_t r0 = (blockIdx.x / tilesC) * T64;
  const int64_t c0 = (blockIdx.x % tilesC) * T64;
  const int tid = threadIdx.x;
  const int cv = tid & 7;
  const int rr = tid >> 3;
  const T* g = static_cast<const T*>(me.src);
  T* buf = static_cast<T*>(me.buf);
  XT* Xm = X + (int64_t)e * tab.m * tab.ldn;

  float ss = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = rr + 32 * h;
    const int64_t gr = r0 + r;
    const int64_t gc = c0 + cv * 8;
    int valid = 0;
    if (gr < R && gc < C) valid = clamp8(C - gc);
    float x[8];
    if (valid > 0 && DMUON_IN(tab.status, gr * C + gc, valid, R * C)) {
      const bool v8 = src_vec && valid == 8;
      const int64_t off = gr * C + gc;
      float gv[8];
      load8<T>(g + off, gv, v8, valid);
      if (CLIP) {
        const float k = *clip_coef;
#pragma unroll
        for (int i = 0; i < 8; ++i) gv[i] = round_to<T>(__fmul_rn(gv[i], k));
      }
      if (MODE == (int)ElemMode::kMomentum) {
        float bv[8], nb[8];
        load8<T>(buf + off, bv, v8, valid);
#pragma unroll
        for (int i = 0; i < 8; ++i) nb[i] = __fadd_rn(__fmul_rn(mu, bv[i]), gv[i]);
        store8<T>(buf + off, nb, v8, valid);
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = nesterov ? __fadd_rn(gv[i], __fmul_rn(mu, nb[i])) : nb[i];
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = gv[i];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        x[i] = (i < valid) ? round_to<T>(x[i]) : 0.f;
        ss = fmaf(x[i], x[i], ss);
      }
      if (!tr && DMUON_IN(tab.status, gc, valid, tab.ldn) &&
          DMUON_IN(tab.status, (int64_t)e * tab.m * tab.ldn + gr * tab.ldn + gc, valid,
                   (int64_t)tab.count * tab.m * tab.ldn))
        store8<XT>(Xm + gr * tab.ldn + gc, x, dst_vec && valid == 8, valid);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = 0.f;
    }
    if (tr) {
#pragma unroll
      for (int i = 0; i < 8; ++i) s[r][cv * 8 + i] = x[i];
    }
  }
  if (tr) {
    __syncthreads();
    // oriented row = source column c0 + i, oriented columns = source rows r0 + j
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = rr + 32 * h;
      const int j0 = cv * 8;
      if (c0 + i < C && r0 + j0 < R) {
        const int valid = clamp8(R - (r0 + j0));
        float y[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) y[k] = s[j0 + k][i];
        if (DMUON_IN(tab.status, r0 + j0, valid, tab.ldn) &&
            DMUON_IN(tab.status, (int64_t)e * tab.m * tab.ldn + (c0 + i) * tab.ldn + r0 + j0, valid,
                     (int64_t)tab.count * tab.m * tab.ldn))
          store8<XT>(Xm + (c0 + i) * tab.ldn + r0 + j0, y, dst_vec && valid == 8, valid);
      }
    }
  }
  ss = warp_sum(ss);
  if ((tid & 31) == 0) red[tid >> 5] = ss;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) t += red[w];
    partials[(int64_t)e * tab.tiles_per_mat + blockIdx.x] = t;
  }
}

__global__ void __launch_bounds__(kThreads)
    k_norm_finalize(const float* __restrict__ partials, int tpm, float* __restrict__ scale,
                    double* __restrict__ sumsq) {
  __shared__ double red[kThreads];
  const int e = blockIdx.x;
  double acc = 0.0;
  for (int i = threadIdx.x; i < tpm; i += kThreads) acc += (double)partials[(int64_t)e * tpm + i];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = kThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double sum = red[0];
    if (scale) scale[e] = (float)(1.0 / (sqrt(sum) + (double)DMUON_NORM_EPS));
    if (sumsq) sumsq[e] = sum;
  }
}

// XT: element type of O in the workspace; an fp32 O of a bf16 matrix is
// rounded to bf16 first, the value dmuon_ns would return for it.
template <typename T, typename XT, int MODE>
__global__ void __launch_bounds__(kThreads)
    k_update(const __grid_constant__ ElemTable tab, const XT* __restrict__ O,
             const float* __restrict__ scale, float decay, float step_scale, int o_vec) {
  __shared__ float s[T64][T64 + 1];
  const int e = blockIdx.y;
  const MatEntry& me = tab.e[e];
  const bool tr = me.transposed != 0;
  const bool dst_vec = (me.pad & 2) != 0;
  const int64_t R = tr ? tab.n : tab.m;
  const int64_t C = tr ? tab.m : tab.n;
  const int64_t tilesC = (C + T64 - 1) / T64;
  const int64_t r0 = (blockIdx.x / tilesC) * T64;
  const int64_t c0 = (blockIdx.x % tilesC) * T64;
  const int tid = threadIdx.x;
  const int cv = tid & 7;
  const int rr = tid >> 3;
  const XT* Om = O + (int64_t)e * tab.m * tab.ldn;
  T* p = static_cast<T*>(me.dst);
  const float sc = scale ? scale[e] : 1.f;

  if (tr) {
    // stage the oriented block rows c0.., columns r0.. into s[i][j]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = rr + 32 * h;
      const int j0 = cv * 8;
      float y[8];
      const int valid = (c0 + i < C && r0 + j0 < R) ? clamp8(R - (r0 + j0)) : 0;
      if (valid > 0 && DMUON_IN(tab.status, r0 + j0, valid, tab.ldn) &&
          DMUON_IN(tab.status, (int64_t)e * tab.m * tab.ldn + (c0 + i) * tab.ldn + r0 + j0, valid,
                   (int64_t)tab.count * tab.m * tab.ldn)) {
        load8<XT>(Om + (c0 + i) * tab.ldn + r0 + j0, y, o_vec && valid == 8, valid);
        if (!std::is_same<T, XT>::value) {
#pragma unroll
          for (int k = 0; k < 8; ++k) y[k] = round_to<T>(y[k]);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) y[k] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) s[j0 + k][i] = y[k];
    }
    __syncthreads();
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = rr + 32 * h;
    const int64_t gr = r0 + r;
    const int64_t gc = c0 + cv * 8;
    if (gr >= R || gc >= C) continue;
    const int valid = clamp8(C - gc);
    if (!DMUON_IN(tab.status, gr * C + gc, valid, R * C)) continue;
    float o[8];
    if (tr) {
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = s[r][cv * 8 + i];
    } else if (DMUON_IN(tab.status, gc, valid, tab.ldn) &&
               DMUON_IN(tab.status, (int64_t)e * tab.m * tab.ldn + gr * tab.ldn + gc, valid,
                        (int64_t)tab.count * tab.m * tab.ldn)) {
      load8<XT>(Om + gr * tab.ldn + gc, o, o_vec && valid == 8, valid);
      if (!std::is_same<T, XT>::value) {
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = round_to<T>(o[i]);
      }
    } else {
      continue;
    }
    if (scale) {
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = __fmul_rn(o[i], sc);
    }
    const int64_t off = gr * C + gc;
    const bool v8 = dst_vec && valid == 8;
    float out[8];
    if (MODE == (int)ElemMode::kUpdate) {
      float pv[8];
      load8<T>(p + off, pv, v8, valid);
#pragma unroll
      for (int i = 0; i < 8; ++i) out[i] = __fsub_rn(__fmul_rn(pv[i], decay), __fmul_rn(step_scale, o[i]));
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) out[i] = o[i];
    }
    store8<T>(p + off, out, v8, valid);
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

template <typename T, typename XT>
void momentum_kernels(const ElemTable& t, ElemMode mode, XT* x, float* partials, float mu, int nesterov,
                      int dst_vec, const float* clip_coef, cudaStream_t st) {
  dim3 grid((unsigned)t.tiles_per_mat, (unsigned)t.count);
  if (clip_coef)
    k_momentum<T, XT, 0, true><<<grid, kThreads, 0, st>>>(t, x, partials, mu, nesterov, dst_vec, clip_coef);
  else if (mode == ElemMode::kMomentum)
    k_momentum<T, XT, 0, false><<<grid, kThreads, 0, st>>>(t, x, partials, mu, nesterov, dst_vec, nullptr);
  else
    k_momentum<T, XT, 1, false><<<grid, kThreads, 0, st>>>(t, x, partials, mu, nesterov, dst_vec, nullptr);
}

cudaError_t launch_momentum(const ElemTable& t, int dtype, ElemMode mode, void* X, float* partials,
                            float mu, int nesterov, cudaStream_t st, const float* clip_coef, int xdtype) {
  if (t.count == 0) return cudaSuccess;
  if (clip_coef && mode != ElemMode::kMomentum) return cudaErrorInvalidValue;
  if (xdtype < 0) xdtype = dtype;
  if (dtype == DMUON_F32 && xdtype != DMUON_F32) return cudaErrorInvalidValue;
  const size_t es = xdtype == DMUON_BF16 ? 2 : 4;
  const int dst_vec = ((t.ldn * (int64_t)es) % 16 == 0) && aligned16(X);
  if (dtype == DMUON_BF16 && xdtype == DMUON_BF16)
    momentum_kernels<__nv_bfloat16>(t, mode, static_cast<__nv_bfloat16*>(X), partials, mu, nesterov, dst_vec,
                                    clip_coef, st);
  else if (dtype == DMUON_BF16)
    momentum_kernels<__nv_bfloat16>(t, mode, static_cast<float*>(X), partials, mu, nesterov, dst_vec, clip_coef,
                                    st);
  else
    momentum_kernels<float>(t, mode, static_cast<float*>(X), partials, mu, nesterov, dst_vec, clip_coef, st);
  return cudaGetLastError();
}

cudaError_t launch_norm_finalize(const float* partials, int count, int tiles_per_mat, float* scale,
                                 double* sumsq, cudaStream_t st) {
  if (count == 0) return cudaSuccess;
  k_norm_finalize<<<count, kThreads, 0, st>>>(partials, tiles_per_mat, scale, sumsq);
  return cudaGetLastError();
}

void update_coeffs(float lr, float wd, int64_t scale_dim, float* decay, float* step_scale) {
  // fp32, each operation rounded once, in this order (no contraction):
  volatile float lw = lr * wd;
  *decay = 1.0f - lw;
  *step_scale = (float)((double)lr * 0.2 * sqrt((double)scale_dim));
}

template <typename T, typename XT>
void update_kernels(const ElemTable& t, ElemMode mode, const XT* o, const float* scale, float decay,
                    float step_scale, int o_vec, cudaStream_t st) {
  dim3 grid((unsigned)t.tiles_per_mat, (unsigned)t.count);
  if (mode == ElemMode::kUpdate)
    k_update<T, XT, 2><<<grid, kThreads, 0, st>>>(t, o, scale, decay, step_scale, o_vec);
  else
    k_update<T, XT, 3><<<grid, kThreads, 0, st>>>(t, o, scale, decay, step_scale, o_vec);
}

cudaError_t launch_update(const ElemTable& t, int dtype, ElemMode mode, const void* O,
                          const float* scale, float lr, float wd, int64_t scale_dim,
                          cudaStream_t st, int xdtype) {
  if (t.count == 0) return cudaSuccess;
  if (xdtype < 0) xdtype = dtype;
  if (dtype == DMUON_F32 && xdtype != DMUON_F32) return cudaErrorInvalidValue;
  const size_t es = xdtype == DMUON_BF16 ? 2 : 4;
  const int o_vec = ((t.ldn * (int64_t)es) % 16 == 0) && aligned16(O);
  float decay, step_scale;
  update_coeffs(lr, wd, scale_dim, &decay, &step_scale);
  if (dtype == DMUON_BF16 && xdtype == DMUON_BF16)
    update_kernels<__nv_bfloat16>(t, mode, static_cast<const __nv_bfloat16*>(O), scale, decay, step_scale, o_vec,
                                  st);
  else if (dtype == DMUON_BF16)
    update_kernels<__nv_bfloat16>(t, mode, static_cast<const float*>(O), scale, decay, step_scale, o_vec, st);
  else
    update_kernels<float>(t, mode, static_cast<const float*>(O), scale, decay, step_scale, o_vec, st);
  return cudaGetLastError();
}

}  // namespace dmuon
