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
#include <memory>

#include "common.cuh"
#include "internal.h"

namespace dmuon {
namespace {

constexpr int SB = 64;
constexpr int SK = 32;
constexpr int kBlockSlices = 8;  // k-slices per accumulation block (256 k)
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

// COH: the data was written earlier in the same launch (the fused chain), so
// it is read through L2 (ld.global.cg), never from a possibly stale L1 line.
template <typename T, bool COH = false>
__device__ __forceinline__ float ld(const T* p, int64_t i) {
  if constexpr (COH) {
    if constexpr (sizeof(T) == 2)
      return Elt<T>::to_f(__ushort_as_bfloat16(__ldcg(reinterpret_cast<const unsigned short*>(p + i))));
    else
      return __ldcg(reinterpret_cast<const float*>(p + i));
  } else {
    return Elt<T>::to_f(p[i]);
  }
}

// linear triangle index l -> (ti, tj) with tj <= ti
__device__ __forceinline__ void tri_decode(int l, int& ti, int& tj) {
  int t = (int)((sqrtf(8.f * (float)l + 1.f) - 1.f) * 0.5f);
  while ((t + 1) * (t + 2) / 2 <= l) ++t;
  while (t * (t + 1) / 2 > l) --t;
  ti = t;
  tj = l - t * (t + 1) / 2;
}

// One 64 x 64 output tile `tile` of matrix b (all 256 threads).  The k loop
// runs over slices of 32 in two shared-memory buffers: the next slice's
// global loads are issued before the current slice is multiplied, so their
// latency overlaps the arithmetic (one barrier per slice).  Each thread keeps
// a 4 x 4 register tile and adds k in ascending order, in blocks of 256.
template <typename TA, typename TB, typename TE, typename TC, int MODE, bool COH>
__device__ __forceinline__ void simt_tile(const SimtArgs& a, int tile, int b, float (&As)[2][SK][SB + 4],
                                          float (&Bs)[2][SK][SB + 4]) {
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

  // per slice each thread moves 8 elements of A (row tid/4, k (tid%4)*8..+7)
  // and 8 of B: k-major rows like A, or (apply) row k tid/8, columns (tid%8)*8..+7
  const int arow = tid / 4, akq = (tid % 4) * 8;
  const int bkk = tid / 8, bjq = (tid % 8) * 8;
  float ra[8], rb[8];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int gr = i0 + arow, gk = k0 + akq + e;
      ra[e] = (gr < a.m && gk < a.k &&
               DMUON_IN(a.status, (int64_t)b * a.sA + (int64_t)gr * a.lda + gk, 1, a.batch * a.sA) &&
               DMUON_IN(a.status, gk, 1, a.lda))
                  ? ld<TA, COH>(A, (int64_t)gr * a.lda + gk)
                  : 0.f;
    }
    if (MODE == kApply) {  // B is k x n row-major
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int gk = k0 + bkk, gj = j0 + bjq + e;
        rb[e] = (gk < a.k && gj < a.n &&
                 DMUON_IN(a.status, (int64_t)b * a.sB + (int64_t)gk * a.ldb + gj, 1, a.batch * a.sB) &&
                 DMUON_IN(a.status, gj, 1, a.ldb))
                    ? ld<TB, COH>(B, (int64_t)gk * a.ldb + gj)
                    : 0.f;
      }
    } else {  // B rows j0.. (k-major, like A)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int gr = j0 + arow, gk = k0 + akq + e;
        rb[e] = (gr < a.n && gk < a.k &&
                 DMUON_IN(a.status, (int64_t)b * a.sB + (int64_t)gr * a.ldb + gk, 1, a.batch * a.sB) &&
                 DMUON_IN(a.status, gk, 1, a.ldb))
                    ? ld<TB, COH>(B, (int64_t)gr * a.ldb + gk)
                    : 0.f;
      }
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int e = 0; e < 8; ++e) As[buf][akq + e][arow] = ra[e];
    if (MODE == kApply) {
#pragma unroll
      for (int e = 0; e < 8; ++e) Bs[buf][bkk][bjq + e] = rb[e];
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) Bs[buf][akq + e][arow] = rb[e];
    }
  };

  fetch(0);
  stash(0);
  __syncthreads();
  int slices = 0;
  for (int k0 = 0, cur = 0; k0 < a.k; k0 += SK, cur ^= 1) {
    const bool more = k0 + SK < a.k;
    if (more) fetch(k0 + SK);  // in flight while this slice is multiplied
#pragma unroll
    for (int kk = 0; kk < SK; ++kk) {
      // 16-byte shared-memory loads (rows of 68 floats keep them aligned)
      const float4 a4 = *reinterpret_cast<const float4*>(&As[cur][kk][ty * 4]);
      const float4 b4 = *reinterpret_cast<const float4*>(&Bs[cur][kk][tx * 4]);
      const float av[4] = {a4.x, a4.y, a4.z, a4.w};
      const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = fmaf(av[i], bv[j], part[i][j]);
    }
    if (++slices == kBlockSlices || !more) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] += part[i][j];
          part[i][j] = 0.f;
        }
      slices = 0;
    }
    if (more) stash(cur ^ 1);  // every thread finished the other buffer at the last barrier
    __syncthreads();
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
        v = fmaf(a.p1, acc[i][j], a.p0 * ld<TE, COH>(Em, (int64_t)r * a.lde + c));
      } else {
        v = alpha * fmaf(a.p0, ld<TE, COH>(Em, (int64_t)r * a.lde + c), acc[i][j]);
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

template <typename TA, typename TB, typename TE, typename TC, int MODE>
__global__ void __launch_bounds__(kThreads) k_simt(const SimtArgs a) {
  __shared__ __align__(16) float As[2][SK][SB + 4];
  __shared__ __align__(16) float Bs[2][SK][SB + 4];
  simt_tile<TA, TB, TE, TC, MODE, false>(a, blockIdx.x, blockIdx.y, As, Bs);
}

// ------------------------------------------------------------ fused chain
// The whole FFMA chain of a chunk in one launch: every product of every
// iteration forms one tile list, phase by phase, matrix by matrix.  A CTA
// claims the next tile index from a global counter, waits (thread 0,
// acquire, bounded) until its matrix's counter shows every tile of the
// earlier phases done, computes the tile exactly as the per-product kernel
// would, and adds 1 (release) to the counter.  Tiles are claimed in order by
// running CTAs only, so the smallest unfinished tile can always proceed.  The
// small chains this path serves (fp32, small near-square bf16) otherwise pay
// one launch per product for a few dozen tiles each.
constexpr int kMaxSimtPhases = 48;
struct SimtPhase {
  SimtArgs a;
  int mode;
  int tile_start;  // global index of the phase's first tile
  uint32_t dep;    // counter value (per matrix) the phase's tiles wait for
};
struct SimtChain {
  SimtPhase ph[kMaxSimtPhases];
  unsigned* counters;  // one per matrix, then the tile counter; zero at launch
  int* status;
  uint64_t limit_ns;
  int nphases, total_tiles, batch;
};

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait until *c >= target; false when the limit ran out (recorded as
// DMUON_ERR_TIMEOUT) or another CTA already failed.
__device__ __noinline__ bool wait_count(const unsigned* c, uint32_t target, int* status, uint64_t limit_ns) {
  if (ld_acquire_u32(c) >= target) return true;
  const uint64_t t0 = global_timer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
      if (ld_acquire_u32(c) >= target) return true;
      __nanosleep(64);
    }
    if (*reinterpret_cast<volatile int*>(status) != 0) return false;
    if (global_timer() - t0 > limit_ns) {
      atomicCAS(status, 0, (int)DMUON_ERR_TIMEOUT);
      return false;
    }
  }
}

// XT: element type of X (fp32, or bf16 for thin bf16 matrices)
template <typename XT>
__global__ void __launch_bounds__(kThreads) k_simt_chain(const __grid_constant__ SimtChain P) {
  __shared__ __align__(16) float As[2][SK][SB + 4];
  __shared__ __align__(16) float Bs[2][SK][SB + 4];
  __shared__ int s_tile;
  unsigned* next = P.counters + P.batch;
  while (true) {
    if (threadIdx.x == 0) {
      int t = (int)atomicAdd(next, 1u);
      if (t >= P.total_tiles) {
        t = -1;
      } else {
        int j = 0;
        while (j + 1 < P.nphases && t >= P.ph[j + 1].tile_start) ++j;
        const int b = (t - P.ph[j].tile_start) / P.ph[j].a.tiles_per_mat;
        if (P.ph[j].dep != 0 && !wait_count(P.counters + b, P.ph[j].dep, P.status, P.limit_ns)) t = -1;
      }
      s_tile = t;
    }
    __syncthreads();
    const int t = s_tile;
    if (t < 0) break;
    int j = 0;
    while (j + 1 < P.nphases && t >= P.ph[j + 1].tile_start) ++j;
    const int mode = P.ph[j].mode;
    const SimtArgs a = P.ph[j].a;  // local: stores below must not force reloads
    const int local = t - P.ph[j].tile_start;
    const int b = local / a.tiles_per_mat;
    const int tile = local - b * a.tiles_per_mat;
    if (mode == kGram)
      simt_tile<XT, XT, float, float, kGram, true>(a, tile, b, As, Bs);
    else if (mode == kPoly)
      simt_tile<float, float, float, float, kPoly, true>(a, tile, b, As, Bs);
    else
      simt_tile<float, XT, XT, XT, kApply, true>(a, tile, b, As, Bs);
    __syncthreads();  // every store of the tile issued
    if (threadIdx.x == 0) {
      __threadfence();
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(P.counters + b) : "memory");
    }
  }
}

int tri_tiles(int m) {
  const int t = (m + SB - 1) / SB;
  return t * (t + 1) / 2;
}

SimtArgs gram_sargs(const void* X, void* G, int batch, int m, int n, int64_t ldx, int64_t ldg, float alpha,
                    const float* scale, int* status) {
  SimtArgs a{};
  a.batch = batch; a.status = status;
  a.A = X; a.B = X; a.E = nullptr; a.C = G;
  a.sA = a.sB = (int64_t)m * ldx; a.sC = (int64_t)m * ldg;
  a.lda = a.ldb = ldx; a.ldc = ldg;
  a.m = m; a.n = m; a.k = n;
  a.p0 = alpha; a.scale = scale;
  a.tiles_per_mat = tri_tiles(m);
  return a;
}

SimtArgs poly_sargs(const void* G, void* P, int batch, int m, int64_t ldg, int64_t ldp, float b, float c,
                    int* status) {
  SimtArgs a{};
  a.batch = batch; a.status = status;
  a.A = G; a.B = G; a.E = G; a.C = P;
  a.sA = a.sB = a.sE = (int64_t)m * ldg; a.sC = (int64_t)m * ldp;
  a.lda = a.ldb = a.lde = ldg; a.ldc = ldp;
  a.m = m; a.n = m; a.k = m;
  a.p0 = b; a.p1 = c;
  a.tiles_per_mat = tri_tiles(m);
  return a;
}

SimtArgs apply_sargs(const void* P, const void* X, void* Y, int batch, int m, int n, int64_t ldp, int64_t ldx,
                     int64_t ldy, float a_coef, float alpha, const float* scale, int* status) {
  SimtArgs a{};
  a.batch = batch; a.status = status;
  a.A = P; a.B = X; a.E = X; a.C = Y;
  a.sA = (int64_t)m * ldp; a.sB = a.sE = (int64_t)m * ldx; a.sC = (int64_t)m * ldy;
  a.lda = ldp; a.ldb = a.lde = ldx; a.ldc = ldy;
  a.m = m; a.n = n; a.k = m;
  a.p0 = a_coef; a.p1 = alpha; a.scale = scale;
  a.tiles_n = (n + SB - 1) / SB;
  a.tiles_per_mat = ((m + SB - 1) / SB) * a.tiles_n;
  return a;
}

}  // namespace

cudaError_t simt_gram(const void* X, void* G, int batch, int m, int n, int64_t ldx, int64_t ldg,
                      float alpha, const float* scale, bool xbf16, cudaStream_t st, int* status) {
  if (batch == 0) return cudaSuccess;
  const SimtArgs a = gram_sargs(X, G, batch, m, n, ldx, ldg, alpha, scale, status);
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
  const SimtArgs a = poly_sargs(G, P, batch, m, ldg, ldp, b, c, status);
  dim3 grid(a.tiles_per_mat, batch);
  k_simt<float, float, float, float, kPoly><<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t simt_apply(const void* P, const void* X, void* Y, int batch, int m, int n, int64_t ldp,
                       int64_t ldx, int64_t ldy, float a_coef, float alpha, const float* scale,
                       bool xbf16, cudaStream_t st, int* status) {
  if (batch == 0) return cudaSuccess;
  const SimtArgs a = apply_sargs(P, X, Y, batch, m, n, ldp, ldx, ldy, a_coef, alpha, scale, status);
  dim3 grid(a.tiles_per_mat, batch);
  if (xbf16)
    k_simt<float, __nv_bfloat16, __nv_bfloat16, __nv_bfloat16, kApply><<<grid, kThreads, 0, st>>>(a);
  else
    k_simt<float, float, float, float, kApply><<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t simt_chain(void* const* x, void* G, void* P, int batch, int m, int n, int64_t ldx, int64_t ldg,
                       int32_t steps, const float* sched, const float* scale, bool xbf16, unsigned* counters,
                       int* status, int num_sms, bool inject_timeout, cudaStream_t st, int* result_x) {
  *result_x = 0;
  if (batch == 0 || steps == 0) return cudaSuccess;
  if (3 * steps > kMaxSimtPhases || !counters) return cudaErrorNotSupported;
  std::unique_ptr<SimtChain> C(new SimtChain());
  int j = 0;
  int64_t tiles = 0, per_matrix = 0;
  auto add = [&](const SimtArgs& a, int mode) {
    SimtPhase& ph = C->ph[j++];
    ph.a = a;
    ph.mode = mode;
    ph.tile_start = (int)tiles;
    ph.dep = (uint32_t)per_matrix;  // one increment per finished tile
    tiles += (int64_t)a.tiles_per_mat * batch;
    per_matrix += a.tiles_per_mat;
  };
  int cur = 0;
  for (int k = 0; k < steps; ++k) {
    const float* sc = k == 0 ? scale : nullptr;
    const float* c = sched + 3 * k;
    add(gram_sargs(x[cur], G, batch, m, n, ldx, ldg, 1.f, sc, status), kGram);
    add(poly_sargs(G, P, batch, m, ldg, ldg, c[1], c[2], status), kPoly);
    add(apply_sargs(P, x[cur], x[1 - cur], batch, m, n, ldg, ldx, ldx, c[0], 1.f, sc, status), kApply);
    cur = 1 - cur;
  }
  if (tiles > 0x7fffffff) return cudaErrorNotSupported;
  C->nphases = j;
  C->total_tiles = (int)tiles;
  C->counters = counters;
  C->status = status;
  C->batch = batch;
  C->limit_ns = 4000000000ull;
  if (inject_timeout) {
    C->ph[j - 1].dep += 1;  // never met: the last phase's waits run out
    C->limit_ns = 20000000ull;
  }
  *result_x = cur;
  cudaError_t e = cudaMemsetAsync(counters, 0, (size_t)(batch + 1) * sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = xbf16 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_simt_chain<__nv_bfloat16>, kThreads, 0)
            : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_simt_chain<float>, kThreads, 0);
  if (e != cudaSuccess || per_sm <= 0) {
    cudaGetLastError();
    per_sm = 1;
  }
  // no more CTAs than the largest product has tiles: the rest would only wait
  int64_t widest = 0;
  for (int i = 0; i < j; ++i) {
    const int64_t w = (int64_t)C->ph[i].a.tiles_per_mat * batch;
    widest = w > widest ? w : widest;
  }
  const int64_t most = (int64_t)num_sms * per_sm;
  const int grid = (int)(widest < most ? widest : most);
  if (xbf16)
    k_simt_chain<__nv_bfloat16><<<grid, kThreads, 0, st>>>(*C);
  else
    k_simt_chain<float><<<grid, kThreads, 0, st>>>(*C);
  return cudaGetLastError();
}

}  // namespace dmuon
