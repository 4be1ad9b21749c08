// FFMA (CUDA-core) kernels of the Gram Newton-Schulz chain.
//
// Used for the fp32 dtype (the tensor cores have no fp32-exact product; tf32
// would lose the 1e-4 budget), for small near-square bf16 matrices (min side
// < 256, max side < 3 x min), whose X, G and p(G) stay in fp32, and for thin
// bf16 matrices (min side <= 64) too wide for the clustered kernel, whose G
// and p(G) stay in fp32: bf16 rounding of G and p(G) alone exceeds the error
// budget at those sizes.  The three kernels are the three products
// of one iteration (Gram Newton-Schulz, as the DMuon FAQ's related-work
// entry names the default "gram" backend):
//   gram:  G = alpha * X X^T           (one triangle of tiles, mirrored)
//   poly:  P = b G + c G G             (G symmetric, so G G = G G^T)
//   apply: Y = alpha * (a X + P X)
// Output tiles of 64 x 64 (256 threads, a 4 x 4 register tile each, k in
// slices of 32) or, for chains too small to fill the GPU with those, 32 x 32
// (128 threads, 2 x 4 each, slices of 64: four times the tiles).  fp32
// accumulation in a fixed order, blocked: each run of 256 k is summed on its
// own and then added to the total, so the rounding error grows with
// 256 + k / 256 rather than k (a 1 x 2^20 fp32 vector: 6e-4 relative error
// unblocked, well inside 1e-4 blocked).  For k <= 256 the result is the plain
// running sum.  Every output element is the same sum in the same order
// whatever the tile shape, so both shapes give the same bits.
#include <algorithm>
#include <cstdlib>
#include <memory>

#include "common.cuh"
#include "internal.h"

namespace dmuon {
namespace {

// BM x BM output tiles, THREADS threads with an RM x 4 register tile each,
// k in slices of SK.  Operands move from global memory in runs of 16 bytes
// (4 fp32 or 8 bf16 elements) along their contiguous dimension; run s of a
// thread is number tid + THREADS * s of the slice, so a warp reads whole
// 64- to 256-byte row segments.
template <int BM_, int THREADS_, int RM_, int SK_>
struct SimtCfg {
  static constexpr int BM = BM_, kThreads = THREADS_, RM = RM_, RN = 4, SK = SK_;
  static constexpr int TX = BM / RN;               // threads across a tile's columns
  static constexpr int kBlockSlices = 256 / SK;    // slices per accumulation block (256 k)
  static constexpr int kPerThread = BM * SK / kThreads;  // elements of each operand per slice
  static constexpr int kPitch = BM + 4;            // floats per shared-memory row
  static_assert((kThreads / TX) * RM == BM, "register tiles cover the output tile");
  static_assert(256 % SK == 0 && BM % 4 == 0, "slices divide the accumulation block");
};
using Wide = SimtCfg<64, 256, 4, 32>;
using Narrow = SimtCfg<32, 128, 2, 64>;

enum { kGram = 0, kPoly = 1, kApply = 2 };

struct SimtArgs {
  const void* A;    // left operand rows (X for gram, G for poly, P for apply)
  const void* B;    // right operand (X for gram, G for poly, X for apply)
  const void* E;    // epilogue operand (G for poly, X for apply)
  void* C;          // output
  int64_t sA, sB, sE, sC;  // batch strides (elements)
  int64_t lda, ldb, ldc, lde;
  int m, n, k;      // output m x n, reduction length k
  float p0, p1;     // gram: alpha; poly: b, c; apply: a, alpha
  const float* scale;
  int tiles_n, tiles_per_mat;
  int batch;
  int vec;          // bit 0: A, bit 1: B start every 16-byte run on a 16-byte boundary
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

// One 16-byte run (4 fp32 or 8 bf16 elements) at p, 16-byte aligned, as fp32.
template <typename T, bool COH>
__device__ __forceinline__ void ld_run(const T* p, float* v) {
  if constexpr (sizeof(T) == 4) {
    const float4 f = COH ? __ldcg(reinterpret_cast<const float4*>(p)) : *reinterpret_cast<const float4*>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  } else {
    const uint4 u = COH ? __ldcg(reinterpret_cast<const uint4*>(p)) : *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
}

// Fetches this thread's runs of the NR x NC region at (r0, c0) of the
// row-major operand M (leading dimension ldm, rows x cols valid; base and
// extent locate M inside its buffer for the bounds checks of debug builds)
// into v; elements outside the valid extent read as 0.  Run s is number
// u = tid + THREADS * s of the region, at row u / (NC / R), column
// (u % (NC / R)) * R.  vec: every run may be read as one aligned 16-byte load.
template <typename T, bool COH, int NR, int NC, int THREADS>
__device__ __forceinline__ void fetch_runs(const T* M, int64_t ldm, int rows, int cols, int r0, int c0, bool vec,
                                           float* v, int* status, int64_t base, int64_t extent) {
  constexpr int R = 16 / (int)sizeof(T);
  constexpr int kRowRuns = NC / R;
  constexpr int kRuns = NR * NC / (R * THREADS);
  static_assert(kRuns * R * THREADS == NR * NC, "runs cover the region");
#pragma unroll
  for (int s = 0; s < kRuns; ++s) {
    const int u = threadIdx.x + THREADS * s;
    const int gr = r0 + u / kRowRuns, gc = c0 + (u % kRowRuns) * R;
    float* w = v + s * R;
    const int64_t off = (int64_t)gr * ldm + gc;
    if (vec && gr < rows && gc + R <= cols && DMUON_IN(status, base + off, R, extent) &&
        DMUON_IN(status, gc, R, ldm)) {
      ld_run<T, COH>(M + off, w);
    } else {
#pragma unroll
      for (int e = 0; e < R; ++e)
        w[e] = (gr < rows && gc + e < cols && DMUON_IN(status, base + off + e, 1, extent) &&
                DMUON_IN(status, gc + e, 1, ldm))
                   ? ld<T, COH>(M, off + e)
                   : 0.f;
    }
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

// Shared-memory column of tile row (or column) r in k row kk of a transposed
// (k-major) operand slice: groups of 4 consecutive rows are permuted by an
// XOR with kk / 4, so that the transposing stores of a warp spread over the
// banks while each thread's 4 (or 2) rows stay contiguous for vector reads.
template <class CFG>
__device__ __forceinline__ int swz(int kk, int r) {
  return ((((r >> 2) ^ (kk >> 2)) & (CFG::BM / 4 - 1)) << 2) | (r & 3);
}

template <class CFG>
struct SimtSmem {
  float As[2][CFG::SK][CFG::kPitch];
  float Bs[2][CFG::SK][CFG::kPitch];
};

// Transposing store of this thread's runs of a k-contiguous BM x SK slice
// (fetched by fetch_runs with runs of R elements): element (row r, k kk)
// goes to [kk][swz(kk, r)].
template <class CFG, int R>
__device__ __forceinline__ void stash_t(float (*S)[CFG::kPitch], const float* v) {
  constexpr int kRowRuns = CFG::SK / R;
#pragma unroll
  for (int e = 0; e < CFG::kPerThread; ++e) {
    const int u = threadIdx.x + CFG::kThreads * (e / R);
    const int r = u / kRowRuns, kk = (u % kRowRuns) * R + e % R;
    S[kk][swz<CFG>(kk, r)] = v[e];
  }
}

// One BM x BM output tile `tile` of matrix b (all threads of the CTA).  The k
// loop runs over slices in two shared-memory buffers: the next slice's global
// loads are issued before the current slice is multiplied, so their latency
// overlaps the arithmetic (one barrier per slice).  Each thread keeps an
// RM x 4 register tile and adds k in ascending order, in blocks of 256.
template <class CFG, typename TA, typename TB, typename TE, typename TC, int MODE, bool COH>
__device__ __forceinline__ void simt_tile(const SimtArgs& a, int tile, int b, SimtSmem<CFG>& sm) {
  constexpr int BM = CFG::BM, SK = CFG::SK, RM = CFG::RM, T = CFG::kThreads, PT = CFG::kPerThread;
  int ti, tj;
  if (MODE == kApply) {
    ti = tile / a.tiles_n;
    tj = tile % a.tiles_n;
  } else {
    tri_decode(tile, ti, tj);
  }
  const int i0 = ti * BM, j0 = tj * BM;
  const TA* A = static_cast<const TA*>(a.A) + (int64_t)b * a.sA;
  const TB* B = static_cast<const TB*>(a.B) + (int64_t)b * a.sB;
  const int tid = threadIdx.x;
  const int ty = tid / CFG::TX, tx = tid % CFG::TX;
  float acc[RM][4], part[RM][4];
#pragma unroll
  for (int i = 0; i < RM; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = part[i][j] = 0.f;

  // A: rows i0.. of a row-major m x k operand (k contiguous); B: rows j0.. of
  // the same kind (gram, poly), or (apply) a k x n row-major operand
  const bool vecA = a.vec & 1, vecB = (a.vec >> 1) & 1;
  const int arows = a.m, brows = MODE == kApply ? a.k : a.n;
  float ra[PT], rb[PT];
  auto fetch = [&](int k0) {
    fetch_runs<TA, COH, BM, SK, T>(A, a.lda, arows, a.k, i0, k0, vecA, ra, a.status, (int64_t)b * a.sA,
                                   (int64_t)a.batch * a.sA);
    if (MODE == kApply)
      fetch_runs<TB, COH, SK, BM, T>(B, a.ldb, brows, a.n, k0, j0, vecB, rb, a.status, (int64_t)b * a.sB,
                                     (int64_t)a.batch * a.sB);
    else
      fetch_runs<TB, COH, BM, SK, T>(B, a.ldb, brows, a.k, j0, k0, vecB, rb, a.status, (int64_t)b * a.sB,
                                     (int64_t)a.batch * a.sB);
  };
  auto stash = [&](int buf) {
    stash_t<CFG, 16 / (int)sizeof(TA)>(sm.As[buf], ra);
    if (MODE == kApply) {  // already k-major: 16-byte stores of whole runs
      constexpr int R = 16 / (int)sizeof(TB);
#pragma unroll
      for (int e = 0; e < PT; e += 4) {
        const int u = tid + T * (e / R);
        const int kk = u / (BM / R), c = (u % (BM / R)) * R + e % R;
        *reinterpret_cast<float4*>(&sm.Bs[buf][kk][c]) = make_float4(rb[e], rb[e + 1], rb[e + 2], rb[e + 3]);
      }
    } else {
      stash_t<CFG, 16 / (int)sizeof(TB)>(sm.Bs[buf], rb);
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
      float av[RM], bv[4];
      if constexpr (RM == 4) {
        const float4 a4 = *reinterpret_cast<const float4*>(&sm.As[cur][kk][swz<CFG>(kk, ty * 4)]);
        av[0] = a4.x; av[1] = a4.y; av[2] = a4.z; av[3] = a4.w;
      } else {
        const float2 a2 = *reinterpret_cast<const float2*>(&sm.As[cur][kk][swz<CFG>(kk, ty * 2)]);
        av[0] = a2.x; av[1] = a2.y;
      }
      const float4 b4 = *reinterpret_cast<const float4*>(
          &sm.Bs[cur][kk][MODE == kApply ? tx * 4 : swz<CFG>(kk, tx * 4)]);
      bv[0] = b4.x; bv[1] = b4.y; bv[2] = b4.z; bv[3] = b4.w;
#pragma unroll
      for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = fmaf(av[i], bv[j], part[i][j]);
    }
    if (++slices == CFG::kBlockSlices || !more) {
#pragma unroll
      for (int i = 0; i < RM; ++i)
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
  for (int i = 0; i < RM; ++i) {
    const int r = i0 + ty * RM + i;
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
__global__ void __launch_bounds__(Wide::kThreads) k_simt(const SimtArgs a) {
  __shared__ __align__(16) SimtSmem<Wide> sm;
  simt_tile<Wide, TA, TB, TE, TC, MODE, false>(a, blockIdx.x, blockIdx.y, sm);
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

// XT: element type of X (fp32, or bf16 for thin bf16 matrices); CFG: tile shape
template <typename XT, class CFG>
__global__ void __launch_bounds__(CFG::kThreads) k_simt_chain(const __grid_constant__ SimtChain P) {
  __shared__ __align__(16) SimtSmem<CFG> sm;
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
      simt_tile<CFG, XT, XT, float, float, kGram, true>(a, tile, b, sm);
    else if (mode == kPoly)
      simt_tile<CFG, float, float, float, float, kPoly, true>(a, tile, b, sm);
    else
      simt_tile<CFG, float, XT, XT, XT, kApply, true>(a, tile, b, sm);
    __syncthreads();  // every store of the tile issued
    if (threadIdx.x == 0) {
      __threadfence();
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(P.counters + b) : "memory");
    }
  }
}

int tri_tiles(int m, int bm) {
  const int t = (m + bm - 1) / bm;
  return t * (t + 1) / 2;
}

// Every 16-byte run of an operand (element size sz, leading dimension ld,
// batch stride st, runs starting at multiples of 16 bytes within a row)
// starts on a 16-byte boundary.
bool runs_aligned(const void* p, int64_t ld, int64_t st, int64_t sz) {
  return reinterpret_cast<uintptr_t>(p) % 16 == 0 && (ld * sz) % 16 == 0 && (st * sz) % 16 == 0;
}

SimtArgs gram_sargs(const void* X, void* G, int batch, int m, int n, int64_t ldx, int64_t ldg, float alpha,
                    const float* scale, int64_t xsz, int bm, int* status) {
  SimtArgs a{};
  a.batch = batch; a.status = status;
  a.A = X; a.B = X; a.E = nullptr; a.C = G;
  a.sA = a.sB = (int64_t)m * ldx; a.sC = (int64_t)m * ldg;
  a.lda = a.ldb = ldx; a.ldc = ldg;
  a.m = m; a.n = m; a.k = n;
  a.p0 = alpha; a.scale = scale;
  a.tiles_per_mat = tri_tiles(m, bm);
  a.vec = runs_aligned(X, ldx, a.sA, xsz) ? 3 : 0;
  return a;
}

SimtArgs poly_sargs(const void* G, void* P, int batch, int m, int64_t ldg, int64_t ldp, float b, float c,
                    int bm, int* status) {
  SimtArgs a{};
  a.batch = batch; a.status = status;
  a.A = G; a.B = G; a.E = G; a.C = P;
  a.sA = a.sB = a.sE = (int64_t)m * ldg; a.sC = (int64_t)m * ldp;
  a.lda = a.ldb = a.lde = ldg; a.ldc = ldp;
  a.m = m; a.n = m; a.k = m;
  a.p0 = b; a.p1 = c;
  a.tiles_per_mat = tri_tiles(m, bm);
  a.vec = runs_aligned(G, ldg, a.sA, 4) ? 3 : 0;
  return a;
}

SimtArgs apply_sargs(const void* P, const void* X, void* Y, int batch, int m, int n, int64_t ldp, int64_t ldx,
                     int64_t ldy, float a_coef, float alpha, const float* scale, int64_t xsz, int bm,
                     int* status) {
  SimtArgs a{};
  a.batch = batch; a.status = status;
  a.A = P; a.B = X; a.E = X; a.C = Y;
  a.sA = (int64_t)m * ldp; a.sB = a.sE = (int64_t)m * ldx; a.sC = (int64_t)m * ldy;
  a.lda = ldp; a.ldb = a.lde = ldx; a.ldc = ldy;
  a.m = m; a.n = n; a.k = m;
  a.p0 = a_coef; a.p1 = alpha; a.scale = scale;
  a.tiles_n = (n + bm - 1) / bm;
  a.tiles_per_mat = ((m + bm - 1) / bm) * a.tiles_n;
  a.vec = (runs_aligned(P, ldp, a.sA, 4) ? 1 : 0) | (runs_aligned(X, ldx, a.sB, xsz) ? 2 : 0);
  return a;
}

// Chains whose widest product has fewer 64 x 64 tiles than the GPU has SMs
// run 32 x 32 tiles (DMUON_FFMA_TILE=64 or =32 forces one shape).
bool narrow_chain(int batch, int m, int n, int num_sms) {
  if (const char* v = std::getenv("DMUON_FFMA_TILE")) {
    if (v[0] == '6') return false;
    if (v[0] == '3') return true;
  }
  const int64_t t = (m + Wide::BM - 1) / Wide::BM, u = (n + Wide::BM - 1) / Wide::BM;
  return t * u * batch < num_sms;
}

template <class CFG, typename XT>
cudaError_t launch_chain(const SimtChain& C, int64_t widest, int num_sms, cudaStream_t st) {
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_simt_chain<XT, CFG>, CFG::kThreads, 0);
  if (e != cudaSuccess || per_sm <= 0) {
    cudaGetLastError();
    per_sm = 1;
  }
  // no more CTAs than the largest product has tiles: the rest would only wait
  const int64_t most = (int64_t)num_sms * per_sm;
  const int grid = (int)(widest < most ? widest : most);
  k_simt_chain<XT, CFG><<<grid, CFG::kThreads, 0, st>>>(C);
  return cudaGetLastError();
}

}  // namespace

cudaError_t simt_gram(const void* X, void* G, int batch, int m, int n, int64_t ldx, int64_t ldg,
                      float alpha, const float* scale, bool xbf16, cudaStream_t st, int* status) {
  if (batch == 0) return cudaSuccess;
  const SimtArgs a = gram_sargs(X, G, batch, m, n, ldx, ldg, alpha, scale, xbf16 ? 2 : 4, Wide::BM, status);
  dim3 grid(a.tiles_per_mat, batch);
  if (xbf16)
    k_simt<__nv_bfloat16, __nv_bfloat16, float, float, kGram><<<grid, Wide::kThreads, 0, st>>>(a);
  else
    k_simt<float, float, float, float, kGram><<<grid, Wide::kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t simt_poly(const void* G, void* P, int batch, int m, int64_t ldg, int64_t ldp, float b,
                      float c, cudaStream_t st, int* status) {
  if (batch == 0) return cudaSuccess;
  const SimtArgs a = poly_sargs(G, P, batch, m, ldg, ldp, b, c, Wide::BM, status);
  dim3 grid(a.tiles_per_mat, batch);
  k_simt<float, float, float, float, kPoly><<<grid, Wide::kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t simt_apply(const void* P, const void* X, void* Y, int batch, int m, int n, int64_t ldp,
                       int64_t ldx, int64_t ldy, float a_coef, float alpha, const float* scale,
                       bool xbf16, cudaStream_t st, int* status) {
  if (batch == 0) return cudaSuccess;
  const SimtArgs a =
      apply_sargs(P, X, Y, batch, m, n, ldp, ldx, ldy, a_coef, alpha, scale, xbf16 ? 2 : 4, Wide::BM, status);
  dim3 grid(a.tiles_per_mat, batch);
  if (xbf16)
    k_simt<float, __nv_bfloat16, __nv_bfloat16, __nv_bfloat16, kApply><<<grid, Wide::kThreads, 0, st>>>(a);
  else
    k_simt<float, float, float, float, kApply><<<grid, Wide::kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t simt_chain(void* const* x, void* G, void* P, int batch, int m, int n, int64_t ldx, int64_t ldg,
                       int32_t steps, const float* sched, const float* scale, bool xbf16, unsigned* counters,
                       int* status, int num_sms, bool inject_timeout, cudaStream_t st, int* result_x) {
  *result_x = 0;
  if (batch == 0 || steps == 0) return cudaSuccess;
  if (3 * steps > kMaxSimtPhases || !counters) return cudaErrorNotSupported;
  const bool narrow = narrow_chain(batch, m, n, num_sms);
  const int bm = narrow ? Narrow::BM : Wide::BM;
  const int64_t xsz = xbf16 ? 2 : 4;
  std::unique_ptr<SimtChain> C(new SimtChain());
  int j = 0;
  int64_t tiles = 0, per_matrix = 0, widest = 0;
  auto add = [&](const SimtArgs& a, int mode) {
    SimtPhase& ph = C->ph[j++];
    ph.a = a;
    ph.mode = mode;
    ph.tile_start = (int)tiles;
    ph.dep = (uint32_t)per_matrix;  // one increment per finished tile
    tiles += (int64_t)a.tiles_per_mat * batch;
    per_matrix += a.tiles_per_mat;
    widest = std::max(widest, (int64_t)a.tiles_per_mat * batch);
  };
  int cur = 0;
  for (int k = 0; k < steps; ++k) {
    const float* sc = k == 0 ? scale : nullptr;
    const float* c = sched + 3 * k;
    add(gram_sargs(x[cur], G, batch, m, n, ldx, ldg, 1.f, sc, xsz, bm, status), kGram);
    add(poly_sargs(G, P, batch, m, ldg, ldg, c[1], c[2], bm, status), kPoly);
    add(apply_sargs(P, x[cur], x[1 - cur], batch, m, n, ldg, ldx, ldx, c[0], 1.f, sc, xsz, bm, status), kApply);
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
  if (narrow)
    return xbf16 ? launch_chain<Narrow, __nv_bfloat16>(*C, widest, num_sms, st)
                 : launch_chain<Narrow, float>(*C, widest, num_sms, st);
  return xbf16 ? launch_chain<Wide, __nv_bfloat16>(*C, widest, num_sms, st)
               : launch_chain<Wide, float>(*C, widest, num_sms, st);
}

}  // namespace dmuon
