// tcgen05 tensor-core kernels of the Gram Newton-Schulz chain (sm_100a).
//
// One iteration of Gram Newton-Schulz (the DMuon FAQ's related-work entry
// for the default "gram" backend; Training Guide, ns_steps / ns_backend
// rows) is three products over an m x n matrix X (m <= n):
//   gram:  G = alpha X X^T        m x m, K = n   (symmetric: one triangle)
//   poly:  P = b G + c G G        m x m, K = m   (G symmetric => G G = G G^T,
//                                                  one triangle again)
// The poly kernel is the general symmetric product C = p1 (A B) + p0 E + p2 I
// for symmetric, commuting A and B (so A B is symmetric and B's rows are its
// columns): the Gram-space form of the chain multiplies polynomials of one
// Gram matrix this way.
//   apply: Y = alpha (a X + P X)  m x n, K = m   (X is the MN-major operand)
//
// Two kernels share the tile decode and the epilogue:
//
// k_tc2 (m >= 256): a CTA pair (cluster of 2) computes 256 x 256 tiles with
//   tcgen05.mma.cta_group::2 (M=256, N=256, K=16).  Each CTA stages its own
//   128 rows of A and its own 128 columns of B (6 stages of 32 KB), so every
//   byte brought into shared memory feeds twice the MMA work of a one-CTA
//   128 x 256 tile.  Both CTAs' TMA copies complete on the leader CTA's
//   full barrier (mapa address, .cta_group::2 copies); the leader's single
//   MMA thread issues the pair's MMAs and its commits multicast to both CTAs'
//   stage-release and accumulator-ready barriers; each CTA's epilogue reads
//   its own 128 TMEM lanes and reports back to the leader.
// k_tc (m < 256): one CTA per SM, 128 x 256 tiles, tcgen05.mma.cta_group::1
//   (M=128), 4 stages of 48 KB.
//
// Both are persistent (one CTA, or CTA pair, per SM / SM pair), warp
// specialised (warp 0 TMA producer, warp 1 TMEM allocator + single MMA
// thread, warps 2-5 epilogue), with two TMEM accumulators (2 x 256 fp32
// columns) so the epilogue of one tile overlaps the MMAs of the next.  The
// polynomial terms (alpha, b G, a X) are fused into the epilogue.  For gram
// and poly only tiles that touch the lower triangle are computed; every
// element r >= c is stored, and r > c also at its mirror (c, r), so each
// element is written exactly once and G, P are exactly symmetric.
//
// Every mbarrier wait is bounded (%globaltimer); a wait that runs out records
// DMUON_ERR_TIMEOUT in the status word, the CTA waits (bounded) for its own
// copies and MMAs in flight, frees its TMEM and exits.  No TMA load uses
// cluster multicast.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bounds.cuh"
#include "internal.h"

namespace dmuon {
namespace {

constexpr int BN = 256;
constexpr int BK = 64;  // 64 bf16 = one 128-byte swizzle row
constexpr int UK = 16;  // K of one tcgen05.mma kind::f16
constexpr int TMEM_COLS = 2 * BN;
constexpr int kThreads = 192;
constexpr uint64_t kTimeoutNs = 4000000000ull;  // 4 s per wait

// one-CTA kernel
constexpr int BM1 = 128;
constexpr int STAGES1 = 4;
constexpr int A1_BYTES = BM1 * BK * 2;   // 16 KB
constexpr int B1_BYTES = BN * BK * 2;    // 32 KB
constexpr int STAGE1_BYTES = A1_BYTES + B1_BYTES;
// CTA-pair kernel (per CTA: 128 rows of A, 128 columns of B)
constexpr int BM2 = 256;
constexpr int STAGES2 = 6;
constexpr int A2_BYTES = 128 * BK * 2;   // 16 KB
constexpr int B2_BYTES = 128 * BK * 2;   // 16 KB
constexpr int STAGE2_BYTES = A2_BYTES + B2_BYTES;

constexpr int kMaxStages = STAGES2 > STAGES1 ? STAGES2 : STAGES1;
constexpr int kBarriers = 2 * kMaxStages + 2 + 2 + 1;
constexpr int SMEM1_BYTES = STAGES1 * STAGE1_BYTES + 1024 + 256;
constexpr int SMEM2_BYTES = STAGES2 * STAGE2_BYTES + 1024 + 256;

enum { kGram = 0, kPoly = 1, kApply = 2 };

// The update table is a kernel parameter only of the fused apply + update
// instantiation; the others take an empty one.
struct NoUpd {};
template <bool UPD> struct UpdSel { using type = NoUpd; };
template <> struct UpdSel<true> { using type = UpdTable; };

struct TcArgs {
  __nv_bfloat16* C;
  const __nv_bfloat16* E;
  int64_t sC, sE, ldc, lde;
  int m, n, k;
  int tm;  // tile rows: 128 (one CTA) or 256 (CTA pair)
  int tiles_m, tiles_n, tiles_per_mat, total_tiles;
  float p0, p1, p2;  // gram: alpha; poly: p1 (A B) + p0 E + p2 I; apply: alpha (p0 X + P X)
  const float* scale;
  int* status;
};

// Matrices in the launch (extent checks of debug builds).
[[maybe_unused]] __device__ __forceinline__ int64_t batch_of(const TcArgs& a) { return a.total_tiles / a.tiles_per_mat; }

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// arrive on a barrier given by its shared::cluster address (own or peer CTA)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; false when the limit ran out or another thread already failed.
__device__ __noinline__ bool wait_bar_limit(uint32_t bar, uint32_t parity, int* status, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 128; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile int*>(status) != 0) return false;
    if (global_timer() - t0 > limit_ns) {
      atomicCAS(status, 0, (int)DMUON_ERR_TIMEOUT);
      return false;
    }
  }
}
// The common case (the phase already completed) stays inline: one poll, no
// call; only a wait that has to spin goes to the bounded loop.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_bar_limit(bar, parity, status, kTimeoutNs);
}

// Self-test of the bounded wait: one thread waits on a barrier that nothing
// arrives on; the wait gives up after limit_ns and records the timeout.
__global__ void k_wait_selftest(int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  wait_bar_limit(b, 0, status, limit_ns);
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// CTA-pair copy into this CTA's shared memory, completing on the barrier at
// `bar_cluster` (the leader CTA's full barrier).
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
template <int G>
__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t cols) {
  if (G == 1)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(cols));
  else
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(cols));
}
template <int G>
__device__ __forceinline__ void tmem_relinquish() {
  if (G == 1)
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  else
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
}
template <int G>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  if (G == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols));
  else
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols));
}
template <int G>
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  if (G == 1)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
// Completion of this thread's prior MMAs arrives on `bar` (own CTA) ...
template <int G>
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  if (G == 1)
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
  else
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
// ... or on the barrier at the same offset in every CTA of `mask`.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          bar),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 layout: start
// address, leading and stride byte offsets in 16-byte units, version 1 at
// bit 46, swizzle mode 2 at bits 61-63).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Instruction descriptor, kind::f16: fp32 D, bf16 A and B, A K-major,
// B K-major or MN-major, N = 256, M = 128 (one CTA) or 256 (CTA pair).
__host__ __device__ constexpr uint32_t make_idesc(bool b_mn_major, int M) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Tile t -> (matrix b, row block I, column block J).
template <int MODE>
__device__ __forceinline__ void decode_tile(const TcArgs& a, int t, int& b, int& I, int& J) {
  b = t / a.tiles_per_mat;
  int l = t - b * a.tiles_per_mat;
  if (MODE == kApply) {
    // column panels of X outermost, so concurrently running CTAs share them
    I = l % a.tiles_m;
    J = l / a.tiles_m;
  } else {
    // row block i holds the column blocks that reach the diagonal
    int i = 0;
    while (true) {
      const int c = min(a.tiles_n, (i * a.tm + a.tm - 1) / BN + 1);
      if (l < c) break;
      l -= c;
      ++i;
    }
    I = i;
    J = l;
  }
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& raw, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 v = __bfloat1622float2(h[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}
__device__ __forceinline__ uint4 pack_bf16x8(const float* f) {
  uint4 raw;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return raw;
}

// Fused update, one 32-column chunk of oriented row r (< m), columns c0 ..
// c0 + 31 (< n) of matrix b: p <- bf16(p * decay - step_scale * bf16(v)).
// Non-transposed rows are contiguous runs of p; transposed ones are a column
// of p, and across the warp (consecutive r) each j is one 64-byte run.  The
// parameters (and the a X term) of a chunk are loaded one chunk ahead into
// packed bf16 pairs, so their latency hides behind the previous chunk.
struct UpdChunk {
  uint32_t p[16];  // 32 bf16 parameters
  uint32_t e[16];  // 32 bf16 of X (only when a != 0)
};

__device__ __forceinline__ uint32_t pack2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}
__device__ __forceinline__ float half_of(const uint32_t* w, int j) {
  const uint32_t x = w[j >> 1];
  return __uint_as_float((j & 1) ? (x & 0xffff0000u) : (x << 16));
}

__device__ __forceinline__ void load_upd_chunk(const UpdTable& u, const TcArgs& a, int b, int r, int c0,
                                               UpdChunk& k) {
  const int m = a.m, n = a.n;
  const __nv_bfloat16* p = static_cast<const __nv_bfloat16*>(u.p[b]);
  const bool tr = (u.tmask[b >> 5] >> (b & 31)) & 1u;
  const bool full = c0 + 32 <= n;
  [[maybe_unused]] const int len = full ? 32 : n - c0;
  [[maybe_unused]] const int64_t pext = (int64_t)m * n;
  if (tr) {
    const __nv_bfloat16* q = p + (int64_t)c0 * m + r;
    const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const __nv_bfloat16 lo =
          (c0 + j < n && DMUON_IN(a.status, (int64_t)(c0 + j) * m + r, 1, pext)) ? *q : z;
      q += m;
      const __nv_bfloat16 hi =
          (c0 + j + 1 < n && DMUON_IN(a.status, (int64_t)(c0 + j + 1) * m + r, 1, pext)) ? *q : z;
      q += m;
      k.p[j >> 1] = pack2(lo, hi);
    }
  } else if (!DMUON_IN(a.status, (int64_t)r * n + c0, len, pext) || !DMUON_IN(a.status, c0, len, n)) {
#pragma unroll
    for (int j = 0; j < 16; ++j) k.p[j] = 0u;
  } else if (full && ((u.vmask[b >> 5] >> (b & 31)) & 1u)) {
    const uint4* q = reinterpret_cast<const uint4*>(p + (int64_t)r * n + c0);
#pragma unroll
    for (int i = 0; i < 4; ++i) reinterpret_cast<uint4*>(k.p)[i] = q[i];
  } else {
    const __nv_bfloat16* q = p + (int64_t)r * n + c0;
    const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
#pragma unroll
    for (int j = 0; j < 32; j += 2)
      k.p[j >> 1] = pack2((c0 + j < n) ? q[j] : z, (c0 + j + 1 < n) ? q[j + 1] : z);
  }
  if (a.p0 != 0.f) {
    const __nv_bfloat16* ep = a.E + (int64_t)b * a.sE + (int64_t)r * a.lde + c0;
    if (!DMUON_IN(a.status, (int64_t)b * a.sE + (int64_t)r * a.lde + c0, len, batch_of(a) * a.sE) ||
        !DMUON_IN(a.status, c0, len, a.lde)) {
#pragma unroll
      for (int j = 0; j < 16; ++j) k.e[j] = 0u;
    } else if (full) {
#pragma unroll
      for (int i = 0; i < 4; ++i) reinterpret_cast<uint4*>(k.e)[i] = __ldg(reinterpret_cast<const uint4*>(ep) + i);
    } else {
      const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
#pragma unroll
      for (int j = 0; j < 32; j += 2)
        k.e[j >> 1] = pack2((c0 + j < n) ? ep[j] : z, (c0 + j + 1 < n) ? ep[j + 1] : z);
    }
  }
}

// v: the accumulator chunk (fp32); applies alpha (a X + .), rounds the result
// to bf16 as the plain apply would store it, and updates the parameters.
__device__ __forceinline__ void store_upd_chunk(const UpdTable& u, const TcArgs& a, int b, int r, int c0,
                                                float alpha, const UpdChunk& k, float* v) {
  const int m = a.m, n = a.n;
  if (a.p0 != 0.f) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = alpha * fmaf(a.p0, half_of(k.e, j), v[j]);
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = alpha * v[j];
  }
  float* pv = v;  // in place: v[j] becomes the new parameter
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float o = __bfloat162float(__float2bfloat16_rn(v[j]));
    pv[j] = __fsub_rn(__fmul_rn(half_of(k.p, j), u.decay), __fmul_rn(u.step_scale, o));
  }
  __nv_bfloat16* p = static_cast<__nv_bfloat16*>(u.p[b]);
  const bool tr = (u.tmask[b >> 5] >> (b & 31)) & 1u;
  [[maybe_unused]] const int64_t pext = (int64_t)m * n;
  if (tr) {
    __nv_bfloat16* q = p + (int64_t)c0 * m + r;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (c0 + j < n && DMUON_IN(a.status, (int64_t)(c0 + j) * m + r, 1, pext)) *q = __float2bfloat16_rn(pv[j]);
      q += m;
    }
  } else if (!DMUON_IN(a.status, (int64_t)r * n + c0, c0 + 32 <= n ? 32 : n - c0, pext)) {
    return;
  } else if (c0 + 32 <= n && ((u.vmask[b >> 5] >> (b & 31)) & 1u)) {
    uint4* q = reinterpret_cast<uint4*>(p + (int64_t)r * n + c0);
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = pack_bf16x8(pv + 8 * i);
  } else {
    __nv_bfloat16* q = p + (int64_t)r * n + c0;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (c0 + j < n) q[j] = __float2bfloat16_rn(pv[j]);
  }
}

// Epilogue of one apply tile with the fused update (see epilogue_row).
__device__ __forceinline__ void epilogue_row_update(const TcArgs& a, const UpdTable& u, uint32_t taddr, int b,
                                                    int r, int J) {
  const bool row_ok = r < a.m;
  const float alpha = a.p1 * (a.scale ? a.scale[b] : 1.f);
  const int cbase = J * BN;
  UpdChunk k0, k1;
  if (row_ok) load_upd_chunk(u, a, b, r, cbase, k0);
  // one chunk: load the next chunk's operands, then drain this one
  auto chunk = [&](int ch, const UpdChunk& cur, UpdChunk& nxt) -> bool {
    const int c0 = cbase + ch * 32;
    if (c0 >= a.n) return false;  // warp-uniform
    if (row_ok && ch + 1 < BN / 32 && c0 + 32 < a.n) load_upd_chunk(u, a, b, r, c0 + 32, nxt);
    uint32_t raw[32];
    tmem_ld32(taddr + (uint32_t)(ch * 32), raw);
    tmem_ld_wait();
    if (row_ok) store_upd_chunk(u, a, b, r, c0, alpha, cur, reinterpret_cast<float*>(raw));
    return true;
  };
#pragma unroll 1
  for (int ch = 0; ch < BN / 32; ch += 2) {
    if (!chunk(ch, k0, k1)) break;
    if (!chunk(ch + 1, k1, k0)) break;
  }
}

// Before an update tile's accumulator is ready: pull the parameters it
// rewrites into L2 (oriented rows [r0, r0 + 32) of this warp, columns
// [col0, col0 + 256)), so the epilogue's loads do not wait on DRAM.
__device__ __forceinline__ void prefetch_update_tile(const UpdTable& u, int b, int r0, int col0, int m, int n,
                                                     int lane) {
  const char* p = static_cast<const char*>(u.p[b]);
  const bool tr = (u.tmask[b >> 5] >> (b & 31)) & 1u;
  if (r0 >= m) return;
  if (tr) {
    // source rows col0 .. col0 + 255, 64 bytes (32 columns from r0) each: 8 per lane
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = col0 + lane * 8 + i;
      if (c < n) asm volatile("prefetch.global.L2 [%0];" ::"l"(p + ((int64_t)c * m + r0) * 2));
    }
  } else {
    // row r0 + lane, 512 bytes from col0: four 128-byte lines
    const int r = r0 + lane;
    if (r < m) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = col0 + i * 64;
        if (c < n) asm volatile("prefetch.global.L2 [%0];" ::"l"(p + ((int64_t)r * n + c) * 2));
      }
    }
  }
}

// Epilogue of one tile for one accumulator row: TMEM lane quarter `wq` of
// accumulator columns [col0, col0 + 256), output row r, output columns from
// J * 256.  Warp-collective (tcgen05.ld).  UPD (apply only): update the
// parameters instead of storing the result.
template <int MODE, bool UPD>
__device__ __forceinline__ void epilogue_row(const TcArgs& a, const typename UpdSel<UPD>::type& u, uint32_t taddr,
                                             int b, int r, int J) {
  if constexpr (UPD) {
    epilogue_row_update(a, u, taddr, b, r, J);
    return;
  }
  const bool row_ok = r < a.m;
  float alpha = 1.f;
  if (MODE == kGram) {
    const float s = a.scale ? a.scale[b] : 1.f;
    alpha = a.p0 * (s * s);
  } else if (MODE == kApply) {
    alpha = a.p1 * (a.scale ? a.scale[b] : 1.f);
  }
  __nv_bfloat16* Cm = a.C + (int64_t)b * a.sC;
  const __nv_bfloat16* Em = a.E ? a.E + (int64_t)b * a.sE : nullptr;
#pragma unroll 1
  for (int ch = 0; ch < BN / 32; ++ch) {
    const int c0 = J * BN + ch * 32;
    if (c0 >= a.n) break;  // warp-uniform
    uint32_t raw[32];
    tmem_ld32(taddr + (uint32_t)(ch * 32), raw);
    tmem_ld_wait();
    if (!row_ok) continue;
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(raw[j]);
    const bool full_chunk = c0 + 32 <= a.n;
    [[maybe_unused]] const int len = full_chunk ? 32 : a.n - c0;
    if ((MODE == kApply && a.p0 != 0.f) || (MODE == kPoly && Em != nullptr)) {
      float e[32];
      const __nv_bfloat16* ep = Em + (int64_t)r * a.lde + c0;
      if (!DMUON_IN(a.status, (int64_t)b * a.sE + (int64_t)r * a.lde + c0, len, batch_of(a) * a.sE) ||
          !DMUON_IN(a.status, c0, len, a.lde)) {
#pragma unroll
        for (int j = 0; j < 32; ++j) e[j] = 0.f;
      } else if (full_chunk) {
#pragma unroll
        for (int q = 0; q < 4; ++q) unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(ep) + q), e + 8 * q);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) e[j] = (c0 + j < a.n) ? __bfloat162float(ep[j]) : 0.f;
      }
      if (MODE == kApply) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = alpha * fmaf(a.p0, e[j], v[j]);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = fmaf(a.p1, v[j], a.p0 * e[j]);
      }
    } else if (MODE == kPoly) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = a.p1 * v[j];
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = alpha * v[j];
    }
    if (MODE == kPoly && a.p2 != 0.f && r >= c0 && r < c0 + 32) {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (c0 + j == r) v[j] += a.p2;
    }
    __nv_bfloat16* rowp = Cm + (int64_t)r * a.ldc + c0;
    if (!DMUON_IN(a.status, (int64_t)b * a.sC + (int64_t)r * a.ldc + c0, len, batch_of(a) * a.sC) ||
        !DMUON_IN(a.status, c0, len, a.ldc))
      continue;
    if (MODE == kApply) {
      if (full_chunk) {
#pragma unroll
        for (int q = 0; q < 4; ++q) reinterpret_cast<uint4*>(rowp)[q] = pack_bf16x8(v + 8 * q);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j < a.n) rowp[j] = __float2bfloat16_rn(v[j]);
      }
    } else {
      // lower triangle incl. diagonal at (r, c); strictly lower also at (c, r)
      __nv_bfloat16 h[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) h[j] = __float2bfloat16_rn(v[j]);
      if (full_chunk && r > c0 + 31) {
#pragma unroll
        for (int q = 0; q < 4; ++q) reinterpret_cast<uint4*>(rowp)[q] = pack_bf16x8(v + 8 * q);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (DMUON_IN(a.status, (int64_t)b * a.sC + (int64_t)(c0 + j) * a.ldc + r, 1, batch_of(a) * a.sC) &&
              DMUON_IN(a.status, r, 1, a.ldc))
            Cm[(int64_t)(c0 + j) * a.ldc + r] = h[j];
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int c = c0 + j;
          if (c < a.n && r >= c) {
            rowp[j] = h[j];
            if (r > c && DMUON_IN(a.status, (int64_t)b * a.sC + (int64_t)c * a.ldc + r, 1, batch_of(a) * a.sC) &&
                DMUON_IN(a.status, r, 1, a.ldc))
              Cm[(int64_t)c * a.ldc + r] = h[j];
          }
        }
      }
    }
  }
}

struct Bars {
  uint32_t full0, empty0, tfull0, tempty0, done;
};
__device__ __forceinline__ Bars bar_layout(uint64_t* bars) {
  Bars b;
  b.full0 = smem_u32(bars);
  b.empty0 = smem_u32(bars + kMaxStages);
  b.tfull0 = smem_u32(bars + 2 * kMaxStages);
  b.tempty0 = smem_u32(bars + 2 * kMaxStages + 2);
  b.done = smem_u32(bars + 2 * kMaxStages + 4);
  return b;
}

// ================================================================ one CTA
template <int MODE, bool UPD>
__global__ void __launch_bounds__(kThreads, 1)
    k_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
         const TcArgs a, const __grid_constant__ typename UpdSel<UPD>::type u) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES1 * STAGE1_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBarriers);
  const Bars B = bar_layout(bars);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES1; ++s) {
      mbar_init(B.full0 + 8 * s, 1);
      mbar_init(B.empty0 + 8 * s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(B.tfull0 + 8 * s, 1);
      mbar_init(B.tempty0 + 8 * s, 4);  // one arrival per epilogue warp
    }
    mbar_init(B.done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
  }
  if (warp == 1) {
    tmem_alloc<1>(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = (a.k + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < a.total_tiles; t += gridDim.x) {
        int b, I, J;
        decode_tile<MODE>(a, t, b, I, J);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait_bar(B.empty0 + 8 * stage, phase ^ 1u, a.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = B.full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, STAGE1_BYTES);
          const uint32_t sa = smem_u32(smem + stage * STAGE1_BYTES);
          const uint32_t sb = sa + A1_BYTES;
          tma_load_3d(sa, &tmA, fb, kb * BK, I * BM1, b);
          if (MODE == kApply) {
#pragma unroll
            for (int q = 0; q < BN / 64; ++q) tma_load_3d(sb + q * 8192, &tmB, fb, J * BN + q * 64, kb * BK, b);
          } else {
            tma_load_3d(sb, &tmB, fb, kb * BK, J * BN, b);
          }
          ++issued;
          if (++stage == STAGES1) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // wait for the copies still in flight (all have landed on the normal path)
      const int64_t first = issued > STAGES1 ? issued - STAGES1 : 0;
      for (int64_t i = first; i < issued; ++i) {
        if (!wait_bar(B.full0 + 8 * (int)(i % STAGES1), (uint32_t)((i / STAGES1) & 1), a.status)) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ----------------------------------------------------------------- MMA
      constexpr uint32_t idesc = make_idesc(MODE == kApply, BM1);
      // stage 0, k-step 0; every other descriptor adds an offset to these
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t b_desc0 = (MODE == kApply) ? sdesc_sw128(smem_u32(smem) + A1_BYTES, 8192, 1024)
                                                : sdesc_sw128(smem_u32(smem) + A1_BYTES, 16, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < a.total_tiles; t += gridDim.x) {
        if (!wait_bar(B.tempty0 + 8 * acc, acc_phase ^ 1u, a.status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait_bar(B.full0 + 8 * stage, phase, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptors of this stage: the bases plus the stage offset (16-byte units)
          const uint64_t soff = (uint64_t)((stage * STAGE1_BYTES) >> 4);
#pragma unroll
          for (int k = 0; k < BK / UK; ++k) {
            const uint64_t ad = a_desc0 + soff + (uint64_t)(k * (UK * 2 / 16));
            const uint64_t bd = b_desc0 + soff + (uint64_t)(k * ((MODE == kApply ? UK * 128 : UK * 2) / 16));
            tc_mma<1>(d, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit<1>(B.empty0 + 8 * stage);
          if (++stage == STAGES1) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit<1>(B.tfull0 + 8 * acc);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // all MMAs issued by this thread complete before the CTA frees TMEM
      tc_commit<1>(B.done);
      wait_bar(B.done, 0, a.status);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    const int wq = warp & 3;  // TMEM lanes 32*wq .. 32*wq+31
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < a.total_tiles; t += gridDim.x) {
      int b, I, J;
      decode_tile<MODE>(a, t, b, I, J);
      if constexpr (UPD) {
        // this CTA's first tile now, then always the next one during this epilogue
        if (t == (int)blockIdx.x) prefetch_update_tile(u, b, I * BM1 + wq * 32, J * BN, a.m, a.n, lane);
        if (t + (int)gridDim.x < a.total_tiles) {
          int b2, I2, J2;
          decode_tile<MODE>(a, t + (int)gridDim.x, b2, I2, J2);
          prefetch_update_tile(u, b2, I2 * BM1 + wq * 32, J2 * BN, a.m, a.n, lane);
        }
      }
      if (!wait_bar(B.tfull0 + 8 * acc, acc_phase, a.status)) break;
      tc_fence_after();
      epilogue_row<MODE, UPD>(a, u, tmem_base + ((uint32_t)(wq * 32) << 16) + (uint32_t)(acc * BN), b,
                         I * BM1 + wq * 32 + lane, J);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(B.tempty0 + 8 * acc);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<1>(tmem_base, TMEM_COLS);
  }
}

// =============================================================== CTA pair
template <int MODE, bool UPD>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    k_tc2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
          const TcArgs a, const __grid_constant__ typename UpdSel<UPD>::type u) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES2 * STAGE2_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBarriers);
  const Bars B = bar_layout(bars);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES2; ++s) {
      mbar_init(B.full0 + 8 * s, 1);   // used in the leader: its arrive.expect_tx
      mbar_init(B.empty0 + 8 * s, 1);  // the leader's MMA commit, multicast to both
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(B.tfull0 + 8 * s, 1);   // the leader's commit, multicast to both
      mbar_init(B.tempty0 + 8 * s, 8);  // in the leader: one per epilogue warp of both CTAs
    }
    mbar_init(B.done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
  }
  if (warp == 1) {
    tmem_alloc<2>(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish<2>();
  }
  tc_fence_before();
  cluster_sync();  // barrier initialisation and TMEM address visible in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = (a.k + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------- producer (both CTAs)
      const uint32_t full_leader0 = mapa_shared(B.full0, 0);
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int t = pair; ok && t < a.total_tiles; t += npairs) {
        int b, I, J;
        decode_tile<MODE>(a, t, b, I, J);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait_bar(B.empty0 + 8 * stage, phase ^ 1u, a.status)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(B.full0 + 8 * stage, 2 * STAGE2_BYTES);
          const uint32_t fb = full_leader0 + 8 * stage;
          const uint32_t sa = smem_u32(smem + stage * STAGE2_BYTES);
          const uint32_t sb = sa + A2_BYTES;
          tma_load_3d_pair(sa, &tmA, fb, kb * BK, I * BM2 + (int)rank * 128, b);
          if (MODE == kApply) {
#pragma unroll
            for (int q = 0; q < 2; ++q)
              tma_load_3d_pair(sb + q * 8192, &tmB, fb, J * BN + (int)rank * 128 + q * 64, kb * BK, b);
          } else {
            tma_load_3d_pair(sb, &tmB, fb, kb * BK, J * BN + (int)rank * 128, b);
          }
          ++issued;
          if (++stage == STAGES2) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // the leader sees both CTAs' copies land on its full barriers
      if (leader) {
        const int64_t first = issued > STAGES2 ? issued - STAGES2 : 0;
        for (int64_t i = first; i < issued; ++i) {
          if (!wait_bar(B.full0 + 8 * (int)(i % STAGES2), (uint32_t)((i / STAGES2) & 1), a.status)) break;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------ MMA (leader)
      constexpr uint32_t idesc = make_idesc(MODE == kApply, BM2);
      // stage 0, k-step 0; every other descriptor adds an offset to these
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t b_desc0 = (MODE == kApply) ? sdesc_sw128(smem_u32(smem) + A2_BYTES, 8192, 1024)
                                                : sdesc_sw128(smem_u32(smem) + A2_BYTES, 16, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = pair; ok && t < a.total_tiles; t += npairs) {
        if (!wait_bar(B.tempty0 + 8 * acc, acc_phase ^ 1u, a.status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!wait_bar(B.full0 + 8 * stage, phase, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptors of this stage: the bases plus the stage offset (16-byte units)
          const uint64_t soff = (uint64_t)((stage * STAGE2_BYTES) >> 4);
#pragma unroll
          for (int k = 0; k < BK / UK; ++k) {
            const uint64_t ad = a_desc0 + soff + (uint64_t)(k * (UK * 2 / 16));
            const uint64_t bd = b_desc0 + soff + (uint64_t)(k * ((MODE == kApply ? UK * 128 : UK * 2) / 16));
            tc_mma<2>(d, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit_pair(B.empty0 + 8 * stage, 0x3);
          if (++stage == STAGES2) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(B.tfull0 + 8 * acc, 0x3);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // all MMAs of the pair complete before either CTA frees TMEM
      tc_commit<2>(B.done);
      wait_bar(B.done, 0, a.status);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------- epilogue (both CTAs)
    const int wq = warp & 3;
    const uint32_t tempty_leader0 = mapa_shared(B.tempty0, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < a.total_tiles; t += npairs) {
      int b, I, J;
      decode_tile<MODE>(a, t, b, I, J);
      if constexpr (UPD) {
        if (t == pair) prefetch_update_tile(u, b, I * BM2 + (int)rank * 128 + wq * 32, J * BN, a.m, a.n, lane);
        if (t + npairs < a.total_tiles) {
          int b2, I2, J2;
          decode_tile<MODE>(a, t + npairs, b2, I2, J2);
          prefetch_update_tile(u, b2, I2 * BM2 + (int)rank * 128 + wq * 32, J2 * BN, a.m, a.n, lane);
        }
      }
      if (!wait_bar(B.tfull0 + 8 * acc, acc_phase, a.status)) break;
      tc_fence_after();
      epilogue_row<MODE, UPD>(a, u, tmem_base + ((uint32_t)(wq * 32) << 16) + (uint32_t)(acc * BN), b,
                         I * BM2 + (int)rank * 128 + wq * 32 + lane, J);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8 * acc);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }
  tc_fence_before();
  cluster_sync();  // no CTA leaves while the pair may still signal its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<2>(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3D bf16 map: (inner, rows, batch), row pitch ld, batch pitch rows*ld.
cudaError_t make_map(CUtensorMap* map, const void* base, int64_t inner, int64_t rows, int64_t batch,
                     int64_t ld, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), (cuuint64_t)(rows * ld * 2)};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int tri_tiles(int tiles_m, int tiles_n, int tm) {
  int t = 0;
  for (int i = 0; i < tiles_m; ++i) {
    const int c = (i * tm + tm - 1) / BN + 1;
    t += tiles_n < c ? tiles_n : c;
  }
  return t;
}

// DMUON_TC_CTA_PAIR=0 forces the one-CTA kernel (for comparisons).
// CTA pair (256-row tiles) or one CTA (128-row tiles).  The pair runs about
// 6 % faster per computed tile element (apply at 4096^2: 1378 vs 1300
// TFLOP/s), so it is used unless the 128-row tiling computes enough less
// area: m just above a multiple of 256 (e.g. 1408, 5.5 pair tiles).
// Triangle kernels (gram, poly) compare their lower-triangle tile sets.
bool use_pair(int m, bool triangle) {
  static int mode = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    const char* e = std::getenv("DMUON_TC_CTA_PAIR");
    mode = (e && std::strcmp(e, "0") == 0) ? 0 : 1;
  });
  if (mode != 1 || m < 256) return false;
  constexpr double kOneCtaCost = 1.06;
  double pair_area, one_area;
  if (triangle) {
    const int tn = (m + BN - 1) / BN;
    pair_area = tri_tiles((m + BM2 - 1) / BM2, tn, BM2) * (double)BM2;
    one_area = tri_tiles((m + BM1 - 1) / BM1, tn, BM1) * (double)BM1;
  } else {
    pair_area = (double)((m + BM2 - 1) / BM2) * BM2;
    one_area = (double)((m + BM1 - 1) / BM1) * BM1;
  }
  return one_area * kOneCtaCost >= pair_area;
}

template <int MODE, bool UPD = false>
cudaError_t launch(const CUtensorMap& ma, const CUtensorMap& mb, TcArgs& a, int batch, int num_sms, bool pair,
                   cudaStream_t st, const typename UpdSel<UPD>::type& u = {}) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(k_tc<MODE, UPD>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM1_BYTES);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(k_tc2<MODE, UPD>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM2_BYTES);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int64_t total = (int64_t)a.tiles_per_mat * batch;
  if (total <= 0) return cudaSuccess;
  if (total > 0x7fffffff) return cudaErrorInvalidValue;
  a.total_tiles = (int)total;
  if (pair) {
    const int64_t pairs = total < num_sms / 2 ? total : num_sms / 2;
    k_tc2<MODE, UPD><<<(int)(2 * pairs), kThreads, SMEM2_BYTES, st>>>(ma, mb, a, u);
  } else {
    const int grid = (int)(total < num_sms ? total : num_sms);
    k_tc<MODE, UPD><<<grid, kThreads, SMEM1_BYTES, st>>>(ma, mb, a, u);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t tc_gram(const void* X, void* G, int batch, int m, int n, int64_t ldx, int64_t ldg, float alpha,
                    const float* scale, int* status, int num_sms, cudaStream_t st) {
  if (batch == 0) return cudaSuccess;
  const bool pair = use_pair(m, true);
  CUtensorMap ma, mb;
  // A: 128 rows per CTA; B: 256 rows (one CTA) or 128 rows per CTA (pair)
  cudaError_t e = make_map(&ma, X, n, m, batch, ldx, BK, 128);
  if (e == cudaSuccess) e = make_map(&mb, X, n, m, batch, ldx, BK, pair ? 128 : BN);
  if (e != cudaSuccess) return e;
  TcArgs a{};
  a.C = static_cast<__nv_bfloat16*>(G);
  a.E = nullptr;
  a.sC = (int64_t)m * ldg;
  a.ldc = ldg;
  a.m = m; a.n = m; a.k = n;
  a.tm = pair ? BM2 : BM1;
  a.tiles_m = (m + a.tm - 1) / a.tm;
  a.tiles_n = (m + BN - 1) / BN;
  a.tiles_per_mat = tri_tiles(a.tiles_m, a.tiles_n, a.tm);
  a.p0 = alpha;
  a.scale = scale;
  a.status = status;
  return launch<kGram>(ma, mb, a, batch, num_sms, pair, st);
}

cudaError_t tc_symm(const void* A, const void* B, const void* E, void* C, int batch, int m, int64_t lda,
                    int64_t ldb, int64_t lde, int64_t ldc, float p0, float p1, float p2, int* status, int num_sms,
                    cudaStream_t st) {
  if (batch == 0) return cudaSuccess;
  const bool pair = use_pair(m, true);
  CUtensorMap ma, mb;
  cudaError_t e = make_map(&ma, A, m, m, batch, lda, BK, 128);
  if (e == cudaSuccess) e = make_map(&mb, B, m, m, batch, ldb, BK, pair ? 128 : BN);
  if (e != cudaSuccess) return e;
  TcArgs a{};
  a.C = static_cast<__nv_bfloat16*>(C);
  a.E = static_cast<const __nv_bfloat16*>(E);
  a.sC = (int64_t)m * ldc;
  a.sE = (int64_t)m * lde;
  a.ldc = ldc;
  a.lde = lde;
  a.m = m; a.n = m; a.k = m;
  a.tm = pair ? BM2 : BM1;
  a.tiles_m = (m + a.tm - 1) / a.tm;
  a.tiles_n = (m + BN - 1) / BN;
  a.tiles_per_mat = tri_tiles(a.tiles_m, a.tiles_n, a.tm);
  a.p0 = p0;
  a.p1 = p1;
  a.p2 = p2;
  a.status = status;
  return launch<kPoly>(ma, mb, a, batch, num_sms, pair, st);
}

cudaError_t tc_poly(const void* G, void* P, int batch, int m, int64_t ldg, int64_t ldp, float b, float c,
                    int* status, int num_sms, cudaStream_t st) {
  return tc_symm(G, G, G, P, batch, m, ldg, ldg, ldg, ldp, b, c, 0.f, status, num_sms, st);
}

cudaError_t tc_apply(const void* P, const void* X, void* Y, int batch, int m, int n, int64_t ldp,
                     int64_t ldx, int64_t ldy, float a_coef, float alpha, const float* scale, int* status,
                     int num_sms, cudaStream_t st) {
  if (batch == 0) return cudaSuccess;
  const bool pair = use_pair(m, false);
  CUtensorMap ma, mb;
  cudaError_t e = make_map(&ma, P, m, m, batch, ldp, BK, 128);
  if (e == cudaSuccess) e = make_map(&mb, X, n, m, batch, ldx, 64, BK);
  if (e != cudaSuccess) return e;
  TcArgs a{};
  a.C = static_cast<__nv_bfloat16*>(Y);
  a.E = static_cast<const __nv_bfloat16*>(X);
  a.sC = (int64_t)m * ldy;
  a.sE = (int64_t)m * ldx;
  a.ldc = ldy;
  a.lde = ldx;
  a.m = m; a.n = n; a.k = m;
  a.tm = pair ? BM2 : BM1;
  a.tiles_m = (m + a.tm - 1) / a.tm;
  a.tiles_n = (n + BN - 1) / BN;
  a.tiles_per_mat = a.tiles_m * a.tiles_n;
  a.p0 = a_coef;
  a.p1 = alpha;
  a.scale = scale;
  a.status = status;
  return launch<kApply>(ma, mb, a, batch, num_sms, pair, st);
}

cudaError_t tc_apply_update(const void* P, const void* X, int batch, int m, int n, int64_t ldp, int64_t ldx,
                            float a_coef, float alpha, const float* scale, const UpdTable& u, int* status,
                            int num_sms, cudaStream_t st) {
  if (batch == 0) return cudaSuccess;
  if (batch > kMaxTable) return cudaErrorInvalidValue;
  const bool pair = use_pair(m, false);
  CUtensorMap ma, mb;
  cudaError_t e = make_map(&ma, P, m, m, batch, ldp, BK, 128);
  if (e == cudaSuccess) e = make_map(&mb, X, n, m, batch, ldx, 64, BK);
  if (e != cudaSuccess) return e;
  TcArgs a{};
  a.C = nullptr;  // nothing stored but the parameters
  a.E = static_cast<const __nv_bfloat16*>(X);
  a.sE = (int64_t)m * ldx;
  a.lde = ldx;
  a.m = m; a.n = n; a.k = m;
  a.tm = pair ? BM2 : BM1;
  a.tiles_m = (m + a.tm - 1) / a.tm;
  a.tiles_n = (n + BN - 1) / BN;
  a.tiles_per_mat = a.tiles_m * a.tiles_n;
  a.p0 = a_coef;
  a.p1 = alpha;
  a.scale = scale;
  a.status = status;
  return launch<kApply, true>(ma, mb, a, batch, num_sms, pair, st, u);
}

cudaError_t wait_selftest(int* status, int64_t limit_us, cudaStream_t st) {
  k_wait_selftest<<<1, 1, 0, st>>>(status, (uint64_t)limit_us * 1000ull);
  return cudaGetLastError();
}

const char* tc_config_string() {
  return "tcgen05 bf16->fp32: CTA-pair kernel (cta_group::2, M256xN256xK16, 6 x 32 KB stages per CTA) for "
         "m >= 256 unless 128-row tiles compute over 6 % less area, one-CTA kernel (cta_group::1, "
         "M128xN256xK16, 4 x 48 KB stages) otherwise; BK=64 SW128, 2 TMEM accumulators, persistent "
         "192-thread CTAs (TMA warp, MMA warp, 4 epilogue warps); last apply of a chain fused with the update";
}

}  // namespace dmuon
