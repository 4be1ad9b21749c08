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
// columns): the chain stores p(G) = a I + b G + c G G this way, and its
// Gram-space form multiplies polynomials of one Gram matrix.
//   apply: Y = alpha (a X + P X)  m x n, K = m   (X is the MN-major operand;
//                                                  the chain passes a = 0)
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
// thread, warps 2-5 epilogue, 2-9 for reductions up to 2048), with two TMEM
// accumulators (2 x 256 fp32 columns) so the epilogue of one tile overlaps
// the MMAs of the next.  The
// polynomial terms (alpha, b G, a I, a X) are fused into the epilogue.  For
// gram and poly only tiles that touch the lower triangle are computed; every
// element r >= c is stored, and r > c also at its mirror (c, r), so G and P
// are exactly symmetric.  Inside a chain the mirror is written only within
// the diagonal 256 x 256 blocks (lower-stored matrices, see TcArgs::lower):
// the consumers read an operand's blocks right of its own 256-row block as
// the transposed lower block.
//
// Every mbarrier wait is bounded (%globaltimer); a wait that runs out records
// DMUON_ERR_TIMEOUT in the status word, the CTA waits (bounded) for its own
// copies and MMAs in flight, frees its TMEM and exits.  No TMA load uses
// cluster multicast.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <memory>
#include <mutex>
#include <type_traits>

#include "bounds.cuh"
#include "internal.h"

namespace dmuon {
namespace {

constexpr int BN = 256;
constexpr int BK = 64;  // 64 bf16 = one 128-byte swizzle row
constexpr int UK = 16;  // K of one tcgen05.mma kind::f16
constexpr int TMEM_COLS = 2 * BN;
// Warp roles: 0 TMA producer, 1 TMEM allocator + MMA issuer, 2.. epilogue.
// A warp reaches only the TMEM lane quarter (warp index mod 4).  EPI = 4: one
// epilogue warp per quarter drains all 256 accumulator columns.  EPI = 8: two
// warps per quarter, 128 columns each, twice the drain rate, which short
// reductions need to keep the MMAs busy (a 128 x 256 x 1408 tile's MMAs take
// about half as long as four warps take to drain it).  Long reductions keep
// four: the extra warps share issue slots with the MMA-issuing warp and
// leave fewer registers to a co-resident elementwise kernel.
template <int EPI>
struct Epi {
  static_assert(EPI == 4 || EPI == 8, "four or eight epilogue warps");
  static constexpr int kCols = BN / (EPI / 4);  // accumulator columns per epilogue warp
  static constexpr int kChunks = kCols / 32;    // 32-column chunks per epilogue warp
  static constexpr int kThreads = 64 + 32 * EPI;
};
// Reductions up to this length use eight epilogue warps.
constexpr int kShortK = 2048;
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
  // Symmetric matrices inside a chain are stored as their lower 256-column
  // blocks only: an element (r, c) is written where c / 256 <= r / 256 (the
  // diagonal 256 x 256 blocks in full).  lower: this launch's symmetric output
  // is stored that way (no mirror stores outside the diagonal blocks).  sym
  // bit 0 / bit 1: operand A / B is such a matrix; its k-blocks right of the
  // operand's own 256-block are read as the transposed lower block.
  int lower, sym;
};

// First k-block (of BK = 64) of a tile's operand that lies right of the
// operand's 256-row block, i.e. in the unstored upper part: from there on the
// operand is read transposed (MN-major).  Beyond every k-block when the
// operand is stored in full.
__device__ __forceinline__ int upper_kb(bool sym, int row0) { return sym ? 4 * ((row0 >> 8) + 1) : 0x7fffffff; }

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
// Operand-major bits of the instruction descriptor (bit 15: A, bit 16: B).
constexpr uint32_t kIdescAMn = 1u << 15, kIdescBMn = 1u << 16;

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

// Loads of the epilogue's E operand (b G, a X).  COH: the operand was written
// earlier in the same kernel (the fused chain), so it is read through L2
// (ld.global.cg), never from a possibly stale L1 line or the non-coherent
// read-only path; otherwise through the read-only path.
template <bool COH>
__device__ __forceinline__ uint4 ld_e16(const __nv_bfloat16* p) {
  return COH ? __ldcg(reinterpret_cast<const uint4*>(p)) : __ldg(reinterpret_cast<const uint4*>(p));
}
template <bool COH>
__device__ __forceinline__ __nv_bfloat16 ld_e1(const __nv_bfloat16* p) {
  return COH ? __ushort_as_bfloat16(__ldcg(reinterpret_cast<const unsigned short*>(p))) : *p;
}

template <bool COH>
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
      for (int i = 0; i < 4; ++i) reinterpret_cast<uint4*>(k.e)[i] = ld_e16<COH>(ep + 8 * i);
    } else {
      const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
#pragma unroll
      for (int j = 0; j < 32; j += 2)
        k.e[j >> 1] = pack2((c0 + j < n) ? ld_e1<COH>(ep + j) : z, (c0 + j + 1 < n) ? ld_e1<COH>(ep + j + 1) : z);
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
template <bool COH, int NCH>
__device__ __forceinline__ void epilogue_row_update(const TcArgs& a, const UpdTable& u, uint32_t taddr, int b,
                                                    int r, int cbase) {
  const bool row_ok = r < a.m;
  const float alpha = a.p1 * (a.scale ? a.scale[b] : 1.f);
  UpdChunk k0, k1;
  if (row_ok) load_upd_chunk<COH>(u, a, b, r, cbase, k0);
  // one chunk: load the next chunk's operands, then drain this one
  auto chunk = [&](int ch, const UpdChunk& cur, UpdChunk& nxt) -> bool {
    const int c0 = cbase + ch * 32;
    if (c0 >= a.n) return false;  // warp-uniform
    if (row_ok && ch + 1 < NCH && c0 + 32 < a.n) load_upd_chunk<COH>(u, a, b, r, c0 + 32, nxt);
    uint32_t raw[32];
    tmem_ld32(taddr + (uint32_t)(ch * 32), raw);
    tmem_ld_wait();
    if (row_ok) store_upd_chunk(u, a, b, r, c0, alpha, cur, reinterpret_cast<float*>(raw));
    return true;
  };
#pragma unroll 1
  for (int ch = 0; ch < NCH; ch += 2) {
    if (!chunk(ch, k0, k1)) break;
    if (!chunk(ch + 1, k1, k0)) break;
  }
}

// Epilogue of one tile for one accumulator row: NCH chunks of 32 accumulator
// columns from taddr (TMEM lane quarter of the warp), output row r, output
// columns from cbase.  Warp-collective (tcgen05.ld).  UPD (apply only):
// update the parameters instead of storing the result.
template <int MODE, bool UPD, bool COH, int NCH>
__device__ __forceinline__ void epilogue_row(const TcArgs& a, const typename UpdSel<UPD>::type& u, uint32_t taddr,
                                             int b, int r, int cbase) {
  if constexpr (UPD) {
    epilogue_row_update<COH, NCH>(a, u, taddr, b, r, cbase);
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
  for (int ch = 0; ch < NCH; ++ch) {
    const int c0 = cbase + ch * 32;
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
        for (int q = 0; q < 4; ++q) unpack_bf16x8(ld_e16<COH>(ep + 8 * q), e + 8 * q);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) e[j] = (c0 + j < a.n) ? __bfloat162float(ld_e1<COH>(ep + j)) : 0.f;
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
        if (a.lower && (c0 >> 8) != (r >> 8)) continue;  // the mirror lies outside the stored blocks
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

// MMAs of k-blocks [k0, k1) of one tile into accumulator d, with descriptors
// that do not change inside the range and compile-time k-steps (AT / BT:
// operand A / B is MN-major, 2048 bytes per 16-row k-step, else K-major, 32
// bytes): the single issuing thread must keep up with the tensor pipe, so
// its loop carries nothing but the stage wait, the MMAs and the release.
// Returns false if a wait ran out.
template <int G, int STAGES, int STAGE_BYTES, bool AT, bool BT>
__device__ __forceinline__ bool mma_range(int k0, int k1, uint32_t d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, const Bars& B, int& stage, uint32_t& phase, int* status) {
  constexpr uint32_t astep = AT ? UK * 128 / 16 : UK * 2 / 16;
  constexpr uint32_t bstep = BT ? UK * 128 / 16 : UK * 2 / 16;
  for (int kb = k0; kb < k1; ++kb) {
    if (!wait_bar(B.full0 + 8 * stage, phase, status)) return false;
    tc_fence_after();
    // descriptors of this stage: the bases plus the stage offset (16-byte units)
    const uint64_t soff = (uint64_t)((stage * STAGE_BYTES) >> 4);
#pragma unroll
    for (int k = 0; k < BK / UK; ++k)
      tc_mma<G>(d, adesc + soff + (uint64_t)(k * astep), bdesc + soff + (uint64_t)(k * bstep), idesc,
                (kb | k) != 0 ? 1u : 0u);
    if constexpr (G == 2)
      tc_commit_pair(B.empty0 + 8 * stage, 0x3);
    else
      tc_commit<1>(B.empty0 + 8 * stage);
    if (++stage == STAGES) {
      stage = 0;
      phase ^= 1u;
    }
  }
  return true;
}

// The k-block ranges of one tile: operand A is read transposed (MN-major,
// from its lower-stored copy) from k-block ka on, B from kb_t on (never when
// beyond num_kb), so a tile is at most three ranges in which neither changes.
// Calls f(A transposed, B transposed, k0, k1) per range, as std::bool_constant
// tags so that each range's loop is compiled with a fixed pattern (a branch
// per k-block in the producer's or the MMA thread's loop costs several per
// cent of the kernel); stops when f returns false.
template <typename F>
__device__ __forceinline__ bool for_each_kb_range(int num_kb, int ka, int kb_t, F&& f) {
  using T = std::true_type;
  using N = std::false_type;
  const int x = ka < num_kb ? ka : num_kb, y = kb_t < num_kb ? kb_t : num_kb;
  const int k1 = x < y ? x : y, k2 = x < y ? y : x;
  if (!f(N{}, N{}, 0, k1)) return false;
  if (k1 == num_kb) return true;
  if (x <= k1 && y <= k1) return f(T{}, T{}, k1, num_kb);
  const bool ok = x <= k1 ? f(T{}, N{}, k1, k2) : f(N{}, T{}, k1, k2);
  if (!ok || k2 == num_kb) return ok;
  return f(T{}, T{}, k2, num_kb);
}

// All k-blocks of one tile.  a, b: the untransposed base descriptors (b is
// MN-major when BMN, the apply's X); a_t, b_t: the MN-major ones; idesc: the
// untransposed instruction descriptor.
template <int G, int STAGES, int STAGE_BYTES, bool BMN>
__device__ __forceinline__ bool mma_tile(int num_kb, int ka, int kb_t, uint32_t d, uint64_t a, uint64_t a_t,
                                         uint64_t b, uint64_t b_t, uint32_t idesc, const Bars& B, int& stage,
                                         uint32_t& phase, int* status) {
  return for_each_kb_range(num_kb, ka, kb_t, [&](auto at, auto bt, int k0, int k1) {
    constexpr bool AT = decltype(at)::value, BT = decltype(bt)::value;
    return mma_range<G, STAGES, STAGE_BYTES, AT, BT || BMN>(
        k0, k1, d, AT ? a_t : a, BT ? b_t : b, idesc | (AT ? kIdescAMn : 0u) | (BT ? kIdescBMn : 0u), B, stage,
        phase, status);
  });
}

// ================================================================ one CTA
template <int MODE, bool UPD, int EPI>
__global__ void __launch_bounds__(Epi<EPI>::kThreads, 1)
    k_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
         const __grid_constant__ CUtensorMap tmAt, const __grid_constant__ CUtensorMap tmBt, const TcArgs a,
         const __grid_constant__ typename UpdSel<UPD>::type u) {
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
      mbar_init(B.tempty0 + 8 * s, EPI);  // one arrival per epilogue warp
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
        const int ka = upper_kb(MODE != kGram && (a.sym & 1), I * BM1);
        const int kbt = upper_kb(MODE == kPoly && (a.sym & 2), J * BN);
        ok = for_each_kb_range(num_kb, ka, kbt, [&](auto at, auto bt, int k0, int k1) {
          for (int kb = k0; kb < k1; ++kb) {
            if (!wait_bar(B.empty0 + 8 * stage, phase ^ 1u, a.status)) return false;
            const uint32_t fb = B.full0 + 8 * stage;
            mbar_arrive_expect_tx(fb, STAGE1_BYTES);
            const uint32_t sa = smem_u32(smem + stage * STAGE1_BYTES);
            const uint32_t sb = sa + A1_BYTES;
            if constexpr (decltype(at)::value) {
#pragma unroll
              for (int q = 0; q < 2; ++q) tma_load_3d(sa + q * 8192, &tmAt, fb, I * BM1 + q * 64, kb * BK, b);
            } else {
              tma_load_3d(sa, &tmA, fb, kb * BK, I * BM1, b);
            }
            if constexpr (MODE == kApply) {
#pragma unroll
              for (int q = 0; q < BN / 64; ++q) tma_load_3d(sb + q * 8192, &tmB, fb, J * BN + q * 64, kb * BK, b);
            } else if constexpr (decltype(bt)::value) {
#pragma unroll
              for (int q = 0; q < BN / 64; ++q) tma_load_3d(sb + q * 8192, &tmBt, fb, J * BN + q * 64, kb * BK, b);
            } else {
              tma_load_3d(sb, &tmB, fb, kb * BK, J * BN, b);
            }
            ++issued;
            if (++stage == STAGES1) {
              stage = 0;
              phase ^= 1u;
            }
          }
          return true;
        });
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
      // (K-major: 16-row k-steps are 32 bytes apart; MN-major: 2048 bytes)
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t a_desc0_t = sdesc_sw128(smem_u32(smem), 8192, 1024);
      const uint64_t b_desc0 = (MODE == kApply) ? sdesc_sw128(smem_u32(smem) + A1_BYTES, 8192, 1024)
                                                : sdesc_sw128(smem_u32(smem) + A1_BYTES, 16, 1024);
      const uint64_t b_desc0_t = sdesc_sw128(smem_u32(smem) + A1_BYTES, 8192, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < a.total_tiles; t += gridDim.x) {
        // the k-blocks from which a lower-stored symmetric operand is read transposed
        int ka = 0x7fffffff, kbt = 0x7fffffff;
        if (MODE != kGram && a.sym) {
          int b, I, J;
          decode_tile<MODE>(a, t, b, I, J);
          ka = upper_kb(a.sym & 1, I * BM1);
          kbt = upper_kb(MODE == kPoly && (a.sym & 2), J * BN);
        }
        if (!wait_bar(B.tempty0 + 8 * acc, acc_phase ^ 1u, a.status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * BN);
        ok = mma_tile<1, STAGES1, STAGE1_BYTES, MODE == kApply>(num_kb, ka, kbt, d, a_desc0, a_desc0_t, b_desc0,
                                                                 b_desc0_t, idesc, B, stage, phase, a.status);
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
    using E = Epi<EPI>;
    const int wq = warp & 3;                     // TMEM lanes 32*wq .. 32*wq+31
    const int half = ((warp - 2) >> 2) * E::kCols;  // this warp's accumulator columns from half
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < a.total_tiles; t += gridDim.x) {
      int b, I, J;
      decode_tile<MODE>(a, t, b, I, J);
      if (!wait_bar(B.tfull0 + 8 * acc, acc_phase, a.status)) break;
      tc_fence_after();
      epilogue_row<MODE, UPD, false, E::kChunks>(a, u, tmem_base + ((uint32_t)(wq * 32) << 16) +
                                                         (uint32_t)(acc * BN + half),
                                                 b, I * BM1 + wq * 32 + lane, J * BN + half);
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
template <int MODE, bool UPD, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Epi<EPI>::kThreads, 1)
    k_tc2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
          const __grid_constant__ CUtensorMap tmAt, const __grid_constant__ CUtensorMap tmBt, const TcArgs a,
          const __grid_constant__ typename UpdSel<UPD>::type u) {
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
      mbar_init(B.tempty0 + 8 * s, 2 * EPI);  // in the leader: one per epilogue warp of both CTAs
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
        const int ka = upper_kb(MODE != kGram && (a.sym & 1), I * BM2);
        const int kbt = upper_kb(MODE == kPoly && (a.sym & 2), J * BN);
        const int r0 = I * BM2 + (int)rank * 128, n0 = J * BN + (int)rank * 128;
        ok = for_each_kb_range(num_kb, ka, kbt, [&](auto at, auto bt, int k0, int k1) {
          for (int kb = k0; kb < k1; ++kb) {
            if (!wait_bar(B.empty0 + 8 * stage, phase ^ 1u, a.status)) return false;
            if (leader) mbar_arrive_expect_tx(B.full0 + 8 * stage, 2 * STAGE2_BYTES);
            const uint32_t fb = full_leader0 + 8 * stage;
            const uint32_t sa = smem_u32(smem + stage * STAGE2_BYTES);
            const uint32_t sb = sa + A2_BYTES;
            if constexpr (decltype(at)::value) {
#pragma unroll
              for (int q = 0; q < 2; ++q) tma_load_3d_pair(sa + q * 8192, &tmAt, fb, r0 + q * 64, kb * BK, b);
            } else {
              tma_load_3d_pair(sa, &tmA, fb, kb * BK, r0, b);
            }
            if constexpr (MODE == kApply) {
#pragma unroll
              for (int q = 0; q < 2; ++q) tma_load_3d_pair(sb + q * 8192, &tmB, fb, n0 + q * 64, kb * BK, b);
            } else if constexpr (decltype(bt)::value) {
#pragma unroll
              for (int q = 0; q < 2; ++q) tma_load_3d_pair(sb + q * 8192, &tmBt, fb, n0 + q * 64, kb * BK, b);
            } else {
              tma_load_3d_pair(sb, &tmB, fb, kb * BK, n0, b);
            }
            ++issued;
            if (++stage == STAGES2) {
              stage = 0;
              phase ^= 1u;
            }
          }
          return true;
        });
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
      // (K-major: 16-row k-steps are 32 bytes apart; MN-major: 2048 bytes)
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t a_desc0_t = sdesc_sw128(smem_u32(smem), 8192, 1024);
      const uint64_t b_desc0 = (MODE == kApply) ? sdesc_sw128(smem_u32(smem) + A2_BYTES, 8192, 1024)
                                                : sdesc_sw128(smem_u32(smem) + A2_BYTES, 16, 1024);
      const uint64_t b_desc0_t = sdesc_sw128(smem_u32(smem) + A2_BYTES, 8192, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = pair; ok && t < a.total_tiles; t += npairs) {
        // the k-blocks from which a lower-stored symmetric operand is read
        // transposed (the same for both CTAs: their rows share a 256-block)
        int ka = 0x7fffffff, kbt = 0x7fffffff;
        if (MODE != kGram && a.sym) {
          int b, I, J;
          decode_tile<MODE>(a, t, b, I, J);
          ka = upper_kb(a.sym & 1, I * BM2);
          kbt = upper_kb(MODE == kPoly && (a.sym & 2), J * BN);
        }
        if (!wait_bar(B.tempty0 + 8 * acc, acc_phase ^ 1u, a.status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * BN);
        ok = mma_tile<2, STAGES2, STAGE2_BYTES, MODE == kApply>(num_kb, ka, kbt, d, a_desc0, a_desc0_t, b_desc0,
                                                                 b_desc0_t, idesc, B, stage, phase, a.status);
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
    using E = Epi<EPI>;
    const int wq = warp & 3;
    const int half = ((warp - 2) >> 2) * E::kCols;
    const uint32_t tempty_leader0 = mapa_shared(B.tempty0, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < a.total_tiles; t += npairs) {
      int b, I, J;
      decode_tile<MODE>(a, t, b, I, J);
      if (!wait_bar(B.tfull0 + 8 * acc, acc_phase, a.status)) break;
      tc_fence_after();
      epilogue_row<MODE, UPD, false, E::kChunks>(a, u, tmem_base + ((uint32_t)(wq * 32) << 16) +
                                                         (uint32_t)(acc * BN + half),
                                                 b, I * BM2 + (int)rank * 128 + wq * 32 + lane, J * BN + half);
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

// ====================================================== fused chain kernel
// One persistent launch for a chunk's whole Newton-Schulz chain.  The phases
// (every gram, polynomial / Gram-space product and apply of the chain, in
// order) form one tile list, phase by phase and matrix by matrix within a
// phase.  A tile of phase j of matrix b needs every tile of phases < j of that
// matrix: each epilogue warp, after its stores, adds 1 (release) to the
// matrix's counter, and the TMA producer waits (acquire, bounded by
// %globaltimer) until the counter holds epilogue warps x CTAs-per-tile x
// (tiles of the earlier phases) before it loads the tile's operands.
//
// Tiles are claimed in increasing order from one global counter (the
// producer of each CTA, or of the pair's leader, takes the next index and
// passes it to its MMA and epilogue warps, and to the peer CTA, through a
// ring of 4 shared-memory slots).  Every dependency points to a lower index
// and only running CTAs claim tiles, so the smallest unfinished tile always
// has its inputs done and a running CTA to finish it, however many CTAs are
// resident (other kernels, or a second chain on another stream, included).
// The tail of one phase overlaps the head of the next for the matrices
// already done, and the chain pays one launch instead of one per product.
constexpr int kMaxPhases = 32;
constexpr int kRing = 4;
enum { kMapX0 = 0, kMapX1 = 1, kMapS0 = 2, kMapX0mn = 7, kMapX1mn = 8, kMapS0t = 9, kChainMaps = 14 };

struct PhaseDesc {
  TcArgs a;
  int mode;        // kGram, kPoly (symmetric products) or kApply
  int upd;         // apply whose epilogue updates the parameters
  int mapA, mapB;  // tensor maps of the operands
  int mapAt, mapBt;  // their MN-major maps, for the transposed reads of lower-stored operands
  int tile_start;  // global index of the phase's first tile
  uint32_t dep;    // counter value (per matrix) the phase's tiles wait for
};

struct ChainParams {
  CUtensorMap maps[kChainMaps];  // K-major {64 x 128} for X0, X1, S0..S4; MN-major {64 x 64} for X0, X1, S0..S4
  PhaseDesc ph[kMaxPhases];
  UpdTable u;
  unsigned* counters;  // one per matrix, then the tile counter; all zero at launch
  int* status;
  uint64_t dep_limit_ns;
  int nphases, total_tiles, batch;
};

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(unsigned* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// orders this thread's generic-proxy accesses with its later async-proxy
// (TMA) accesses of global memory
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
// store to the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait with cluster-scope acquire (the slot was written by the peer CTA).
__device__ __noinline__ bool wait_bar_cluster(uint32_t bar, uint32_t parity, int* status) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 128; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*reinterpret_cast<volatile int*>(status) != 0) return false;
    if (global_timer() - t0 > kTimeoutNs) {
      atomicCAS(status, 0, (int)DMUON_ERR_TIMEOUT);
      return false;
    }
  }
}

// Bounded wait until *c >= target; false when the limit ran out (recorded as
// DMUON_ERR_TIMEOUT) or another thread already failed.
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

__device__ __forceinline__ int find_phase(const ChainParams& P, int t) {
  int j = 0;
  while (j + 1 < P.nphases && t >= P.ph[j + 1].tile_start) ++j;
  return j;
}
__device__ __forceinline__ void decode_phase_tile(const PhaseDesc& ph, int t, int& b, int& I, int& J) {
  if (ph.mode == kApply)
    decode_tile<kApply>(ph.a, t - ph.tile_start, b, I, J);
  else
    decode_tile<kGram>(ph.a, t - ph.tile_start, b, I, J);
}

// G = 1: one CTA, 128 x 256 tiles (cta_group::1); G = 2: CTA pair, 256 x 256
// tiles (cta_group::2).  Both load K-major operands as boxes of 128 rows (the
// one-CTA kernel's 256 B rows as two), so one set of tensor maps serves both.
template <int G, int EPI>
__global__ void __launch_bounds__(Epi<EPI>::kThreads, 1) k_chain(const __grid_constant__ ChainParams P) {
  constexpr int STAGES = G == 2 ? STAGES2 : STAGES1;
  constexpr int STAGE_BYTES = G == 2 ? STAGE2_BYTES : STAGE1_BYTES;
  constexpr int A_BYTES = G == 2 ? A2_BYTES : A1_BYTES;
  constexpr int TM = G == 2 ? BM2 : BM1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* qbars = bars + kBarriers;                        // ring: full[kRing], empty[kRing]
  int* ring = reinterpret_cast<int*>(qbars + 2 * kRing);    // tile index per slot
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring + kRing);
  const Bars B = bar_layout(bars);
  const uint32_t qfull0 = smem_u32(qbars), qempty0 = smem_u32(qbars + kRing);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = G == 2 ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  int* status = P.status;
  unsigned* next_tile = P.counters + P.batch;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(B.full0 + 8 * s, 1);
      mbar_init(B.empty0 + 8 * s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(B.tfull0 + 8 * s, 1);
      mbar_init(B.tempty0 + 8 * s, EPI * G);  // one arrival per epilogue warp (of both CTAs)
    }
    mbar_init(B.done, 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(qfull0 + 8 * s, 1);              // the leader's producer
      // MMA + the epilogue warps (+ the peer's producer and epilogue warps)
      mbar_init(qempty0 + 8 * s, G * (1 + EPI));
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int i = 0; i < kChainMaps; ++i)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&P.maps[i])) : "memory");
  }
  if (warp == 1) {
    tmem_alloc<G>(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish<G>();
  }
  tc_fence_before();
  if (G == 2)
    cluster_sync();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the leader's ring-empty barriers (every consumer of both CTAs arrives there)
  const uint32_t qempty_leader0 = G == 2 ? mapa_shared(qempty0, 0) : qempty0;
  // next tile of the ring for a consumer: wait for the slot, read it, free it
  auto take = [&](int& qs, uint32_t& qph, bool remote_writer) -> int {
    const bool ok = remote_writer ? wait_bar_cluster(qfull0 + 8 * qs, qph, status)
                                  : wait_bar(qfull0 + 8 * qs, qph, status);
    const int t = ok ? *reinterpret_cast<volatile int*>(ring + qs) : -1;
    return t;
  };
  auto release = [&](int qs) {
    if (G == 2)
      mbar_arrive_cluster(qempty_leader0 + 8 * qs);
    else
      mbar_arrive(qempty0 + 8 * qs);
  };
  auto advance = [](int& qs, uint32_t& qph) {
    if (++qs == kRing) {
      qs = 0;
      qph ^= 1u;
    }
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const uint32_t full_base = G == 2 ? mapa_shared(B.full0, 0) : B.full0;
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      int qs = 0;
      uint32_t qph = 0;
      bool ok = true;
      while (ok) {
        int t;
        if (leader) {
          // claim the next tile and publish it to this CTA (and the peer)
          // (every consumer has read this slot; the peer's arrivals are remote)
          const bool free = G == 2 ? wait_bar_cluster(qempty0 + 8 * qs, qph ^ 1u, status)
                                   : wait_bar(qempty0 + 8 * qs, qph ^ 1u, status);
          if (!free) break;
          t = (int)atomicAdd(next_tile, 1u);
          if (t >= P.total_tiles) t = -1;
          ring[qs] = t;
          if (G == 2) st_cluster_u32(mapa_shared(smem_u32(ring + qs), 1), (uint32_t)t);
          mbar_arrive(qfull0 + 8 * qs);
          if (G == 2) mbar_arrive_cluster(mapa_shared(qfull0 + 8 * qs, 1));
        } else {
          t = take(qs, qph, true);
          release(qs);
        }
        advance(qs, qph);
        if (t < 0) break;
        const PhaseDesc& ph = P.ph[find_phase(P, t)];
        int b, I, J;
        decode_phase_tile(ph, t, b, I, J);
        if (ph.dep != 0) {
          if (!wait_count(P.counters + b, ph.dep, status, P.dep_limit_ns)) break;
          fence_proxy_async_global();  // the operands were written by generic stores
        }
        const CUtensorMap* mA = &P.maps[ph.mapA];
        const CUtensorMap* mB = &P.maps[ph.mapB];
        const CUtensorMap* mAt = &P.maps[ph.mapAt];
        const CUtensorMap* mBt = &P.maps[ph.mapBt];
        const int ka = upper_kb(ph.a.sym & 1, I * TM);
        const int kbt = upper_kb(ph.mode == kPoly && (ph.a.sym & 2), J * BN);
        const int num_kb = (ph.a.k + BK - 1) / BK;
        const bool apply_b = ph.mode == kApply;  // B is X, MN-major
        ok = for_each_kb_range(num_kb, ka, kbt, [&](auto at, auto bt, int k0, int k1) {
          for (int kb = k0; kb < k1; ++kb) {
            if (!wait_bar(B.empty0 + 8 * stage, phase ^ 1u, status)) return false;
            if (leader) mbar_arrive_expect_tx(B.full0 + 8 * stage, G * STAGE_BYTES);
            const uint32_t fb = full_base + 8 * stage;
            const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES;
            if constexpr (G == 2) {
              const int r0 = I * TM + (int)rank * 128, n0 = J * BN + (int)rank * 128;
              if constexpr (decltype(at)::value) {
#pragma unroll
                for (int q = 0; q < 2; ++q) tma_load_3d_pair(sa + q * 8192, mAt, fb, r0 + q * 64, kb * BK, b);
              } else {
                tma_load_3d_pair(sa, mA, fb, kb * BK, r0, b);
              }
              if (apply_b || decltype(bt)::value) {
#pragma unroll
                for (int q = 0; q < 2; ++q)
                  tma_load_3d_pair(sb + q * 8192, apply_b ? mB : mBt, fb, n0 + q * 64, kb * BK, b);
              } else {
                tma_load_3d_pair(sb, mB, fb, kb * BK, n0, b);
              }
            } else {
              if constexpr (decltype(at)::value) {
#pragma unroll
                for (int q = 0; q < 2; ++q) tma_load_3d(sa + q * 8192, mAt, fb, I * TM + q * 64, kb * BK, b);
              } else {
                tma_load_3d(sa, mA, fb, kb * BK, I * TM, b);
              }
              if (apply_b || decltype(bt)::value) {
#pragma unroll
                for (int q = 0; q < BN / 64; ++q)
                  tma_load_3d(sb + q * 8192, apply_b ? mB : mBt, fb, J * BN + q * 64, kb * BK, b);
              } else {
#pragma unroll
                for (int h = 0; h < 2; ++h) tma_load_3d(sb + h * 16384, mB, fb, kb * BK, J * BN + h * 128, b);
              }
            }
            ++issued;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          return true;
        });
        if (!ok) break;
      }
      if (leader) {
        const int64_t first = issued > STAGES ? issued - STAGES : 0;
        for (int64_t i = first; i < issued; ++i) {
          if (!wait_bar(B.full0 + 8 * (int)(i % STAGES), (uint32_t)((i / STAGES) & 1), status)) break;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ----------------------------------------------------------------- MMA
      constexpr uint32_t idesc_k = make_idesc(false, TM);
      constexpr uint32_t idesc_mn = make_idesc(true, TM);
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t b_desc0_k = sdesc_sw128(smem_u32(smem) + A_BYTES, 16, 1024);
      const uint64_t b_desc0_mn = sdesc_sw128(smem_u32(smem) + A_BYTES, 8192, 1024);
      const uint64_t a_desc0_mn = sdesc_sw128(smem_u32(smem), 8192, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      int qs = 0;
      uint32_t qph = 0;
      bool ok = true;
      while (ok) {
        const int t = take(qs, qph, false);
        release(qs);
        advance(qs, qph);
        if (t < 0) break;
        const PhaseDesc& ph = P.ph[find_phase(P, t)];
        const bool mn = ph.mode == kApply;
        const uint32_t idesc = mn ? idesc_mn : idesc_k;
        // the k-blocks from which a lower-stored symmetric operand is read transposed
        int ka = 0x7fffffff, kbt = 0x7fffffff;
        if (ph.a.sym) {
          int b, I, J;
          decode_phase_tile(ph, t, b, I, J);
          ka = upper_kb(ph.a.sym & 1, I * TM);
          kbt = upper_kb(ph.mode == kPoly && (ph.a.sym & 2), J * BN);
        }
        const int num_kb = (ph.a.k + BK - 1) / BK;
        if (!wait_bar(B.tempty0 + 8 * acc, acc_phase ^ 1u, status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * BN);
        ok = mn ? mma_tile<G, STAGES, STAGE_BYTES, true>(num_kb, ka, kbt, d, a_desc0, a_desc0_mn, b_desc0_mn,
                                                         b_desc0_mn, idesc, B, stage, phase, status)
                : mma_tile<G, STAGES, STAGE_BYTES, false>(num_kb, ka, kbt, d, a_desc0, a_desc0_mn, b_desc0_k,
                                                          b_desc0_mn, idesc, B, stage, phase, status);
        if (!ok) break;
        if constexpr (G == 2)
          tc_commit_pair(B.tfull0 + 8 * acc, 0x3);
        else
          tc_commit<1>(B.tfull0 + 8 * acc);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc_commit<G>(B.done);
      wait_bar(B.done, 0, status);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    using E = Epi<EPI>;
    const int wq = warp & 3;
    const int half = ((warp - 2) >> 2) * E::kCols;
    const uint32_t tempty0 = G == 2 ? mapa_shared(B.tempty0, 0) : B.tempty0;
    int acc = 0;
    uint32_t acc_phase = 0;
    int qs = 0;
    uint32_t qph = 0;
    int t = take(qs, qph, G == 2 && !leader);
    __syncwarp();
    if (lane == 0) release(qs);
    advance(qs, qph);
    while (t >= 0) {
      const PhaseDesc& ph = P.ph[find_phase(P, t)];
      int b, I, J;
      decode_phase_tile(ph, t, b, I, J);
      const int r0 = I * TM + (int)rank * 128 + wq * 32;
      // the next tile's index (claimed ahead by the producer), read now so the
      // ring slot frees early
      const int tn = take(qs, qph, G == 2 && !leader);
      __syncwarp();
      if (lane == 0) release(qs);
      advance(qs, qph);
      if (!wait_bar(B.tfull0 + 8 * acc, acc_phase, status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(wq * 32) << 16) + (uint32_t)(acc * BN + half);
      const int c0 = J * BN + half;
      const NoUpd none{};
      // a local copy: read from the indexed parameter table, the arguments would
      // be reloaded after every store of the epilogue (which might alias them)
      const TcArgs a = ph.a;
      if (ph.upd)
        epilogue_row<kApply, true, true, E::kChunks>(a, P.u, taddr, b, r0 + lane, c0);
      else if (ph.mode == kApply)
        epilogue_row<kApply, false, true, E::kChunks>(a, none, taddr, b, r0 + lane, c0);
      else if (ph.mode == kPoly)
        epilogue_row<kPoly, false, true, E::kChunks>(a, none, taddr, b, r0 + lane, c0);
      else
        epilogue_row<kGram, false, true, E::kChunks>(a, none, taddr, b, r0 + lane, c0);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        // this warp's part of the tile is stored: publish it, then free the accumulator
        red_release_add(P.counters + b, 1u);  // release: after the warp's stores (ordered by the __syncwarp)
        if constexpr (G == 2)
          mbar_arrive_cluster(tempty0 + 8 * acc);
        else
          mbar_arrive(tempty0 + 8 * acc);
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
      t = tn;
    }
  }
  tc_fence_before();
  if (G == 2)
    cluster_sync();
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<G>(tmem_base, TMEM_COLS);
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

// Largest number of CTA pairs (clusters of 2 at the pair kernels' shared
// memory) that can be resident at once on the current device: SMs / 2 unless
// the GPCs leave some SMs unpaired.  Persistent pair launches use no more,
// so no pair starts only after others finish, and the fused chain (whose CTAs
// wait on one another) relies on it.
int max_pair_units(int num_sms) {
  static std::mutex mu;
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return num_sms / 2;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] > 0) return cached[dev];
  int n = 0;
  cudaError_t e = cudaFuncSetAttribute(k_chain<2, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM2_BYTES);
  if (e == cudaSuccess) {
    // shared memory allows one CTA per SM whatever the epilogue width
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(num_sms & ~1));
    cfg.blockDim = dim3(Epi<8>::kThreads);
    cfg.dynamicSmemBytes = SMEM2_BYTES;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    e = cudaOccupancyMaxActiveClusters(&n, (void*)k_chain<2, 8>, &cfg);
  }
  if (e != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = num_sms / 2;
  }
  cached[dev] = n < num_sms / 2 ? n : num_sms / 2;
  return cached[dev];
}

// Epilogue warps for a reduction of length k; DMUON_EPI_WARPS=4 or 8 forces
// one width (for measurements).
int epi_warps(int64_t k) {
  const char* v = std::getenv("DMUON_EPI_WARPS");
  const int forced = v ? std::atoi(v) : 0;
  if (forced == 4 || forced == 8) return forced;
  return k <= kShortK ? 8 : 4;
}

template <int MODE, bool UPD, int EPI>
cudaError_t launch_epi(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mat, const CUtensorMap& mbt,
                       const TcArgs& a, int64_t total, int num_sms, bool pair, cudaStream_t st,
                       const typename UpdSel<UPD>::type& u) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(k_tc<MODE, UPD, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM1_BYTES);
    if (attr_err == cudaSuccess)
      attr_err =
          cudaFuncSetAttribute(k_tc2<MODE, UPD, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM2_BYTES);
  });
  if (attr_err != cudaSuccess) return attr_err;
  if (pair) {
    const int units = max_pair_units(num_sms);
    const int64_t pairs = total < units ? total : units;
    k_tc2<MODE, UPD, EPI><<<(int)(2 * pairs), Epi<EPI>::kThreads, SMEM2_BYTES, st>>>(ma, mb, mat, mbt, a, u);
  } else {
    const int grid = (int)(total < num_sms ? total : num_sms);
    k_tc<MODE, UPD, EPI><<<grid, Epi<EPI>::kThreads, SMEM1_BYTES, st>>>(ma, mb, mat, mbt, a, u);
  }
  return cudaGetLastError();
}

// mat / mbt: MN-major {64 x 64} maps of operands A / B, read where a.sym
// says they are lower-stored symmetric matrices (otherwise unused).
template <int MODE, bool UPD = false>
cudaError_t launch(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mat, const CUtensorMap& mbt,
                   TcArgs& a, int batch, int num_sms, bool pair, cudaStream_t st,
                   const typename UpdSel<UPD>::type& u = {}) {
  const int64_t total = (int64_t)a.tiles_per_mat * batch;
  if (total <= 0) return cudaSuccess;
  if (total > 0x7fffffff) return cudaErrorInvalidValue;
  a.total_tiles = (int)total;
  if (epi_warps(a.k) == 8) return launch_epi<MODE, UPD, 8>(ma, mb, mat, mbt, a, total, num_sms, pair, st, u);
  return launch_epi<MODE, UPD, 4>(ma, mb, mat, mbt, a, total, num_sms, pair, st, u);
}

// Arguments of each product; the per-product launches and the fused chain
// build them the same way, so both compute the same tiles with the same
// epilogues.
TcArgs gram_args(void* G, int batch, int m, int n, int64_t ldg, float alpha, const float* scale, int* status,
                 bool pair) {
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
  a.total_tiles = a.tiles_per_mat * batch;
  a.p0 = alpha;
  a.scale = scale;
  a.status = status;
  return a;
}

TcArgs symm_args(const void* E, void* C, int batch, int m, int64_t lde, int64_t ldc, float p0, float p1, float p2,
                 int* status, bool pair) {
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
  a.total_tiles = a.tiles_per_mat * batch;
  a.p0 = p0;
  a.p1 = p1;
  a.p2 = p2;
  a.status = status;
  return a;
}

// Y may be NULL (the fused update stores nothing but the parameters).
TcArgs apply_args(const void* X, void* Y, int batch, int m, int n, int64_t ldx, int64_t ldy, float a_coef,
                  float alpha, const float* scale, int* status, bool pair) {
  TcArgs a{};
  a.C = static_cast<__nv_bfloat16*>(Y);
  a.E = static_cast<const __nv_bfloat16*>(X);
  a.sC = Y ? (int64_t)m * ldy : 0;
  a.sE = (int64_t)m * ldx;
  a.ldc = Y ? ldy : 0;
  a.lde = ldx;
  a.m = m; a.n = n; a.k = m;
  a.tm = pair ? BM2 : BM1;
  a.tiles_m = (m + a.tm - 1) / a.tm;
  a.tiles_n = (n + BN - 1) / BN;
  a.tiles_per_mat = a.tiles_m * a.tiles_n;
  a.total_tiles = a.tiles_per_mat * batch;
  a.p0 = a_coef;
  a.p1 = alpha;
  a.scale = scale;
  a.status = status;
  return a;
}

}  // namespace

cudaError_t tc_gram(const void* X, void* G, int batch, int m, int n, int64_t ldx, int64_t ldg, float alpha,
                    const float* scale, int* status, int num_sms, cudaStream_t st, bool lower) {
  if (batch == 0) return cudaSuccess;
  const bool pair = use_pair(m, true);
  CUtensorMap ma, mb;
  // A: 128 rows per CTA; B: 256 rows (one CTA) or 128 rows per CTA (pair)
  cudaError_t e = make_map(&ma, X, n, m, batch, ldx, BK, 128);
  if (e == cudaSuccess) e = make_map(&mb, X, n, m, batch, ldx, BK, pair ? 128 : BN);
  if (e != cudaSuccess) return e;
  TcArgs a = gram_args(G, batch, m, n, ldg, alpha, scale, status, pair);
  a.lower = lower ? 1 : 0;
  return launch<kGram>(ma, mb, ma, mb, a, batch, num_sms, pair, st);
}

cudaError_t tc_symm(const void* A, const void* B, const void* E, void* C, int batch, int m, int64_t lda,
                    int64_t ldb, int64_t lde, int64_t ldc, float p0, float p1, float p2, int* status, int num_sms,
                    cudaStream_t st, bool lower) {
  if (batch == 0) return cudaSuccess;
  const bool pair = use_pair(m, true);
  CUtensorMap ma, mb, mat, mbt;
  cudaError_t e = make_map(&ma, A, m, m, batch, lda, BK, 128);
  if (e == cudaSuccess) e = make_map(&mb, B, m, m, batch, ldb, BK, pair ? 128 : BN);
  // lower-stored operands: their upper k-blocks are read as transposed {64 x 64} boxes
  if (e == cudaSuccess && lower) e = make_map(&mat, A, m, m, batch, lda, 64, BK);
  if (e == cudaSuccess && lower) e = make_map(&mbt, B, m, m, batch, ldb, 64, BK);
  if (e != cudaSuccess) return e;
  TcArgs a = symm_args(E, C, batch, m, lde, ldc, p0, p1, p2, status, pair);
  a.lower = lower ? 1 : 0;
  a.sym = lower ? 3 : 0;
  return lower ? launch<kPoly>(ma, mb, mat, mbt, a, batch, num_sms, pair, st)
               : launch<kPoly>(ma, mb, ma, mb, a, batch, num_sms, pair, st);
}

cudaError_t tc_poly(const void* G, void* P, int batch, int m, int64_t ldg, int64_t ldp, float b, float c,
                    int* status, int num_sms, cudaStream_t st) {
  return tc_symm(G, G, G, P, batch, m, ldg, ldg, ldg, ldp, b, c, 0.f, status, num_sms, st, false);
}

cudaError_t tc_apply(const void* P, const void* X, void* Y, int batch, int m, int n, int64_t ldp,
                     int64_t ldx, int64_t ldy, float a_coef, float alpha, const float* scale, int* status,
                     int num_sms, cudaStream_t st, bool lower_p) {
  if (batch == 0) return cudaSuccess;
  const bool pair = use_pair(m, false);
  CUtensorMap ma, mb, mat;
  cudaError_t e = make_map(&ma, P, m, m, batch, ldp, BK, 128);
  if (e == cudaSuccess) e = make_map(&mb, X, n, m, batch, ldx, 64, BK);
  if (e == cudaSuccess && lower_p) e = make_map(&mat, P, m, m, batch, ldp, 64, BK);
  if (e != cudaSuccess) return e;
  TcArgs a = apply_args(X, Y, batch, m, n, ldx, ldy, a_coef, alpha, scale, status, pair);
  a.sym = lower_p ? 1 : 0;
  return launch<kApply>(ma, mb, lower_p ? mat : ma, mb, a, batch, num_sms, pair, st);
}

cudaError_t tc_apply_update(const void* P, const void* X, int batch, int m, int n, int64_t ldp, int64_t ldx,
                            float a_coef, float alpha, const float* scale, const UpdTable& u, int* status,
                            int num_sms, cudaStream_t st, bool lower_p) {
  if (batch == 0) return cudaSuccess;
  if (batch > kMaxTable) return cudaErrorInvalidValue;
  const bool pair = use_pair(m, false);
  CUtensorMap ma, mb, mat;
  cudaError_t e = make_map(&ma, P, m, m, batch, ldp, BK, 128);
  if (e == cudaSuccess) e = make_map(&mb, X, n, m, batch, ldx, 64, BK);
  if (e == cudaSuccess && lower_p) e = make_map(&mat, P, m, m, batch, ldp, 64, BK);
  if (e != cudaSuccess) return e;
  TcArgs a = apply_args(X, nullptr, batch, m, n, ldx, 0, a_coef, alpha, scale, status, pair);
  a.sym = lower_p ? 1 : 0;
  return launch<kApply, true>(ma, mb, lower_p ? mat : ma, mb, a, batch, num_sms, pair, st, u);
}

bool tc_chain_fusable(int m, const std::vector<int>& blocks) {
  int nph = 0;
  for (int len : blocks) nph += len == 1 ? 3 : (len == 2 ? 7 : 11);
  return nph > 0 && nph <= kMaxPhases && use_pair(m, true) == use_pair(m, false);
}

bool tc_chain_small(int batch, int m, int n, const std::vector<int>& blocks) {
  // tiles of each product kind for this chunk (the grouping the chain uses)
  const bool pair = use_pair(m, false);
  const TcArgs g = gram_args(nullptr, batch, m, n, m, 1.f, nullptr, nullptr, pair);
  const TcArgs sy = symm_args(nullptr, nullptr, batch, m, m, m, 0.f, 1.f, 0.f, nullptr, pair);
  const TcArgs ap = apply_args(nullptr, nullptr, batch, m, n, n, n, 0.f, 1.f, nullptr, nullptr, pair);
  int64_t tiles = 0, nph = 0;
  for (int len : blocks) {
    const int products = len == 1 ? 1 : (len == 2 ? 5 : 9);
    tiles += g.total_tiles + (int64_t)products * sy.total_tiles + ap.total_tiles;
    nph += 2 + products;
  }
  // B200: 74 CTA pairs or 148 CTAs
  const int64_t units = pair ? 74 : 148;
  return nph > 0 && tiles <= 2 * units * nph;
}

cudaError_t tc_chain(const ChainBuffers& buf, int batch, int m, int n, int64_t ldn, int64_t ldm,
                     const std::vector<int>& blocks, const float* sched, const float* scale, const UpdTable* upd,
                     int* status, int num_sms, bool inject_timeout, cudaStream_t st, int* result_x) {
  *result_x = 0;
  if (batch == 0) return cudaSuccess;
  // one CTA grouping for every product, the one the per-product launches
  // would pick for each of them (so both schedules give the same bits)
  const bool pair = use_pair(m, false);
  if (!tc_chain_fusable(m, blocks) || batch > kMaxTable || !buf.counters) return cudaErrorNotSupported;
  const bool blocked = false == std::all_of(blocks.begin(), blocks.end(), [](int l) { return l == 1; });
  if (blocked && !(buf.slot[2] && buf.slot[3] && buf.slot[4])) return cudaErrorNotSupported;
  const int G = pair ? 2 : 1;
  // every product but the Gram matrix reduces over m
  const int EPI = epi_warps(m);

  std::unique_ptr<ChainParams> P(new ChainParams());
  cudaError_t e = make_map(&P->maps[kMapX0], buf.x[0], n, m, batch, ldn, BK, 128);
  if (e == cudaSuccess) e = make_map(&P->maps[kMapX1], buf.x[1], n, m, batch, ldn, BK, 128);
  for (int i = 0; i < 5 && e == cudaSuccess; ++i)
    e = make_map(&P->maps[kMapS0 + i], buf.slot[i] ? buf.slot[i] : buf.slot[0], m, m, batch, ldm, BK, 128);
  if (e == cudaSuccess) e = make_map(&P->maps[kMapX0mn], buf.x[0], n, m, batch, ldn, 64, BK);
  if (e == cudaSuccess) e = make_map(&P->maps[kMapX1mn], buf.x[1], n, m, batch, ldn, 64, BK);
  for (int i = 0; i < 5 && e == cudaSuccess; ++i)
    e = make_map(&P->maps[kMapS0t + i], buf.slot[i] ? buf.slot[i] : buf.slot[0], m, m, batch, ldm, 64, BK);
  if (e != cudaSuccess) return e;
  // the symmetric matrices are stored as their lower 256-column blocks, as in
  // the per-product launches (DMUON_LOWER_STORE=0: in full)
  const bool low = !(std::getenv("DMUON_LOWER_STORE") && std::getenv("DMUON_LOWER_STORE")[0] == '0');

  int j = 0;
  int64_t tiles = 0, per_matrix = 0;
  auto add = [&](const TcArgs& a, int mode, int mapA, int mapB, int u) {
    PhaseDesc& ph = P->ph[j++];
    ph.a = a;
    ph.mode = mode;
    ph.upd = u;
    ph.mapA = mapA;
    ph.mapB = mapB;
    // operands from the S slots are symmetric; gram and poly outputs too
    const bool sa = mapA >= kMapS0 && mapA < kMapS0 + 5, sb = mapB >= kMapS0 && mapB < kMapS0 + 5;
    ph.mapAt = sa ? mapA - kMapS0 + kMapS0t : mapA;
    ph.mapBt = sb ? mapB - kMapS0 + kMapS0t : mapB;
    ph.a.lower = low && mode != kApply ? 1 : 0;
    ph.a.sym = low ? (sa ? 1 : 0) | (sb && mode == kPoly ? 2 : 0) : 0;
    ph.tile_start = (int)tiles;
    ph.dep = (uint32_t)(EPI * G * per_matrix);  // every epilogue warp of every CTA of a tile adds 1
    tiles += a.total_tiles;
    per_matrix += a.tiles_per_mat;
  };
  int steps = 0;
  for (int len : blocks) steps += len;
  auto S = [&](int i) { return buf.slot[i]; };
  int cur = 0, k = 0;
  for (int len : blocks) {
    const float* sc = k == 0 ? scale : nullptr;
    const bool last = k + len == steps;
    const bool fuse = last && upd != nullptr;
    const float* c = sched + 3 * k;
    if (len == 1) {
      // G, P = a I + b G + c G G, X <- P X (the per-product launches' schedule)
      add(gram_args(S(0), batch, m, n, ldm, 1.f, sc, status, pair), kGram, kMapX0 + cur, kMapX0 + cur, 0);
      add(symm_args(S(0), S(1), batch, m, ldm, ldm, c[1], c[2], c[0], status, pair), kPoly, kMapS0, kMapS0, 0);
      add(apply_args(buf.x[cur], fuse ? nullptr : buf.x[1 - cur], batch, m, n, ldn, ldn, 0.f, 1.f, sc, status, pair),
          kApply, kMapS0 + 1, kMapX0mn + cur, fuse ? 1 : 0);
    } else {
      const float* c1 = sched + 3 * (k + 1);
      add(gram_args(S(0), batch, m, n, ldm, 1.f, sc, status, pair), kGram, kMapX0 + cur, kMapX0 + cur, 0);
      add(symm_args(S(0), S(1), batch, m, ldm, ldm, c[1], c[2], c[0], status, pair), kPoly, kMapS0, kMapS0, 0);  // P0
      add(symm_args(nullptr, S(2), batch, m, ldm, ldm, 0.f, 1.f, 0.f, status, pair), kPoly, kMapS0 + 1, kMapS0, 0);  // T = P0 G
      add(symm_args(nullptr, S(0), batch, m, ldm, ldm, 0.f, 1.f, 0.f, status, pair), kPoly, kMapS0 + 2, kMapS0 + 1,
          0);  // G1 = T P0
      add(symm_args(S(0), S(3), batch, m, ldm, ldm, c1[1], c1[2], c1[0], status, pair), kPoly, kMapS0, kMapS0, 0);  // P1
      add(symm_args(nullptr, S(4), batch, m, ldm, ldm, 0.f, 1.f, 0.f, status, pair), kPoly, kMapS0 + 3, kMapS0 + 1,
          0);  // Q = P1 P0
      int q = 4;
      if (len == 3) {
        const float* c2 = sched + 3 * (k + 2);
        add(symm_args(nullptr, S(2), batch, m, ldm, ldm, 0.f, 1.f, 0.f, status, pair), kPoly, kMapS0 + 3, kMapS0,
            0);  // T = P1 G1
        add(symm_args(nullptr, S(0), batch, m, ldm, ldm, 0.f, 1.f, 0.f, status, pair), kPoly, kMapS0 + 2, kMapS0 + 3,
            0);  // G2 = T P1
        add(symm_args(S(0), S(1), batch, m, ldm, ldm, c2[1], c2[2], c2[0], status, pair), kPoly, kMapS0, kMapS0,
            0);  // P2
        add(symm_args(nullptr, S(2), batch, m, ldm, ldm, 0.f, 1.f, 0.f, status, pair), kPoly, kMapS0 + 1, kMapS0 + 4,
            0);  // Q2 = P2 Q
        q = 2;
      }
      add(apply_args(buf.x[cur], fuse ? nullptr : buf.x[1 - cur], batch, m, n, ldn, ldn, 0.f, 1.f, sc, status, pair),
          kApply, kMapS0 + q, kMapX0mn + cur, fuse ? 1 : 0);  // X <- Q X
    }
    cur = 1 - cur;
    k += len;
  }
  if (tiles <= 0) return cudaSuccess;
  if (tiles > 0x7fffffff) return cudaErrorNotSupported;
  P->nphases = j;
  P->total_tiles = (int)tiles;
  P->counters = buf.counters;
  P->batch = batch;
  P->status = status;
  P->dep_limit_ns = kTimeoutNs;
  if (inject_timeout) {
    // a dependency nothing will meet: the last phase's waits run out
    P->ph[j - 1].dep += 1;
    P->dep_limit_ns = 20000000ull;
  }
  if (upd) P->u = *upd;
  *result_x = (upd != nullptr) ? -1 : cur;

  e = cudaMemsetAsync(buf.counters, 0, (size_t)(batch + 1) * sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    const int one = SMEM1_BYTES, two = SMEM2_BYTES;
    attr_err = cudaFuncSetAttribute(k_chain<1, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, one);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(k_chain<1, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, one);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(k_chain<2, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, two);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(k_chain<2, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, two);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int max_units = pair ? max_pair_units(num_sms) : num_sms;
  const int units = (int)(tiles < max_units ? tiles : max_units);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(G * units));
  cfg.blockDim = dim3(EPI == 8 ? Epi<8>::kThreads : Epi<4>::kThreads);
  cfg.dynamicSmemBytes = pair ? SMEM2_BYTES : SMEM1_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = pair ? 2 : 1;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = pair ? 1 : 0;
  if (EPI == 8)
    e = pair ? cudaLaunchKernelEx(&cfg, k_chain<2, 8>, *P) : cudaLaunchKernelEx(&cfg, k_chain<1, 8>, *P);
  else
    e = pair ? cudaLaunchKernelEx(&cfg, k_chain<2, 4>, *P) : cudaLaunchKernelEx(&cfg, k_chain<1, 4>, *P);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t wait_selftest(int* status, int64_t limit_us, cudaStream_t st) {
  k_wait_selftest<<<1, 1, 0, st>>>(status, (uint64_t)limit_us * 1000ull);
  return cudaGetLastError();
}

const char* tc_config_string() {
  return "tcgen05 bf16->fp32: CTA-pair kernel (cta_group::2, M256xN256xK16, 6 x 32 KB stages per CTA) for "
         "m >= 256 unless 128-row tiles compute over 6 % less area, one-CTA kernel (cta_group::1, "
         "M128xN256xK16, 4 x 48 KB stages) otherwise; BK=64 SW128, 2 TMEM accumulators, persistent "
         "CTAs (TMA warp, MMA warp, 4 epilogue warps, 8 for reductions up to 2048); last apply of a chain "
         "fused with the update";
}

}  // namespace dmuon
