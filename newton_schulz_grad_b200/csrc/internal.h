// Internal host-side interfaces between the translation units of the library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "dmuon.h"

namespace dmuon {

// Tile edge of the elementwise kernels (source-layout tiles, 64 x 64).
constexpr int kElemTile = 64;
// Matrices per elementwise launch (size of the pointer table in the kernel
// parameters: 256 entries x 32 bytes).
constexpr int kMaxTable = 256;
// Largest min(rows, cols) that runs the FFMA chain with fp32 Gram matrices in
// the bf16 path (bf16 rounding of G and p(G) is too coarse for such thin
// matrices to meet the 2e-2 budget).
constexpr int kSmallM = 64;
// Below this min(rows, cols), bf16 matrices that are also near-square
// (max < kNearSquare * min) keep X in fp32 as well: their many tiny singular
// values are not resolved by bf16 storage of X (measured: the tensor-core
// chain exceeds 2e-2 on low-rank-plus-noise inputs there, e.g. 96 x 200 and
// 128 x 160), and at these sizes the FFMA chain costs well under a
// millisecond.
constexpr int kF32XBelowM = 256;
constexpr int kNearSquare = 3;

// One matrix of an elementwise launch.  `src` is the gradient (momentum
// stage) or the input matrix (load stage); `buf` the momentum buffer or NULL;
// `dst` the parameter (update stage) or the output matrix (copy-out stage).
struct MatEntry {
  const void* src;
  void* buf;
  void* dst;
  int32_t transposed;  // 1: source is n x m and is transposed into m x n
  int32_t pad;         // bit 0: src and buf allow 16-byte vectors; bit 1: dst does
};

// All entries of one launch share the oriented shape m x n (m <= n) and the
// workspace row pitch ldn; source shape is (m, n) or (n, m) per entry.
struct ElemTable {
  int64_t m, n, ldn;
  int32_t count;
  int32_t tiles_per_mat;  // ceil(m/64) * ceil(n/64)
  int* status = nullptr;  // device status word (debug builds record bounds errors)
  MatEntry e[kMaxTable];
};

enum class ElemMode : int { kMomentum = 0, kLoad = 1, kUpdate = 2, kCopyOut = 3 };

// Storage type of the Newton-Schulz chain.
enum class Path : int {
  kTensorBf16 = 0,   // bf16 X, G, P on tcgen05 tensor cores
  kSmallBf16 = 1,    // bf16 X, fp32 G, P on FFMA
  kF32 = 2,          // fp32 X, G, P on FFMA
  kBf16F32 = 3       // bf16 matrix, fp32 X, G, P on FFMA (small, near-square)
};

// ---- elementwise.cu --------------------------------------------------------
// Momentum (or load) stage: writes x0 into X (batch pitch m*ldn elements,
// transposed where the entry says so) and one fp32 sum-of-squares partial per
// 64x64 tile into `partials` (tiles_per_mat per matrix).
// clip_coef (device float, kMomentum only): scale each gradient by it first.
// xdtype: storage type of X in the workspace (-1: dtype; DMUON_F32 for a bf16
// matrix whose chain keeps X in fp32, see Path::kBf16F32).
cudaError_t launch_momentum(const ElemTable& t, int dtype, ElemMode mode, void* X,
                            float* partials, float mu, int nesterov, cudaStream_t st,
                            const float* clip_coef = nullptr, int xdtype = -1);
// Sum the partials of each matrix in a fixed order; scale[i] = 1/(sqrt(sum)+eps).
// sumsq (optional) receives the sums in fp64.
cudaError_t launch_norm_finalize(const float* partials, int count, int tiles_per_mat,
                                 float* scale, double* sumsq, cudaStream_t st);
// Update (or copy-out) stage.  O is the oriented m x n result in the
// workspace (pitch ldn); `scale` (optional, per matrix) multiplies O first.
// The update uses lr * 0.2 * sqrt(scale_dim) (scale_dim = max(rows, cols)).
// xdtype as for launch_momentum; an fp32 O of a bf16 matrix is rounded to
// bf16 before it is used.
cudaError_t launch_update(const ElemTable& t, int dtype, ElemMode mode, const void* O,
                          const float* scale, float lr, float wd, int64_t scale_dim,
                          cudaStream_t st, int xdtype = -1);

// ---- simt_gemm.cu -----------------------------------------------------------
// FFMA chain kernels, batched over `batch` matrices with element batch strides.
// xbf16: X is bf16 (else fp32); G and P are bf16 only when gbf16 (stage calls
// of the bf16 dtype never come here; gbf16 is always false in practice).
// status: device status word (debug builds record bounds errors there).
cudaError_t simt_gram(const void* X, void* G, int batch, int m, int n, int64_t ldx, int64_t ldg,
                      float alpha, const float* scale, bool xbf16, cudaStream_t st, int* status);
cudaError_t simt_poly(const void* G, void* P, int batch, int m, int64_t ldg, int64_t ldp,
                      float b, float c, cudaStream_t st, int* status);
cudaError_t simt_apply(const void* P, const void* X, void* Y, int batch, int m, int n,
                       int64_t ldp, int64_t ldx, int64_t ldy, float a, float alpha,
                       const float* scale, bool xbf16, cudaStream_t st, int* status);

// The whole FFMA chain (steps x (gram, poly, apply), per-iteration form) of a
// chunk in one launch, tiles ordered phase by phase with per-matrix
// dependency counters (the same tiles and arithmetic as the three kernels
// above, so the same bits).  x[0] holds X at entry, x[1] is the ping-pong
// buffer; counters has batch + 1 entries (zeroed here); *result_x: the x
// buffer holding the result.  cudaErrorNotSupported: more than 16 iterations
// (run product by product).  inject_timeout: a test hook whose last
// dependency is never met, so its bounded waits run out (DMUON_ERR_TIMEOUT).
cudaError_t simt_chain(void* const* x, void* G, void* P, int batch, int m, int n, int64_t ldx, int64_t ldg,
                       int32_t steps, const float* sched, const float* scale, bool xbf16, unsigned* counters,
                       int* status, int num_sms, bool inject_timeout, cudaStream_t st, int* result_x);

// ---- clip.cu --------------------------------------------------------------------
// Each matrix is read as a flat array of rows * cols elements; one partial per
// chunk of kClipChunk elements (ceil(rows * cols / kClipChunk) per matrix).
constexpr int kClipChunk = 4096;
// Global p-norm clipping (p = 0 means the infinity norm).  Tables hold
// matrices of one source shape (m = rows, n = cols, not oriented; tiles_per_mat
// = chunks per matrix); `src` is read for the norm, `buf` scaled in place; pad
// bit 0: the base is 16-byte aligned.
cudaError_t launch_clip_partials(const ElemTable& t, int dtype, int p, float* partials, cudaStream_t st);
cudaError_t launch_clip_coef(const float* partials, int64_t count, int p, float max_norm, float* coef,
                             double* total, cudaStream_t st);
cudaError_t launch_clip_scale(const ElemTable& t, int dtype, const float* coef, cudaStream_t st);
// Bucketed clipping: bucket k owns partials [off[k], off[k + 1]) and gets its
// own coefficient (coefs[k]) and total (total[k] when total is not null).
constexpr int kMaxClipBuckets = 128;
struct ClipBuckets {
  int64_t off[kMaxClipBuckets + 1];
  float max_norm[kMaxClipBuckets];
  int32_t p[kMaxClipBuckets];  // 2, 1, or 0 for the infinity norm
  double* total;
};
cudaError_t launch_clip_coef_buckets(const float* partials, const ClipBuckets& b, int num_buckets, float* coefs,
                                     cudaStream_t st);

// ---- small_ns.cu -------------------------------------------------------------
// The whole chain for min side m <= 64 in one launch: one cluster of 8 CTAs per
// matrix, X's columns split over the CTAs and kept in shared memory, the fp32
// Gram matrix all-reduced over distributed shared memory each iteration.  X (in
// place, batch pitch m*ld) holds x0 on entry and the result on exit.
// Valid for steps <= 16 and n <= small_ns_max_n(m, element size).
int small_ns_max_n(int m, size_t es);
cudaError_t small_ns(void* X, int batch, int m, int n, int64_t ld, int steps, const float* coeffs,
                     const float* scale, bool xbf16, cudaStream_t st, int* status);

// ---- tc_gemm.cu -------------------------------------------------------------
// tcgen05 chain kernels (bf16 in/out, fp32 accumulation in TMEM).
// Inside a chain the symmetric matrices (G, p(G) and the Gram-space products)
// may be stored as their lower 256-column blocks only (lower = true: the
// producer skips the mirror stores outside the diagonal blocks) and read so
// by their consumers (lower / lower_p = true: the operand's upper k-blocks
// are loaded as the transposed lower block).  The stage calls store and read
// full matrices.
cudaError_t tc_gram(const void* X, void* G, int batch, int m, int n, int64_t ldx, int64_t ldg,
                    float alpha, const float* scale, int* status, int num_sms, cudaStream_t st, bool lower = false);
cudaError_t tc_poly(const void* G, void* P, int batch, int m, int64_t ldg, int64_t ldp, float b,
                    float c, int* status, int num_sms, cudaStream_t st);
// C = p1 (A B) + p0 E + p2 I for symmetric, commuting A, B (E may be NULL);
// one triangle computed, mirrored.
cudaError_t tc_symm(const void* A, const void* B, const void* E, void* C, int batch, int m, int64_t lda,
                    int64_t ldb, int64_t lde, int64_t ldc, float p0, float p1, float p2, int* status,
                    int num_sms, cudaStream_t st, bool lower = false);
cudaError_t tc_apply(const void* P, const void* X, void* Y, int batch, int m, int n, int64_t ldp,
                     int64_t ldx, int64_t ldy, float a, float alpha, const float* scale,
                     int* status, int num_sms, cudaStream_t st, bool lower_p = false);

// The parameter update fused into the last apply of the chain: for matrix b
// of the launch, O = bf16(alpha (a X + P X)) (the value tc_apply would store)
// and p_b <- bf16(p_b * decay - step_scale * O), p_b in its source layout
// (n x m, i.e. O transposed, where the tmask bit is set).  Same arithmetic and
// rounding as launch_update on the stored O, so the two paths agree bit for bit.
struct UpdTable {
  void* p[kMaxTable];
  uint32_t tmask[kMaxTable / 32];  // source is n x m
  uint32_t vmask[kMaxTable / 32];  // source rows allow 16-byte vectors
  float decay, step_scale;
};
cudaError_t tc_apply_update(const void* P, const void* X, int batch, int m, int n, int64_t ldp, int64_t ldx,
                            float a, float alpha, const float* scale, const UpdTable& u, int* status,
                            int num_sms, cudaStream_t st, bool lower_p = false);
// The whole chain of a chunk in one persistent launch (tensor path): every
// product of the iteration blocks `blocks` (chain_blocks) in order, per-matrix
// dependency counters between them.  x[0] holds X at entry; slot[0..4] are
// the m x m buffers (slots 2-4 only for Gram-space blocks); counters has
// batch + 1 entries (zeroed here: one per matrix, then the tile counter).  upd: the last apply updates the parameters.
// *result_x: the x buffer holding the result (-1 when fused with the update).
// cudaErrorNotSupported: this chain cannot run fused (too many products, or
// its products would pick different CTA groupings); run it product by
// product instead.  inject_timeout: a test hook whose last dependency is never
// met, so its bounded waits run out (DMUON_ERR_TIMEOUT).
struct ChainBuffers {
  void* x[2];
  void* slot[5];
  unsigned* counters;
};
bool tc_chain_fusable(int m, const std::vector<int>& blocks);
// True when the chain's products average at most two waves of tiles on a
// B200 (74 CTA pairs or 148 CTAs): launched one by one they would be
// dominated by launch, ramp-up and tail, so the fused launch pays off.  Large
// chunks run one launch per product (measured faster there).
bool tc_chain_small(int batch, int m, int n, const std::vector<int>& blocks);
cudaError_t tc_chain(const ChainBuffers& buf, int batch, int m, int n, int64_t ldn, int64_t ldm,
                     const std::vector<int>& blocks, const float* sched, const float* scale, const UpdTable* upd,
                     int* status, int num_sms, bool inject_timeout, cudaStream_t st, int* result_x);
// decay = 1 - lr wd and step_scale = fl32(lr 0.2 sqrt(scale_dim)), each rounded
// as the update kernels use them.
void update_coeffs(float lr, float wd, int64_t scale_dim, float* decay, float* step_scale);
const char* tc_config_string();
// One-thread kernel whose bounded wait runs out after limit_us (status word).
cudaError_t wait_selftest(int* status, int64_t limit_us, cudaStream_t st);

// ---- api.cu -------------------------------------------------------------------
// Sets the message returned by dmuon_get_last_error on this thread; returns s.
dmuon_status_t record_error(dmuon_status_t s, const std::string& msg);
struct ChunkLayout;
struct ChunkOffsets;
// The Newton-Schulz chain that dmuon_ns_ex and dmuon_step run, over a chunk of
// `b` oriented m x n matrices whose x0 is in the workspace `ws` (laid out by
// chunk_offsets, per-matrix scales filled in); sched holds 3 * steps
// coefficients (a, b, c per iteration); *result receives the buffer holding
// the result.  `status` is the device status word the kernels'
// bounded waits report to; `sms` the device's SM count.
dmuon_status_t ns_chain(const ChunkLayout& L, int b, int64_t m, int64_t n, char* ws, const ChunkOffsets& off,
                        int32_t steps, const float* sched, int* status, int sms, cudaStream_t st,
                        void** result);

// ---- plan.cpp -----------------------------------------------------------------
struct Group {
  int64_t rows, cols;
  int32_t dtype;
  std::vector<int32_t> members;  // ascending indices
};
// Groups by (rows, cols, dtype) in order of first appearance.
std::vector<Group> plan_groups(const dmuon_shape_t* shapes, int32_t count);

// A launch class: groups with the same oriented shape (m, n) and dtype.
struct LaunchClass {
  int64_t m, n;
  int32_t dtype;
  std::vector<int32_t> members;  // in group order, ascending within a group
};
std::vector<LaunchClass> plan_classes(const std::vector<Group>& groups);

// Per-chunk workspace layout of a launch class.
struct ChunkLayout {
  Path path;
  bool blocked;            // Gram-space blocks of iterations (tensor path, n >= 1.25 m)
  int gslots;              // m x m buffers: 2 (G, P) or 5 (blocked)
  int64_t ldn, ldm;        // row pitches (elements) of X and of G/P
  int64_t xbytes, gbytes;  // bytes of one X (one matrix) and of one G
  int64_t tiles_per_mat;   // elementwise tiles
  int64_t per_matrix;      // workspace bytes per matrix in a chunk
};
// allow_blocked = false keeps the per-iteration form (two m x m buffers).
ChunkLayout chunk_layout(int64_t m, int64_t n, int32_t dtype, bool allow_blocked = true);
// Storage type of X in the workspace of a layout.
inline int32_t x_dtype(const ChunkLayout& L, int32_t dtype) {
  return L.path == Path::kBf16F32 ? (int32_t)DMUON_F32 : dtype;
}
// Iteration blocks of the chain for `steps` iterations: all 1 in the
// per-iteration form; otherwise the Gram-space schedule of DMUON_GRAM_BLOCKS
// (default: per-iteration steps, then the last two iterations as one block;
// "2": blocks of 2, 3, 3, ...).
std::vector<int> chain_blocks(const ChunkLayout& L, int32_t steps);
int64_t workspace_cap_bytes();
int64_t chunk_size(const ChunkLayout& L, int64_t members, int64_t cap);
// Offsets of the pieces of a chunk of `b` matrices inside the workspace.
struct ChunkOffsets {
  int64_t x0, x1, g, p, partials, scale, counters, total;  // counters: fused-chain dependencies
};
ChunkOffsets chunk_offsets(const ChunkLayout& L, int64_t b);

// The chunks of one dmuon_step in execution order.  With two or more chunks
// (and DMUON_OVERLAP not "0") the step runs overlapped: two workspace buffers
// of half the cap each, chunk i in buffer i % 2, the elementwise stages of
// neighbouring chunks on an auxiliary stream under the Newton-Schulz chain.
struct ChunkRef {
  size_t cls;    // launch class
  size_t start;  // first member of the class in this chunk
  int b;         // matrices in the chunk
};
struct StepPlan {
  std::vector<LaunchClass> classes;
  std::vector<ChunkLayout> layouts;
  std::vector<ChunkRef> chunks;
  bool overlap = false;
  int64_t buffer_bytes = 0;  // one buffer (two are used when overlapping)
};
StepPlan make_step_plan(const dmuon_shape_t* shapes, int32_t count);
// Dedicated ownership of `count` matrices over `world` ranks (see
// dmuon_assign_owners); loads has `world` entries.
void assign_owners(const dmuon_shape_t* shapes, int32_t count, int32_t world, int32_t* owner_of, double* loads);

}  // namespace dmuon
