// C ABI of the Muon-step library: argument validation, device state,
// workspace cache and the orchestration of one step.
//
// dmuon_step (DMuon Training Guide, "Step 4": momentum + NS + update for the
// dedicated parameters) runs, per launch class (same oriented shape and
// dtype) and per chunk of at most 256 matrices that fits the workspace cap:
//   momentum+norm partials -> norm finalise -> the Newton-Schulz chain
//   (ns_steps x (gram, poly, apply); wide matrices on the tensor path run
//   their last two iterations as one Gram-space block) -> update
// With several chunks the elementwise stages run on an internal stream
// underneath the chains of neighbouring chunks (two workspace buffers), the
// chains on a second, higher-priority internal stream, ordered by events and
// joined back into the caller's stream; there is no host synchronisation.
//
// Environment switches (read per call): DMUON_WS_CAP_MB (workspace cap,
// default 8 GiB), DMUON_OVERLAP=0 (serial schedule), DMUON_GRAM_BLOCKS=0|2
// (per-iteration form | Gram-space blocks of 2, 3, 3, ...),
// DMUON_TC_CTA_PAIR=0 (one-CTA tensor-core kernel only, read once),
// DMUON_SMALL_CHAIN=0 (thin matrices on the per-product FFMA kernels),
// DMUON_FAULT_INJECT=alloc (workspace allocation fails) or =launch (dmuon_step
// reports a failed launch before its first chain), for tests;
// DMUON_NVTX=1 (NVTX ranges per step, chunk chain and clip stage, for
// profilers: `ncu --nvtx --nvtx-include "dmuon_step/"`).
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "bounds.cuh"
#include "internal.h"

namespace dmuon {
namespace {

thread_local std::string g_last_error;

dmuon_status_t fail(dmuon_status_t s, const std::string& msg) {
  g_last_error = msg;
  return s;
}

dmuon_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(DMUON_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

struct DeviceState {
  int sm_count = 0;
  int major = 0, minor = 0;
  int* status_word = nullptr;
};

std::mutex g_mu;
std::map<int, DeviceState> g_devices;
std::map<std::pair<int, uintptr_t>, std::pair<void*, size_t>> g_workspace;

dmuon_status_t device_state(DeviceState* out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_devices.find(dev);
  if (it == g_devices.end()) {
    DeviceState ds;
    e = cudaDeviceGetAttribute(&ds.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&ds.major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&ds.minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    if (ds.major != 10)
      return fail(DMUON_ERR_UNSUPPORTED, "device is sm_" + std::to_string(ds.major) +
                                             std::to_string(ds.minor) + "; this library is built for sm_100a");
    e = cudaMalloc(&ds.status_word, sizeof(int));
    if (e != cudaSuccess) return fail(DMUON_ERR_OOM, "status word allocation failed");
    e = cudaMemset(ds.status_word, 0, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset");
    it = g_devices.emplace(dev, ds).first;
  }
  *out = it->second;
  return DMUON_OK;
}

bool env_is(const char* name, char first) {
  const char* e = std::getenv(name);
  return e && e[0] == first;
}

// An NVTX range for the scope when DMUON_NVTX=1 (a no-op without a tool attached).
struct NvtxRange {
  bool on;
  explicit NvtxRange(const std::string& name) : on(env_is("DMUON_NVTX", '1')) {
    if (on) nvtxRangePushA(name.c_str());
  }
  ~NvtxRange() {
    if (on) nvtxRangePop();
  }
};

// One check of element offset 1 in a one-element extent; no memory is
// touched in either build (release: the check is the constant true).
__global__ void k_bounds_selftest(int* status) { (void)DMUON_IN(status, 1, 1, 1); }

bool fault_injected(const char* what) {
  const char* e = std::getenv("DMUON_FAULT_INJECT");
  return e && std::strcmp(e, what) == 0;
}
// DMUON_FAULT_INJECT=chain_wait: the fused chain's last dependency is never
// met, so its bounded waits run out (for the failure-detection test)
bool env_is_inject_chain() { return fault_injected("chain_wait"); }

// Stream-ordered, grow-only workspace per (device, stream).
dmuon_status_t get_workspace(size_t bytes, cudaStream_t st, void** out) {
  if (fault_injected("alloc")) return fail(DMUON_ERR_OOM, "workspace allocation failed (injected)");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_mu);
  auto key = std::make_pair(dev, reinterpret_cast<uintptr_t>(st));
  auto& slot = g_workspace[key];
  if (slot.first && slot.second >= bytes) {
    *out = slot.first;
    return DMUON_OK;
  }
  // growing inside a stream capture would make the cached workspace memory
  // owned by the graph: the first call with these shapes must run uncaptured
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) {
    cudaGetLastError();
    cap = cudaStreamCaptureStatusNone;
  }
  if (cap != cudaStreamCaptureStatusNone)
    return fail(DMUON_ERR_INVALID_ARG, "the stream is capturing and its workspace needs " + std::to_string(bytes) +
                                           " bytes it does not have yet: make one call with these shapes on this "
                                           "stream before capturing");
  if (slot.first) {
    cudaFreeAsync(slot.first, st);
    slot = {nullptr, 0};
  }
  void* p = nullptr;
  e = cudaMallocAsync(&p, bytes, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(DMUON_ERR_OOM, "workspace allocation of " + std::to_string(bytes) + " bytes failed: " +
                                   cudaGetErrorString(e));
  }
  slot = {p, bytes};
  *out = p;
  return DMUON_OK;
}

// Internal streams per (device, caller stream) of an overlapped step: `aux`
// (least priority) for the elementwise stages, `chain` (greatest priority) for
// the Newton-Schulz chains.  The priorities matter when a chain kernel is
// launched while a momentum kernel still has blocks waiting: the block
// scheduler then places the chain kernel's persistent CTAs first, instead of
// letting the waiting momentum blocks take the SMs as they free up (which
// delayed the chain kernel by about the momentum kernel's whole duration).
struct SideStreams {
  cudaStream_t aux = nullptr, chain = nullptr, chain2 = nullptr;
};
std::map<std::pair<int, uintptr_t>, SideStreams> g_side;

dmuon_status_t get_side_streams(cudaStream_t st, SideStreams* out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_mu);
  auto key = std::make_pair(dev, reinterpret_cast<uintptr_t>(st));
  auto it = g_side.find(key);
  if (it == g_side.end()) {
    int least = 0, greatest = 0;
    e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    SideStreams ss;
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&ss.aux, cudaStreamNonBlocking, least);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&ss.chain, cudaStreamNonBlocking, greatest);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&ss.chain2, cudaStreamNonBlocking, greatest);
    if (e != cudaSuccess) {
      if (ss.aux) cudaStreamDestroy(ss.aux);
      if (ss.chain) cudaStreamDestroy(ss.chain);
      return cuda_fail(e, "cudaStreamCreateWithPriority");
    }
    it = g_side.emplace(key, ss).first;
  }
  *out = it->second;
  return DMUON_OK;
}

// `waiter` waits for everything enqueued so far on `signaller`.
cudaError_t stream_after(cudaStream_t waiter, cudaStream_t signaller) {
  cudaEvent_t ev;
  cudaError_t e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
  if (e != cudaSuccess) return e;
  e = cudaEventRecord(ev, signaller);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(waiter, ev, 0);
  cudaEventDestroy(ev);  // released once the recorded work completes
  return e;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t esize(int32_t dtype) { return dtype == DMUON_BF16 ? 2 : 4; }
bool dtype_ok(int32_t d) { return d == DMUON_F32 || d == DMUON_BF16; }

// ------------------------------------------------------------ kernel timing
enum Kind { kMomentum, kNorm, kGramTc, kPolyTc, kApplyTc, kGramFfma, kPolyFfma, kApplyFfma, kUpdate,
            kLoad, kCopyOut, kSymmTc, kChainSmall, kClipNorm, kClipScale, kApplyUpdTc, kChainTc, kChainFfma,
            kNumKinds };
const char* const kKindNames[kNumKinds] = {"momentum", "norm", "gram_tc", "poly_tc", "apply_tc",
                                           "gram_ffma", "poly_ffma", "apply_ffma", "update", "load",
                                           "copy_out", "symm_tc", "chain_small", "clip_norm", "clip_scale",
                                           "apply_update_tc", "chain_tc", "chain_ffma"};
struct ProfRec {
  int kind;
  cudaEvent_t a, b;
  double flops, bytes;
};
thread_local bool g_prof_on = false;
thread_local std::vector<ProfRec> g_prof;
// Event pairs reused from one profiling window to the next, so that a window
// whose launches were seen before creates no events (only records them).
thread_local std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_prof_pool;

// Brackets one kernel launch with events when profiling is on.
struct Prof {
  bool on;
  ProfRec r;
  Prof(int kind, cudaStream_t st, double flops, double bytes) : on(g_prof_on) {
    if (!on) return;
    r = ProfRec{kind, nullptr, nullptr, flops, bytes};
    const size_t i = g_prof.size();
    if (i < g_prof_pool.size()) {
      r.a = g_prof_pool[i].first;
      r.b = g_prof_pool[i].second;
    } else {
      if (cudaEventCreate(&r.a) != cudaSuccess) {
        on = false;
        return;
      }
      if (cudaEventCreate(&r.b) != cudaSuccess) {
        cudaEventDestroy(r.a);
        on = false;
        return;
      }
      g_prof_pool.emplace_back(r.a, r.b);
    }
    cudaEventRecord(r.a, st);
  }
  void done(cudaStream_t st) {
    if (!on) return;
    cudaEventRecord(r.b, st);
    g_prof.push_back(r);
    on = false;
  }
};

constexpr int64_t kMaxSide = int64_t(1) << 20;
constexpr int64_t kMaxElems = (int64_t(1) << 31) - 1;

dmuon_status_t check_shape(int64_t rows, int64_t cols, const char* what) {
  if (rows <= 0 || cols <= 0 || rows > kMaxSide || cols > kMaxSide || rows * cols > kMaxElems)
    return fail(DMUON_ERR_INVALID_ARG, std::string(what) + ": shape " + std::to_string(rows) + "x" +
                                           std::to_string(cols) + " out of range (sides 1..2^20, < 2^31 elements)");
  return DMUON_OK;
}

dmuon_status_t coeff_schedule(int32_t steps, const float* coeffs, std::vector<float>& out) {
  out.resize(3 * (size_t)steps);
  for (int32_t k = 0; k < steps; ++k) {
    if (coeffs) {
      out[3 * k] = coeffs[3 * k];
      out[3 * k + 1] = coeffs[3 * k + 1];
      out[3 * k + 2] = coeffs[3 * k + 2];
    } else {
      out[3 * k] = DMUON_DEFAULT_A;
      out[3 * k + 1] = DMUON_DEFAULT_B;
      out[3 * k + 2] = DMUON_DEFAULT_C;
    }
  }
  return DMUON_OK;
}

struct Interval {
  uintptr_t lo, hi;
  int who;
};

// True if any two intervals overlap.
bool any_overlap(std::vector<Interval>& v) {
  std::sort(v.begin(), v.end(), [](const Interval& a, const Interval& b) { return a.lo < b.lo; });
  for (size_t i = 1; i < v.size(); ++i)
    if (v[i].lo < v[i - 1].hi) return true;
  return false;
}

// The Newton-Schulz chain over a chunk of `b` oriented m x n matrices in the
// workspace; returns the buffer that holds the result.
// Thin matrices (m <= 64, FFMA path) whose chain runs as one clustered launch.
bool thin_chain(const ChunkLayout& L, int64_t m, int64_t n, int32_t steps) {
  return L.path != Path::kTensorBf16 && m <= kSmallM && steps >= 1 && steps <= 16 &&
         n <= small_ns_max_n((int)m, L.path == Path::kSmallBf16 ? 2 : 4) && !env_is("DMUON_SMALL_CHAIN", '0');
}

// The tensor-path chain of a chunk runs as one persistent launch when its
// products are small (tc_chain_small) and the chain can (tc_chain_fusable);
// DMUON_FUSED_CHAIN=1 fuses every chain that can be fused, =0 none.
// FFMA chains always fuse (their products are small: a few dozen tiles per
// launch otherwise), up to 16 iterations, unless DMUON_FUSED_CHAIN=0.
bool fuse_ffma_chain(const ChunkLayout& L, int32_t steps) {
  return L.path != Path::kTensorBf16 && steps >= 1 && steps <= 16 && !env_is("DMUON_FUSED_CHAIN", '0');
}

bool fuse_chain(const ChunkLayout& L, int b, int64_t m, int64_t n, int32_t steps) {
  if (L.path != Path::kTensorBf16 || env_is("DMUON_FUSED_CHAIN", '0')) return false;
  const std::vector<int> blocks = chain_blocks(L, steps);
  if (!tc_chain_fusable((int)m, blocks)) return false;
  return env_is("DMUON_FUSED_CHAIN", '1') || tc_chain_small(b, (int)m, (int)n, blocks);
}

// The chunk's whole chain is one launch (thin, FFMA or small tensor chain).
// Such chains are latency-bound (a few waves of tiles per product at most),
// so two consecutive ones run on two chain streams and share the GPU;
// DMUON_CHAIN_STREAMS=1 keeps one stream.  Large chains keep one stream: two
// of them at once only draw more power under the cap.
bool one_launch_chain(const ChunkLayout& L, int b, int64_t m, int64_t n, int32_t steps) {
  if (env_is("DMUON_CHAIN_STREAMS", '1')) return false;
  return thin_chain(L, m, n, steps) || fuse_ffma_chain(L, steps) || fuse_chain(L, b, m, n, steps);
}

// Executed flops of a tensor-path chain: gram m^2 n, symmetric products m^3,
// applies 2 m^2 n per matrix (one triangle of every symmetric product).
double chain_flops(const std::vector<int>& blocks, double m, double n) {
  double f = 0.0;
  for (int len : blocks)
    f += m * m * n + (len == 1 ? 1.0 : (len == 2 ? 5.0 : 9.0)) * m * m * m + 2.0 * m * m * n;
  return f;
}

// The tensor path ends with a tensor-core apply, whose epilogue can update
// the parameters directly (DMUON_FUSED_UPDATE=0 keeps the separate pass).
bool fuses_update(const ChunkLayout& L, int32_t steps) {
  return L.path == Path::kTensorBf16 && steps >= 1 && !env_is("DMUON_FUSED_UPDATE", '0');
}

// upd (optional, only where fuses_update): the last apply updates the
// parameters in its epilogue and stores no result (*result = nullptr).
dmuon_status_t run_chain(const ChunkLayout& L, int b, int64_t m, int64_t n, char* ws,
                         const ChunkOffsets& off, int32_t steps, const float* sched,
                         int* sw, int sms, cudaStream_t st, void** result,
                         const UpdTable* upd = nullptr) {
  void* cur = ws + off.x0;
  void* nxt = ws + off.x1;
  void* G = ws + off.g;
  void* P = ws + off.p;
  const float* scale = reinterpret_cast<const float*>(ws + off.scale);
  const bool tc = L.path == Path::kTensorBf16;
  const bool xbf16 = L.path == Path::kSmallBf16;
  const double fm = (double)m, fn = (double)n, fb = (double)b;
  const int mi = (int)m, ni = (int)n;
  cudaError_t e = cudaSuccess;
  // the chain's symmetric matrices are stored as their lower 256-column blocks
  // and read back so (DMUON_LOWER_STORE=0: stored in full)
  const bool low = !env_is("DMUON_LOWER_STORE", '0');
  // m x m slot s of the chunk (slot 0 is G, the rest follow P)
  auto slot = [&](int s) -> char* { return s == 0 ? (char*)G : (char*)P + (int64_t)(s - 1) * ((off.p - off.g)); };
  auto gram = [&](const void* X, void* out, const float* sc) {
    Prof p(tc ? kGramTc : kGramFfma, st, fb * fm * fm * fn, 0.0);
    e = tc ? tc_gram(X, out, b, mi, ni, L.ldn, L.ldm, 1.f, sc, sw, sms, st, low)
           : simt_gram(X, out, b, mi, ni, L.ldn, L.ldm, 1.f, sc, xbf16, st, sw);
    p.done(st);
  };
  bool fused = false;
  auto apply = [&](const void* Pm, const void* X, void* Y, float a, const float* sc, bool last) {
    if (tc && last && upd) {
      // update bytes: read and write p
      Prof p(kApplyUpdTc, st, 2.0 * fb * fm * fm * fn, 4.0 * fb * fm * fn);
      e = tc_apply_update(Pm, X, b, mi, ni, L.ldm, L.ldn, a, 1.f, sc, *upd, sw, sms, st, low);
      p.done(st);
      fused = true;
      return;
    }
    Prof p(tc ? kApplyTc : kApplyFfma, st, 2.0 * fb * fm * fm * fn, 0.0);
    e = tc ? tc_apply(Pm, X, Y, b, mi, ni, L.ldm, L.ldn, L.ldn, a, 1.f, sc, sw, sms, st, low)
           : simt_apply(Pm, X, Y, b, mi, ni, L.ldm, L.ldn, L.ldn, a, 1.f, sc, xbf16, st, sw);
    p.done(st);
  };
  // C = p1 (A B) + p0 E + p2 I on the tensor path (A, B symmetric and commuting)
  auto symm = [&](const void* A, const void* B, const void* E, void* C, float p0, float p1, float p2, int kind) {
    Prof p(kind, st, fb * fm * fm * fm, 0.0);
    e = tc_symm(A, B, E, C, b, mi, L.ldm, L.ldm, L.ldm, L.ldm, p0, p1, p2, sw, sms, st, low);
    p.done(st);
  };
  const auto coef = [&](int k, int i) { return sched[3 * k + i]; };

  // thin matrices: the whole chain in one clustered launch, in place on X0
  if (thin_chain(L, m, n, steps)) {
    Prof p(kChainSmall, st, fb * (3.0 * fm * fm * fn + fm * fm * fm) * steps, 0.0);
    e = small_ns(cur, b, mi, ni, L.ldn, steps, sched, scale, xbf16, st, sw);
    p.done(st);
    if (e != cudaSuccess) return cuda_fail(e, "Newton-Schulz launch");
    *result = cur;
    return DMUON_OK;
  }

  // FFMA chains (fp32, small near-square bf16, thin bf16 beyond the clustered
  // kernel): every product in one launch (same tiles, same arithmetic, same bits)
  if (!tc && fuse_ffma_chain(L, steps)) {
    void* xs[2] = {cur, nxt};
    int rx = 0;
    Prof p(kChainFfma, st, fb * (3.0 * fm * fm * fn + fm * fm * fm) * steps, 0.0);
    e = simt_chain(xs, G, P, b, mi, ni, L.ldn, L.ldm, steps, sched, scale, xbf16,
                   reinterpret_cast<unsigned*>(ws + off.counters), sw, sms, env_is_inject_chain(), st, &rx);
    p.done(st);
    if (e == cudaSuccess) {
      *result = rx == 0 ? cur : nxt;
      return DMUON_OK;
    }
    if (e != cudaErrorNotSupported) return cuda_fail(e, "fused FFMA chain launch");
    e = cudaSuccess;  // too many iterations: product by product below
  }

  // the whole chain in one persistent launch (same tiles, same epilogues, same bits)
  if (tc && fuse_chain(L, b, m, n, steps)) {
    const std::vector<int> blocks = chain_blocks(L, steps);
    ChainBuffers cb{};
    cb.x[0] = cur;
    cb.x[1] = nxt;
    for (int i = 0; i < L.gslots && i < 5; ++i) cb.slot[i] = slot(i);
    cb.counters = reinterpret_cast<unsigned*>(ws + off.counters);
    int rx = 0;
    Prof p(kChainTc, st, fb * chain_flops(blocks, fm, fn), upd ? 4.0 * fb * fm * fn : 0.0);
    e = tc_chain(cb, b, mi, ni, L.ldn, L.ldm, blocks, sched, scale, upd, sw, sms, env_is_inject_chain(), st, &rx);
    p.done(st);
    if (e == cudaSuccess) {
      *result = rx < 0 ? nullptr : (rx == 0 ? cur : nxt);
      return DMUON_OK;
    }
    if (e != cudaErrorNotSupported) return cuda_fail(e, "fused chain launch");
    e = cudaSuccess;  // not fusable: the chain runs product by product below
  }

  // Blocks of iterations (chain_blocks).  A block of one is the iteration as
  // written: G = X X^T, then X <- p(G) X.  The tensor path stores p(G) =
  // a I + b G + c G G (the identity term in the polynomial's epilogue) and
  // applies it as one product; the FFMA path keeps P = b G + c G G and adds
  // a X in the apply's epilogue (X <- a X + P X).  In a longer block
  // every matrix is a polynomial of the block's Gram matrix G:
  //   P_j = p_j(G_j) (with a I),  G_{j+1} = P_j G_j P_j,  Q = P_j ... P_0,
  // and the block ends with X <- Q X (a fresh G starts the next block).
  int k = 0;
  for (int len : chain_blocks(L, steps)) {
    if (e != cudaSuccess) break;
    const float* sc = k == 0 ? scale : nullptr;
    if (len == 1) {
      gram(cur, G, sc);
      if (e != cudaSuccess) break;
      if (tc) {
        symm(G, G, G, P, coef(k, 1), coef(k, 2), coef(k, 0), kPolyTc);  // P = a I + b G + c G G
      } else {
        Prof p(kPolyFfma, st, fb * fm * fm * fm, 0.0);
        e = simt_poly(G, P, b, mi, L.ldm, L.ldm, coef(k, 1), coef(k, 2), st, sw);
        p.done(st);
      }
      if (e != cudaSuccess) break;
      apply(P, cur, nxt, tc ? 0.f : coef(k, 0), sc, k + 1 == steps);
      std::swap(cur, nxt);
      k += 1;
      continue;
    }
    char* S0 = slot(0);  // G, G1, G2
    char* S1 = slot(1);  // P0, P2
    char* S2 = slot(2);  // T, Q2
    char* S3 = slot(3);  // P1
    char* S4 = slot(4);  // Q
    gram(cur, S0, sc);
    void* Q = S4;
    if (e == cudaSuccess) symm(S0, S0, S0, S1, coef(k, 1), coef(k, 2), coef(k, 0), kPolyTc);  // P0
    if (e == cudaSuccess) symm(S1, S0, nullptr, S2, 0.f, 1.f, 0.f, kSymmTc);                 // T = P0 G
    if (e == cudaSuccess) symm(S2, S1, nullptr, S0, 0.f, 1.f, 0.f, kSymmTc);                 // G1 = T P0
    if (e == cudaSuccess) symm(S0, S0, S0, S3, coef(k + 1, 1), coef(k + 1, 2), coef(k + 1, 0), kPolyTc);  // P1
    if (e == cudaSuccess) symm(S3, S1, nullptr, S4, 0.f, 1.f, 0.f, kSymmTc);                 // Q = P1 P0
    if (len == 3) {
      if (e == cudaSuccess) symm(S3, S0, nullptr, S2, 0.f, 1.f, 0.f, kSymmTc);  // T = P1 G1
      if (e == cudaSuccess) symm(S2, S3, nullptr, S0, 0.f, 1.f, 0.f, kSymmTc);  // G2 = T P1
      if (e == cudaSuccess) symm(S0, S0, S0, S1, coef(k + 2, 1), coef(k + 2, 2), coef(k + 2, 0), kPolyTc);  // P2
      if (e == cudaSuccess) symm(S1, S4, nullptr, S2, 0.f, 1.f, 0.f, kSymmTc);  // Q2 = P2 Q
      Q = S2;
    }
    if (e == cudaSuccess) apply(Q, cur, nxt, 0.f, sc, k + len == steps);  // X <- Q X (scaled by s when k == 0)
    std::swap(cur, nxt);
    k += len;
  }
  if (e != cudaSuccess) return cuda_fail(e, "Newton-Schulz launch");
  *result = fused ? nullptr : cur;
  return DMUON_OK;
}

// Kernels one chunk launches: momentum, norm, the chain, update (unless fused).
int64_t chunk_launches_for(const ChunkLayout& L, int b, int64_t m, int64_t n, int32_t steps) {
  int64_t k = fuses_update(L, steps) ? 2 : 3;
  if (thin_chain(L, m, n, steps)) return k + 1;
  if (fuse_ffma_chain(L, steps) || fuse_chain(L, b, m, n, steps)) return k + 1;
  for (int len : chain_blocks(L, steps)) k += len == 1 ? 3 : (len == 2 ? 7 : 11);  // gram + products + apply
  return k;
}

// ----------------------------------------------------------- gradient clipping

struct ClipReq {
  int p;            // 2, 1, or 0 for the infinity norm
  float max_norm;
  double* total;    // device, optional
};

dmuon_status_t parse_clip(float max_norm, float norm_type, int* p) {
  if (!std::isfinite(max_norm) || max_norm < 0.f) return fail(DMUON_ERR_INVALID_ARG, "max_norm must be finite and >= 0");
  if (norm_type == 2.f) *p = 2;
  else if (norm_type == 1.f) *p = 1;
  else if (std::isinf(norm_type) && norm_type > 0.f) *p = 0;
  else return fail(DMUON_ERR_UNSUPPORTED, "norm_type must be 1, 2 or inf");
  return DMUON_OK;
}

int64_t tiles_of(int64_t rows, int64_t cols) { return (rows * cols + kClipChunk - 1) / kClipChunk; }

int64_t clip_tiles(const std::vector<Group>& groups) {
  int64_t t = 0;
  for (const Group& g : groups) t += (int64_t)g.members.size() * tiles_of(g.rows, g.cols);
  return t;
}

// Bytes of clip workspace: one fp32 partial per 64x64 tile, then the coefficient.
size_t clip_ws_bytes(int64_t tiles) { return (size_t)(((tiles * 4 + 15) / 16) * 16 + 16); }
float* clip_coef_ptr(void* ws, int64_t tiles) {
  return reinterpret_cast<float*>(static_cast<char*>(ws) + ((tiles * 4 + 15) / 16) * 16);
}

// Calls fn(table, dtype, partials offset, bytes) for every table of at most
// kMaxTable matrices of one source shape (src = buf = the gradient).
template <typename Fn>
cudaError_t for_each_clip_table(const std::vector<Group>& groups, const void* const* grads, ElemTable* tab, Fn&& fn) {
  int64_t offset = 0;
  for (const Group& g : groups) {
    const size_t es = esize(g.dtype);
    const int32_t tpm = (int32_t)tiles_of(g.rows, g.cols);
    for (size_t start = 0; start < g.members.size(); start += kMaxTable) {
      const int b = (int)std::min<size_t>(kMaxTable, g.members.size() - start);
      tab->m = g.rows;
      tab->n = g.cols;
      tab->ldn = g.cols;
      tab->count = b;
      tab->tiles_per_mat = tpm;
      for (int j = 0; j < b; ++j) {
        const int32_t i = g.members[start + j];
        tab->e[j] = MatEntry{grads[i], const_cast<void*>(grads[i]), nullptr, 0, aligned16(grads[i]) ? 1 : 0};
      }
      cudaError_t e = fn(*tab, g.dtype, offset, (double)b * (double)g.rows * (double)g.cols * (double)es);
      if (e != cudaSuccess) return e;
      offset += (int64_t)b * tpm;
    }
  }
  return cudaSuccess;
}

// The norm pass and the coefficient: coef = min(1, max_norm / (total + 1e-6)).
cudaError_t clip_norm_stage(const std::vector<Group>& groups, const void* const* grads, const ClipReq& req,
                            void* ws, int64_t tiles, ElemTable* tab, cudaStream_t st) {
  NvtxRange range("clip norm");
  float* partials = static_cast<float*>(ws);
  cudaError_t e = for_each_clip_table(groups, grads, tab, [&](const ElemTable& t, int32_t dtype, int64_t off, double bytes) {
    Prof pr(kClipNorm, st, 0.0, bytes);
    cudaError_t r = launch_clip_partials(t, dtype, req.p, partials + off, st);
    pr.done(st);
    return r;
  });
  if (e == cudaSuccess) e = launch_clip_coef(partials, tiles, req.p, req.max_norm, clip_coef_ptr(ws, tiles), req.total, st);
  return e;
}


dmuon_status_t step_impl(void* const* params, const void* const* grads, void* const* mom_bufs,
                         const dmuon_shape_t* shapes, int32_t count, float lr, float momentum,
                         int32_t nesterov, int32_t ns_steps, const float* coeffs, float wd,
                         const ClipReq* clip, dmuon_stream_t stream) {
  NvtxRange range(clip ? "dmuon_step_clipped" : "dmuon_step");
  // ---------------------------------------------------------- validation
  if (count < 0) return fail(DMUON_ERR_INVALID_ARG, "count < 0");
  if (ns_steps < 0 || ns_steps > 1000) return fail(DMUON_ERR_INVALID_ARG, "ns_steps must be in 0..1000");
  if (nesterov != 0 && nesterov != 1) return fail(DMUON_ERR_INVALID_ARG, "nesterov must be 0 or 1");
  if (!std::isfinite(lr) || !std::isfinite(momentum) || !std::isfinite(wd))
    return fail(DMUON_ERR_INVALID_ARG, "lr, momentum and wd must be finite");
  if (count == 0) return DMUON_OK;
  if (!params || !grads || !mom_bufs || !shapes) return fail(DMUON_ERR_INVALID_ARG, "null array argument");
  std::vector<Interval> iv;
  iv.reserve(3 * (size_t)count);
  for (int32_t i = 0; i < count; ++i) {
    const dmuon_shape_t& s = shapes[i];
    dmuon_status_t st = check_shape(s.rows, s.cols, "dmuon_step");
    if (st != DMUON_OK) return st;
    if (!dtype_ok(s.dtype)) return fail(DMUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": bad dtype");
    if (s.reserved != 0) return fail(DMUON_ERR_INVALID_ARG, "reserved shape field must be 0");
    if (!params[i] || !grads[i] || !mom_bufs[i])
      return fail(DMUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": null pointer");
    const uintptr_t bytes = (uintptr_t)(s.rows * s.cols) * esize(s.dtype);
    iv.push_back({(uintptr_t)params[i], (uintptr_t)params[i] + bytes, i});
    iv.push_back({(uintptr_t)grads[i], (uintptr_t)grads[i] + bytes, i});
    iv.push_back({(uintptr_t)mom_bufs[i], (uintptr_t)mom_bufs[i] + bytes, i});
  }
  if (any_overlap(iv)) return fail(DMUON_ERR_INVALID_ARG, "params, grads and momentum buffers must not overlap");
  std::vector<float> sched;
  coeff_schedule(ns_steps, coeffs, sched);

  // ------------------------------------------------------------- planning
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DeviceState ds;
  dmuon_status_t rc = device_state(&ds);
  if (rc != DMUON_OK) return rc;
  const StepPlan P = make_step_plan(shapes, count);
  const int nbuf = P.overlap ? 2 : 1;
  // clipping: one fp32 partial per gradient tile and the coefficient, after the chunk buffers
  std::vector<Group> clip_groups;
  int64_t clip_tile_count = 0;
  const size_t clip_off = (((size_t)P.buffer_bytes * nbuf + 255) / 256) * 256;
  if (clip) {
    clip_groups = plan_groups(shapes, count);
    clip_tile_count = clip_tiles(clip_groups);
  }
  void* wsv = nullptr;
  rc = get_workspace(clip ? clip_off + clip_ws_bytes(clip_tile_count) : (size_t)(P.buffer_bytes * nbuf), st, &wsv);
  if (rc != DMUON_OK) return rc;
  std::unique_ptr<ElemTable[]> tabs(new ElemTable[2]);
  tabs[0].status = tabs[1].status = ds.status_word;
  const float* clip_coef = nullptr;
  if (clip) {
    void* cws = static_cast<char*>(wsv) + clip_off;
    cudaError_t e = clip_norm_stage(clip_groups, grads, *clip, cws, clip_tile_count, &tabs[0], st);
    if (e != cudaSuccess) return cuda_fail(e, "clip norm launch");
    clip_coef = clip_coef_ptr(cws, clip_tile_count);
  }
  // when overlapping, the elementwise stages run on `aux` and the chains on
  // `cs` (or `cs2`, see one_launch_chain); otherwise everything runs on the
  // caller's stream
  cudaStream_t aux = st, cs = st, cs2 = st;
  if (P.overlap) {
    SideStreams ss;
    rc = get_side_streams(st, &ss);
    if (rc != DMUON_OK) return rc;
    aux = ss.aux;
    cs = ss.chain;
    cs2 = ss.chain2;
    cudaError_t e = stream_after(aux, st);
    if (e == cudaSuccess) e = stream_after(cs, st);
    if (e == cudaSuccess) e = stream_after(cs2, st);
    if (e != cudaSuccess) {
      stream_after(st, aux);
      stream_after(st, cs);
      return cuda_fail(e, "stream fork");
    }
  }
  // Every return after the fork leaves the caller's stream ordered after both
  // internal streams, so a call that fails part-way leaves none of its work
  // unordered.
  struct JoinSide {
    cudaStream_t st, aux, cs, cs2;
    bool on;
    ~JoinSide() {
      if (on) {
        stream_after(st, aux);
        stream_after(st, cs);
        stream_after(st, cs2);
      }
    }
  } join{st, aux, cs, cs2, P.overlap};
  std::vector<void*> results(P.chunks.size(), nullptr);
  std::unique_ptr<UpdTable> upd_tab(new UpdTable());

  auto fill_table = [&](const ChunkRef& ck, ElemTable& tab) {
    const LaunchClass& c = P.classes[ck.cls];
    const size_t es = esize(c.dtype);
    tab.m = c.m;
    tab.n = c.n;
    tab.ldn = P.layouts[ck.cls].ldn;
    tab.count = ck.b;
    tab.tiles_per_mat = (int32_t)P.layouts[ck.cls].tiles_per_mat;
    for (int j = 0; j < ck.b; ++j) {
      const int32_t i = c.members[ck.start + j];
      MatEntry& e = tab.e[j];
      e.src = grads[i];
      e.buf = mom_bufs[i];
      e.dst = params[i];
      e.transposed = shapes[i].rows > shapes[i].cols ? 1 : 0;
      const bool row16 = ((int64_t)shapes[i].cols * (int64_t)es) % 16 == 0;
      e.pad = ((row16 && aligned16(grads[i]) && aligned16(mom_bufs[i])) ? 1 : 0) |
              ((row16 && aligned16(params[i])) ? 2 : 0);
    }
  };
  auto buffer = [&](size_t i) { return static_cast<char*>(wsv) + (int64_t)(i % nbuf) * P.buffer_bytes; };
  // the parameter update of chunk i, unless its last apply already did it
  auto update = [&](size_t i) -> dmuon_status_t {
    if (!results[i]) return DMUON_OK;
    const ChunkRef& ck = P.chunks[i];
    const LaunchClass& c = P.classes[ck.cls];
    const ChunkOffsets off = chunk_offsets(P.layouts[ck.cls], ck.b);
    const float* scale = reinterpret_cast<const float*>(buffer(i) + off.scale);
    const double elems = (double)ck.b * (double)c.m * (double)c.n;
    Prof pu(kUpdate, aux, 0.0, 3.0 * elems * (double)esize(c.dtype));
    cudaError_t e = launch_update(tabs[i % 2], c.dtype, ElemMode::kUpdate, results[i], ns_steps == 0 ? scale : nullptr,
                                  lr, wd, c.n, aux, x_dtype(P.layouts[ck.cls], c.dtype));
    pu.done(aux);
    return e == cudaSuccess ? DMUON_OK : cuda_fail(e, "update launch");
  };

  // ------------------------------------------------------------ execution
  // aux: M0 N0 | M1 N1 U0 | M2 N2 U1 | ...   cs: chain0 | chain1 | ...
  // U(i-1) waits only for chain(i-1) (event recorded when it was enqueued);
  // M(i+1) comes after that wait, so it overwrites buffer (i+1) % 2 only once
  // chain(i-1), which used it, is done.  A one-launch chain whose predecessor
  // ran on cs runs on cs2: it waits for its own momentum (so for chain(i-2))
  // but not for chain(i-1), which uses the other buffer.  Without overlap,
  // cs, cs2 and aux are the caller's stream.
  cudaEvent_t chain_done = nullptr;
  cudaStream_t prev_cs = cs2;  // stream of the previous chunk's chain
  auto drop = [&]() {
    if (chain_done) cudaEventDestroy(chain_done);  // released once complete
    chain_done = nullptr;
  };
  for (size_t i = 0; i < P.chunks.size(); ++i) {
    const ChunkRef& ck = P.chunks[i];
    const LaunchClass& c = P.classes[ck.cls];
    const ChunkLayout& L = P.layouts[ck.cls];
    const ChunkOffsets off = chunk_offsets(L, ck.b);
    char* ws = buffer(i);
    fill_table(ck, tabs[i % 2]);
    float* partials = reinterpret_cast<float*>(ws + off.partials);
    float* scale = reinterpret_cast<float*>(ws + off.scale);
    const double elems = (double)ck.b * (double)c.m * (double)c.n;
    Prof pm(kMomentum, aux, 0.0, 4.0 * elems * (double)esize(c.dtype));
    cudaError_t e = launch_momentum(tabs[i % 2], c.dtype, ElemMode::kMomentum, ws + off.x0, partials, momentum,
                                    nesterov, aux, clip_coef, x_dtype(L, c.dtype));
    pm.done(aux);
    if (e != cudaSuccess) {
      drop();
      return cuda_fail(e, "momentum launch");
    }
    Prof pn(kNorm, aux, 0.0, 4.0 * (double)ck.b * (double)L.tiles_per_mat);
    e = launch_norm_finalize(partials, ck.b, (int)L.tiles_per_mat, scale, nullptr, aux);
    pn.done(aux);
    const cudaStream_t csi =
        (P.overlap && prev_cs == cs && one_launch_chain(L, ck.b, c.m, c.n, ns_steps)) ? cs2 : cs;
    prev_cs = csi;
    if (e == cudaSuccess && P.overlap) e = stream_after(csi, aux);
    if (e != cudaSuccess) {
      drop();
      return cuda_fail(e, "norm launch / stream join");
    }
    const UpdTable* upd = nullptr;
    if (fuses_update(L, ns_steps)) {
      UpdTable& u = *upd_tab;
      update_coeffs(lr, wd, c.n, &u.decay, &u.step_scale);
      std::memset(u.tmask, 0, sizeof(u.tmask));
      std::memset(u.vmask, 0, sizeof(u.vmask));
      for (int j = 0; j < ck.b; ++j) {
        const int32_t mi = c.members[ck.start + j];
        u.p[j] = params[mi];
        if (shapes[mi].rows > shapes[mi].cols) u.tmask[j >> 5] |= 1u << (j & 31);
        if ((shapes[mi].cols * (int64_t)esize(c.dtype)) % 16 == 0 && aligned16(params[mi]))
          u.vmask[j >> 5] |= 1u << (j & 31);
      }
      upd = &u;
    }
    if (i == 0 && fault_injected("launch")) {
      drop();
      return cuda_fail(cudaErrorLaunchFailure, "first chain launch (injected failure)");
    }
    {
      NvtxRange r("chain " + std::to_string(c.m) + "x" + std::to_string(c.n) + " x" + std::to_string(ck.b));
      rc = run_chain(L, ck.b, c.m, c.n, ws, off, ns_steps, sched.data(), ds.status_word, ds.sm_count, csi,
                     &results[i], upd);
    }
    if (rc != DMUON_OK) {
      drop();
      return rc;
    }
    if (!P.overlap) {
      rc = update(i);
      if (rc != DMUON_OK) return rc;
      continue;
    }
    if (i >= 1) {
      e = cudaStreamWaitEvent(aux, chain_done, 0);
      if (e != cudaSuccess) {
        drop();
        return cuda_fail(e, "stream fork");
      }
      rc = update(i - 1);
      if (rc != DMUON_OK) {
        drop();
        return rc;
      }
    }
    drop();
    e = cudaEventCreateWithFlags(&chain_done, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(chain_done, csi);
    if (e != cudaSuccess) {
      drop();
      return cuda_fail(e, "chain event");
    }
  }
  if (P.overlap) {
    cudaError_t e = cudaStreamWaitEvent(aux, chain_done, 0);
    drop();
    if (e != cudaSuccess) return cuda_fail(e, "stream fork");
    rc = update(P.chunks.size() - 1);
    if (rc != DMUON_OK) return rc;
    join.on = false;
    e = stream_after(st, aux);
    if (e == cudaSuccess) e = stream_after(st, cs);
    if (e == cudaSuccess) e = stream_after(st, cs2);
    if (e != cudaSuccess) return cuda_fail(e, "stream join");
  }
  return DMUON_OK;
}

}  // namespace

dmuon_status_t record_error(dmuon_status_t s, const std::string& msg) { return fail(s, msg); }

dmuon_status_t ns_chain(const ChunkLayout& L, int b, int64_t m, int64_t n, char* ws, const ChunkOffsets& off,
                        int32_t steps, const float* sched, int* status, int sms, cudaStream_t st,
                        void** result) {
  return run_chain(L, b, m, n, ws, off, steps, sched, status, sms, st, result);
}

}  // namespace dmuon

using namespace dmuon;

// Shapes, dtypes and pointers of the gradients of a clip; none may overlap.
static dmuon_status_t check_clip_grads(void* const* grads, const dmuon_shape_t* shapes, int32_t count, const char* what) {
  if (!grads || !shapes) return fail(DMUON_ERR_INVALID_ARG, "null array argument");
  std::vector<Interval> iv;
  for (int32_t i = 0; i < count; ++i) {
    dmuon_status_t rc = check_shape(shapes[i].rows, shapes[i].cols, what);
    if (rc != DMUON_OK) return rc;
    if (!dtype_ok(shapes[i].dtype) || shapes[i].reserved != 0)
      return fail(DMUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": bad dtype or reserved field");
    if (!grads[i]) return fail(DMUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": null pointer");
    const uintptr_t bytes = (uintptr_t)(shapes[i].rows * shapes[i].cols) * esize(shapes[i].dtype);
    iv.push_back({(uintptr_t)grads[i], (uintptr_t)grads[i] + bytes, i});
  }
  if (any_overlap(iv)) return fail(DMUON_ERR_INVALID_ARG, "gradients must not overlap");
  return DMUON_OK;
}

extern "C" {

const char* dmuon_get_last_error(void) { return g_last_error.c_str(); }

const char* dmuon_build_info(void) {
  static std::string s = std::string("dmuon-b200 0.1.0; sm_100a; ") + tc_config_string() +
                         "; FFMA chain (64x64 or 32x32 tiles) for fp32, for bf16 with min side < 256 and max side < 3 x min,"
                         " and for bf16 with min side <= 64 beyond the clustered kernel; elementwise 64x64 tiles" +
#ifdef DMUON_DEBUG
                         "; debug bounds checks";
#else
                         "; release";
#endif
  return s.c_str();
}

dmuon_status_t dmuon_plan_groups(const dmuon_shape_t* shapes, int32_t count, int32_t* group_of,
                                 int32_t* order, int32_t* num_groups) {
  if (count < 0) return fail(DMUON_ERR_INVALID_ARG, "count < 0");
  if (!num_groups || (count > 0 && (!shapes || !group_of || !order)))
    return fail(DMUON_ERR_INVALID_ARG, "null pointer argument");
  std::vector<Group> groups = plan_groups(shapes, count);
  int32_t pos = 0;
  for (size_t g = 0; g < groups.size(); ++g)
    for (int32_t i : groups[g].members) {
      group_of[i] = (int32_t)g;
      order[pos++] = i;
    }
  *num_groups = (int32_t)groups.size();
  return DMUON_OK;
}

dmuon_status_t dmuon_assign_owners(const dmuon_shape_t* shapes, int32_t count, int32_t world, int32_t* owner_of,
                                   double* loads, double* imbalance) {
  if (count < 0) return fail(DMUON_ERR_INVALID_ARG, "count < 0");
  if (world < 1) return fail(DMUON_ERR_INVALID_ARG, "world must be >= 1");
  if (!loads || !imbalance || (count > 0 && (!shapes || !owner_of)))
    return fail(DMUON_ERR_INVALID_ARG, "null pointer argument");
  for (int32_t i = 0; i < count; ++i) {
    dmuon_status_t rc = check_shape(shapes[i].rows, shapes[i].cols, "dmuon_assign_owners");
    if (rc != DMUON_OK) return rc;
  }
  assign_owners(shapes, count, world, owner_of, loads);
  double total = 0.0, most = 0.0;
  for (int32_t r = 0; r < world; ++r) {
    total += loads[r];
    most = std::max(most, loads[r]);
  }
  *imbalance = total > 0.0 ? most / (total / world) - 1.0 : 0.0;
  return DMUON_OK;
}

int64_t dmuon_workspace_bytes(const dmuon_shape_t* shapes, int32_t count, int32_t ns_steps) {
  (void)ns_steps;
  if (count <= 0 || !shapes) return 0;
  const StepPlan P = make_step_plan(shapes, count);
  return P.buffer_bytes * (P.overlap ? 2 : 1);
}

int64_t dmuon_step_launches(const dmuon_shape_t* shapes, int32_t count, int32_t ns_steps) {
  if (count <= 0 || !shapes) return 0;
  const StepPlan P = make_step_plan(shapes, count);
  int64_t n = 0;
  for (const ChunkRef& ck : P.chunks)
    n += chunk_launches_for(P.layouts[ck.cls], ck.b, P.classes[ck.cls].m, P.classes[ck.cls].n, ns_steps);
  return n;
}



dmuon_status_t dmuon_step(void* const* params, const void* const* grads, void* const* mom_bufs,
                          const dmuon_shape_t* shapes, int32_t count, float lr, float momentum,
                          int32_t nesterov, int32_t ns_steps, const float* coeffs, float wd,
                          dmuon_stream_t stream) {
  return step_impl(params, grads, mom_bufs, shapes, count, lr, momentum, nesterov, ns_steps, coeffs, wd,
                   nullptr, stream);
}

dmuon_status_t dmuon_step_clipped(void* const* params, const void* const* grads, void* const* mom_bufs,
                                  const dmuon_shape_t* shapes, int32_t count, float lr, float momentum,
                                  int32_t nesterov, int32_t ns_steps, const float* coeffs, float wd,
                                  float max_norm, float norm_type, double* total_norm,
                                  dmuon_stream_t stream) {
  ClipReq req{0, max_norm, total_norm};
  dmuon_status_t rc = parse_clip(max_norm, norm_type, &req.p);
  if (rc != DMUON_OK) return rc;
  return step_impl(params, grads, mom_bufs, shapes, count, lr, momentum, nesterov, ns_steps, coeffs, wd,
                   &req, stream);
}

dmuon_status_t dmuon_clip_grad_norm_buckets(void* const* grads, const dmuon_shape_t* shapes, int32_t count,
                                            const int32_t* bucket_of, int32_t num_buckets, const float* max_norms,
                                            const float* norm_types, double* total_norms, dmuon_stream_t stream) {
  if (count < 0) return fail(DMUON_ERR_INVALID_ARG, "count < 0");
  if (num_buckets < 1 || num_buckets > kMaxClipBuckets)
    return fail(DMUON_ERR_INVALID_ARG, "num_buckets must be in 1.." + std::to_string(kMaxClipBuckets));
  if (!max_norms || !norm_types) return fail(DMUON_ERR_INVALID_ARG, "null max_norms or norm_types");
  std::unique_ptr<ClipBuckets> B(new ClipBuckets());
  for (int32_t k = 0; k < num_buckets; ++k) {
    int p = 0;
    dmuon_status_t rc = parse_clip(max_norms[k], norm_types[k], &p);
    if (rc != DMUON_OK) return fail(rc, "bucket " + std::to_string(k) + ": " + dmuon_get_last_error());
    B->max_norm[k] = max_norms[k];
    B->p[k] = p;
  }
  if (count > 0 && !bucket_of) return fail(DMUON_ERR_INVALID_ARG, "null bucket_of");
  for (int32_t i = 0; i < count; ++i)
    if (bucket_of[i] < 0 || bucket_of[i] >= num_buckets)
      return fail(DMUON_ERR_INVALID_ARG, "matrix " + std::to_string(i) + ": bucket out of range");
  dmuon_status_t rc = count > 0 ? check_clip_grads(grads, shapes, count, "dmuon_clip_grad_norm_buckets") : DMUON_OK;
  if (rc != DMUON_OK) return rc;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DeviceState ds;
  rc = device_state(&ds);
  if (rc != DMUON_OK) return rc;
  // each bucket's launch classes, grouped exactly as a separate clip of that
  // bucket would group them (member indices mapped back to the whole list)
  std::vector<std::vector<Group>> groups(num_buckets);
  int64_t tiles = 0;
  for (int32_t k = 0; k < num_buckets; ++k) {
    std::vector<int32_t> idx;
    std::vector<dmuon_shape_t> sub;
    for (int32_t i = 0; i < count; ++i)
      if (bucket_of[i] == k) {
        idx.push_back(i);
        sub.push_back(shapes[i]);
      }
    groups[k] = plan_groups(sub.data(), (int32_t)sub.size());
    for (Group& g : groups[k])
      for (int32_t& m : g.members) m = idx[m];
    B->off[k] = tiles;
    tiles += clip_tiles(groups[k]);
  }
  B->off[num_buckets] = tiles;
  B->total = total_norms;
  // partials, then one coefficient per bucket
  const size_t coef_off = (((size_t)tiles * 4 + 255) / 256) * 256;
  void* ws = nullptr;
  rc = get_workspace(coef_off + (size_t)num_buckets * sizeof(float), st, &ws);
  if (rc != DMUON_OK) return rc;
  float* partials = static_cast<float*>(ws);
  float* coefs = reinterpret_cast<float*>(static_cast<char*>(ws) + coef_off);
  std::unique_ptr<ElemTable> tab(new ElemTable());
  tab->status = ds.status_word;
  const void* const* cg = const_cast<const void* const*>(grads);
  NvtxRange range("clip buckets");
  cudaError_t e = cudaSuccess;
  for (int32_t k = 0; k < num_buckets && e == cudaSuccess; ++k)
    e = for_each_clip_table(groups[k], cg, tab.get(), [&](const ElemTable& t, int32_t dtype, int64_t off, double bytes) {
      Prof pr(kClipNorm, st, 0.0, bytes);
      cudaError_t r = launch_clip_partials(t, dtype, B->p[k], partials + B->off[k] + off, st);
      pr.done(st);
      return r;
    });
  // an empty bucket reduces nothing: total 0, coefficient 1
  if (e == cudaSuccess) e = launch_clip_coef_buckets(partials, *B, num_buckets, coefs, st);
  for (int32_t k = 0; k < num_buckets && e == cudaSuccess; ++k)
    e = for_each_clip_table(groups[k], cg, tab.get(), [&](const ElemTable& t, int32_t dtype, int64_t, double bytes) {
      Prof pr(kClipScale, st, 0.0, 2.0 * bytes);
      cudaError_t r = launch_clip_scale(t, dtype, coefs + k, st);
      pr.done(st);
      return r;
    });
  return e == cudaSuccess ? DMUON_OK : cuda_fail(e, "dmuon_clip_grad_norm_buckets");
}

dmuon_status_t dmuon_clip_grad_norm(void* const* grads, const dmuon_shape_t* shapes, int32_t count,
                                    float max_norm, float norm_type, double* total_norm,
                                    dmuon_stream_t stream) {
  if (count < 0) return fail(DMUON_ERR_INVALID_ARG, "count < 0");
  ClipReq req{0, max_norm, total_norm};
  dmuon_status_t rc = parse_clip(max_norm, norm_type, &req.p);
  if (rc != DMUON_OK) return rc;
  if (count == 0) return DMUON_OK;
  rc = check_clip_grads(grads, shapes, count, "dmuon_clip_grad_norm");
  if (rc != DMUON_OK) return rc;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DeviceState ds;
  rc = device_state(&ds);
  if (rc != DMUON_OK) return rc;
  const std::vector<Group> groups = plan_groups(shapes, count);
  const int64_t tiles = clip_tiles(groups);
  void* ws = nullptr;
  rc = get_workspace(clip_ws_bytes(tiles), st, &ws);
  if (rc != DMUON_OK) return rc;
  std::unique_ptr<ElemTable> tab(new ElemTable());
  tab->status = ds.status_word;
  const void* const* cg = const_cast<const void* const*>(grads);
  cudaError_t e = clip_norm_stage(groups, cg, req, ws, tiles, tab.get(), st);
  if (e == cudaSuccess)
    e = for_each_clip_table(groups, cg, tab.get(), [&](const ElemTable& t, int32_t dtype, int64_t, double bytes) {
      Prof pr(kClipScale, st, 0.0, 2.0 * bytes);
      cudaError_t r = launch_clip_scale(t, dtype, clip_coef_ptr(ws, tiles), st);
      pr.done(st);
      return r;
    });
  return e == cudaSuccess ? DMUON_OK : cuda_fail(e, "dmuon_clip_grad_norm");
}

dmuon_status_t dmuon_ns_ex(const void* X, void* out, int64_t rows, int64_t cols, int32_t steps,
                           const float* coeffs, int32_t dtype, dmuon_stream_t stream) {
  if (!X || !out) return fail(DMUON_ERR_INVALID_ARG, "null pointer argument");
  dmuon_status_t rc = check_shape(rows, cols, "dmuon_ns");
  if (rc != DMUON_OK) return rc;
  if (!dtype_ok(dtype)) return fail(DMUON_ERR_INVALID_ARG, "bad dtype");
  if (steps < 0 || steps > 1000) return fail(DMUON_ERR_INVALID_ARG, "steps must be in 0..1000");
  const uintptr_t bytes = (uintptr_t)(rows * cols) * esize(dtype);
  const uintptr_t x = (uintptr_t)X, o = (uintptr_t)out;
  if (x < o + bytes && o < x + bytes) return fail(DMUON_ERR_INVALID_ARG, "out may not overlap X");
  std::vector<float> sched;
  coeff_schedule(steps, coeffs, sched);

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DeviceState ds;
  rc = device_state(&ds);
  if (rc != DMUON_OK) return rc;
  const int64_t m = std::min(rows, cols), n = std::max(rows, cols);
  const ChunkLayout L = chunk_layout(m, n, dtype);
  const ChunkOffsets off = chunk_offsets(L, 1);
  void* wsv = nullptr;
  rc = get_workspace((size_t)off.total, st, &wsv);
  if (rc != DMUON_OK) return rc;
  char* ws = static_cast<char*>(wsv);
  std::unique_ptr<ElemTable> tab(new ElemTable());
  tab->status = ds.status_word;
  tab->m = m;
  tab->n = n;
  tab->ldn = L.ldn;
  tab->count = 1;
  tab->tiles_per_mat = (int32_t)L.tiles_per_mat;
  MatEntry& e0 = tab->e[0];
  e0.src = X;
  e0.buf = nullptr;
  e0.dst = out;
  e0.transposed = rows > cols ? 1 : 0;
  const bool row16 = (cols * (int64_t)esize(dtype)) % 16 == 0;
  e0.pad = ((row16 && aligned16(X)) ? 1 : 0) | ((row16 && aligned16(out)) ? 2 : 0);
  float* partials = reinterpret_cast<float*>(ws + off.partials);
  float* scale = reinterpret_cast<float*>(ws + off.scale);
  const double elems = (double)m * (double)n, es = (double)esize(dtype);
  Prof pl(kLoad, st, 0.0, 2.0 * elems * es);
  cudaError_t e = launch_momentum(*tab, dtype, ElemMode::kLoad, ws + off.x0, partials, 0.f, 0, st, nullptr,
                                  x_dtype(L, dtype));
  pl.done(st);
  if (e != cudaSuccess) return cuda_fail(e, "load launch");
  Prof pn(kNorm, st, 0.0, 4.0 * (double)L.tiles_per_mat);
  e = launch_norm_finalize(partials, 1, (int)L.tiles_per_mat, scale, nullptr, st);
  pn.done(st);
  if (e != cudaSuccess) return cuda_fail(e, "norm launch");
  void* result = nullptr;
  rc = run_chain(L, 1, m, n, ws, off, steps, sched.data(), ds.status_word, ds.sm_count, st, &result);
  if (rc != DMUON_OK) return rc;
  Prof pc(kCopyOut, st, 0.0, 2.0 * elems * es);
  e = launch_update(*tab, dtype, ElemMode::kCopyOut, result, steps == 0 ? scale : nullptr, 0.f, 0.f, n, st,
                    x_dtype(L, dtype));
  pc.done(st);
  if (e != cudaSuccess) return cuda_fail(e, "copy-out launch");
  return DMUON_OK;
}

dmuon_status_t dmuon_ns(const void* X, void* out, int64_t rows, int64_t cols, int32_t steps,
                        const float* coeffs, dmuon_stream_t stream) {
  return dmuon_ns_ex(X, out, rows, cols, steps, coeffs, DMUON_BF16, stream);
}

// ---------------------------------------------------------------- stage calls
static dmuon_status_t check_stage(const void* const* ptrs, int np, int64_t batch, int64_t m, int64_t n,
                                  const int64_t* lds, const int64_t* ldmin, int nl, int32_t dtype) {
  for (int i = 0; i < np; ++i)
    if (!ptrs[i]) return fail(DMUON_ERR_INVALID_ARG, "null pointer argument");
  if (batch < 0 || batch > 65535) return fail(DMUON_ERR_INVALID_ARG, "batch must be in 0..65535");
  dmuon_status_t rc = check_shape(m, n, "stage call");
  if (rc != DMUON_OK) return rc;
  if (!dtype_ok(dtype)) return fail(DMUON_ERR_INVALID_ARG, "bad dtype");
  for (int i = 0; i < nl; ++i)
    if (lds[i] < ldmin[i]) return fail(DMUON_ERR_INVALID_ARG, "leading dimension smaller than the row");
  if (dtype == DMUON_BF16) {
    for (int i = 0; i < np; ++i)
      if (!aligned16(ptrs[i])) return fail(DMUON_ERR_INVALID_ARG, "bf16 stage calls need 16-byte aligned pointers");
    for (int i = 0; i < nl; ++i)
      if (lds[i] % 8 != 0) return fail(DMUON_ERR_INVALID_ARG, "bf16 stage calls need leading dimensions % 8 == 0");
  }
  return DMUON_OK;
}

dmuon_status_t dmuon_gram(const void* X, void* G, int64_t batch, int64_t m, int64_t n, int64_t ldx,
                          int64_t ldg, float alpha, int32_t dtype, dmuon_stream_t stream) {
  const void* ptrs[2] = {X, G};
  const int64_t lds[2] = {ldx, ldg}, mins[2] = {n, m};
  dmuon_status_t rc = check_stage(ptrs, 2, batch, m, n, lds, mins, 2, dtype);
  if (rc != DMUON_OK) return rc;
  if (batch == 0) return DMUON_OK;
  DeviceState ds;
  rc = device_state(&ds);
  if (rc != DMUON_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = dtype == DMUON_BF16
                      ? tc_gram(X, G, (int)batch, (int)m, (int)n, ldx, ldg, alpha, nullptr, ds.status_word,
                                ds.sm_count, st)
                      : simt_gram(X, G, (int)batch, (int)m, (int)n, ldx, ldg, alpha, nullptr, false, st, ds.status_word);
  return e == cudaSuccess ? DMUON_OK : cuda_fail(e, "dmuon_gram");
}

dmuon_status_t dmuon_gram_poly(const void* G, void* P, int64_t batch, int64_t m, int64_t ldg, int64_t ldp,
                               float b, float c, int32_t dtype, dmuon_stream_t stream) {
  const void* ptrs[2] = {G, P};
  const int64_t lds[2] = {ldg, ldp}, mins[2] = {m, m};
  dmuon_status_t rc = check_stage(ptrs, 2, batch, m, m, lds, mins, 2, dtype);
  if (rc != DMUON_OK) return rc;
  if (batch == 0) return DMUON_OK;
  DeviceState ds;
  rc = device_state(&ds);
  if (rc != DMUON_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = dtype == DMUON_BF16
                      ? tc_poly(G, P, (int)batch, (int)m, ldg, ldp, b, c, ds.status_word, ds.sm_count, st)
                      : simt_poly(G, P, (int)batch, (int)m, ldg, ldp, b, c, st, ds.status_word);
  return e == cudaSuccess ? DMUON_OK : cuda_fail(e, "dmuon_gram_poly");
}

dmuon_status_t dmuon_poly_apply(const void* P, const void* X, void* Y, int64_t batch, int64_t m, int64_t n,
                                int64_t ldp, int64_t ldx, int64_t ldy, float a, float alpha, int32_t dtype,
                                dmuon_stream_t stream) {
  const void* ptrs[3] = {P, X, Y};
  const int64_t lds[3] = {ldp, ldx, ldy}, mins[3] = {m, n, n};
  dmuon_status_t rc = check_stage(ptrs, 3, batch, m, n, lds, mins, 3, dtype);
  if (rc != DMUON_OK) return rc;
  if (batch == 0) return DMUON_OK;
  DeviceState ds;
  rc = device_state(&ds);
  if (rc != DMUON_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = dtype == DMUON_BF16
                      ? tc_apply(P, X, Y, (int)batch, (int)m, (int)n, ldp, ldx, ldy, a, alpha, nullptr,
                                 ds.status_word, ds.sm_count, st)
                      : simt_apply(P, X, Y, (int)batch, (int)m, (int)n, ldp, ldx, ldy, a, alpha, nullptr, false,
                                   st, ds.status_word);
  return e == cudaSuccess ? DMUON_OK : cuda_fail(e, "dmuon_poly_apply");
}

dmuon_status_t dmuon_momentum(void* buf, const void* grad, void* x0, int64_t rows, int64_t cols, float momentum,
                              int32_t nesterov, int32_t dtype, double* sumsq, dmuon_stream_t stream) {
  if (!buf || !grad || !x0) return fail(DMUON_ERR_INVALID_ARG, "null pointer argument");
  dmuon_status_t rc = check_shape(rows, cols, "dmuon_momentum");
  if (rc != DMUON_OK) return rc;
  if (!dtype_ok(dtype)) return fail(DMUON_ERR_INVALID_ARG, "bad dtype");
  if (nesterov != 0 && nesterov != 1) return fail(DMUON_ERR_INVALID_ARG, "nesterov must be 0 or 1");
  DeviceState ds;
  rc = device_state(&ds);
  if (rc != DMUON_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  std::unique_ptr<ElemTable> tab(new ElemTable());
  tab->status = ds.status_word;
  tab->m = rows;
  tab->n = cols;
  tab->ldn = cols;
  tab->count = 1;
  tab->tiles_per_mat = (int32_t)(((rows + kElemTile - 1) / kElemTile) * ((cols + kElemTile - 1) / kElemTile));
  const size_t es = esize(dtype);
  const bool row16 = (cols * (int64_t)es) % 16 == 0;
  tab->e[0] = MatEntry{grad, buf, x0, 0, (row16 && aligned16(grad) && aligned16(buf)) ? 1 : 0};
  void* wsv = nullptr;
  rc = get_workspace((size_t)tab->tiles_per_mat * 4 + 256, st, &wsv);
  if (rc != DMUON_OK) return rc;
  float* partials = static_cast<float*>(wsv);
  cudaError_t e = launch_momentum(*tab, dtype, ElemMode::kMomentum, x0, partials, momentum, nesterov, st);
  if (e == cudaSuccess && sumsq) e = launch_norm_finalize(partials, 1, tab->tiles_per_mat, nullptr, sumsq, st);
  return e == cudaSuccess ? DMUON_OK : cuda_fail(e, "dmuon_momentum");
}

dmuon_status_t dmuon_update(void* param, const void* O, int64_t rows, int64_t cols, float lr, float wd,
                            int32_t dtype, dmuon_stream_t stream) {
  if (!param || !O) return fail(DMUON_ERR_INVALID_ARG, "null pointer argument");
  dmuon_status_t rc = check_shape(rows, cols, "dmuon_update");
  if (rc != DMUON_OK) return rc;
  if (!dtype_ok(dtype)) return fail(DMUON_ERR_INVALID_ARG, "bad dtype");
  if (!std::isfinite(lr) || !std::isfinite(wd)) return fail(DMUON_ERR_INVALID_ARG, "lr and wd must be finite");
  DeviceState ds;
  rc = device_state(&ds);
  if (rc != DMUON_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  std::unique_ptr<ElemTable> tab(new ElemTable());
  tab->status = ds.status_word;
  // not oriented: the table's (m, n) is the matrix itself
  const int64_t n = std::max(rows, cols);
  tab->m = rows;
  tab->n = cols;
  tab->ldn = cols;
  tab->count = 1;
  tab->tiles_per_mat = (int32_t)(((rows + kElemTile - 1) / kElemTile) * ((cols + kElemTile - 1) / kElemTile));
  const bool row16 = (cols * (int64_t)esize(dtype)) % 16 == 0;
  tab->e[0] = MatEntry{nullptr, nullptr, param, 0, (row16 && aligned16(param)) ? 2 : 0};
  cudaError_t e = launch_update(*tab, dtype, ElemMode::kUpdate, O, nullptr, lr, wd, n, st);
  return e == cudaSuccess ? DMUON_OK : cuda_fail(e, "dmuon_update");
}

dmuon_status_t dmuon_profile_start(void) {
  g_prof.clear();  // the events stay in the pool
  g_prof_on = true;
  return DMUON_OK;
}

int32_t dmuon_profile_stop_launches(dmuon_launch_record_t* recs, int32_t max_recs) {
  g_prof_on = false;
  bool ok = true;
  if (!g_prof.empty() && cudaEventSynchronize(g_prof.back().b) != cudaSuccess) ok = false;
  int32_t n = 0;
  for (size_t i = 0; i < g_prof.size(); ++i) {
    ProfRec& r = g_prof[i];
    float t = 0.f, t0 = 0.f;
    if (ok && (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess ||
               cudaEventElapsedTime(&t0, g_prof.front().a, r.a) != cudaSuccess))
      ok = false;
    if (ok && recs && n < max_recs) {
      dmuon_launch_record_t& o = recs[n];
      std::memset(&o, 0, sizeof(o));
      std::strncpy(o.name, kKindNames[r.kind], sizeof(o.name) - 1);
      o.start_ms = t0;
      o.ms = t;
      o.flops = r.flops;
      o.bytes = r.bytes;
    }
    ++n;
  }
  g_prof.clear();
  if (!ok) {
    fail(DMUON_ERR_CUDA, "profile events failed");
    return -1;
  }
  return n;
}

int32_t dmuon_profile_stop(dmuon_kernel_stat_t* stats, int32_t max_stats) {
  g_prof_on = false;
  double ms[kNumKinds] = {0}, fl[kNumKinds] = {0}, by[kNumKinds] = {0};
  int64_t cnt[kNumKinds] = {0};
  bool ok = true;
  if (!g_prof.empty() && cudaEventSynchronize(g_prof.back().b) != cudaSuccess) ok = false;
  for (ProfRec& r : g_prof) {
    float t = 0.f;
    if (ok && cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&t, r.a, r.b) == cudaSuccess) {
      ms[r.kind] += t;
      fl[r.kind] += r.flops;
      by[r.kind] += r.bytes;
      cnt[r.kind] += 1;
    } else {
      ok = false;
    }
  }
  g_prof.clear();
  if (!ok) {
    fail(DMUON_ERR_CUDA, "profile events failed");
    return -1;
  }
  int32_t n = 0;
  for (int k = 0; k < kNumKinds; ++k) {
    if (cnt[k] == 0) continue;
    if (stats && n < max_stats) {
      dmuon_kernel_stat_t& s = stats[n];
      std::memset(&s, 0, sizeof(s));
      std::strncpy(s.name, kKindNames[k], sizeof(s.name) - 1);
      s.launches = cnt[k];
      s.total_ms = ms[k];
      s.flops = fl[k];
      s.bytes = by[k];
    }
    ++n;
  }
  return n;
}

dmuon_status_t dmuon_selftest_timeout(int32_t limit_us, dmuon_stream_t stream) {
  if (limit_us < 1 || limit_us > 2000000) return fail(DMUON_ERR_INVALID_ARG, "limit_us must be in 1..2000000");
  DeviceState ds;
  dmuon_status_t rc = device_state(&ds);
  if (rc != DMUON_OK) return rc;
  cudaError_t e = wait_selftest(ds.status_word, limit_us, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DMUON_OK : cuda_fail(e, "self-test launch");
}

dmuon_status_t dmuon_selftest_bounds(dmuon_stream_t stream) {
  DeviceState ds;
  dmuon_status_t rc = device_state(&ds);
  if (rc != DMUON_OK) return rc;
  k_bounds_selftest<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(ds.status_word);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DMUON_OK : cuda_fail(e, "self-test launch");
}

dmuon_status_t dmuon_stream_status(dmuon_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stream");
  DeviceState ds;
  dmuon_status_t rc = device_state(&ds);
  if (rc != DMUON_OK) return rc;
  int word = 0;
  e = cudaMemcpy(&word, ds.status_word, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (word != 0) {
    cudaMemset(ds.status_word, 0, sizeof(int));
    return fail((dmuon_status_t)word, word == DMUON_ERR_BOUNDS
                                          ? "a kernel access fell outside its buffer (debug build: skipped)"
                                          : "a device-side wait ran out (kernel gave up and returned)");
  }
  return DMUON_OK;
}

void dmuon_release_workspace(void) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  cudaDeviceSynchronize();
  std::lock_guard<std::mutex> lock(g_mu);
  for (auto it = g_workspace.begin(); it != g_workspace.end();) {
    if (it->first.first == dev) {
      if (it->second.first) cudaFree(it->second.first);
      it = g_workspace.erase(it);
    } else {
      ++it;
    }
  }
  for (auto it = g_side.begin(); it != g_side.end();) {
    if (it->first.first == dev) {
      cudaStreamDestroy(it->second.aux);
      cudaStreamDestroy(it->second.chain);
      it = g_side.erase(it);
    } else {
      ++it;
    }
  }
}

}  // extern "C"
