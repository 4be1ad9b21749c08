// dmuon_ns_noalloc: the Newton-Schulz call for callers that cannot allocate
// device memory.
//
// Some callers cannot call cudaMalloc: a framework that has given the whole
// device to its own caching allocator (a hidden allocation would fail or
// fragment its pool), or a loop that must not allocate after start-up
// (cudaMalloc may synchronise the device and costs an unpredictable time).
// This entry point gives them dmuon_ns_ex without any allocation: its
// workspace is one fixed array in device memory, reserved when the library is
// loaded, and the kernels are the same ones dmuon_ns_ex launches.
//
// The array is shared by every call on a device and keeps whatever the last
// call left in it.  Only the status word has to start at zero and is cleared
// at the start of each call; everything else is written before it is read.
// Calls that may overlap on the GPU race on the array.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace dmuon {
namespace {

// The scratch array: a 256-byte header (the status word when the caller
// passes none) followed by the workspace of one matrix.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DMUON_NOALLOC_SCRATCH_BYTES];
constexpr size_t kHeader = 256;

// Per-device set-up with that device current: the device address of the array
// (host code only holds a stand-in for it) and the SM count.  It is marked done
// only once it succeeded, so a failed first attempt (for instance one made
// while a stream was capturing) is retried by the next call.
constexpr int kMaxDevices = 64;
struct DeviceSetup {
  bool done = false;
  void* scratch = nullptr;
  int sm_count = 0;
  int major = 0;
};
std::mutex g_setup_mu;
DeviceSetup g_setup[kMaxDevices];

cudaError_t setup_device(int dev, DeviceSetup* out) {
  std::lock_guard<std::mutex> lock(g_setup_mu);
  DeviceSetup& d = g_setup[dev];
  if (!d.done) {
    DeviceSetup t;
    cudaError_t e = cudaGetSymbolAddress(&t.scratch, g_noalloc_scratch);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&t.sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&t.major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) {
      cudaGetLastError();  // not sticky: the next call tries again
      return e;
    }
    t.done = true;
    d = t;
  }
  *out = d;
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dmuon_status_t cuda_error(cudaError_t e, const char* what) {
  return record_error(DMUON_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

}  // namespace
}  // namespace dmuon

using namespace dmuon;

extern "C" dmuon_status_t dmuon_ns_noalloc(const void* X, void* out, int64_t rows, int64_t cols,
                                           int32_t steps, const float* coeffs, int32_t dtype,
                                           int32_t* status, dmuon_stream_t stream) {
  // ------------------------------------------------------------ validation
  if (!X || !out) return record_error(DMUON_ERR_INVALID_ARG, "null pointer argument");
  if (rows <= 0 || cols <= 0 || rows > (int64_t(1) << 20) || cols > (int64_t(1) << 20) ||
      rows * cols > (int64_t(1) << 31) - 1)
    return record_error(DMUON_ERR_INVALID_ARG, "dmuon_ns_noalloc: shape out of range");
  if (dtype != DMUON_F32 && dtype != DMUON_BF16) return record_error(DMUON_ERR_INVALID_ARG, "bad dtype");
  if (steps < 0 || steps > 1000) return record_error(DMUON_ERR_INVALID_ARG, "steps must be in 0..1000");
  const int64_t es = dtype == DMUON_BF16 ? 2 : 4;
  const uintptr_t bytes = (uintptr_t)(rows * cols * es), x = (uintptr_t)X, o = (uintptr_t)out;
  if (x < o + bytes && o < x + bytes) return record_error(DMUON_ERR_INVALID_ARG, "out may not overlap X");
  const int64_t m = std::min(rows, cols), n = std::max(rows, cols);
  // the layout and schedule of dmuon_ns_ex, so both give the same bits
  const ChunkLayout L = chunk_layout(m, n, dtype);
  const ChunkOffsets off = chunk_offsets(L, 1);
  const size_t need = kHeader + (size_t)off.total;
  if (need > (size_t)DMUON_NOALLOC_SCRATCH_BYTES)
    return record_error(DMUON_ERR_INVALID_ARG,
                        "dmuon_ns_noalloc: a " + std::to_string(rows) + "x" + std::to_string(cols) +
                            " matrix needs " + std::to_string(need) + " bytes of scratch; the fixed array holds " +
                            std::to_string((size_t)DMUON_NOALLOC_SCRATCH_BYTES));
  float sched[3 * 1000];  // on the stack
  for (int32_t k = 0; k < steps; ++k) {
    sched[3 * k] = coeffs ? coeffs[3 * k] : DMUON_DEFAULT_A;
    sched[3 * k + 1] = coeffs ? coeffs[3 * k + 1] : DMUON_DEFAULT_B;
    sched[3 * k + 2] = coeffs ? coeffs[3 * k + 2] : DMUON_DEFAULT_C;
  }

  // ---------------------------------------------------------------- set-up
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return record_error(DMUON_ERR_UNSUPPORTED, "device ordinal beyond 63");
  DeviceSetup d;
  e = setup_device(dev, &d);
  if (e != cudaSuccess) return cuda_error(e, "scratch address lookup");
  if (d.major != 10) return record_error(DMUON_ERR_UNSUPPORTED, "this library is built for sm_100a");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(d.scratch);
  int* status_word = status ? status : reinterpret_cast<int*>(base);
  char* ws = base + kHeader;
  e = cudaMemsetAsync(status_word, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_error(e, "status clear");

  // ------------------------------------------------- the dmuon_ns_ex kernels
  ElemTable tab;  // on the stack: no host or device allocation
  tab.status = status_word;
  tab.m = m;
  tab.n = n;
  tab.ldn = L.ldn;
  tab.count = 1;
  tab.tiles_per_mat = (int32_t)L.tiles_per_mat;
  const bool row16 = (cols * es) % 16 == 0;
  tab.e[0] = MatEntry{X, nullptr, out, rows > cols ? 1 : 0,
                      ((row16 && aligned16(X)) ? 1 : 0) | ((row16 && aligned16(out)) ? 2 : 0)};
  float* partials = reinterpret_cast<float*>(ws + off.partials);
  float* scale = reinterpret_cast<float*>(ws + off.scale);
  e = launch_momentum(tab, dtype, ElemMode::kLoad, ws + off.x0, partials, 0.f, 0, st, nullptr, x_dtype(L, dtype));
  if (e == cudaSuccess) e = launch_norm_finalize(partials, 1, (int)L.tiles_per_mat, scale, nullptr, st);
  if (e != cudaSuccess) return cuda_error(e, "dmuon_ns_noalloc launch");
  void* result = nullptr;
  const dmuon_status_t rc = ns_chain(L, 1, m, n, ws, off, steps, sched, status_word, d.sm_count, st, &result);
  if (rc != DMUON_OK) return rc;
  e = launch_update(tab, dtype, ElemMode::kCopyOut, result, steps == 0 ? scale : nullptr, 0.f, 0.f, n, st,
                    x_dtype(L, dtype));
  if (e != cudaSuccess) return cuda_error(e, "dmuon_ns_noalloc launch");
  return DMUON_OK;
}
