// Bounds checks of debug builds, shared by every kernel file.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "dmuon.h"

namespace dmuon {

// Debug builds (-DDMUON_DEBUG): an access of `len` elements at element offset
// `off` of a buffer of `extent` elements is made only if it lies inside; one
// that does not is skipped and the status word records DMUON_ERR_BOUNDS.  In
// release builds the check is the constant true and its arguments are not
// evaluated.
#ifdef DMUON_DEBUG
__device__ __forceinline__ bool dbg_in(int* status, int64_t off, int64_t len, int64_t extent) {
  const bool ok = off >= 0 && len >= 0 && off + len <= extent;
  if (!ok && status) atomicCAS(status, 0, (int)DMUON_ERR_BOUNDS);
  return ok;
}
#define DMUON_IN(status, off, len, extent) ::dmuon::dbg_in((status), (off), (len), (extent))
#else
#define DMUON_IN(status, off, len, extent) true
#endif

}  // namespace dmuon
