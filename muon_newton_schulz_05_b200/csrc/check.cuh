// Bounds checks of the debug build (nvcc -DMUON_CHECK, `build.py --check`):
// an index outside its buffer is recorded in the device status word as
// MUON_ERR_BOUNDS and the access is skipped. Without the macro every check is
// the constant true and compiles away.
#pragma once

#include "muon_b200.h"

namespace muon {

#ifdef MUON_CHECK
__device__ __forceinline__ bool in_bounds(bool ok, int* status) {
  if (!ok && status) atomicExch(status, MUON_ERR_BOUNDS);
  return ok;
}
#else
__device__ __forceinline__ constexpr bool in_bounds(bool, int*) { return true; }
#endif

}  // namespace muon
