// bounds.cuh -- index checks of the debug-bounds build.
//
// Compiled with -DDA2_DEBUG_BOUNDS (the library libdiffattn_v2_debug.so), every checked
// shared-memory offset, tensor-memory column and global index is compared with the extent of
// what it addresses before the access. A violation records kErrBounds in the device error
// word (the first error recorded wins) and the access is skipped; the kernel never traps. A
// skipped copy leaves its barrier short, so the waits on it give up after their time limit
// and the kernel leaves through its abort path. In the normal build `checked` is the
// constant true and the comparisons compile away.
#pragma once

#include "ptx.cuh"

namespace da2 {

#ifdef DA2_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif

// `ok` is the bounds condition of one access: true lets it happen.
__device__ __forceinline__ bool checked(bool ok, int* err) {
  if constexpr (kDebugBounds) {
    if (!ok) atomicCAS(err, 0, kErrBounds);
    return ok;
  } else {
    (void)ok;
    (void)err;
    return true;
  }
}

// [lo, lo + len) inside [base, base + extent)
__device__ __forceinline__ bool within(uint64_t lo, uint64_t len, uint64_t base, uint64_t extent) {
  return lo >= base && lo + len <= base + extent;
}

}  // namespace da2
