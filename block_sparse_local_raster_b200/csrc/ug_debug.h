// Range checks of the debug build (compiled with -DUG_DEBUG=1; the release
// build compiles them away).  Every global index a kernel computes -- list
// entries, token rows of permutations and scatters, RoPE table rows -- is
// checked against the extent of what it indexes before the access; a failed
// check records UG_ERR_INVALID_ARG in the plan's error word (read by
// ug_check_error) and the access is skipped.  With the canary regions the
// GPU tests place around every output, this stands in for a device memory
// checker.
#pragma once

#include "ug.h"

#ifndef UG_DEBUG
#define UG_DEBUG 0
#endif

namespace ug {

// true when the condition holds (always, in the release build); otherwise
// records the failure in *err.
__device__ __forceinline__ bool dbg_ok(bool cond, int* err) {
#if UG_DEBUG
  if (!cond) atomicCAS(err, 0, (int)UG_ERR_INVALID_ARG);
  return cond;
#else
  (void)cond;
  (void)err;
  return true;
#endif
}

}  // namespace ug
