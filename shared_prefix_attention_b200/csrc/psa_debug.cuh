// Device-side bounds checks of the debug build.
//
// Compiled with -DPSA_DEBUG=1 (python -m shared_prefix_attention_b200.build
// --debug, which writes libpsa_debug.so), psa_in_bounds(cond, status)
// reports PSA_ERR_BOUNDS to the caller's status word when an index taken from
// caller data -- a schedule item, tile entry or rectangle range, a prefix
// offset, a tree-mask offset -- falls outside its buffer, and the kernel
// skips the access.  Nothing traps, so a bad input shows up as a status
// instead of a fault.  In the release build it is the constant true and
// compiles away.
#pragma once

#include <stdint.h>

#include "psa.h"

#ifndef PSA_DEBUG
#define PSA_DEBUG 0
#endif

namespace psa {

__device__ __forceinline__ bool psa_in_bounds(bool cond, int32_t* dev_status) {
#if PSA_DEBUG
  if (!cond && dev_status) atomicCAS(dev_status, 0, int32_t(PSA_ERR_BOUNDS));
  return cond;
#else
  (void)cond;
  (void)dev_status;
  return true;
#endif
}

}  // namespace psa
