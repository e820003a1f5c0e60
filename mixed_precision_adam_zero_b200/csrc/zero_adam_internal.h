// zero_adam_internal.h -- helpers shared between the library's translation
// units; not part of the C ABI.
#pragma once

#include <stdint.h>

namespace zadam_host {

// params16[e] = round-to-nearest-even(master[e - state_offset]) for every e
// in [lo, hi), on `stream`.  master holds elements from state_offset on
// (a multiple of 8, at most lo); master and params16 are 16-byte aligned.
// Returns a ZERO_* status.
int cast_slice(const float* master, uint64_t state_offset, void* params16, int32_t param_dtype, uint64_t lo,
               uint64_t hi, void* stream);

}  // namespace zadam_host
