// zero_adam_host.cpp -- the pure host functions of the C ABI (no CUDA):
// ownership bounds, per-rank state accounting and status texts.
#include <cstdint>

#include "zero_adam.h"

extern "C" {

// "Deep dive: DeepSpeed", "Reduce first, then update the owned slice":
// owner r keeps [floor(P*r/R), floor(P*(r+1)/R)); 128-bit products so that
// P*r never wraps.
int zero_partition_bounds(uint64_t P, uint32_t R, uint64_t* lo, uint64_t* hi) {
    if (R == 0 || lo == nullptr || hi == nullptr) return ZERO_EINVAL;
    const unsigned __int128 p = P;
    for (uint32_t r = 0; r < R; ++r) {
        lo[r] = (uint64_t)((p * r) / R);
        hi[r] = (uint64_t)((p * (r + 1u)) / R);
    }
    return ZERO_OK;
}

// "Deep dive: DeepSpeed", "Count state before choosing a stage": each stage
// keeps a 1/R share of one more kind of state (optimizer, then gradient,
// then weight).  Returned multiplied by R so the values stay integers.
int zero_state_bytes(uint64_t P, uint32_t R, uint32_t param_b, uint32_t grad_b, uint32_t opt_b,
                     uint64_t out_times_R[4]) {
    if (P == 0 || R == 0 || param_b == 0 || grad_b == 0 || opt_b == 0 || out_times_R == nullptr)
        return ZERO_EINVAL;
    const uint32_t width[3] = {opt_b, grad_b, param_b};  // the order the stages shard them
    for (int stage = 0; stage < 4; ++stage) {
        unsigned __int128 total = 0;
        for (int k = 0; k < 3; ++k) {
            // replicated: P*width bytes (R*P*width after scaling by R);
            // sharded: P*width/R bytes (P*width after scaling by R)
            unsigned __int128 term = (unsigned __int128)P * width[k];
            if (k >= stage) term *= R;
            total += term;
        }
        if (total > (unsigned __int128)UINT64_MAX) return ZERO_EOVERFLOW;
        out_times_R[stage] = (uint64_t)total;
    }
    return ZERO_OK;
}

// "Deep dive: DeepSpeed", "Stage 3 needs a live working set": each rank
// keeps of a tensor of n elements a shard of ceil(n/R) elements (the last
// shards padded), rank r holding elements [r*s, min((r+1)*s, n)).
int zero3_shard_bounds(uint64_t n, uint32_t R, uint32_t r, uint64_t* lo, uint64_t* hi, uint64_t* shard) {
    if (R == 0 || r >= R || lo == nullptr || hi == nullptr || shard == nullptr) return ZERO_EINVAL;
    const uint64_t s = n / R + (n % R != 0 ? 1u : 0u);
    const unsigned __int128 a = (unsigned __int128)s * r, b = (unsigned __int128)s * (r + 1u);
    *shard = s;
    *lo = a < n ? (uint64_t)a : n;
    *hi = b < n ? (uint64_t)b : n;
    return ZERO_OK;
}

// The same section's storage model, in elements: resident shards of every
// tensor, plus one separate full padded buffer (R shards) per live tensor.
int zero_parameter_storage(const uint64_t* sizes, uint32_t T, uint32_t R, const uint32_t* live, uint32_t n_live,
                           uint64_t out[3]) {
    if (sizes == nullptr || T == 0 || R == 0 || out == nullptr || (n_live > 0 && live == nullptr))
        return ZERO_EINVAL;
    unsigned __int128 resident = 0, gathered = 0;
    for (uint32_t j = 0; j < T; ++j) {
        if (sizes[j] == 0) return ZERO_EINVAL;
        resident += sizes[j] / R + (sizes[j] % R != 0 ? 1u : 0u);
    }
    for (uint32_t i = 0; i < n_live; ++i) {
        if (live[i] >= T) return ZERO_EINVAL;
        for (uint32_t k = 0; k < i; ++k)
            if (live[k] == live[i]) return ZERO_EINVAL;
        const uint64_t n = sizes[live[i]];
        gathered += (unsigned __int128)(n / R + (n % R != 0 ? 1u : 0u)) * R;
    }
    const unsigned __int128 total = resident + gathered;
    if (total > (unsigned __int128)UINT64_MAX) return ZERO_EOVERFLOW;
    out[0] = (uint64_t)resident;
    out[1] = (uint64_t)gathered;
    out[2] = (uint64_t)total;
    return ZERO_OK;
}

const char* zero_status_string(int status) {
    switch (status) {
        case ZERO_OK: return "ok";
        case ZERO_EINVAL: return "invalid argument (NULL pointer, unknown dtype, bad count or hyperparameter)";
        case ZERO_EALIGN: return "device pointer not 16-byte aligned";
        case ZERO_EOVERFLOW: return "byte size overflows 64 bits";
        case ZERO_ERANGE: return "count beyond a documented limit";
        case ZERO_ECUDA: return "CUDA runtime error (see zero_last_cuda_error)";
        case ZERO_EIO: return "checkpoint file error (see zero_checkpoint_error)";
        default: return "unknown status";
    }
}

}  // extern "C"
