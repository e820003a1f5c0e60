// zero_adam_ckpt.cpp -- checkpoint files of the optimizer state ("Deep dive:
// DeepSpeed", "Resume training and export weights separately": resuming needs
// the weights, both moments and the step counter, an export needs only the
// consolidated weights).
//
// One file per owner slice ("shard"): a fixed header, then the slice of the
// fp32 master weights, first moment and second moment, then a 64-bit FNV-1a
// checksum of everything before it.  All integers little-endian.
//
//   offset  size  field
//   0       8     magic "ZADAMCK1"
//   8       4     header bytes (128)
//   12      4     R (ranks)
//   16      8     P (parameters of the whole vector)
//   24      4     owner (-1: the whole vector in one file)
//   28      4     reserved (0)
//   32      8     lo (first element of the slice)
//   40      8     hi (one past the last element)
//   48      40    zero_ctrl (step, skipped, loss scale, growth, parity 0, ...)
//   88      40    reserved (0)
//   128     ...   master[hi-lo], exp_avg[hi-lo], exp_avg_sq[hi-lo] (fp32)
//   end     8     FNV-1a 64 of bytes [0, end)
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <utility>
#include <cstring>
#include <vector>

#include "zero_adam.h"
#include "zero_adam_internal.h"

namespace {

constexpr char kMagic[8] = {'Z', 'A', 'D', 'A', 'M', 'C', 'K', '1'};
constexpr uint32_t kHeaderBytes = 128;
constexpr size_t kChunk = size_t(1) << 24;  // elements per staged copy (64 MB of fp32)

struct Header {
    char magic[8];
    uint32_t header_bytes;
    uint32_t R;
    uint64_t P;
    int32_t owner;
    uint32_t reserved0;
    uint64_t lo, hi;
    zero_ctrl ctrl;
    unsigned char reserved1[40];
};
static_assert(sizeof(Header) == kHeaderBytes, "checkpoint header layout");

struct Fnv {
    uint64_t h = 1469598103934665603ull;
    void add(const void* p, size_t n) {
        const unsigned char* b = static_cast<const unsigned char*>(p);
        for (size_t i = 0; i < n; ++i) {
            h ^= b[i];
            h *= 1099511628211ull;
        }
    }
};

thread_local char g_ckpt_error[256] = "no error";

int cuda_fail(cudaError_t e) {
    std::snprintf(g_ckpt_error, sizeof g_ckpt_error, "%s", cudaGetErrorString(e));
    return ZERO_ECUDA;
}

int io_fail(const char* what, const char* path) {
    std::snprintf(g_ckpt_error, sizeof g_ckpt_error, "%s: %s", what, path ? path : "(null)");
    return ZERO_EIO;
}

void slice_of(const zero_step_args* a, uint64_t* lo, uint64_t* hi) {
    if (a->owner < 0) {
        *lo = 0;
        *hi = a->P;
        return;
    }
    const unsigned __int128 P = a->P;
    *lo = (uint64_t)((P * (uint32_t)a->owner) / a->R);
    *hi = (uint64_t)((P * ((uint32_t)a->owner + 1u)) / a->R);
}

int check_args(const zero_step_args* a, const char* path) {
    if (a == nullptr || path == nullptr || a->R == 0 || a->ctrl == nullptr) return ZERO_EINVAL;
    if (a->owner < -1 || a->owner >= (int64_t)a->R) return ZERO_EINVAL;
    if (a->P > (UINT64_MAX >> 3)) return ZERO_EOVERFLOW;
    if (a->P > 0 && (a->master[0] == nullptr || a->exp_avg[0] == nullptr || a->exp_avg_sq[0] == nullptr))
        return ZERO_EINVAL;
    const bool two = a->master[1] != nullptr || a->exp_avg[1] != nullptr || a->exp_avg_sq[1] != nullptr;
    if (two && (a->master[1] == nullptr || a->exp_avg[1] == nullptr || a->exp_avg_sq[1] == nullptr))
        return ZERO_EINVAL;
    if ((a->state_offset & 7u) != 0) return ZERO_EALIGN;
    uint64_t lo, hi;
    slice_of(a, &lo, &hi);
    if (a->state_offset > lo && lo < hi) return ZERO_EINVAL;
    return ZERO_OK;
}

// Copy n floats device -> FILE through a host staging buffer, feeding the checksum.
int write_array(FILE* f, const float* dev, uint64_t n, std::vector<float>& stage, Fnv& sum, cudaStream_t st,
                const char* path) {
    for (uint64_t done = 0; done < n;) {
        const size_t k = (size_t)((n - done) < kChunk ? (n - done) : kChunk);
        cudaError_t e = cudaMemcpyAsync(stage.data(), dev + done, k * sizeof(float), cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e);
        sum.add(stage.data(), k * sizeof(float));
        if (std::fwrite(stage.data(), sizeof(float), k, f) != k) return io_fail("write failed", path);
        done += k;
    }
    return ZERO_OK;
}

int read_array(FILE* f, float* dev, uint64_t n, std::vector<float>& stage, Fnv& sum, cudaStream_t st,
               const char* path) {
    for (uint64_t done = 0; done < n;) {
        const size_t k = (size_t)((n - done) < kChunk ? (n - done) : kChunk);
        if (std::fread(stage.data(), sizeof(float), k, f) != k) return io_fail("file too short", path);
        sum.add(stage.data(), k * sizeof(float));
        if (dev != nullptr) {
            cudaError_t e = cudaMemcpyAsync(dev + done, stage.data(), k * sizeof(float), cudaMemcpyHostToDevice, st);
            if (e == cudaSuccess) e = cudaStreamSynchronize(st);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        done += k;
    }
    return ZERO_OK;
}

int read_header(FILE* f, Header* h, Fnv& sum, const char* path) {
    if (std::fread(h, sizeof(Header), 1, f) != 1) return io_fail("cannot read header", path);
    if (std::memcmp(h->magic, kMagic, 8) != 0 || h->header_bytes != kHeaderBytes)
        return io_fail("not a checkpoint shard of this format", path);
    if (h->hi < h->lo || h->hi > h->P) return io_fail("corrupt slice bounds", path);
    sum.add(h, sizeof(Header));
    return ZERO_OK;
}

int read_checksum(FILE* f, const Fnv& sum, const char* path) {
    uint64_t stored = 0;
    if (std::fread(&stored, sizeof stored, 1, f) != 1) return io_fail("file too short", path);
    if (stored != sum.h) return io_fail("checksum mismatch", path);
    return ZERO_OK;
}

}  // namespace

extern "C" {

const char* zero_checkpoint_error(void) { return g_ckpt_error; }

int zero_checkpoint_save(const char* path, const zero_step_args* a, void* stream) {
    int rc = check_args(a, path);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Header h;
    std::memset(&h, 0, sizeof h);
    std::memcpy(h.magic, kMagic, 8);
    h.header_bytes = kHeaderBytes;
    h.R = a->R;
    h.P = a->P;
    h.owner = a->owner;
    slice_of(a, &h.lo, &h.hi);
    cudaError_t e = cudaMemcpyAsync(&h.ctrl, a->ctrl, sizeof(zero_ctrl), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e);
    const bool two = a->master[1] != nullptr;
    const int set = two ? (int)(h.ctrl.parity & 1u) : 0;
    h.ctrl.parity = 0;  // a restore always lands in set 0
    FILE* f = std::fopen(path, "wb");
    if (f == nullptr) return io_fail("cannot open for writing", path);
    Fnv sum;
    sum.add(&h, sizeof h);
    if (std::fwrite(&h, sizeof h, 1, f) != 1) {
        std::fclose(f);
        return io_fail("write failed", path);
    }
    const uint64_t n = h.hi - h.lo;
    std::vector<float> stage((size_t)(n < kChunk ? (n > 0 ? n : 1) : kChunk));
    const float* arrays[3] = {a->master[set], a->exp_avg[set], a->exp_avg_sq[set]};
    for (const float* arr : arrays) {
        if ((rc = write_array(f, arr + (h.lo - a->state_offset), n, stage, sum, st, path))) {
            std::fclose(f);
            return rc;
        }
    }
    const uint64_t c = sum.h;
    const bool ok = std::fwrite(&c, sizeof c, 1, f) == 1;
    if (std::fclose(f) != 0 || !ok) return io_fail("write failed", path);
    return ZERO_OK;
}

int zero_checkpoint_load(const char* path, const zero_step_args* a, void* stream) {
    int rc = check_args(a, path);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    FILE* f = std::fopen(path, "rb");
    if (f == nullptr) return io_fail("cannot open for reading", path);
    Header h;
    Fnv sum;
    if ((rc = read_header(f, &h, sum, path))) {
        std::fclose(f);
        return rc;
    }
    uint64_t lo, hi;
    slice_of(a, &lo, &hi);
    if (h.P != a->P || h.R != a->R || h.owner != a->owner || h.lo != lo || h.hi != hi) {
        std::fclose(f);
        return io_fail("shard does not match P, R and owner of the arguments", path);
    }
    const uint64_t n = hi - lo;
    std::vector<float> stage((size_t)(n < kChunk ? (n > 0 ? n : 1) : kChunk));
    float* arrays[3] = {a->master[0], a->exp_avg[0], a->exp_avg_sq[0]};
    for (float* arr : arrays) {
        if ((rc = read_array(f, arr + (lo - a->state_offset), n, stage, sum, st, path))) {
            std::fclose(f);
            return rc;
        }
    }
    rc = read_checksum(f, sum, path);
    std::fclose(f);
    if (rc) return rc;
    if ((rc = zero_ctrl_set(a->ctrl, &h.ctrl, stream))) return rc;
    if (a->params16 != nullptr && n > 0) {
        // The 16-bit parameters of exactly the slice follow from the restored
        // masters; nothing outside [lo, hi) is read or written, so the arrays
        // may hold only the slice (state_offset) and the other owners'
        // elements of the replica are left to their own restores.
        return zadam_host::cast_slice(a->master[0], a->state_offset, a->params16, a->param_dtype, lo, hi, stream);
    }
    return ZERO_OK;
}

int zero_checkpoint_consolidate(const char* const* paths, uint32_t n_paths, float* weights, uint64_t P) {
    if (paths == nullptr || n_paths == 0 || (P > 0 && weights == nullptr)) return ZERO_EINVAL;
    std::vector<std::pair<uint64_t, uint64_t>> slices;
    for (uint32_t i = 0; i < n_paths; ++i) {
        FILE* f = std::fopen(paths[i], "rb");
        if (f == nullptr) return io_fail("cannot open for reading", paths[i]);
        Header h;
        Fnv sum;
        int rc = read_header(f, &h, sum, paths[i]);
        if (!rc && h.P != P) rc = io_fail("shard belongs to a vector of another size", paths[i]);
        const uint64_t n = rc ? 0 : h.hi - h.lo;
        // masters go straight to the output; the moments are read only for the checksum
        if (!rc && n > 0) {
            if (std::fread(weights + h.lo, sizeof(float), n, f) != n) rc = io_fail("file too short", paths[i]);
            else sum.add(weights + h.lo, n * sizeof(float));
        }
        if (!rc) {
            std::vector<float> skip((size_t)(n < kChunk ? (n > 0 ? n : 1) : kChunk));
            for (int k = 0; k < 2 && !rc; ++k) {
                for (uint64_t done = 0; done < n && !rc;) {
                    const size_t c = (size_t)((n - done) < kChunk ? (n - done) : kChunk);
                    if (std::fread(skip.data(), sizeof(float), c, f) != c) rc = io_fail("file too short", paths[i]);
                    else sum.add(skip.data(), c * sizeof(float));
                    done += c;
                }
            }
        }
        if (!rc) rc = read_checksum(f, sum, paths[i]);
        std::fclose(f);
        if (rc) return rc;
        if (n > 0) slices.emplace_back(h.lo, h.hi);
    }
    // the slices must tile [0, P) exactly: no gap, no overlap
    std::sort(slices.begin(), slices.end());
    uint64_t next = 0;
    for (const auto& sl : slices) {
        if (sl.first != next) {
            std::snprintf(g_ckpt_error, sizeof g_ckpt_error, "shards leave a gap or overlap at element %llu",
                          (unsigned long long)next);
            return ZERO_EIO;
        }
        next = sl.second;
    }
    if (next != P) {
        std::snprintf(g_ckpt_error, sizeof g_ckpt_error, "shards end at element %llu of %llu",
                      (unsigned long long)next, (unsigned long long)P);
        return ZERO_EIO;
    }
    return ZERO_OK;
}

}  // extern "C"
