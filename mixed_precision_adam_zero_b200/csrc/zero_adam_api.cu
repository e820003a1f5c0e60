// zero_adam_api.cu -- the exported C ABI around the sm_100a kernels:
// argument checks, launch shapes and kernel selection.  Declarations and
// the contract of every entry point: include/zero_adam.h.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "zero_adam.h"
#include "zero_adam_internal.h"
#include "zero_adam_kernels.cuh"
#include "zero_adam_bulk.cuh"

using namespace zadam;

namespace {

thread_local char g_cuda_error[256] = "no error";

// Remember the text of a failed CUDA call for zero_last_cuda_error().
int zadam_record_cuda(cudaError_t e) {
    std::snprintf(g_cuda_error, sizeof g_cuda_error, "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return ZERO_ECUDA;
}

// ------------------------------------------------------------ launch shapes

struct OccEntry {
    const void* fn;
    int device;
    int ctas;  // max CTAs resident on the whole device
};

// A kernel, its block size and the dynamic shared memory it is launched with.
struct Kern {
    const void* fn;
    unsigned smem;
    int threads;
};

std::mutex g_occ_mu;
std::vector<OccEntry> g_occ;

// Resident CTAs of `fn` on the current device (SMs x CTAs per SM), cached.
// A kernel with dynamic shared memory gets its opt-in limit raised first.
int resident_ctas(const void* fn, int* err, unsigned smem = 0, int threads = kThreads) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) { *err = zadam_record_cuda(e); return 0; }
    {
        std::lock_guard<std::mutex> lk(g_occ_mu);
        for (const OccEntry& o : g_occ)
            if (o.fn == fn && o.device == dev) return o.ctas;
    }
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess && smem > 0)
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem);
    if (e != cudaSuccess) { *err = zadam_record_cuda(e); return 0; }
    if (per_sm < 1) per_sm = 1;
    const int ctas = sms * per_sm;
    std::lock_guard<std::mutex> lk(g_occ_mu);
    g_occ.push_back({fn, dev, ctas});
    return ctas;
}

struct Shape {
    uint64_t base, chunk;
    unsigned grid;
};

// Split [lo, hi) into at most max_ctas contiguous CTA ranges whose inner
// boundaries are multiples of 64 elements (absolute index: 128-byte aligned
// for 16-bit arrays), each at least one vector per thread long.
constexpr uint64_t kChunkAlign = 64;

Shape make_shape(uint64_t lo, uint64_t hi, int max_ctas) {
    Shape s;
    s.base = lo & ~(kChunkAlign - 1);
    if (hi <= lo) { s.chunk = kChunkAlign; s.grid = 1; return s; }
    const uint64_t n = hi - s.base;
    const uint64_t min_chunk = (uint64_t)kThreads * kVec;
    uint64_t g = (n + min_chunk - 1) / min_chunk;
    if (g > (uint64_t)max_ctas) g = (uint64_t)max_ctas;
    if (g < 1) g = 1;
    uint64_t ch = (n + g - 1) / g;
    ch = (ch + kChunkAlign - 1) & ~(kChunkAlign - 1);
    s.chunk = ch;
    s.grid = (unsigned)((n + ch - 1) / ch);
    return s;
}

// Every kernel is launched with programmatic stream serialization: it may
// start while the kernel before it in the stream finishes, and waits for
// that kernel's completion (griddepcontrol.wait) before it touches global
// memory, so the launch latency and its prologue overlap the earlier
// kernel's tail.
int launch(const void* fn, const Shape& sh, void* params, cudaStream_t st, unsigned smem = 0,
           int threads = kThreads) {
    void* args[] = {params};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sh.grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
    if (e != cudaSuccess) return zadam_record_cuda(e);
    return ZERO_OK;
}

// ------------------------------------------------------------ kernel tables

// Calls with a compiled rank count stage their tiles through shared memory
// with bulk copies (step_bulk_kernel); calls with any other count stream each
// tile's ranks through the same kind of ring, eight at a time
// (step_chunked_kernel); the register kernel takes every call that asks for
// it.  PUSH: flat calls that also store the
// 16-bit values into other replicas.
enum class StepKind { Register, Staged, Chunked };

template <class G, class Pm, int RC, bool LIST, bool PUSH>
Kern bulk_kern() {
    return Kern{(const void*)step_bulk_kernel<G, Pm, RC, LIST, PUSH>, BulkShape<G, RC>::kSmem, kBulkThreads};
}

template <class G, class Pm, bool LIST, bool PUSH>
Kern step_kern_rc(uint32_t R, StepKind kind) {
    if (kind == StepKind::Chunked)
        return Kern{(const void*)step_chunked_kernel<G, Pm, LIST, PUSH>, ChunkShape<G>::kSmem, kBulkThreads};
    if (kind == StepKind::Staged) {
        switch (R) {
            case 1: return bulk_kern<G, Pm, 1, LIST, PUSH>();
            case 2: return bulk_kern<G, Pm, 2, LIST, PUSH>();
            case 4: return bulk_kern<G, Pm, 4, LIST, PUSH>();
            case 8: return bulk_kern<G, Pm, 8, LIST, PUSH>();
            case 16:
                if constexpr (sizeof(G) == 2) return bulk_kern<G, Pm, 16, LIST, PUSH>();
                break;
            default: break;
        }
    }
    return Kern{(const void*)step_kernel<G, Pm, 0, LIST, PUSH>, 0u, kThreads};
}

template <class G, bool LIST, bool PUSH>
Kern step_kern_pm(int32_t param_dtype, uint32_t R, StepKind kind) {
    return param_dtype == ZERO_BF16 ? step_kern_rc<G, __nv_bfloat16, LIST, PUSH>(R, kind)
                                    : step_kern_rc<G, __half, LIST, PUSH>(R, kind);
}

template <bool LIST, bool PUSH>
Kern step_kern_gd(int32_t grad_dtype, int32_t param_dtype, uint32_t R, StepKind kind) {
    switch (grad_dtype) {
        case ZERO_F32: return step_kern_pm<float, LIST, PUSH>(param_dtype, R, kind);
        case ZERO_BF16: return step_kern_pm<__nv_bfloat16, LIST, PUSH>(param_dtype, R, kind);
        default: return step_kern_pm<__half, LIST, PUSH>(param_dtype, R, kind);
    }
}

// Rank counts with a compiled staged instance: 1, 2, 4 and 8, and 16 for
// 16-bit gradients (two 88 KB stages; with fp32 gradients one stage would not
// leave room for a second).
bool has_staged(uint32_t R, int32_t grad_dtype) {
    return R == 1 || R == 2 || R == 4 || R == 8 || (R == 16 && grad_dtype != ZERO_F32);
}

// The step kernel for a path (ZERO_PATH_*): AUTO and STAGED take the staged
// instance compiled for R, else the chunked kernel; REGISTER the register
// kernel.
Kern step_kern(bool list, bool push, int32_t grad_dtype, int32_t param_dtype, uint32_t R, uint32_t path) {
    StepKind kind = StepKind::Register;
    if (path != ZERO_PATH_REGISTER) {
        if (has_staged(R, grad_dtype)) kind = StepKind::Staged;
        else kind = StepKind::Chunked;
    }
    if (list) return step_kern_gd<true, false>(grad_dtype, param_dtype, R, kind);
    return push ? step_kern_gd<false, true>(grad_dtype, param_dtype, R, kind)
                : step_kern_gd<false, false>(grad_dtype, param_dtype, R, kind);
}

template <bool LIST>
const void* scan_fn(int32_t grad_dtype) {
    switch (grad_dtype) {
        case ZERO_F32: return (const void*)scan_kernel<float, LIST>;
        case ZERO_BF16: return (const void*)scan_kernel<__nv_bfloat16, LIST>;
        default: return (const void*)scan_kernel<__half, LIST>;
    }
}

template <bool LIST>
const void* gather_fn(int32_t param_dtype) {
    return param_dtype == ZERO_BF16 ? (const void*)gather_kernel<__nv_bfloat16, LIST>
                                    : (const void*)gather_kernel<__half, LIST>;
}

// Accumulation: when the caller gives a workspace, the bulk kernel compiled
// for R or, for any other R, the chunked one; else the register kernel.
// Measured on a B200 (R = 8 bf16, a window of one first and three continuing
// micro-batches):
// the staged kernel is 10 % faster at 4.2M elements, 4 % at 6.3M, equal at
// 10.5M, 3 % faster at 12.6M and 7 % at 16.8M; only near 8.4M is the
// register kernel ahead (4 %).
template <class G, int RC>
Kern accum_bulk_kern() {
    return Kern{(const void*)accum_bulk_kernel<G, RC>, AccumShape<G, RC>::kSmem, kBulkThreads};
}

template <class G>
Kern accum_kern_rc(uint32_t R, bool bulk) {
    if (bulk) {
        switch (R) {
            case 1: return accum_bulk_kern<G, 1>();
            case 2: return accum_bulk_kern<G, 2>();
            case 4: return accum_bulk_kern<G, 4>();
            case 8: return accum_bulk_kern<G, 8>();
            case 16:
                if constexpr (sizeof(G) == 2) return accum_bulk_kern<G, 16>();
                break;
            default: break;
        }
        // any other rank count: the ranks streamed eight at a time
        return Kern{(const void*)accum_chunked_kernel<G>, AccumChunkShape<G>::kSmem, kBulkThreads};
    }
    switch (R) {
        case 1: return Kern{(const void*)accum_kernel<G, 1>, 0u, kThreads};
        case 2: return Kern{(const void*)accum_kernel<G, 2>, 0u, kThreads};
        case 4: return Kern{(const void*)accum_kernel<G, 4>, 0u, kThreads};
        case 8: return Kern{(const void*)accum_kernel<G, 8>, 0u, kThreads};
        default: return Kern{(const void*)accum_kernel<G, 0>, 0u, kThreads};
    }
}

Kern accum_kern(int32_t grad_dtype, uint32_t R, bool bulk) {
    switch (grad_dtype) {
        case ZERO_F32: return accum_kern_rc<float>(R, bulk);
        case ZERO_BF16: return accum_kern_rc<__nv_bfloat16>(R, bulk);
        default: return accum_kern_rc<__half>(R, bulk);
    }
}

// ------------------------------------------------------------ argument checks

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool finite_nonneg(double x) { return std::isfinite(x) && x >= 0.0; }

int check_hparams(const zero_adam_hparams& h) {
    if (!finite_nonneg(h.lr) || !finite_nonneg(h.eps) || !finite_nonneg(h.weight_decay)) return ZERO_EINVAL;
    if (!(h.beta1 >= 0.0 && h.beta1 < 1.0) || !(h.beta2 >= 0.0 && h.beta2 < 1.0)) return ZERO_EINVAL;
    return ZERO_OK;
}

bool is_grad_dtype(int32_t d) { return d == ZERO_F32 || d == ZERO_BF16 || d == ZERO_F16; }
uint64_t grad_bytes(int32_t d) { return d == ZERO_F32 ? 4u : 2u; }
bool is_param_dtype(int32_t d) { return d == ZERO_BF16 || d == ZERO_F16; }

// Checks shared by the flat and the list step; fills the rank weights, the
// hyperparameters and the state pointers of `kp`.
int check_common(const zero_step_args* a, StepParams* kp) {
    if (a == nullptr) return ZERO_EINVAL;
    if (a->R == 0) return ZERO_EINVAL;
    if (a->R > ZERO_MAX_RANKS) return ZERO_ERANGE;
    if (a->owner < -1 || a->owner >= (int64_t)a->R) return ZERO_EINVAL;
    if (!is_grad_dtype(a->grad_dtype) || !is_param_dtype(a->param_dtype)) return ZERO_EINVAL;
    if (a->check_nonfinite < 0 || a->check_nonfinite > 2) return ZERO_EINVAL;
    if (a->n_push > ZERO_MAX_PUSH) return ZERO_ERANGE;
    if (a->n_push > 0 && a->push_params16 == nullptr) return ZERO_EINVAL;
    if (a->path != ZERO_PATH_AUTO && a->path != ZERO_PATH_REGISTER && a->path != ZERO_PATH_STAGED)
        return ZERO_EINVAL;
    if ((a->state_offset & 7u) != 0 || (a->grad_offset & 7u) != 0) return ZERO_EALIGN;
    if (a->n_grads > ZERO_MAX_RANKS) return ZERO_ERANGE;
    if (a->reserved2 != 0u || (a->grad_offset != 0 && a->check_nonfinite == 1)) return ZERO_EINVAL;
    if (a->P > (UINT64_MAX >> 3)) return ZERO_EOVERFLOW;
    if (a->P > ZERO_MAX_ELEMENTS) return ZERO_ERANGE;
    int rc = check_hparams(a->hp);
    if (rc) return rc;
    if (a->ctrl == nullptr || a->workspace == nullptr) return ZERO_EINVAL;
    if ((reinterpret_cast<uintptr_t>(a->ctrl) & 7u) != 0 || !aligned16(a->workspace)) return ZERO_EALIGN;
    const bool two = a->master[1] != nullptr || a->exp_avg[1] != nullptr || a->exp_avg_sq[1] != nullptr;
    if (two && (a->master[1] == nullptr || a->exp_avg[1] == nullptr || a->exp_avg_sq[1] == nullptr))
        return ZERO_EINVAL;
    const int sets = two ? 2 : 1;
    for (int k = 0; k < sets; ++k) {
        if (a->P > 0 && (a->master[k] == nullptr || a->exp_avg[k] == nullptr || a->exp_avg_sq[k] == nullptr))
            return ZERO_EINVAL;
        if (!aligned16(a->master[k]) || !aligned16(a->exp_avg[k]) || !aligned16(a->exp_avg_sq[k])) return ZERO_EALIGN;
    }
    if (!aligned16(a->reduced_out)) return ZERO_EALIGN;

    // Rank weights as given (float64) and their sum, in rank order, over the
    // gradient buffers the call reduces (the R ranks', or n_grads of them).
    const uint32_t ng = a->n_grads ? a->n_grads : a->R;
    double wsum = 0.0;
    for (uint32_t r = 0; r < ng; ++r) {
        const double wr = a->rank_weights ? a->rank_weights[r] : 1.0;
        if (!finite_nonneg(wr)) return ZERO_EINVAL;
        wsum += wr;
    }
    if (!(wsum > 0.0) || !std::isfinite(wsum)) return ZERO_EINVAL;
    std::memset(kp, 0, sizeof(*kp));
    for (uint32_t r = 0; r < ng; ++r) kp->wt[r] = a->rank_weights ? a->rank_weights[r] : 1.0;
    kp->wsum = wsum;

    // State arrays that start at flat index state_offset: the kernels index
    // them by the flat index, so hand them pointers moved back by that much
    // (only indices >= state_offset are ever dereferenced).
    const uintptr_t back = (uintptr_t)(a->state_offset * sizeof(float));
    auto shift = [back](float* q) { return q ? reinterpret_cast<float*>(reinterpret_cast<uintptr_t>(q) - back) : q; };
    for (int k = 0; k < 2; ++k) {
        const int src = two ? k : 0;
        kp->w[k] = shift(a->master[src]);
        kp->m[k] = shift(a->exp_avg[src]);
        kp->v[k] = shift(a->exp_avg_sq[src]);
    }
    kp->reduced = shift(a->reduced_out);
    for (uint32_t i = 0; i < a->n_push; ++i) {
        if (a->P > 0 && a->push_params16[i] == nullptr) return ZERO_EINVAL;
        if (!aligned16(a->push_params16[i])) return ZERO_EALIGN;
        kp->push[i] = a->push_params16[i];
    }
    kp->npush = a->n_push;
    // Push targets hold the other ranks' replicas of one owner's slice.  An
    // all-owner call may take its skip decision in the same pass that stores
    // the 16-bit values (two-set mode), and only the local replica is
    // restored after a skip; so pushes need an owner.
    if (a->n_push > 0 && a->owner < 0) return ZERO_EINVAL;
    const zero_adam_hparams& h = a->hp;
    kp->h.b1 = (float)h.beta1;
    kp->h.b2 = (float)h.beta2;
    kp->h.omb1 = (float)(1.0 - h.beta1);
    kp->h.omb2 = (float)(1.0 - h.beta2);
    kp->h.eps = (float)h.eps;
    kp->h.lr_wd = (float)(h.lr * h.weight_decay);
    kp->h.lr = h.lr;
    kp->h.b1d = h.beta1;
    kp->h.b2d = h.beta2;
    kp->ctrl = static_cast<zero_ctrl*>(a->ctrl);
    kp->ws = static_cast<Workspace*>(a->workspace);
    kp->R = ng;  // the reduction's length; the partition is a->R (owner_range)
    kp->growth_interval = a->growth_interval;
    kp->two_set = two ? 1 : 0;
    return ZERO_OK;
}

// Range of the launch: every slice, or one owner's.
void owner_range(const zero_step_args* a, uint64_t* lo, uint64_t* hi) {
    if (a->owner < 0) { *lo = 0; *hi = a->P; return; }
    const unsigned __int128 P = a->P;
    *lo = (uint64_t)((P * (uint32_t)a->owner) / a->R);
    *hi = (uint64_t)((P * ((uint32_t)a->owner + 1u)) / a->R);
}

// The launch sequence shared by the flat and list calls.
template <bool LIST>
int run_step(const zero_step_args* a, StepParams* kp, cudaStream_t st) {
    uint64_t lo, hi;
    owner_range(a, &lo, &hi);
    if ((a->state_offset > lo || a->grad_offset > lo) && lo < hi) return ZERO_EINVAL;
    kp->lo = lo;
    kp->hi = hi;
    int err = ZERO_OK;
    const bool check = a->check_nonfinite != 0;
    const bool single_pass = a->check_nonfinite == 1 && kp->two_set && a->owner < 0;
    if (a->check_nonfinite == 2) {
        kp->check = 2;  // zero_scan_nonfinite calls (and the caller) decided
    } else if (check && !single_pass) {
        // Scan every rank's whole gradient first; the step then reads the flag.
        StepParams sp = *kp;
        const void* sfn = scan_fn<LIST>(a->grad_dtype);
        const int ctas = resident_ctas(sfn, &err);
        if (err) return err;
        const Shape sh = make_shape(0, a->P, ctas);
        sp.lo = 0;
        sp.hi = a->P;
        sp.base = sh.base;
        sp.chunk = sh.chunk;
        if ((err = launch(sfn, sh, &sp, st))) return err;
        kp->check = 2;
    } else {
        kp->check = check ? 1 : 0;
    }
    const Kern k = step_kern(LIST, kp->npush > 0, a->grad_dtype, a->param_dtype, kp->R, a->path);
    const int ctas = resident_ctas(k.fn, &err, k.smem, k.threads);
    if (err) return err;
    const Shape sh = make_shape(lo, hi, ctas);
    kp->base = sh.base;
    kp->chunk = sh.chunk;
    if ((err = launch(k.fn, sh, kp, st, k.smem, k.threads))) return err;
    if (single_pass) {
        // Only if the step was skipped: re-cast the 16-bit parameters from
        // the master set that stayed current.
        GatherParams gp;
        std::memset(&gp, 0, sizeof gp);
        gp.w[0] = kp->w[0];
        gp.w[1] = kp->w[1];
        gp.params16 = kp->params16;
        gp.tab = kp->tab;
        gp.lo = lo;
        gp.hi = hi;
        gp.ctrl = kp->ctrl;
        gp.only_if_skipped = 1;
        const void* gfn = gather_fn<LIST>(a->param_dtype);
        const int gctas = resident_ctas(gfn, &err);
        if (err) return err;
        const Shape gsh = make_shape(lo, hi, gctas);
        gp.base = gsh.base;
        gp.chunk = gsh.chunk;
        if ((err = launch(gfn, gsh, &gp, st))) return err;
    }
    return ZERO_OK;
}

// Host copy of a list's table layout: byte offsets of each array.
struct TableLayout {
    size_t offs, params, grads, flags, tiles, scratch, total;
};

TableLayout table_layout(uint32_t T, uint32_t R) {
    TableLayout L;
    L.offs = 0;
    L.params = L.offs + 8ull * ((size_t)T + 1);
    L.grads = L.params + 8ull * T;
    L.flags = L.grads + 8ull * (size_t)T * R;
    L.tiles = L.flags + ((4ull * T + 15) & ~15ull);
    L.scratch = L.tiles + 8ull * ((size_t)T + 1);
    L.total = L.scratch + 16;
    return L;
}

Table device_table(const zero_tensor_list* l) {
    const TableLayout L = table_layout(l->T, l->R);
    const char* base = static_cast<const char*>(l->table);
    Table t;
    t.offs = reinterpret_cast<const uint64_t*>(base + L.offs);
    t.params = reinterpret_cast<void* const*>(base + L.params);
    t.grads = reinterpret_cast<const void* const*>(base + L.grads);
    t.flags = reinterpret_cast<const uint32_t*>(base + L.flags);
    t.tiles = reinterpret_cast<const uint64_t*>(base + L.tiles);
    t.scratch = reinterpret_cast<unsigned int*>(const_cast<char*>(base) + L.scratch);
    t.T = l->T;
    return t;
}

int check_list(const zero_tensor_list* l) {
    if (l == nullptr || l->table == nullptr || l->T == 0 || l->R == 0) return ZERO_EINVAL;
    if (l->R > ZERO_MAX_RANKS) return ZERO_ERANGE;
    if (!aligned16(l->table)) return ZERO_EALIGN;
    if (l->table_bytes < table_layout(l->T, l->R).total) return ZERO_EINVAL;
    if (!is_grad_dtype(l->grad_dtype) || !is_param_dtype(l->param_dtype)) return ZERO_EINVAL;
    return ZERO_OK;
}

// ------------------------------------------------------------ no-alloc scratch

// Library-owned scratch of zero_step_fused_noalloc: one workspace per device,
// alive until the process exits.  Host code sees only a stand-in symbol; the
// device address comes from cudaGetSymbolAddress with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ZERO_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of this device's scratch array (looked up on first use).
int noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return zadam_record_cuda(e);
    if (dev < 0 || dev >= kMaxDevices) return ZERO_ERANGE;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return zadam_record_cuda(e);
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return ZERO_OK;
}

}  // namespace

// =================================================================== C ABI

int zadam_host::cast_slice(const float* master, uint64_t state_offset, void* params16, int32_t param_dtype,
                           uint64_t lo, uint64_t hi, void* stream) {
    if (!is_param_dtype(param_dtype) || master == nullptr || params16 == nullptr) return ZERO_EINVAL;
    if ((state_offset & 7u) != 0 || !aligned16(master) || !aligned16(params16)) return ZERO_EALIGN;
    if (state_offset > lo) return ZERO_EINVAL;
    if (lo >= hi) return ZERO_OK;
    GatherParams gp;
    std::memset(&gp, 0, sizeof gp);
    const float* w = reinterpret_cast<const float*>(reinterpret_cast<uintptr_t>(master) - state_offset * 4u);
    gp.w[0] = gp.w[1] = w;
    gp.params16 = params16;
    gp.lo = lo;
    gp.hi = hi;
    int err = ZERO_OK;
    const void* fn = gather_fn<false>(param_dtype);
    const int ctas = resident_ctas(fn, &err);
    if (err) return err;
    const Shape sh = make_shape(lo, hi, ctas);
    gp.base = sh.base;
    gp.chunk = sh.chunk;
    return launch(fn, sh, &gp, static_cast<cudaStream_t>(stream));
}

extern "C" {

const char* zero_last_cuda_error(void) { return g_cuda_error; }

size_t zero_ctrl_bytes(void) { return sizeof(zero_ctrl); }
size_t zero_workspace_bytes(void) { return ZERO_WORKSPACE_BYTES; }

size_t zero_list_table_bytes(uint32_t T, uint32_t R) { return table_layout(T, R).total; }

int zero_ctrl_init(void* ctrl, float loss_scale, void* stream) {
    if (!(std::isfinite(loss_scale) && loss_scale > 0.0f)) return ZERO_EINVAL;
    zero_ctrl v;
    std::memset(&v, 0, sizeof v);
    v.loss_scale = loss_scale;
    return zero_ctrl_set(ctrl, &v, stream);
}

int zero_ctrl_set(void* ctrl, const zero_ctrl* value, void* stream) {
    if (ctrl == nullptr || value == nullptr) return ZERO_EINVAL;
    if ((reinterpret_cast<uintptr_t>(ctrl) & 7u) != 0) return ZERO_EALIGN;
    if (!(std::isfinite(value->loss_scale) && value->loss_scale > 0.0f) || value->parity > 1u) return ZERO_EINVAL;
    ctrl_set_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<zero_ctrl*>(ctrl), *value);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ZERO_OK : zadam_record_cuda(e);
}

int zero_ctrl_read(const void* ctrl, zero_ctrl* out, void* stream) {
    if (ctrl == nullptr || out == nullptr) return ZERO_EINVAL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(out, ctrl, sizeof(zero_ctrl), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e == cudaSuccess ? ZERO_OK : zadam_record_cuda(e);
}

int zero_scan_nonfinite(const void* grad, int32_t grad_dtype, uint64_t n, void* workspace, void* stream) {
    if (!is_grad_dtype(grad_dtype) || workspace == nullptr || (n > 0 && grad == nullptr)) return ZERO_EINVAL;
    if (!aligned16(grad) || !aligned16(workspace)) return ZERO_EALIGN;
    if (n > (UINT64_MAX >> 3)) return ZERO_EOVERFLOW;
    if (n == 0) return ZERO_OK;
    StepParams sp;
    std::memset(&sp, 0, sizeof sp);
    sp.grads[0] = grad;
    sp.R = 1;
    sp.ws = static_cast<Workspace*>(workspace);
    sp.lo = 0;
    sp.hi = n;
    int err = ZERO_OK;
    const void* fn = scan_fn<false>(grad_dtype);
    const int ctas = resident_ctas(fn, &err);
    if (err) return err;
    const Shape sh = make_shape(0, n, ctas);
    sp.base = sh.base;
    sp.chunk = sh.chunk;
    return launch(fn, sh, &sp, static_cast<cudaStream_t>(stream));
}

int zero_selftest_wait_timeout(void* ctrl, void* stream) {
    if (ctrl == nullptr) return ZERO_EINVAL;
    if ((reinterpret_cast<uintptr_t>(ctrl) & 7u) != 0) return ZERO_EALIGN;
    Shape sh{0, 0, 1};
    zero_ctrl* c = static_cast<zero_ctrl*>(ctrl);
    return launch((const void*)wait_timeout_probe_kernel, sh, &c, static_cast<cudaStream_t>(stream), 0, 32);
}

int zero_enable_peer_access(int32_t peer_device) {
    if (peer_device < 0) return ZERO_EINVAL;
    int dev = 0, count = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaGetDeviceCount(&count);
    if (e != cudaSuccess) return zadam_record_cuda(e);
    if (peer_device >= count) return ZERO_ERANGE;
    if (peer_device == dev) return ZERO_OK;
    int can = 0;
    if ((e = cudaDeviceCanAccessPeer(&can, dev, peer_device)) != cudaSuccess) return zadam_record_cuda(e);
    if (!can) return ZERO_EINVAL;
    e = cudaDeviceEnablePeerAccess(peer_device, 0);
    if (e == cudaErrorPeerAccessAlreadyEnabled) {
        (void)cudaGetLastError();  // not an error here: clear it from the thread's state
        return ZERO_OK;
    }
    return e == cudaSuccess ? ZERO_OK : zadam_record_cuda(e);
}

int zero_workspace_init(void* workspace, void* stream) {
    if (workspace == nullptr) return ZERO_EINVAL;
    if (!aligned16(workspace)) return ZERO_EALIGN;
    const cudaError_t e = cudaMemsetAsync(workspace, 0, ZERO_WORKSPACE_BYTES, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ZERO_OK : zadam_record_cuda(e);
}

int zero_step_fused(const zero_step_args* a, void* stream) {
    StepParams kp;
    int rc = check_common(a, &kp);
    if (rc) return rc;
    if (a->grads == nullptr) return ZERO_EINVAL;
    if (a->P > 0 && a->params16 == nullptr) return ZERO_EINVAL;
    if (!aligned16(a->params16)) return ZERO_EALIGN;
    // Gradient buffers that start at flat index grad_offset: moved back like
    // the state arrays (only indices >= grad_offset are dereferenced).
    const uintptr_t gback = (uintptr_t)(a->grad_offset * grad_bytes(a->grad_dtype));
    for (uint32_t r = 0; r < kp.R; ++r) {
        if (a->P > 0 && a->grads[r] == nullptr) return ZERO_EINVAL;
        if (!aligned16(a->grads[r])) return ZERO_EALIGN;
        kp.grads[r] = a->grads[r] ? reinterpret_cast<const void*>(reinterpret_cast<uintptr_t>(a->grads[r]) - gback)
                                  : nullptr;
    }
    kp.params16 = a->params16;
    return run_step<false>(a, &kp, static_cast<cudaStream_t>(stream));
}

int zero_step_fused_list(const zero_step_args* a, const zero_tensor_list* l, void* stream) {
    StepParams kp;
    int rc = check_common(a, &kp);
    if (rc) return rc;
    if ((rc = check_list(l))) return rc;
    if (a->grads != nullptr || a->params16 != nullptr) return ZERO_EINVAL;
    if (a->state_offset != 0 || a->n_push != 0 || a->n_grads != 0 || a->grad_offset != 0)
        return ZERO_EINVAL;  // multi-GPU fields: flat calls only
    if (a->P != l->P || a->R != l->R || a->grad_dtype != l->grad_dtype || a->param_dtype != l->param_dtype)
        return ZERO_EINVAL;
    kp.tab = device_table(l);
    kp.whole = a->owner < 0 ? 1 : 0;
    return run_step<true>(a, &kp, static_cast<cudaStream_t>(stream));
}

int zero_accumulate_grads(const zero_accum_args* a, void* stream) {
    if (a == nullptr || a->R == 0 || a->grads == nullptr) return ZERO_EINVAL;
    if (a->R > ZERO_MAX_RANKS) return ZERO_ERANGE;
    if (a->owner < -1 || a->owner >= (int64_t)a->R) return ZERO_EINVAL;
    if (!is_grad_dtype(a->grad_dtype) || (a->first != 0 && a->first != 1)) return ZERO_EINVAL;
    if (!std::isfinite(a->scale)) return ZERO_EINVAL;
    if (a->P > (UINT64_MAX >> 3)) return ZERO_EOVERFLOW;
    if (a->P > ZERO_MAX_ELEMENTS) return ZERO_ERANGE;
    if (a->P > 0 && a->accum == nullptr) return ZERO_EINVAL;
    if (!aligned16(a->accum)) return ZERO_EALIGN;
    if ((a->workspace == nullptr) != (a->ctrl == nullptr)) return ZERO_EINVAL;
    if (a->path != ZERO_PATH_AUTO && a->path != ZERO_PATH_REGISTER && a->path != ZERO_PATH_STAGED)
        return ZERO_EINVAL;
    const bool can_stage = a->workspace != nullptr;  // a staged instance, or the chunked kernel
    // AUTO takes the chunked kernel only where it measured faster than the
    // register kernel on a B200: it pays a fixed cost per tile, so a tile has
    // to carry enough gradient bytes (16-bit gradients from R = 6 on, fp32
    // from R = 9 on; 67M elements: bf16 R = 3 0.72 vs 0.78 of the copy peak,
    // R = 6 0.87 vs 0.75, R = 32 0.86 vs 0.70, fp32 R = 3 0.82 vs 0.94,
    // R = 16 1.06 vs 1.01).
    const bool chunk_pays = a->grad_dtype == ZERO_F32 ? a->R >= 9u : a->R >= 6u;
    if (a->path == ZERO_PATH_STAGED && !can_stage) return ZERO_EINVAL;
    if (!aligned16(a->workspace) || (reinterpret_cast<uintptr_t>(a->ctrl) & 7u) != 0) return ZERO_EALIGN;
    AccumParams ap;
    std::memset(&ap, 0, sizeof ap);
    double wsum = 0.0;
    for (uint32_t r = 0; r < a->R; ++r) {
        if (a->P > 0 && a->grads[r] == nullptr) return ZERO_EINVAL;
        if (!aligned16(a->grads[r])) return ZERO_EALIGN;
        const double wr = a->rank_weights ? a->rank_weights[r] : 1.0;
        if (!finite_nonneg(wr)) return ZERO_EINVAL;
        ap.grads[r] = a->grads[r];
        ap.wt[r] = wr;
        wsum += wr;
    }
    if (!(wsum > 0.0) || !std::isfinite(wsum)) return ZERO_EINVAL;
    ap.inv_wsum = 1.0 / wsum;
    ap.scale = a->scale;
    if ((a->accum_offset & 7u) != 0) return ZERO_EALIGN;
    // An accumulator that starts at flat index accum_offset is moved back like
    // the step's state arrays (only indices >= accum_offset are dereferenced).
    ap.acc = a->accum ? reinterpret_cast<float*>(reinterpret_cast<uintptr_t>(a->accum) - a->accum_offset * 4u)
                      : nullptr;
    ap.ws = static_cast<Workspace*>(a->workspace);
    ap.ctrl = static_cast<zero_ctrl*>(a->ctrl);
    ap.R = a->R;
    ap.first = a->first;
    if (a->owner < 0) {
        ap.lo = 0;
        ap.hi = a->P;
    } else {
        const unsigned __int128 P = a->P;
        ap.lo = (uint64_t)((P * (uint32_t)a->owner) / a->R);
        ap.hi = (uint64_t)((P * ((uint32_t)a->owner + 1u)) / a->R);
    }
    if (ap.lo >= ap.hi) return ZERO_OK;
    if (a->accum_offset > ap.lo) return ZERO_EINVAL;
    int err = ZERO_OK;
    const bool staged = a->path == ZERO_PATH_STAGED ||
                        (a->path == ZERO_PATH_AUTO && can_stage && (has_staged(a->R, a->grad_dtype) || chunk_pays));
    const Kern k = accum_kern(a->grad_dtype, a->R, staged);
    const int ctas = resident_ctas(k.fn, &err, k.smem, k.threads);
    if (err) return err;
    const Shape sh = make_shape(ap.lo, ap.hi, ctas);
    ap.base = sh.base;
    ap.chunk = sh.chunk;
    return launch(k.fn, sh, &ap, static_cast<cudaStream_t>(stream), k.smem, k.threads);
}

int zero_step_fused_noalloc(const zero_step_args* a, void* stream) {
    if (a == nullptr || a->workspace != nullptr) return ZERO_EINVAL;
    // Mode 2 reads an inf/NaN word that zero_scan_nonfinite calls wrote into
    // the caller's workspace; no scan can write into the library's array.
    if (a->check_nonfinite == 2) return ZERO_EINVAL;
    if (ZERO_WORKSPACE_BYTES > ZERO_NOALLOC_SCRATCH_BYTES) return ZERO_ERANGE;
    void* ws = nullptr;
    int rc = noalloc_scratch(&ws);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const cudaError_t e = cudaMemsetAsync(ws, 0, ZERO_WORKSPACE_BYTES, st);
    if (e != cudaSuccess) return zadam_record_cuda(e);
    zero_step_args b = *a;
    b.workspace = ws;
    return zero_step_fused(&b, stream);
}

int zero_list_table_build(uint32_t T, uint32_t R, const uint64_t* numel, void* const* params16,
                          const void* const* grads, int32_t grad_dtype, int32_t param_dtype, void* table,
                          size_t table_bytes, zero_tensor_list* out, void* stream) {
    if (T == 0 || R == 0 || numel == nullptr || params16 == nullptr || grads == nullptr || table == nullptr ||
        out == nullptr)
        return ZERO_EINVAL;
    if (R > ZERO_MAX_RANKS) return ZERO_ERANGE;
    if (!is_grad_dtype(grad_dtype) || !is_param_dtype(param_dtype)) return ZERO_EINVAL;
    if (!aligned16(table)) return ZERO_EALIGN;
    const TableLayout L = table_layout(T, R);
    if (table_bytes < L.total) return ZERO_EINVAL;
    std::vector<unsigned char> buf(L.total, 0);
    uint64_t* offs = reinterpret_cast<uint64_t*>(buf.data() + L.offs);
    void** prm = reinterpret_cast<void**>(buf.data() + L.params);
    const void** grd = reinterpret_cast<const void**>(buf.data() + L.grads);
    uint32_t* flags = reinterpret_cast<uint32_t*>(buf.data() + L.flags);
    uint64_t* tiles = reinterpret_cast<uint64_t*>(buf.data() + L.tiles);
    uint64_t P = 0;
    for (uint32_t j = 0; j < T; ++j) {
        offs[j] = P;
        if (numel[j] > (UINT64_MAX >> 3) - P) return ZERO_EOVERFLOW;
        P += numel[j];
        bool vec_ok = (offs[j] & 7u) == 0;
        if (numel[j] > 0 && params16[j] == nullptr) return ZERO_EINVAL;
        vec_ok = vec_ok && aligned16(params16[j]);
        prm[j] = params16[j];
        for (uint32_t r = 0; r < R; ++r) {
            const void* g = grads[(size_t)r * T + j];
            if (numel[j] > 0 && g == nullptr) return ZERO_EINVAL;
            vec_ok = vec_ok && aligned16(g);
            grd[(size_t)j * R + r] = g;
        }
        flags[j] = vec_ok ? 1u : 0u;
    }
    offs[T] = P;
    // Vector tiles of each tensor's body [offs[j], round_down(offs[j+1], 8)),
    // as running counts (used when a step covers the whole vector).
    tiles[0] = 0;
    for (uint32_t j = 0; j < T; ++j) {
        const uint64_t body_end = offs[j + 1] & ~7ull;
        const uint64_t nt = (flags[j] && body_end > offs[j]) ? (body_end - offs[j] + kTile - 1) / kTile : 0;
        tiles[j + 1] = tiles[j] + nt;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(table, buf.data(), L.total, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return zadam_record_cuda(e);
    out->table = table;
    out->P = P;
    out->T = T;
    out->R = R;
    out->grad_dtype = grad_dtype;
    out->param_dtype = param_dtype;
    out->table_bytes = L.total;
    return ZERO_OK;
}

int zero3_gather_list_build(uint32_t T, uint32_t R, const uint64_t* numel, void* const* full,
                            const void* const* shards, int32_t dtype, void* table, size_t table_bytes,
                            zero_tensor_list* out, void* stream) {
    if (T == 0 || R == 0 || numel == nullptr) return ZERO_EINVAL;
    std::vector<uint64_t> padded(T);
    for (uint32_t j = 0; j < T; ++j) {
        const uint64_t s = numel[j] / R + (numel[j] % R != 0 ? 1u : 0u);
        if (s > (UINT64_MAX >> 4) / R) return ZERO_EOVERFLOW;
        padded[j] = s * R;
    }
    return zero_list_table_build(T, R, padded.data(), full, shards, dtype, dtype, table, table_bytes, out, stream);
}

int zero3_gather(const zero_tensor_list* l, void* stream) {
    int rc = check_list(l);
    if (rc) return rc;
    if (l->grad_dtype != l->param_dtype || l->param_dtype == ZERO_F32) return ZERO_EINVAL;
    if (l->P == 0) return ZERO_OK;
    Z3Params zp;
    std::memset(&zp, 0, sizeof zp);
    zp.tab = device_table(l);
    zp.lo = 0;
    zp.hi = l->P;
    zp.R = l->R;
    int err = ZERO_OK;
    const void* fn = l->param_dtype == ZERO_BF16 ? (const void*)z3_gather_kernel<__nv_bfloat16>
                                                 : (const void*)z3_gather_kernel<__half>;
    const int ctas = resident_ctas(fn, &err);
    if (err) return err;
    const uint64_t nchunks = (l->P + kZ3Chunk - 1) / kZ3Chunk;
    if (nchunks > 0xFFFFFFFFull - 65536ull) return ZERO_EOVERFLOW;  // claims stay below 2^32
    Shape sh{0, kZ3Chunk, (unsigned)(nchunks < (uint64_t)ctas ? nchunks : (uint64_t)ctas)};
    return launch(fn, sh, &zp, static_cast<cudaStream_t>(stream));
}

int zero_gather_params(const float* master, void* params16, int32_t param_dtype, uint64_t P, void* stream) {
    if (!is_param_dtype(param_dtype)) return ZERO_EINVAL;
    if (P > (UINT64_MAX >> 3)) return ZERO_EOVERFLOW;
    if (P > 0 && (master == nullptr || params16 == nullptr)) return ZERO_EINVAL;
    if (!aligned16(master) || !aligned16(params16)) return ZERO_EALIGN;
    if (P == 0) return ZERO_OK;
    GatherParams gp;
    std::memset(&gp, 0, sizeof gp);
    gp.w[0] = gp.w[1] = master;
    gp.params16 = params16;
    gp.lo = 0;
    gp.hi = P;
    int err = ZERO_OK;
    const void* fn = gather_fn<false>(param_dtype);
    const int ctas = resident_ctas(fn, &err);
    if (err) return err;
    const Shape sh = make_shape(0, P, ctas);
    gp.base = sh.base;
    gp.chunk = sh.chunk;
    return launch(fn, sh, &gp, static_cast<cudaStream_t>(stream));
}

int zero_gather_params_list(const float* master, const zero_tensor_list* l, void* stream) {
    int rc = check_list(l);
    if (rc) return rc;
    if (l->P > 0 && master == nullptr) return ZERO_EINVAL;
    if (!aligned16(master)) return ZERO_EALIGN;
    if (l->P == 0) return ZERO_OK;
    GatherParams gp;
    std::memset(&gp, 0, sizeof gp);
    gp.w[0] = gp.w[1] = master;
    gp.tab = device_table(l);
    gp.lo = 0;
    gp.hi = l->P;
    int err = ZERO_OK;
    const void* fn = gather_fn<true>(l->param_dtype);
    const int ctas = resident_ctas(fn, &err);
    if (err) return err;
    const Shape sh = make_shape(0, l->P, ctas);
    gp.base = sh.base;
    gp.chunk = sh.chunk;
    return launch(fn, sh, &gp, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
