// zero_adam_kernels.cuh -- sm_100a kernels of the fused ZeRO-2/3 Adam step.
//
// The step is HBM-bound (about 25 flops against 2R+26 bytes per parameter),
// so it is written as streaming kernels, not as tensor-core work.  This file
// holds the shared arithmetic and the register-staged kernels (the step for
// rank counts without a staged instance, the overflow scan, the 16-bit
// cast, the ZeRO-3 gather, the accumulation); zero_adam_bulk.cuh holds the
// shared-memory staged kernels that the common rank counts run.
//   * register kernels: one CTA per slot of a persistent grid (SMs x
//     resident CTAs), each CTA owning one contiguous range of the flat index
//     space, so every CTA streams sequential addresses and the ranges
//     balance to within 8 elements;
//   * 128-bit loads and stores with the streaming (evict-first) cache hint;
//     one vector is 8 elements: one 16-byte load per 16-bit gradient, two per
//     fp32 array;
//   * the rank reduction is a fixed-order float64 FMA chain over r = 0..R-1
//     of the raw rank weights times the gradients (both exact in float64),
//     scaled once by 1/(sum(w)*S) and rounded once to float32.  A float32
//     chain is not enough: at small step counts Adam moves w by about
//     lr*g/(|g|+eps), whose sensitivity to an absolute error in g reaches
//     lr/eps, so the reduced gradient must be accurate relative to itself
//     even where the ranks' gradients nearly cancel.  The chain is the same
//     in the vector and the scalar path, so results are bitwise reproducible;
//   * grid-level results (the inf/NaN flag, the step counter) use a
//     last-block-done epilogue: each CTA adds its packed arrival (count,
//     inf/NaN, timeout) to one word of the workspace, and the CTA whose
//     atomic completes the count updates the control block and re-zeroes
//     the workspace.  No kernel here spins; the only wait is the grid
//     dependency wait of the programmatic launch (grid_dependency_wait).
//
// Sources of the arithmetic ("Deep dive: DeepSpeed", "Reduce first, then
// update the owned slice"; AdamW of the "ZeRO" documentation page): see
// include/zero_adam.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zero_adam.h"

namespace zadam {

constexpr int kThreads = 256;  // threads per CTA
constexpr int kVec = 8;        // elements per vector

// Scratch of one step call (ZERO_WORKSPACE_BYTES).  All zero between calls.
struct Workspace {
    unsigned long long arrive;  // CTAs of the running launch that have finished, packed (see Arrival)
    unsigned int found;         // two-pass check: the scan kernel saw an inf or NaN
    unsigned int next_tile;     // dynamic tiles: claims made so far
    unsigned int pad[60];
};
static_assert(sizeof(Workspace) == ZERO_WORKSPACE_BYTES, "workspace size");

// A CTA's arrival adds 1 to the count field, and 1 to the found field if it
// saw an inf or NaN, and 1 to the timeout field if one of its bounded waits
// gave up.  One 64-bit atomic carries all three, so the CTA that completes
// the count knows the whole grid's flags from the value its own atomic
// returns, with no fence and no second read (a grid has < 2^21 CTAs).
struct Arrival {
    static constexpr int kBits = 21;
    static constexpr unsigned long long kMask = (1ull << kBits) - 1ull;
    static constexpr unsigned long long kFound = 1ull << kBits;
    static constexpr unsigned long long kTimeout = 1ull << (2 * kBits);
    static __device__ __forceinline__ unsigned long long mine(bool found, bool timeout) {
        return 1ull | (found ? kFound : 0ull) | (timeout ? kTimeout : 0ull);
    }
    static __device__ __forceinline__ unsigned long long count(unsigned long long v) { return v & kMask; }
    static __device__ __forceinline__ bool any_found(unsigned long long v) { return ((v >> kBits) & kMask) != 0ull; }
    static __device__ __forceinline__ bool any_timeout(unsigned long long v) {
        return ((v >> (2 * kBits)) & kMask) != 0ull;
    }
};

// Programmatic dependent launch.  Every kernel the library launches is
// launched so that it may start while the kernel before it in the stream is
// still finishing (its CTAs take each SM as the earlier CTAs leave it), and
// each kernel first waits, with grid_dependency_wait, until that kernel has
// completed and its memory is visible, before its first access to global
// memory; it then lets the kernel after it start early the same way.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

struct Hyper {
    float b1, b2, omb1, omb2, eps, lr_wd;  // float32 per-element constants
    double lr, b1d, b2d;                   // float64, for the bias corrections
};

// Device view of a tensor-list table.
struct Table {
    const uint64_t* offs;       // [T+1] flat start of each tensor, offs[T] = P
    void* const* params;        // [T] 16-bit parameter tensors
    const void* const* grads;   // [T*R] gradients, tensor-major: grads[j*R + r]
    const uint32_t* flags;      // [T] bit 0: vector path allowed
    const uint64_t* tiles;      // [T+1] vector tiles of tensors 0..j-1 (whole-vector calls)
    unsigned int* scratch;      // [4] ZeRO-3 gather: chunks claimed, CTAs finished (zero between calls)
    uint32_t T;
};

struct StepParams {
    const void* grads[ZERO_MAX_RANKS];  // flat call: rank r's gradient [P]
    double wt[ZERO_MAX_RANKS];          // rank weights w_r (1 for the equal mean)
    double wsum;                        // sum of the w_r
    float* w[2];                        // master sets
    float* m[2];
    float* v[2];
    void* params16;                     // flat call: 16-bit parameters [P]
    void* push[ZERO_MAX_PUSH];          // flat call: other ranks' 16-bit parameters [P]
    float* reduced;                     // optional reduced-gradient output
    Table tab;                          // list call
    uint64_t lo, hi;                    // elements this launch updates
    uint64_t base, chunk;               // CTA b: [base + b*chunk, base + (b+1)*chunk) within [lo, hi)
    Hyper h;
    zero_ctrl* ctrl;
    Workspace* ws;
    uint32_t R;
    uint32_t growth_interval;
    int32_t two_set;  // 1: read set ctrl.parity, write the other set
    int32_t check;    // 0: none; 1: detect inf/NaN in this pass; 2: a scan decided
    int32_t whole;    // 1: the launch covers every owner's slice ([0, P))
    uint32_t npush;   // entries of push in use
};

struct GatherParams {
    const float* w[2];
    void* params16;
    Table tab;
    uint64_t lo, hi, base, chunk;
    const zero_ctrl* ctrl;     // non-NULL: read the set at ctrl.parity
    int32_t only_if_skipped;   // 1: do nothing unless ctrl.last_skipped
};

// Per-call scalars derived from the control block.
struct Scal {
    float b1, b2, omb1, omb2, eps, lr_wd;
    float step;          // lr / (1 - b1^t)
    float inv_sqrt_bc2;  // 1 / sqrt(1 - b2^t)
    double inv_ws;       // 1 / (sum(w) * S)
};

// b^e by binary exponentiation (float64).
__device__ __forceinline__ double pow_u64(double b, uint64_t e) {
    double r = 1.0;
    while (e) {
        if (e & 1ull) r *= b;
        b *= b;
        e >>= 1;
    }
    return r;
}

__device__ __forceinline__ Scal make_scal(const Hyper& h, uint64_t t, float S, double wsum) {
    Scal s;
    s.b1 = h.b1;
    s.b2 = h.b2;
    s.omb1 = h.omb1;
    s.omb2 = h.omb2;
    s.eps = h.eps;
    s.lr_wd = h.lr_wd;
    const double bc1 = 1.0 - pow_u64(h.b1d, t);
    const double bc2 = 1.0 - pow_u64(h.b2d, t);
    s.step = (float)(h.lr / bc1);
    s.inv_sqrt_bc2 = (float)(1.0 / sqrt(bc2));
    s.inv_ws = 1.0 / (wsum * (double)S);
    return s;
}

// One element of Adam/AdamW on the reduced, unscaled gradient g.  The
// square root and the division of the step term use the hardware's
// approximate forms (sqrt.approx.f32, a few units in the last place; the
// __fdividef intrinsic, 2 units): the step term lr*m^/(sqrt(v^)+eps) is at
// most about lr, so they add at most ~5e-10 to w per step, against the
// master tolerance of 1e-5*|w| + 1e-7; they save about 60 instructions per
// thread per tile, which is what small launches are bound by (their
// consumer warps are latency-bound).
__device__ __forceinline__ void adam1(float g, float& w, float& m, float& v, const Scal& s) {
    m = fmaf(s.b1, m, s.omb1 * g);
    v = fmaf(s.b2, v, s.omb2 * (g * g));
    float root;
    asm("sqrt.approx.f32 %0, %1;" : "=f"(root) : "f"(v));
    const float denom = fmaf(root, s.inv_sqrt_bc2, s.eps);
    w = w - fmaf(s.step, __fdividef(m, denom), s.lr_wd * w);
}

// ------------------------------------------------------------ gradient I/O

template <class G> struct Raw8;
template <> struct Raw8<float> { uint4 a, b; };
template <> struct Raw8<__nv_bfloat16> { uint4 a; };
template <> struct Raw8<__half> { uint4 a; };

template <class G> __device__ __forceinline__ Raw8<G> load8(const G* p, uint64_t i);
template <> __device__ __forceinline__ Raw8<float> load8<float>(const float* p, uint64_t i) {
    Raw8<float> r;
    r.a = __ldcs(reinterpret_cast<const uint4*>(p + i));
    r.b = __ldcs(reinterpret_cast<const uint4*>(p + i + 4));
    return r;
}
template <> __device__ __forceinline__ Raw8<__nv_bfloat16> load8<__nv_bfloat16>(const __nv_bfloat16* p, uint64_t i) {
    Raw8<__nv_bfloat16> r;
    r.a = __ldcs(reinterpret_cast<const uint4*>(p + i));
    return r;
}
template <> __device__ __forceinline__ Raw8<__half> load8<__half>(const __half* p, uint64_t i) {
    Raw8<__half> r;
    r.a = __ldcs(reinterpret_cast<const uint4*>(p + i));
    return r;
}

__device__ __forceinline__ void bf16x2(uint32_t u, float& lo, float& hi) {
    lo = __uint_as_float(u << 16);
    hi = __uint_as_float(u & 0xFFFF0000u);
}
__device__ __forceinline__ void f16x2(uint32_t u, float& lo, float& hi) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u));
    lo = f.x;
    hi = f.y;
}

__device__ __forceinline__ void unpack8(const Raw8<float>& r, float (&f)[8]) {
    f[0] = __uint_as_float(r.a.x); f[1] = __uint_as_float(r.a.y);
    f[2] = __uint_as_float(r.a.z); f[3] = __uint_as_float(r.a.w);
    f[4] = __uint_as_float(r.b.x); f[5] = __uint_as_float(r.b.y);
    f[6] = __uint_as_float(r.b.z); f[7] = __uint_as_float(r.b.w);
}
__device__ __forceinline__ void unpack8(const Raw8<__nv_bfloat16>& r, float (&f)[8]) {
    bf16x2(r.a.x, f[0], f[1]); bf16x2(r.a.y, f[2], f[3]);
    bf16x2(r.a.z, f[4], f[5]); bf16x2(r.a.w, f[6], f[7]);
}
__device__ __forceinline__ void unpack8(const Raw8<__half>& r, float (&f)[8]) {
    f16x2(r.a.x, f[0], f[1]); f16x2(r.a.y, f[2], f[3]);
    f16x2(r.a.z, f[4], f[5]); f16x2(r.a.w, f[6], f[7]);
}

// Non-finite test on raw bits: exponent field all ones.
__device__ __forceinline__ bool exp_all_ones32(uint32_t u) { return (u & 0x7F800000u) == 0x7F800000u; }
__device__ __forceinline__ bool exp_all_ones2(uint32_t u, uint32_t mask) {
    return __vcmpeq2(u & mask, mask) != 0u;
}
__device__ __forceinline__ bool bad8(const Raw8<float>& r) {
    return exp_all_ones32(r.a.x) | exp_all_ones32(r.a.y) | exp_all_ones32(r.a.z) | exp_all_ones32(r.a.w) |
           exp_all_ones32(r.b.x) | exp_all_ones32(r.b.y) | exp_all_ones32(r.b.z) | exp_all_ones32(r.b.w);
}
__device__ __forceinline__ bool bad8(const Raw8<__nv_bfloat16>& r) {
    const uint32_t k = 0x7F807F80u;
    return exp_all_ones2(r.a.x, k) | exp_all_ones2(r.a.y, k) | exp_all_ones2(r.a.z, k) | exp_all_ones2(r.a.w, k);
}
__device__ __forceinline__ bool bad8(const Raw8<__half>& r) {
    const uint32_t k = 0x7C007C00u;
    return exp_all_ones2(r.a.x, k) | exp_all_ones2(r.a.y, k) | exp_all_ones2(r.a.z, k) | exp_all_ones2(r.a.w, k);
}

template <class G> __device__ __forceinline__ float load1(const G* p, uint64_t i, bool& bad);
template <> __device__ __forceinline__ float load1<float>(const float* p, uint64_t i, bool& bad) {
    const uint32_t u = __ldcs(reinterpret_cast<const unsigned int*>(p + i));
    bad |= exp_all_ones32(u);
    return __uint_as_float(u);
}
template <> __device__ __forceinline__ float load1<__nv_bfloat16>(const __nv_bfloat16* p, uint64_t i, bool& bad) {
    const uint32_t u = __ldcs(reinterpret_cast<const unsigned short*>(p + i));
    bad |= (u & 0x7F80u) == 0x7F80u;
    return __uint_as_float(u << 16);
}
template <> __device__ __forceinline__ float load1<__half>(const __half* p, uint64_t i, bool& bad) {
    const unsigned short u = __ldcs(reinterpret_cast<const unsigned short*>(p + i));
    bad |= (u & 0x7C00u) == 0x7C00u;
    return __half2float(__ushort_as_half(u));
}

// ------------------------------------------------------------ parameter I/O

template <class Pm> __device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}
template <> __device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}
template <class Pm> __device__ __forceinline__ unsigned short cvt1(float x);
template <> __device__ __forceinline__ unsigned short cvt1<__nv_bfloat16>(float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}
template <> __device__ __forceinline__ unsigned short cvt1<__half>(float x) {
    return __half_as_ushort(__float2half_rn(x));
}

// Gradient base pointers of one tensor: registers for a compile-time rank
// count, or read through from parameter/shared memory for any R.
template <class G, int RC> struct GradPtrs {
    const G* p[RC];
    __device__ __forceinline__ explicit GradPtrs(const void* const* src) {
#pragma unroll
        for (int r = 0; r < RC; ++r) p[r] = static_cast<const G*>(src[r]);
    }
    __device__ __forceinline__ const G* operator[](int r) const { return p[r]; }
};
template <class G> struct GradPtrs<G, 0> {
    const void* const* src;
    __device__ __forceinline__ explicit GradPtrs(const void* const* s) : src(s) {}
    __device__ __forceinline__ const G* operator[](int r) const { return static_cast<const G*>(src[r]); }
};

struct StateIO {
    const float* wi;
    const float* mi;
    const float* vi;
    float* wo;
    float* mo;
    float* vo;
};

// ------------------------------------------------------------ step bodies

// One 8-element vector at flat index e (multiple of 8); le = e - tensor start.
template <class G, class Pm, int RC, bool PUSH = false>
__device__ __forceinline__ void vec_step(const StepParams& p, const Scal& s, const GradPtrs<G, RC>& gp,
                                         Pm* pp, uint64_t e, uint64_t le, const StateIO& io, bool& bad) {
    double acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.0;

    float4 w0, w1, m0, m1, v0, v1;
    if constexpr (RC > 0) {
        Raw8<G> raw[RC];
#pragma unroll
        for (int r = 0; r < RC; ++r) raw[r] = load8<G>(gp[r], le);
        w0 = __ldcs(reinterpret_cast<const float4*>(io.wi + e));
        w1 = __ldcs(reinterpret_cast<const float4*>(io.wi + e + 4));
        m0 = __ldcs(reinterpret_cast<const float4*>(io.mi + e));
        m1 = __ldcs(reinterpret_cast<const float4*>(io.mi + e + 4));
        v0 = __ldcs(reinterpret_cast<const float4*>(io.vi + e));
        v1 = __ldcs(reinterpret_cast<const float4*>(io.vi + e + 4));
#pragma unroll
        for (int r = 0; r < RC; ++r) {
            if (p.check == 1) bad |= bad8(raw[r]);
            float f[8];
            unpack8(raw[r], f);
            const double c = p.wt[r];
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] = fma(c, (double)f[k], acc[k]);
        }
    } else {
        w0 = __ldcs(reinterpret_cast<const float4*>(io.wi + e));
        w1 = __ldcs(reinterpret_cast<const float4*>(io.wi + e + 4));
        m0 = __ldcs(reinterpret_cast<const float4*>(io.mi + e));
        m1 = __ldcs(reinterpret_cast<const float4*>(io.mi + e + 4));
        v0 = __ldcs(reinterpret_cast<const float4*>(io.vi + e));
        v1 = __ldcs(reinterpret_cast<const float4*>(io.vi + e + 4));
        const int R = (int)p.R;
        for (int r0 = 0; r0 < R; r0 += 8) {
            Raw8<G> raw[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (r0 + q < R) raw[q] = load8<G>(gp[r0 + q], le);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (r0 + q < R) {
                    if (p.check == 1) bad |= bad8(raw[q]);
                    float f[8];
                    unpack8(raw[q], f);
                    const double c = p.wt[r0 + q];
#pragma unroll
                    for (int k = 0; k < 8; ++k) acc[k] = fma(c, (double)f[k], acc[k]);
                }
            }
        }
    }

    float w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    float m[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
    float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float g[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        g[k] = (float)(acc[k] * s.inv_ws);
        adam1(g[k], w[k], m[k], v[k], s);
    }
    __stcs(reinterpret_cast<float4*>(io.wo + e), make_float4(w[0], w[1], w[2], w[3]));
    __stcs(reinterpret_cast<float4*>(io.wo + e + 4), make_float4(w[4], w[5], w[6], w[7]));
    __stcs(reinterpret_cast<float4*>(io.mo + e), make_float4(m[0], m[1], m[2], m[3]));
    __stcs(reinterpret_cast<float4*>(io.mo + e + 4), make_float4(m[4], m[5], m[6], m[7]));
    __stcs(reinterpret_cast<float4*>(io.vo + e), make_float4(v[0], v[1], v[2], v[3]));
    __stcs(reinterpret_cast<float4*>(io.vo + e + 4), make_float4(v[4], v[5], v[6], v[7]));
    uint4 o;
    o.x = pack2<Pm>(w[0], w[1]);
    o.y = pack2<Pm>(w[2], w[3]);
    o.z = pack2<Pm>(w[4], w[5]);
    o.w = pack2<Pm>(w[6], w[7]);
    __stcs(reinterpret_cast<uint4*>(pp + le), o);
    if constexpr (PUSH)
        for (uint32_t i = 0; i < p.npush; ++i) __stcs(reinterpret_cast<uint4*>(static_cast<Pm*>(p.push[i]) + le), o);
    if (p.reduced != nullptr) {
        __stcs(reinterpret_cast<float4*>(p.reduced + e), make_float4(g[0], g[1], g[2], g[3]));
        __stcs(reinterpret_cast<float4*>(p.reduced + e + 4), make_float4(g[4], g[5], g[6], g[7]));
    }
}

// One element (heads, tails and tensors that cannot take the vector path).
template <class G, class Pm, int RC, bool PUSH = false>
__device__ __forceinline__ void elem_step(const StepParams& p, const Scal& s, const GradPtrs<G, RC>& gp,
                                          Pm* pp, uint64_t e, uint64_t le, const StateIO& io, bool& bad) {
    double acc = 0.0;
    const int R = RC > 0 ? RC : (int)p.R;
    for (int r = 0; r < R; ++r) {
        bool b = false;
        const float x = load1<G>(gp[r], le, b);
        if (p.check == 1) bad |= b;
        acc = fma(p.wt[r], (double)x, acc);
    }
    const float g = (float)(acc * s.inv_ws);
    float w = io.wi[e], m = io.mi[e], v = io.vi[e];
    adam1(g, w, m, v, s);
    io.wo[e] = w;
    io.mo[e] = m;
    io.vo[e] = v;
    const unsigned short h = cvt1<Pm>(w);
    reinterpret_cast<unsigned short*>(pp)[le] = h;
    if constexpr (PUSH)
        for (uint32_t i = 0; i < p.npush; ++i) static_cast<unsigned short*>(p.push[i])[le] = h;
    if (p.reduced != nullptr) p.reduced[e] = g;
}

// Flat range [a, b) of one tensor that starts at flat index toff.
template <class G, class Pm, int RC, bool PUSH = false>
__device__ __forceinline__ void run_segment(const StepParams& p, const Scal& s, const GradPtrs<G, RC>& gp,
                                            Pm* pp, uint64_t toff, uint64_t a, uint64_t b, bool vec_ok,
                                            const StateIO& io, bool& bad) {
    uint64_t va = b, vb = b;
    if (vec_ok) {
        va = (a + 7) & ~7ull;
        if (va > b) va = b;
        vb = b & ~7ull;
        if (vb < va) vb = va;
    }
    for (uint64_t e = a + threadIdx.x; e < va; e += kThreads)
        elem_step<G, Pm, RC, PUSH>(p, s, gp, pp, e, e - toff, io, bad);
    for (uint64_t e = va + (uint64_t)threadIdx.x * kVec; e < vb; e += (uint64_t)kThreads * kVec)
        vec_step<G, Pm, RC, PUSH>(p, s, gp, pp, e, e - toff, io, bad);
    for (uint64_t e = vb + threadIdx.x; e < b; e += kThreads)
        elem_step<G, Pm, RC, PUSH>(p, s, gp, pp, e, e - toff, io, bad);
}

// Index of the tensor holding flat element x (offs[j] <= x < offs[j+1]).
__device__ __forceinline__ uint32_t find_tensor(const Table& t, uint64_t x) {
    uint32_t lo = 0, hi = t.T;
    while (hi - lo > 1) {
        const uint32_t mid = (lo + hi) >> 1;
        if (t.offs[mid] <= x) lo = mid; else hi = mid;
    }
    return lo;
}

// Index of the tensor holding vector tile `tile` (tiles[j] <= tile < tiles[j+1]).
__device__ __forceinline__ uint32_t find_tensor_by_tile(const Table& t, uint64_t tile) {
    uint32_t lo = 0, hi = t.T;
    while (hi - lo > 1) {
        const uint32_t mid = (lo + hi) >> 1;
        if (t.tiles[mid] <= tile) lo = mid; else hi = mid;
    }
    return lo;
}

// The control block after one step call (one thread, once per call), from
// c0, its contents when the call started (no other code writes it during a
// call).
//   found:   an inf/NaN was seen -> skipped: S halves, t and the set stay;
//   timeout: a bounded wait of some CTA gave up, so part of the output was
//            never written -> not applied either (t and parity stay, so a
//            two-set optimizer keeps its last complete set and the restore
//            kernel re-casts the 16-bit parameters from it), S and the
//            growth count stay as they were, and device_error is set;
//   else:    applied: t += 1, the set flips (two-set mode), and with the
//            check on S doubles after growth_interval applied steps in a row.
__device__ __forceinline__ void ctrl_after_step(const zero_ctrl& c0, zero_ctrl* c, bool found, bool timeout,
                                                bool two_set, int check, uint32_t growth_interval) {
    if (timeout) {
        c->device_error = 1u;
        c->last_skipped = 1u;
    } else if (found) {
        c->loss_scale = c0.loss_scale * 0.5f;
        c->growth_tracker = 0u;
        c->skipped = c0.skipped + 1ull;
        c->last_skipped = 1u;
    } else {
        c->step = c0.step + 1ull;
        c->last_skipped = 0u;
        if (two_set) c->parity = c0.parity ^ 1u;
        if (check) {
            uint32_t gt = c0.growth_tracker + 1u;
            if (growth_interval != 0u && gt >= growth_interval) {
                c->loss_scale = c0.loss_scale * 2.0f;
                gt = 0u;
            }
            c->growth_tracker = gt;
        }
    }
}

// What a step launch knew of its control block and workspace when it
// started: the control block, and (mode 2) the inf/NaN word of the scans
// that ran before it.
struct StepStart {
    zero_ctrl ctrl;
    unsigned int found;
};

// Grid-level epilogue: the last CTA to finish updates the control block and
// clears the workspace for the next launch.  Every other access to the
// control block and the workspace in this launch happened before the
// accessing CTA's arrival, and the next launch sees the writes at the kernel
// boundary.  Only thread 0's `timed_out` is used.  `start`: the launch's
// start record in shared memory (written before the CTA's first barrier), or
// null to read the control block and the word here.
template <bool PUSH>
__device__ __forceinline__ void finish_step(const StepParams& p, bool bad, bool timed_out = false,
                                            const StepStart* start = nullptr) {
    // PUSH: no fence for the stores into other GPUs' replicas.  Nothing in
    // the kernel signals a peer; the peers read their replicas only after
    // this kernel has completed (its stores are then performed) and a
    // collective barrier that follows it on the stream.
    const int any = __syncthreads_or(bad ? 1 : 0);
    if (threadIdx.x == 0) {
        Workspace* ws = p.ws;
        const unsigned long long mine = Arrival::mine(any != 0, timed_out);
        const unsigned long long all = atomicAdd(&ws->arrive, mine) + mine;
        if (Arrival::count(all) == gridDim.x) {
            StepStart s0;
            if (start != nullptr) {
                s0 = *start;
            } else {
                s0.ctrl = *p.ctrl;
                s0.found = ws->found;
            }
            const bool found = p.check == 1 ? Arrival::any_found(all) : (p.check == 2 && s0.found != 0u);
            ctrl_after_step(s0.ctrl, p.ctrl, found, Arrival::any_timeout(all), p.two_set != 0, p.check,
                            p.growth_interval);
            ws->found = 0u;
            ws->next_tile = 0u;
            ws->arrive = 0ull;
        }
    }
}

// Two 256-thread CTAs per SM: at most 128 registers a thread.  Without the
// bound the list instances with fp32 gradients took 131 (one CTA per SM);
// with it they spill 16 bytes, and every other instance fits without a spill.
template <class G, class Pm, int RC, bool LIST, bool PUSH = false>
__global__ void __launch_bounds__(kThreads, 2) step_kernel(const __grid_constant__ StepParams p) {
    __shared__ const void* s_gp[LIST ? ZERO_MAX_RANKS : 1];
    grid_dependency_wait();
    allow_dependents();
    const zero_ctrl* c = p.ctrl;
    const uint32_t par = p.two_set ? c->parity : 0u;
    const uint32_t out = par ^ (uint32_t)p.two_set;
    const StateIO io{p.w[par], p.m[par], p.v[par], p.w[out], p.m[out], p.v[out]};
    bool skip = false;
    if (p.check == 2) skip = *reinterpret_cast<volatile const unsigned*>(&p.ws->found) != 0u;
    const Scal s = make_scal(p.h, c->step + 1ull, c->loss_scale, p.wsum);

    uint64_t a = p.base + (uint64_t)blockIdx.x * p.chunk;
    uint64_t b = a + p.chunk;
    if (a < p.lo) a = p.lo;
    if (b > p.hi) b = p.hi;
    bool bad = false;
    if (!skip && a < b) {
        if constexpr (!LIST) {
            const GradPtrs<G, RC> gp(&p.grads[0]);
            run_segment<G, Pm, RC, PUSH>(p, s, gp, static_cast<Pm*>(p.params16), 0ull, a, b, true, io, bad);
        } else {
            uint32_t j = find_tensor(p.tab, a);
            uint64_t x = a;
            while (x < b) {
                const uint64_t t0 = p.tab.offs[j], t1 = p.tab.offs[j + 1];
                const uint64_t sb = t1 < b ? t1 : b;
                if (x < sb) {
                    __syncthreads();
                    for (uint32_t r = threadIdx.x; r < p.R; r += kThreads)
                        s_gp[r] = p.tab.grads[(uint64_t)j * p.R + r];
                    __syncthreads();
                    const GradPtrs<G, RC> gp(s_gp);
                    run_segment<G, Pm, RC>(p, s, gp, static_cast<Pm*>(p.tab.params[j]), t0, x, sb,
                                           (p.tab.flags[j] & 1u) != 0u, io, bad);
                }
                x = sb;
                ++j;
            }
        }
    }
    finish_step<PUSH>(p, bad);
}

// ------------------------------------------------------------ overflow scan

template <class G>
__device__ __forceinline__ void scan_range(const G* g, uint64_t a, uint64_t b, bool vec_ok, bool& bad) {
    uint64_t va = b, vb = b;
    if (vec_ok) {
        va = (a + 7) & ~7ull;
        if (va > b) va = b;
        vb = b & ~7ull;
        if (vb < va) vb = va;
    }
    for (uint64_t e = a + threadIdx.x; e < va; e += kThreads) (void)load1<G>(g, e, bad);
    // four independent 16-byte loads in flight per thread per iteration
    constexpr uint64_t kStride = (uint64_t)kThreads * kVec;
    uint64_t e = va + (uint64_t)threadIdx.x * kVec;
    for (; e + 3 * kStride < vb; e += 4 * kStride) {
        const Raw8<G> r0 = load8<G>(g, e), r1 = load8<G>(g, e + kStride);
        const Raw8<G> r2 = load8<G>(g, e + 2 * kStride), r3 = load8<G>(g, e + 3 * kStride);
        bad |= bad8(r0) | bad8(r1) | bad8(r2) | bad8(r3);
    }
    for (; e < vb; e += kStride) bad |= bad8(load8<G>(g, e));
    for (uint64_t x = vb + threadIdx.x; x < b; x += kThreads) (void)load1<G>(g, x, bad);
}

// Sets ws.found if any gradient of any rank in [lo, hi) is inf or NaN.
template <class G, bool LIST>
__global__ void __launch_bounds__(kThreads) scan_kernel(const __grid_constant__ StepParams p) {
    grid_dependency_wait();
    allow_dependents();
    uint64_t a = p.base + (uint64_t)blockIdx.x * p.chunk;
    uint64_t b = a + p.chunk;
    if (a < p.lo) a = p.lo;
    if (b > p.hi) b = p.hi;
    bool bad = false;
    if (a < b) {
        if constexpr (!LIST) {
            for (uint32_t r = 0; r < p.R; ++r) scan_range<G>(static_cast<const G*>(p.grads[r]), a, b, true, bad);
        } else {
            uint32_t j = find_tensor(p.tab, a);
            uint64_t x = a;
            while (x < b) {
                const uint64_t t0 = p.tab.offs[j], t1 = p.tab.offs[j + 1];
                const uint64_t sb = t1 < b ? t1 : b;
                if (x < sb) {
                    const bool vec_ok = (p.tab.flags[j] & 1u) != 0u;
                    for (uint32_t r = 0; r < p.R; ++r)
                        scan_range<G>(static_cast<const G*>(p.tab.grads[(uint64_t)j * p.R + r]), x - t0, sb - t0,
                                      vec_ok, bad);
                }
                x = sb;
                ++j;
            }
        }
    }
    if (__syncthreads_or(bad ? 1 : 0) && threadIdx.x == 0) atomicOr(&p.ws->found, 1u);
}

// ------------------------------------------------------------ 16-bit cast

template <class Pm>
__device__ __forceinline__ void cast_range(const float* w, Pm* pp, uint64_t toff, uint64_t a, uint64_t b,
                                           bool vec_ok) {
    uint64_t va = b, vb = b;
    if (vec_ok) {
        va = (a + 7) & ~7ull;
        if (va > b) va = b;
        vb = b & ~7ull;
        if (vb < va) vb = va;
    }
    unsigned short* po = reinterpret_cast<unsigned short*>(pp);
    for (uint64_t e = a + threadIdx.x; e < va; e += kThreads) po[e - toff] = cvt1<Pm>(w[e]);
    for (uint64_t e = va + (uint64_t)threadIdx.x * kVec; e < vb; e += (uint64_t)kThreads * kVec) {
        const float4 x = __ldcs(reinterpret_cast<const float4*>(w + e));
        const float4 y = __ldcs(reinterpret_cast<const float4*>(w + e + 4));
        uint4 o;
        o.x = pack2<Pm>(x.x, x.y);
        o.y = pack2<Pm>(x.z, x.w);
        o.z = pack2<Pm>(y.x, y.y);
        o.w = pack2<Pm>(y.z, y.w);
        __stcs(reinterpret_cast<uint4*>(po + (e - toff)), o);
    }
    for (uint64_t e = vb + threadIdx.x; e < b; e += kThreads) po[e - toff] = cvt1<Pm>(w[e]);
}

template <class Pm, bool LIST>
__global__ void __launch_bounds__(kThreads) gather_kernel(const __grid_constant__ GatherParams p) {
    grid_dependency_wait();
    allow_dependents();
    if (p.only_if_skipped && p.ctrl->last_skipped == 0u) return;
    const float* w = p.ctrl != nullptr ? p.w[p.ctrl->parity & 1u] : p.w[0];
    uint64_t a = p.base + (uint64_t)blockIdx.x * p.chunk;
    uint64_t b = a + p.chunk;
    if (a < p.lo) a = p.lo;
    if (b > p.hi) b = p.hi;
    if (a >= b) return;
    if constexpr (!LIST) {
        cast_range<Pm>(w, static_cast<Pm*>(p.params16), 0ull, a, b, true);
    } else {
        uint32_t j = find_tensor(p.tab, a);
        uint64_t x = a;
        while (x < b) {
            const uint64_t t0 = p.tab.offs[j], t1 = p.tab.offs[j + 1];
            const uint64_t sb = t1 < b ? t1 : b;
            if (x < sb)
                cast_range<Pm>(w, static_cast<Pm*>(p.tab.params[j]), t0, x, sb, (p.tab.flags[j] & 1u) != 0u);
            x = sb;
            ++j;
        }
    }
}

// ------------------------------------------------------------ ZeRO-3 gather

// Full padded views of tensors from their R rank shards.  The table is a
// gather list: tensor j's element count is R * s_j (its padded full size),
// params[j] is the full view buffer and grads[j*R + r] rank r's shard of s_j
// elements, so full_j[r*s_j + k] = shard_{r,j}[k].  Launch space: the padded
// concatenation [0, sum_j R*s_j).
struct Z3Params {
    Table tab;
    uint64_t lo, hi;  // the launch covers [lo, hi) of the padded concatenation (lo = 0)
    uint32_t R;
};

// Elements [a, b) of the padded concatenation.
__device__ __forceinline__ void z3_copy_range(const Z3Params& p, uint64_t a, uint64_t b) {
    uint32_t j = find_tensor(p.tab, a);
    uint64_t x = a;
    while (x < b) {
        const uint64_t t0 = p.tab.offs[j], t1 = p.tab.offs[j + 1];
        const uint64_t s = (t1 - t0) / p.R;
        unsigned short* full = static_cast<unsigned short*>(p.tab.params[j]);
        while (x < b && x < t1) {
            const uint64_t pos = x - t0;
            const uint64_t r = pos / s;
            const uint64_t k0 = pos - r * s;
            uint64_t end = t0 + (r + 1) * s;
            if (end > b) end = b;
            const unsigned short* src = static_cast<const unsigned short*>(p.tab.grads[(uint64_t)j * p.R + r]);
            const uint64_t n = end - x;
            const bool vec = (p.tab.flags[j] & 1u) != 0u && (s & 7ull) == 0 && (k0 & 7ull) == 0;
            if (vec) {
                const uint64_t nv = n >> 3;
                const uint4* in = reinterpret_cast<const uint4*>(src + k0);
                uint4* out = reinterpret_cast<uint4*>(full + pos);
                uint64_t v = threadIdx.x;
                for (; v + 3 * kThreads < nv; v += 4 * kThreads) {  // four copies in flight
                    const uint4 x0 = in[v], x1 = in[v + kThreads];
                    const uint4 x2 = in[v + 2 * kThreads], x3 = in[v + 3 * kThreads];
                    out[v] = x0;
                    out[v + kThreads] = x1;
                    out[v + 2 * kThreads] = x2;
                    out[v + 3 * kThreads] = x3;
                }
                for (; v < nv; v += kThreads) out[v] = in[v];
                for (uint64_t e = (nv << 3) + threadIdx.x; e < n; e += kThreads) full[pos + e] = src[k0 + e];
            } else {
                for (uint64_t e = threadIdx.x; e < n; e += kThreads) full[pos + e] = src[k0 + e];
            }
            x = end;
        }
        ++j;
    }
}

// Chunks of kZ3Chunk elements are handed out dynamically: CTA b starts on
// chunk b, then claims chunks from gridDim.x on through the table's scratch
// counter; the last CTA to finish clears the counters for the next call.
constexpr uint64_t kZ3Chunk = 32768;

template <class Pm>
__global__ void __launch_bounds__(kThreads) z3_gather_kernel(const __grid_constant__ Z3Params p) {
    __shared__ uint64_t s_next;
    grid_dependency_wait();
    allow_dependents();
    unsigned int* sc = p.tab.scratch;
    const uint64_t nchunks = (p.hi + kZ3Chunk - 1) / kZ3Chunk;
    uint64_t c = blockIdx.x;
    while (c < nchunks) {
        if (threadIdx.x == 0) s_next = (uint64_t)gridDim.x + atomicAdd(&sc[0], 1u);
        const uint64_t a = c * kZ3Chunk;
        z3_copy_range(p, a, a + kZ3Chunk < p.hi ? a + kZ3Chunk : p.hi);
        __syncthreads();
        c = s_next;
        __syncthreads();
    }
    if (threadIdx.x == 0 && atomicAdd(&sc[1], 1u) == gridDim.x - 1) {
        sc[0] = 0u;
        sc[1] = 0u;
    }
}

// ------------------------------------------------------------ micro-step accumulation

struct AccumParams {
    const void* grads[ZERO_MAX_RANKS];  // rank r's micro-batch gradient [P]
    double wt[ZERO_MAX_RANKS];          // rank weights
    double inv_wsum;                    // 1 / sum(w)
    double scale;                       // multiplies the reduced gradient
    float* acc;                         // fp32 accumulation array [P]
    Workspace* ws;                      // bulk kernel: tile counter and error flag
    zero_ctrl* ctrl;                    // bulk kernel: receives device_error
    uint64_t lo, hi, base, chunk;
    uint32_t R;
    int32_t first;                      // 1: acc starts from zero
};

// acc = (first ? 0 : acc) + scale * (sum_r w_r g_r) / sum(w), float64, one
// rounding, for U vectors at e, e + stride, ...: every load of the U vectors
// is issued before any arithmetic or store.  (U = 2 measured slower than
// U = 1 on a B200: the extra registers cost resident CTAs.)
template <class G, int RC, int U>
__device__ __forceinline__ void accum_vec(const AccumParams& p, const GradPtrs<G, RC>& gp, uint64_t e,
                                          uint64_t stride) {
    float4 a0[U], a1[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        a0[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        a1[u] = a0[u];
    }
    if (!p.first) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            a0[u] = __ldcs(reinterpret_cast<const float4*>(p.acc + e + u * stride));
            a1[u] = __ldcs(reinterpret_cast<const float4*>(p.acc + e + u * stride + 4));
        }
    }
    double acc[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[u][k] = 0.0;
    if constexpr (RC > 0) {
        Raw8<G> raw[U][RC];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int r = 0; r < RC; ++r) raw[u][r] = load8<G>(gp[r], e + u * stride);
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int r = 0; r < RC; ++r) {
                float f[8];
                unpack8(raw[u][r], f);
#pragma unroll
                for (int k = 0; k < 8; ++k) acc[u][k] = fma(p.wt[r], (double)f[k], acc[u][k]);
            }
    } else {
        for (int r = 0; r < (int)p.R; ++r) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                float f[8];
                unpack8(load8<G>(gp[r], e + u * stride), f);
#pragma unroll
                for (int k = 0; k < 8; ++k) acc[u][k] = fma(p.wt[r], (double)f[k], acc[u][k]);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const float prev[8] = {a0[u].x, a0[u].y, a0[u].z, a0[u].w, a1[u].x, a1[u].y, a1[u].z, a1[u].w};
        float out[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) out[k] = (float)((double)prev[k] + p.scale * (acc[u][k] * p.inv_wsum));
        __stcs(reinterpret_cast<float4*>(p.acc + e + u * stride), make_float4(out[0], out[1], out[2], out[3]));
        __stcs(reinterpret_cast<float4*>(p.acc + e + u * stride + 4), make_float4(out[4], out[5], out[6], out[7]));
    }
}

template <class G, int RC>
__device__ __forceinline__ void accum_elem(const AccumParams& p, const GradPtrs<G, RC>& gp, uint64_t e) {
    double acc = 0.0;
    const int R = RC > 0 ? RC : (int)p.R;
    for (int r = 0; r < R; ++r) {
        bool b = false;
        acc = fma(p.wt[r], (double)load1<G>(gp[r], e, b), acc);
    }
    const double prev = p.first ? 0.0 : (double)p.acc[e];
    p.acc[e] = (float)(prev + p.scale * (acc * p.inv_wsum));
}

template <class G, int RC>
__global__ void __launch_bounds__(kThreads) accum_kernel(const __grid_constant__ AccumParams p) {
    grid_dependency_wait();
    allow_dependents();
    uint64_t a = p.base + (uint64_t)blockIdx.x * p.chunk;
    uint64_t b = a + p.chunk;
    if (a < p.lo) a = p.lo;
    if (b > p.hi) b = p.hi;
    if (a >= b) return;
    const GradPtrs<G, RC> gp(&p.grads[0]);
    uint64_t va = (a + 7) & ~7ull, vb = b & ~7ull;
    if (va > b) va = b;
    if (vb < va) vb = va;
    for (uint64_t e = a + threadIdx.x; e < va; e += kThreads) accum_elem<G, RC>(p, gp, e);
    constexpr uint64_t kStride = (uint64_t)kThreads * kVec;
    uint64_t e = va + (uint64_t)threadIdx.x * kVec;
    for (; e < vb; e += kStride) accum_vec<G, RC, 1>(p, gp, e, kStride);
    for (uint64_t x = vb + threadIdx.x; x < b; x += kThreads) accum_elem<G, RC>(p, gp, x);
}

// ------------------------------------------------------------ control block

__global__ void ctrl_set_kernel(zero_ctrl* c, zero_ctrl value) { *c = value; }

}  // namespace zadam
