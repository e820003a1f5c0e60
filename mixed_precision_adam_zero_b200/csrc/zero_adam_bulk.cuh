// zero_adam_bulk.cuh -- the flat step with shared-memory staging by 1-D bulk
// asynchronous copies (the TMA engine's cp.async.bulk, no tensor map, no
// multicast).
//
// Why: the register-staged kernel holds each thread's loads in registers, so
// the bytes a SM keeps in flight are bounded by registers x resident warps.
// Here one thread per CTA streams tiles of every input array (R gradient
// slices and the master, m and v slices) into a ring of shared-memory
// stages, several tiles ahead of the 256 threads that consume them; the bytes
// in flight are set by the ring size (about 170 KB per SM), not by registers.
//
// Per tile of n <= kTile elements (n a multiple of 8, every source 16-byte
// aligned): stage = [R gradient slices][w][m][v], each slice contiguous.
// Thread t consumes two groups of 4 elements, [4t, 4t+4) and
// [n/2 + 4t, n/2 + 4t + 4), so every shared-memory read is conflict-free and
// every global store is coalesced.  The arithmetic per element is exactly
// that of step_kernel (adam1 and the float64 rank reduction), so the two
// kernels give bitwise identical results.
//
// Waits on the stage barriers are bounded (by %globaltimer): a wait that
// gives up records an error in the workspace, the CTA stops consuming, waits
// (again bounded) for the copies it issued, and finishes normally.
#pragma once

#include "zero_adam_kernels.cuh"

namespace zadam {

constexpr int kTile = 2048;                     // elements per stage (256 threads x 8)
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
constexpr int kBarBytes = 128;                  // barrier block at the start of shared memory

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Global -> shared bulk copy completing on `bar` (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0u;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of `bar`; false if it did not complete in time.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1; it < (1u << 30); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0u && global_ns() - t0 > kWaitLimitNs) return false;
    }
    return false;
}

template <class G> struct Raw4;
template <> struct Raw4<float> { uint4 a; };
template <> struct Raw4<__nv_bfloat16> { uint2 a; };
template <> struct Raw4<__half> { uint2 a; };

template <class G> __device__ __forceinline__ Raw4<G> lds4(const unsigned char* p);
template <> __device__ __forceinline__ Raw4<float> lds4<float>(const unsigned char* p) {
    return Raw4<float>{*reinterpret_cast<const uint4*>(p)};
}
template <> __device__ __forceinline__ Raw4<__nv_bfloat16> lds4<__nv_bfloat16>(const unsigned char* p) {
    return Raw4<__nv_bfloat16>{*reinterpret_cast<const uint2*>(p)};
}
template <> __device__ __forceinline__ Raw4<__half> lds4<__half>(const unsigned char* p) {
    return Raw4<__half>{*reinterpret_cast<const uint2*>(p)};
}

__device__ __forceinline__ void unpack4(const Raw4<float>& r, float (&f)[4]) {
    f[0] = __uint_as_float(r.a.x); f[1] = __uint_as_float(r.a.y);
    f[2] = __uint_as_float(r.a.z); f[3] = __uint_as_float(r.a.w);
}
__device__ __forceinline__ void unpack4(const Raw4<__nv_bfloat16>& r, float (&f)[4]) {
    bf16x2(r.a.x, f[0], f[1]); bf16x2(r.a.y, f[2], f[3]);
}
__device__ __forceinline__ void unpack4(const Raw4<__half>& r, float (&f)[4]) {
    f16x2(r.a.x, f[0], f[1]); f16x2(r.a.y, f[2], f[3]);
}
__device__ __forceinline__ bool bad4(const Raw4<float>& r) {
    return exp_all_ones32(r.a.x) | exp_all_ones32(r.a.y) | exp_all_ones32(r.a.z) | exp_all_ones32(r.a.w);
}
__device__ __forceinline__ bool bad4(const Raw4<__nv_bfloat16>& r) {
    return exp_all_ones2(r.a.x, 0x7F807F80u) | exp_all_ones2(r.a.y, 0x7F807F80u);
}
__device__ __forceinline__ bool bad4(const Raw4<__half>& r) {
    return exp_all_ones2(r.a.x, 0x7C007C00u) | exp_all_ones2(r.a.y, 0x7C007C00u);
}

// Bytes of one stage and the number of stages for R ranks of gradient type G.
template <class G, int RC>
struct BulkShape {
    static constexpr uint32_t kGradSlice = kTile * sizeof(G);
    static constexpr uint32_t kStage = RC * kGradSlice + 3u * kTile * 4u;
    static constexpr int kBudget = 200 * 1024;
    static constexpr int kStages = (kBudget / kStage) > 6 ? 6 : (kBudget / kStage);
    static constexpr uint32_t kSmem = kBarBytes + kStages * kStage;
    static_assert(kStages >= 2, "stage too large for the ring");
};

// Four consecutive elements at flat index e (tile-relative offset q in the
// stage), reduced, updated and stored.
template <class G, class Pm, int RC>
__device__ __forceinline__ void bulk_group(const StepParams& p, const Scal& s, const unsigned char* stage,
                                           uint32_t q, uint64_t e, float* wo, float* mo, float* vo, Pm* pp,
                                           bool& bad) {
    using Sh = BulkShape<G, RC>;
    Raw4<G> raw[RC];
#pragma unroll
    for (int r = 0; r < RC; ++r) raw[r] = lds4<G>(stage + r * Sh::kGradSlice + q * sizeof(G));
    const unsigned char* st = stage + RC * Sh::kGradSlice;
    const float4 w4 = *reinterpret_cast<const float4*>(st + q * 4u);
    const float4 m4 = *reinterpret_cast<const float4*>(st + kTile * 4u + q * 4u);
    const float4 v4 = *reinterpret_cast<const float4*>(st + 2u * kTile * 4u + q * 4u);
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int r = 0; r < RC; ++r) {
        if (p.check == 1) bad |= bad4(raw[r]);
        float f[4];
        unpack4(raw[r], f);
        const double c = p.wt[r];
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = fma(c, (double)f[k], acc[k]);
    }
    float w[4] = {w4.x, w4.y, w4.z, w4.w};
    float m[4] = {m4.x, m4.y, m4.z, m4.w};
    float v[4] = {v4.x, v4.y, v4.z, v4.w};
    float g[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        g[k] = (float)(acc[k] * s.inv_ws);
        adam1(g[k], w[k], m[k], v[k], s);
    }
    __stcs(reinterpret_cast<float4*>(wo + e), make_float4(w[0], w[1], w[2], w[3]));
    __stcs(reinterpret_cast<float4*>(mo + e), make_float4(m[0], m[1], m[2], m[3]));
    __stcs(reinterpret_cast<float4*>(vo + e), make_float4(v[0], v[1], v[2], v[3]));
    uint2 o;
    o.x = pack2<Pm>(w[0], w[1]);
    o.y = pack2<Pm>(w[2], w[3]);
    __stcs(reinterpret_cast<uint2*>(pp + e), o);
    if (p.reduced != nullptr) __stcs(reinterpret_cast<float4*>(p.reduced + e), make_float4(g[0], g[1], g[2], g[3]));
}

// Issue the copies of tile k (flat elements [e0, e0+n)) into `stage`.
template <class G, int RC>
__device__ __forceinline__ void bulk_issue(const StepParams& p, const StateIO& io, unsigned char* stage,
                                           uint64_t* bar, uint64_t e0, uint32_t n) {
    using Sh = BulkShape<G, RC>;
    const uint32_t gb = n * (uint32_t)sizeof(G), sb = n * 4u;
    mbar_expect_tx(bar, RC * gb + 3u * sb);
#pragma unroll
    for (int r = 0; r < RC; ++r)
        bulk_g2s(stage + r * Sh::kGradSlice, static_cast<const G*>(p.grads[r]) + e0, gb, bar);
    unsigned char* st = stage + RC * Sh::kGradSlice;
    bulk_g2s(st, io.wi + e0, sb, bar);
    bulk_g2s(st + kTile * 4u, io.mi + e0, sb, bar);
    bulk_g2s(st + 2u * kTile * 4u, io.vi + e0, sb, bar);
}

template <class G, class Pm, int RC>
__global__ void __launch_bounds__(kThreads, 1) step_bulk_kernel(const __grid_constant__ StepParams p) {
    using Sh = BulkShape<G, RC>;
    constexpr int D = Sh::kStages;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    unsigned char* ring = smem + kBarBytes;

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
    bool failed = false;
    if (!skip && a < b) {
        const GradPtrs<G, RC> gp(&p.grads[0]);
        Pm* pp = static_cast<Pm*>(p.params16);
        // ragged head and tail: the register path, same arithmetic
        uint64_t va = (a + 7) & ~7ull, vb = b & ~7ull;
        if (va > b) va = b;
        if (vb < va) vb = va;
        for (uint64_t e = a + threadIdx.x; e < va; e += kThreads) elem_step<G, Pm, RC>(p, s, gp, pp, e, e, io, bad);
        for (uint64_t e = vb + threadIdx.x; e < b; e += kThreads) elem_step<G, Pm, RC>(p, s, gp, pp, e, e, io, bad);

        const uint64_t nt = (vb - va + kTile - 1) / kTile;
        if (threadIdx.x == 0) {
            for (int i = 0; i < D; ++i) mbar_init(&bars[i], 1u);
            fence_mbar_init();
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            for (uint64_t k = 0; k < nt && k < (uint64_t)D; ++k) {
                const uint64_t e0 = va + k * kTile;
                const uint32_t n = (uint32_t)((vb - e0) < (uint64_t)kTile ? (vb - e0) : (uint64_t)kTile);
                bulk_issue<G, RC>(p, io, ring + k * Sh::kStage, &bars[k], e0, n);
            }
        }
        uint64_t k = 0;
        for (; k < nt; ++k) {
            const int st = (int)(k % D);
            const uint32_t phase = (uint32_t)((k / D) & 1u);
            const bool ok = mbar_wait_bounded(&bars[st], phase);
            const uint64_t e0 = va + k * kTile;
            const uint32_t n = (uint32_t)((vb - e0) < (uint64_t)kTile ? (vb - e0) : (uint64_t)kTile);
            const uint32_t half = n >> 1;  // a multiple of 4
            const uint32_t q = 4u * threadIdx.x;
            if (ok && q < half) {
                const unsigned char* stage = ring + st * Sh::kStage;
                bulk_group<G, Pm, RC>(p, s, stage, q, e0 + q, io.wo, io.mo, io.vo, pp, bad);
                bulk_group<G, Pm, RC>(p, s, stage, half + q, e0 + half + q, io.wo, io.mo, io.vo, pp, bad);
            }
            if (!__syncthreads_and(ok ? 1 : 0)) {
                failed = true;
                break;
            }
            if (threadIdx.x == 0 && k + D < nt) {
                const uint64_t e1 = va + (k + D) * kTile;
                const uint32_t n1 = (uint32_t)((vb - e1) < (uint64_t)kTile ? (vb - e1) : (uint64_t)kTile);
                bulk_issue<G, RC>(p, io, ring + st * Sh::kStage, &bars[st], e1, n1);
            }
        }
        if (failed && threadIdx.x == 0) {
            // Do not leave while copies this CTA issued may still land in its
            // shared memory: wait (bounded) for every issued, unconsumed tile.
            atomicOr(&p.ws->error, 1u);
            const uint64_t issued = nt < k + D ? nt : k + D;
            for (uint64_t j = k; j < issued; ++j)
                (void)mbar_wait_bounded(&bars[j % D], (uint32_t)((j / D) & 1u));
        }
        __syncthreads();
    }
    finish_step(p, bad);
}

}  // namespace zadam
