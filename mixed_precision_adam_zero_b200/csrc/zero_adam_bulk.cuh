// zero_adam_bulk.cuh -- the step (flat buffer or tensor list) and the
// micro-step accumulation with shared-memory staging by 1-D bulk
// asynchronous copies (the TMA engine's cp.async.bulk, no tensor map, no
// multicast).
//
// Why: the register-staged kernels hold each thread's loads in registers, so
// the bytes a SM keeps in flight are bounded by registers x resident warps.
// Here one producer thread per CTA streams tiles of every input array (R
// gradient slices and the master, m and v slices) into a ring of
// shared-memory stages, several tiles ahead of the consumer warps; the bytes
// in flight are set by the ring size (up to 200 KB per SM), not by
// registers.
//
// Per tile of n <= kTile elements (n a multiple of 8, every source 16-byte
// aligned): stage = [R gradient slices][w][m][v], each slice contiguous.
// Consumer thread t handles the 4-element groups [4t, 4t+4), [4t + 4C, ...)
// (C consumer threads), so every shared-memory read is conflict-free and
// every global store is coalesced.  The arithmetic per element is exactly
// that of step_kernel (adam1 and the float64 rank reduction), so the two
// kernels give bitwise identical results.
//
// Instances are compiled for R = 1, 2, 4, 8 (and 16 with 16-bit gradients):
// their R loads are unrolled into registers.  Any other R takes the chunked
// kernels at the end of the file, which pass each tile through the ring in
// stages of eight ranks.
//
// Waits on the stage barriers are bounded (by %globaltimer): a wait that
// gives up marks the CTA as timed out, the CTA stops consuming, waits (again
// bounded) for the copies it issued, and finishes normally; the grid's
// epilogue then sets zero_ctrl.device_error.
#pragma once

#include "zero_adam_kernels.cuh"

namespace zadam {

// Consumer threads per CTA: 16 warps, one 4-element group per thread per
// 2048-element tile.  Against 8 warps (two groups per thread) on a B200:
// equal at 16.8M and 64M parameters, +13 % at 4.2M, and +5 to +10 % on the
// 1-3B workloads that run under the power cap at lower SM clocks, where
// more warps hide the longer per-tile arithmetic.
constexpr int kConsumers = 512;
constexpr int kBulkThreads = kConsumers + 32;     // plus one producer warp
constexpr int kTile = 2048;                     // elements per stage
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
constexpr int kBarBytes = 384;                  // full and empty stage barriers (at most 2 x 8 x 8 B), padded
constexpr int kGpBytes = 640;                   // gradient bases of a tensor (scalar pass of a list);
                                                // pads the header so the stage ring starts 1024-B aligned

// Set to 1 by any thread of the CTA whose bounded wait gave up; thread 0
// clears it before the CTA's first wait and folds it into the arrival.
static __shared__ unsigned int s_timed_out;

__device__ __forceinline__ void note_timeout() { s_timed_out = 1u; }

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

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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
    static constexpr int kStages = (kBudget / kStage) > 8 ? 8 : (kBudget / kStage);
    static constexpr uint32_t kSmem = kBarBytes + kGpBytes + kStages * kStage;
    static_assert(kStages >= 2, "stage too large for the ring");
    static_assert((kBarBytes + kGpBytes) % 1024 == 0, "stage ring must start 1024-byte aligned");
    static_assert(kStage % 1024 == 0, "stages must stay 1024-byte aligned");
};

// Four consecutive elements at flat index e (tile-relative offset q in the
// stage, index le within the tensor's 16-bit parameters), reduced, updated
// and stored.
template <class G, class Pm, int RC, bool PUSH = false>
__device__ __forceinline__ void bulk_group(const StepParams& p, const Scal& s, const unsigned char* stage,
                                           uint32_t q, uint64_t e, uint64_t le, float* wo, float* mo, float* vo,
                                           Pm* pp, bool& bad) {
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
    __stcs(reinterpret_cast<uint2*>(pp + le), o);
    if constexpr (PUSH)
        for (uint32_t i = 0; i < p.npush; ++i) __stcs(reinterpret_cast<uint2*>(static_cast<Pm*>(p.push[i]) + le), o);
    if (p.reduced != nullptr) __stcs(reinterpret_cast<float4*>(p.reduced + e), make_float4(g[0], g[1], g[2], g[3]));
}

// Issue the copies of one tile into `stage` (gradient bases already offset
// to the tile's tensor; `le0` = tile start within the tensor).
template <class G, int RC>
__device__ __forceinline__ void bulk_issue(const StateIO& io, const G* const (&gb)[RC], unsigned char* stage,
                                           uint64_t* bar, uint64_t e0, uint64_t le0, uint32_t n) {
    using Sh = BulkShape<G, RC>;
    const uint32_t gbytes = n * (uint32_t)sizeof(G), sbytes = n * 4u;
    mbar_expect_tx(bar, RC * gbytes + 3u * sbytes);
#pragma unroll
    for (int r = 0; r < RC; ++r) bulk_g2s(stage + r * Sh::kGradSlice, gb[r] + le0, gbytes, bar);
    unsigned char* st = stage + RC * Sh::kGradSlice;
    bulk_g2s(st, io.wi + e0, sbytes, bar);
    bulk_g2s(st + kTile * 4u, io.mi + e0, sbytes, bar);
    bulk_g2s(st + 2u * kTile * 4u, io.vi + e0, sbytes, bar);
}

// The walk over a CTA's vector tiles.  Flat: one tensor [0, P).  List:
// tensors in order; a tensor's vector body is its part of [a, b) rounded
// inward to multiples of 8, and only tensors flagged for the vector path
// have one.  Everything outside the bodies is left to the scalar pass, which
// walks the same segments.  Every thread runs the walk in registers (the
// tile sequence is a pure function of the range and the table); the issuing
// thread runs a second copy D tiles ahead that also loads each tensor's
// gradient bases.
template <class G, int RC, bool LIST, bool GRADS>
struct TileWalk {
    uint64_t x, bb;  // next tile start and end of the current vector body
    uint64_t segx;   // list: flat start of the next segment to examine
    uint64_t b;      // end of the CTA's range
    uint32_t j;      // list: next tensor to examine
    const G* gb[GRADS ? RC : 1];
    void* params;
    uint64_t toff;

    __device__ __forceinline__ void start(const StepParams& p, uint64_t a, uint64_t b_) {
        b = b_;
        toff = 0;
        params = p.params16;
        if constexpr (!LIST) {
            x = (a + 7) & ~7ull;
            bb = b & ~7ull;
            if constexpr (GRADS) {
#pragma unroll
                for (int r = 0; r < RC; ++r) gb[r] = static_cast<const G*>(p.grads[r]);
            }
        } else {
            x = bb = 0;
            segx = a;
            j = find_tensor(p.tab, a);
        }
    }

    // List: move to the next segment that has a vector body; the table is
    // read only here, once per tensor.
    __device__ __forceinline__ bool next_body(const StepParams& p) {
        while (segx < b) {
            const uint64_t t0 = p.tab.offs[j], t1 = p.tab.offs[j + 1];
            const uint64_t sb = t1 < b ? t1 : b;
            const uint32_t jt = j++;
            if (segx >= sb) continue;            // empty tensor
            const uint64_t ba = (segx + 7) & ~7ull, be = sb & ~7ull;
            segx = sb;
            if ((p.tab.flags[jt] & 1u) == 0u || ba >= be) continue;  // scalar pass only
            x = ba;
            bb = be;
            toff = t0;
            params = p.tab.params[jt];
            if constexpr (GRADS) {
#pragma unroll
                for (int r = 0; r < RC; ++r) gb[r] = static_cast<const G*>(p.tab.grads[(uint64_t)jt * RC + r]);
            }
            return true;
        }
        return false;
    }

    // Next tile: flat start e0 and length n (a multiple of 8); false at the end.
    __device__ __forceinline__ bool next(const StepParams& p, uint64_t& e0, uint32_t& n) {
        if (x >= bb) {
            if constexpr (!LIST) return false;
            else if (!next_body(p)) return false;
        }
        e0 = x;
        n = (uint32_t)((bb - x) < (uint64_t)kTile ? (bb - x) : (uint64_t)kTile);
        x += n;
        return true;
    }
};

// Scalar pass over everything the tile walk leaves out.
template <class G, class Pm, int RC, bool LIST, bool PUSH = false>
__device__ __forceinline__ void bulk_scalar_pass(const StepParams& p, const Scal& s, uint64_t a, uint64_t b,
                                                 const StateIO& io, bool& bad, const void** s_gp) {
    if constexpr (!LIST) {
        const GradPtrs<G, RC> gp(&p.grads[0]);
        Pm* pp = static_cast<Pm*>(p.params16);
        uint64_t va = (a + 7) & ~7ull, vb = b & ~7ull;
        if (va > b) va = b;
        if (vb < va) vb = va;
        for (uint64_t e = a + threadIdx.x; e < va; e += kBulkThreads)
            elem_step<G, Pm, RC, PUSH>(p, s, gp, pp, e, e, io, bad);
        for (uint64_t e = vb + threadIdx.x; e < b; e += kBulkThreads)
            elem_step<G, Pm, RC, PUSH>(p, s, gp, pp, e, e, io, bad);
    } else {
        uint32_t j = find_tensor(p.tab, a);
        uint64_t x = a;
        while (x < b) {
            const uint64_t t0 = p.tab.offs[j], t1 = p.tab.offs[j + 1];
            const uint64_t sb = t1 < b ? t1 : b;
            if (x < sb) {
                const bool vec = (p.tab.flags[j] & 1u) != 0u;
                uint64_t ba = sb, bb = sb;
                if (vec) {
                    ba = (x + 7) & ~7ull;
                    bb = sb & ~7ull;
                    if (ba > sb) ba = sb;
                    if (bb < ba) bb = ba;
                }
                if (ba > x || bb < sb) {
                    const uint32_t nr = RC > 0 ? (uint32_t)RC : p.R;  // RC == 0: the chunked kernel, any R
                    __syncthreads();
                    for (uint32_t r = threadIdx.x; r < nr; r += kBulkThreads) s_gp[r] = p.tab.grads[(uint64_t)j * nr + r];
                    __syncthreads();
                    const GradPtrs<G, RC> gp(s_gp);
                    Pm* pp = static_cast<Pm*>(p.tab.params[j]);
                    for (uint64_t e = x + threadIdx.x; e < ba; e += kBulkThreads)
                        elem_step<G, Pm, RC>(p, s, gp, pp, e, e - t0, io, bad);
                    for (uint64_t e = bb + threadIdx.x; e < sb; e += kBulkThreads)
                        elem_step<G, Pm, RC>(p, s, gp, pp, e, e - t0, io, bad);
                }
            }
            x = sb;
            ++j;
        }
    }
}


// Input and output state arrays of this step (set ctrl.parity in two-set mode).
__device__ __forceinline__ StateIO state_io(const StepParams& p) {
    const uint32_t par = p.two_set ? p.ctrl->parity : 0u;
    const uint32_t out = par ^ (uint32_t)p.two_set;
    return StateIO{p.w[par], p.m[par], p.v[par], p.w[out], p.m[out], p.v[out]};
}

// Flat calls: tiles are handed out dynamically.  The launch's vector body
// [va, vb) is cut into kTile-element tiles.  CTA b fills its ring with tiles
// b, b + G, ..., b + (D-1) G (G CTAs, D stages) without asking anyone, so
// every stage's copies are in flight at once from the start; after that each
// CTA's producer claims the next tile from a counter in the workspace
// (claims number the tiles from D*G on), one claim ahead of use so the
// atomic's latency overlaps the copies.  All CTAs then finish within about
// one tile of each other, whatever the speed of their SM.  The tile id
// travels to the consumers in a per-stage slot, written before the stage's
// barrier is armed; kEndTile marks the end.
constexpr uint32_t kEndTile = 0xFFFFFFFFu;

__device__ __forceinline__ uint32_t flat_tile_count(uint64_t va, uint64_t vb) {
    return va < vb ? (uint32_t)((vb - va + kTile - 1) / kTile) : 0u;
}

// Producer side (one thread): `issue(st, e0, n)` arms full[st] and starts
// the copies of the tile [e0, e0 + n) into stage st.
template <int D, class Issue>
__device__ __forceinline__ void flat_produce(Workspace* ws, uint64_t va, uint64_t vb, uint64_t* full,
                                             uint64_t* empty, uint32_t* slot, Issue&& issue) {
    const uint32_t ntiles = flat_tile_count(va, vb);
    const uint32_t first_claimed = (uint32_t)D * gridDim.x;
    uint32_t next = 0;
    uint32_t k = 0;
    bool ok = true;
    for (;; ++k) {
        const int st = (int)(k % D);
        if (k >= (uint32_t)D && !mbar_wait_bounded(&empty[st], ((k / D) - 1u) & 1u)) {
            ok = false;
            break;
        }
        // ntiles <= 2^29 (the host refuses more than ZERO_MAX_ELEMENTS), so no tile id here wraps
        const uint32_t tile = k < (uint32_t)D ? blockIdx.x + k * gridDim.x : next;
        if (tile >= ntiles) {
            slot[st] = kEndTile;
            mbar_arrive(&full[st]);
            break;
        }
        if (k + 1u >= (uint32_t)D) next = first_claimed + atomicAdd(&ws->next_tile, 1u);
        slot[st] = tile;
        const uint64_t e0 = va + (uint64_t)tile * kTile;
        const uint32_t n = (uint32_t)((vb - e0) < (uint64_t)kTile ? (vb - e0) : (uint64_t)kTile);
        issue(st, e0, n);
    }
    if (!ok) {
        // Do not leave while copies of this CTA may still land in its shared
        // memory: wait (bounded) for the last tile of every stage.
        note_timeout();
        for (uint32_t j = k > (uint32_t)D ? k - D : 0u; j < k; ++j)
            (void)mbar_wait_bounded(&full[j % D], (j / D) & 1u);
    }
}

// Consumer side (every consumer thread): `consume(st, e0, n)` reads stage st.
template <int D, class Consume>
__device__ __forceinline__ void flat_consume(Workspace* ws, uint64_t va, uint64_t vb, uint64_t* full,
                                             uint64_t* empty, const uint32_t* slot, Consume&& consume) {
    for (uint32_t k = 0;; ++k) {
        const int st = (int)(k % D);
        if (!mbar_wait_bounded(&full[st], (k / D) & 1u)) {
            note_timeout();
            break;
        }
        const uint32_t tile = slot[st];
        if (tile == kEndTile) break;
        const uint64_t e0 = va + (uint64_t)tile * kTile;
        const uint32_t n = (uint32_t)((vb - e0) < (uint64_t)kTile ? (vb - e0) : (uint64_t)kTile);
        consume(st, e0, n);
        __syncwarp();
        if ((threadIdx.x & 31u) == 0u) mbar_arrive(&empty[st]);
    }
}

// The ragged ends of a flat launch, [lo, va) and [vb, hi) outside the vector
// body (at most 7 elements each), one element per lane: lanes `lane` of
// `nlanes` >= 14.
template <class G, class Pm, int RC, bool PUSH>
__device__ __forceinline__ void flat_ends(const StepParams& p, const Scal& s, const StateIO& io, uint32_t lane,
                                          bool& bad) {
    uint64_t va = (p.lo + 7) & ~7ull, vb = p.hi & ~7ull;
    if (va > p.hi) va = p.hi;
    if (vb < va) vb = va;
    const uint64_t nhead = va - p.lo, ntail = p.hi - vb;
    uint64_t e;
    if (lane < nhead) e = p.lo + lane;
    else if (lane - nhead < ntail) e = vb + (lane - nhead);
    else return;
    const GradPtrs<G, RC> gp(&p.grads[0]);
    elem_step<G, Pm, RC, PUSH>(p, s, gp, static_cast<Pm*>(p.params16), e, e, io, bad);
}

// Flat step over [lo, hi): the producer thread, the consumer warps, and --
// in the last CTA, while its ring fills -- the producer warp's other 31
// lanes on the ragged ends, so they cost the launch no time at its end.
template <class G, class Pm, int RC, bool PUSH = false>
__device__ __forceinline__ void flat_dynamic(const StepParams& p, uint64_t* full, uint64_t* empty,
                                             uint32_t* slot, unsigned char* ring, bool& bad) {
    using Sh = BulkShape<G, RC>;
    constexpr int D = Sh::kStages;
    const uint64_t va = (p.lo + 7) & ~7ull;
    const uint64_t vb = p.hi & ~7ull;
    if (threadIdx.x == kConsumers) {
        const StateIO io = state_io(p);
        const G* gb[RC];
#pragma unroll
        for (int r = 0; r < RC; ++r) gb[r] = static_cast<const G*>(p.grads[r]);
        flat_produce<D>(p.ws, va, vb, full, empty, slot, [&](int st, uint64_t e0, uint32_t n) {
            bulk_issue<G, RC>(io, gb, ring + st * Sh::kStage, &full[st], e0, e0, n);
        });
    } else if (threadIdx.x < kConsumers) {
        const StateIO io = state_io(p);
        const Scal s = make_scal(p.h, p.ctrl->step + 1ull, p.ctrl->loss_scale, p.wsum);
        Pm* pp = static_cast<Pm*>(p.params16);
        flat_consume<D>(p.ws, va, vb, full, empty, slot, [&](int st, uint64_t e0, uint32_t n) {
            const unsigned char* stage = ring + st * Sh::kStage;
            for (uint32_t q = 4u * threadIdx.x; q < n; q += 4u * kConsumers)
                bulk_group<G, Pm, RC, PUSH>(p, s, stage, q, e0 + q, e0 + q, io.wo, io.mo, io.vo, pp, bad);
        });
    } else if (blockIdx.x == gridDim.x - 1) {
        const StateIO io = state_io(p);
        const Scal s = make_scal(p.h, p.ctrl->step + 1ull, p.ctrl->loss_scale, p.wsum);
        flat_ends<G, Pm, RC, PUSH>(p, s, io, threadIdx.x - kConsumers - 1u, bad);
    }
}

// Tile descriptor handed from the producer to the consumers through shared
// memory (list calls): written before the stage's barrier is armed.
struct TileDesc {
    uint64_t e0;    // flat index of the tile's first element
    uint64_t toff;  // flat index of the tensor's first element
    void* params;   // the tensor's 16-bit parameters
    uint32_t n;     // elements (a multiple of 8); 0: no more tiles
    uint32_t pad;
};

// List call over the whole vector: the vector body of tensor j (if it may
// take the vector path) is [offs[j], round_down(offs[j+1], 8)); the bodies
// are cut into kTile tiles, numbered across tensors (tab.tiles holds the
// running count), and handed out dynamically like the flat call's tiles.
// As for flat calls, CTA b fills its ring with tiles b, b + G, ... and
// claims the rest.  Tile ids a producer gets only grow, so it finds each
// tile's tensor by scanning forward from the previous one.
template <class G, class Pm, int RC>
__device__ __forceinline__ void list_dynamic(const StepParams& p, uint64_t* full, uint64_t* empty,
                                             TileDesc* desc, unsigned char* ring, bool& bad) {
    using Sh = BulkShape<G, RC>;
    constexpr int D = Sh::kStages;
    const Table& t = p.tab;
    const uint64_t ntiles = t.tiles[t.T];
    if (threadIdx.x == kConsumers) {
        const StateIO io = state_io(p);
        const G* gb[RC];
        uint32_t j = 0xFFFFFFFFu;  // tensor whose pointers are loaded
        uint32_t jn = 0;           // scan position
        uint64_t t0 = 0, bb = 0, tfirst = 0;
        void* params = nullptr;
        const uint64_t first_claimed = (uint64_t)D * gridDim.x;
        uint64_t next = 0;
        if (blockIdx.x < ntiles) jn = find_tensor_by_tile(t, blockIdx.x);
        uint32_t k = 0;
        bool ok = true;
        for (;; ++k) {
            const int st = (int)(k % D);
            if (k >= (uint32_t)D && !mbar_wait_bounded(&empty[st], ((k / D) - 1u) & 1u)) {
                ok = false;
                break;
            }
            const uint64_t tile = k < (uint32_t)D ? (uint64_t)blockIdx.x + (uint64_t)k * gridDim.x : next;
            if (tile >= ntiles) {
                desc[st] = TileDesc{0ull, 0ull, nullptr, 0u, 0u};
                mbar_arrive(&full[st]);
                break;
            }
            if (k + 1u >= (uint32_t)D) next = first_claimed + atomicAdd(&p.ws->next_tile, 1u);
            while (t.tiles[jn + 1] <= tile) ++jn;
            if (jn != j) {
                j = jn;
#pragma unroll
                for (int r = 0; r < RC; ++r) gb[r] = static_cast<const G*>(t.grads[(uint64_t)j * RC + r]);
                params = t.params[j];
                t0 = t.offs[j];
                bb = t.offs[j + 1] & ~7ull;
                tfirst = t.tiles[j];
            }
            const uint64_t e0 = t0 + (tile - tfirst) * kTile;
            const uint32_t n = (uint32_t)((bb - e0) < (uint64_t)kTile ? (bb - e0) : (uint64_t)kTile);
            desc[st] = TileDesc{e0, t0, params, n, 0u};
            bulk_issue<G, RC>(io, gb, ring + st * Sh::kStage, &full[st], e0, e0 - t0, n);
        }
        if (!ok) {
            note_timeout();
            for (uint32_t i = k > (uint32_t)D ? k - D : 0u; i < k; ++i)
                (void)mbar_wait_bounded(&full[i % D], (i / D) & 1u);
        }
    } else if (threadIdx.x < kConsumers) {
        const StateIO io = state_io(p);
        const Scal s = make_scal(p.h, p.ctrl->step + 1ull, p.ctrl->loss_scale, p.wsum);
        for (uint32_t k = 0;; ++k) {
            const int st = (int)(k % D);
            if (!mbar_wait_bounded(&full[st], (k / D) & 1u)) {
                note_timeout();
                break;
            }
            const TileDesc d = desc[st];
            if (d.n == 0u) break;
            const unsigned char* stage = ring + st * Sh::kStage;
            Pm* pp = static_cast<Pm*>(d.params);
            const uint64_t le0 = d.e0 - d.toff;
            for (uint32_t q = 4u * threadIdx.x; q < d.n; q += 4u * kConsumers)
                bulk_group<G, Pm, RC>(p, s, stage, q, d.e0 + q, le0 + q, io.wo, io.mo, io.vo, pp, bad);
            __syncwarp();
            if ((threadIdx.x & 31u) == 0u) mbar_arrive(&empty[st]);
        }
    }
}

// Scalar part of [a, b) for list_dynamic: everything outside the tensors'
// vector bodies.
template <class G, class Pm, int RC>
__device__ __forceinline__ void list_scalar_whole(const StepParams& p, const Scal& s, uint64_t a, uint64_t b,
                                                  const StateIO& io, bool& bad, const void** s_gp) {
    uint32_t j = find_tensor(p.tab, a);
    uint64_t x = a;
    while (x < b) {
        const uint64_t t0 = p.tab.offs[j], t1 = p.tab.offs[j + 1];
        const uint64_t sb = t1 < b ? t1 : b;
        if (x < sb) {
            const bool vec = (p.tab.flags[j] & 1u) != 0u;
            const uint64_t be = vec ? (t1 & ~7ull) : t0;  // body [t0, be)
            const uint64_t from = be > x ? be : x;
            if (from < sb) {
                const uint32_t nr = RC > 0 ? (uint32_t)RC : p.R;  // RC == 0: the chunked kernel, any R
                __syncthreads();
                for (uint32_t r = threadIdx.x; r < nr; r += kBulkThreads) s_gp[r] = p.tab.grads[(uint64_t)j * nr + r];
                __syncthreads();
                const GradPtrs<G, RC> gp(s_gp);
                Pm* pp = static_cast<Pm*>(p.tab.params[j]);
                for (uint64_t e = from + threadIdx.x; e < sb; e += kBulkThreads)
                    elem_step<G, Pm, RC>(p, s, gp, pp, e, e - t0, io, bad);
            }
        }
        x = sb;
        ++j;
    }
}

// List call: each CTA walks its own contiguous range of the concatenation.
template <class G, class Pm, int RC>
__device__ __forceinline__ void list_static(const StepParams& p, uint64_t a, uint64_t b, uint64_t* full,
                                            uint64_t* empty, unsigned char* ring, bool& bad) {
    using Sh = BulkShape<G, RC>;
    constexpr int D = Sh::kStages;
    if (threadIdx.x == kConsumers) {
        const StateIO io = state_io(p);
        TileWalk<G, RC, true, true> pw;
        pw.start(p, a, b);
        uint64_t e0;
        uint32_t n;
        uint32_t k = 0;
        bool ok = true;
        for (; pw.next(p, e0, n); ++k) {
            const int st = (int)(k % D);
            if (k >= (uint32_t)D && !mbar_wait_bounded(&empty[st], ((k / D) - 1u) & 1u)) {
                ok = false;
                break;
            }
            bulk_issue<G, RC>(io, pw.gb, ring + st * Sh::kStage, &full[st], e0, e0 - pw.toff, n);
        }
        if (!ok) {
            // Do not leave while copies of this CTA may still land in its
            // shared memory: wait (bounded) for the last tile of every stage.
            note_timeout();
            for (uint32_t j = k > (uint32_t)D ? k - D : 0u; j < k; ++j)
                (void)mbar_wait_bounded(&full[j % D], (j / D) & 1u);
        }
    } else if (threadIdx.x < kConsumers) {
        const StateIO io = state_io(p);
        const Scal s = make_scal(p.h, p.ctrl->step + 1ull, p.ctrl->loss_scale, p.wsum);
        TileWalk<G, RC, true, false> cw;
        cw.start(p, a, b);
        uint64_t e0;
        uint32_t n;
        for (uint32_t k = 0; cw.next(p, e0, n); ++k) {
            const int st = (int)(k % D);
            if (!mbar_wait_bounded(&full[st], (k / D) & 1u)) {
                note_timeout();
                break;
            }
            const unsigned char* stage = ring + st * Sh::kStage;
            Pm* pp = static_cast<Pm*>(cw.params);
            const uint64_t le0 = e0 - cw.toff;
            for (uint32_t q = 4u * threadIdx.x; q < n; q += 4u * kConsumers)
                bulk_group<G, Pm, RC>(p, s, stage, q, e0 + q, le0 + q, io.wo, io.mo, io.vo, pp, bad);
            __syncwarp();
            if ((threadIdx.x & 31u) == 0u) mbar_arrive(&empty[st]);
        }
    }
}

// PUSH (flat calls only): every 16-bit value is also stored into the
// p.npush other replicas in p.push.
template <class G, class Pm, int RC, bool LIST, bool PUSH = false>
__global__ void __launch_bounds__(kBulkThreads, 1) step_bulk_kernel(const __grid_constant__ StepParams p) {
    static_assert(!(LIST && PUSH), "parameter push is for flat calls");
    using Sh = BulkShape<G, RC>;
    constexpr int D = Sh::kStages;
    constexpr uint32_t kConsumerWarps = kConsumers / 32;
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);        // data of stage s has landed
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + 64);  // every consumer warp is done with stage s
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + 128);  // tile id (flat) or TileDesc (list) of stage s
    const void** s_gp = reinterpret_cast<const void**>(smem + kBarBytes);
    unsigned char* ring = smem + kBarBytes + kGpBytes;

    __shared__ StepStart s_start;
    uint64_t a = p.base + (uint64_t)blockIdx.x * p.chunk;
    uint64_t b = a + p.chunk;
    if (a < p.lo) a = p.lo;
    if (b > p.hi) b = p.hi;
    const bool work = (LIST && !p.whole) ? a < b : p.lo < p.hi;
    // shared memory only until the wait: overlaps the earlier kernel's tail
    if (threadIdx.x == 0) {
        s_timed_out = 0u;
        if (work) {
            for (int i = 0; i < D; ++i) {
                mbar_init(&full[i], 1u);
                mbar_init(&empty[i], kConsumerWarps);
            }
            fence_mbar_init();
        }
    }
    grid_dependency_wait();
    allow_dependents();
    bool skip = false;
    if (p.check == 2) skip = *reinterpret_cast<volatile const unsigned*>(&p.ws->found) != 0u;
    bool bad = false;
    if (!skip && work) {
        __syncthreads();
        // the epilogue's inputs, loaded while the first tiles are in flight
        if (threadIdx.x == 0) s_start = StepStart{*p.ctrl, p.ws->found};
        if constexpr (LIST) {
            if (p.whole) list_dynamic<G, Pm, RC>(p, full, empty, reinterpret_cast<TileDesc*>(slot), ring, bad);
            else list_static<G, Pm, RC>(p, a, b, full, empty, ring, bad);
            __syncthreads();
            // Ragged heads and tails, and tensors that cannot take the vector path.
            const StateIO io = state_io(p);
            const Scal s = make_scal(p.h, p.ctrl->step + 1ull, p.ctrl->loss_scale, p.wsum);
            if (p.whole) {
                if (a < b) list_scalar_whole<G, Pm, RC>(p, s, a, b, io, bad, s_gp);
            } else {
                if (a < b) bulk_scalar_pass<G, Pm, RC, true>(p, s, a, b, io, bad, s_gp);
            }
        } else {
            flat_dynamic<G, Pm, RC, PUSH>(p, full, empty, slot, ring, bad);
        }
    } else if (threadIdx.x == 0) {
        s_start = StepStart{*p.ctrl, p.ws->found};
    }
    finish_step<PUSH>(p, bad, s_timed_out != 0u, &s_start);
}

// ------------------------------------------------------------ any rank count

// Rank counts without a compiled staged instance (3, 5-7, 9-15, 17-256, and
// 16 with fp32 gradients) stream each tile through the ring in chunks of
// kChunkRanks ranks: the stage of chunk c holds the tile's gradient slices of
// ranks [8c, 8c + 8), and the tile's last chunk also its master, m and v.  A
// consumer thread handles the same four elements in every chunk of a tile and
// keeps their float64 sums in registers from the first chunk to the last, so
// the ranks are added in the order 0..R-1 as in the other kernels (the
// results are bitwise theirs); the last chunk applies Adam.  Flat calls and
// list calls over the whole vector hand their tiles out as flat_dynamic and
// list_dynamic do (CTA b starts on tile b and claims the rest from the
// workspace counter one tile ahead); a list call for one owner walks each
// CTA's own range, as list_static does.
constexpr uint32_t kChunkRanks = 8;
static_assert(4 * kConsumers == kTile, "one 4-element group per consumer thread per tile");

template <class G>
using ChunkShape = BulkShape<G, (int)kChunkRanks>;

// Stage descriptor of the chunked kernel, written before the stage's
// barrier is armed.
struct ChunkDesc {
    uint64_t e0;      // flat index of the tile's first element
    uint64_t toff;    // flat index of the tensor's first element (0: flat)
    void* params;     // the tensor's 16-bit parameters
    uint32_t n;       // elements (a multiple of 8); 0: no more tiles
    uint32_t chunk;   // ranks [8 chunk, 8 chunk + 8) of the tile
};
static_assert(sizeof(ChunkDesc) * 8 <= kBarBytes - 128, "stage descriptors must fit the barrier header");

// Copies of one chunk into `stage`: ranks [r0, r0 + rn) of the gradient bases
// `gp` (the tile's tensor), and the state when `last`.
template <class G>
__device__ __forceinline__ void chunk_issue(const StateIO& io, const void* const* gp, uint32_t r0, uint32_t rn,
                                            bool last, unsigned char* stage, uint64_t* bar, uint64_t e0,
                                            uint64_t le0, uint32_t n) {
    using Sh = ChunkShape<G>;
    const uint32_t gbytes = n * (uint32_t)sizeof(G), sbytes = n * 4u;
    mbar_expect_tx(bar, rn * gbytes + (last ? 3u * sbytes : 0u));
    for (uint32_t r = 0; r < rn; ++r)
        bulk_g2s(stage + r * Sh::kGradSlice, static_cast<const G*>(gp[r0 + r]) + le0, gbytes, bar);
    if (last) {
        unsigned char* st = stage + kChunkRanks * Sh::kGradSlice;
        bulk_g2s(st, io.wi + e0, sbytes, bar);
        bulk_g2s(st + kTile * 4u, io.mi + e0, sbytes, bar);
        bulk_g2s(st + 2u * kTile * 4u, io.vi + e0, sbytes, bar);
    }
}

// The producer thread of the chunked kernel.  Flat: tile i is [va + i kTile,
// ...) of the vector body [va, vb).  List: tiles are numbered across the
// tensors' vector bodies (tab.tiles).  Every tile takes ceil(R/8) stages.
template <class G, bool LIST>
__device__ __forceinline__ void chunk_produce(const StepParams& p, uint64_t va, uint64_t vb, uint64_t* full,
                                              uint64_t* empty, ChunkDesc* desc, unsigned char* ring) {
    using Sh = ChunkShape<G>;
    constexpr uint32_t D = (uint32_t)Sh::kStages;
    const StateIO io = state_io(p);
    const Table& t = p.tab;
    const uint32_t C = (p.R + kChunkRanks - 1u) / kChunkRanks;
    const uint64_t ntiles = LIST ? t.tiles[t.T] : (uint64_t)flat_tile_count(va, vb);
    const void* const* gp = &p.grads[0];
    void* params = p.params16;
    uint64_t t0 = 0, bb = vb, tfirst = 0;
    uint32_t j = 0xFFFFFFFFu, jn = 0;
    uint64_t tile = blockIdx.x;
    if (LIST && tile < ntiles) jn = find_tensor_by_tile(t, tile);
    uint32_t k = 0;
    bool ok = true;
    for (;;) {
        const bool have = tile < ntiles;
        uint64_t next = 0;
        uint64_t e0 = 0;
        uint32_t n = 0;
        if (have) {
            next = (uint64_t)gridDim.x + atomicAdd(&p.ws->next_tile, 1u);  // one claim ahead
            if constexpr (LIST) {
                while (t.tiles[jn + 1] <= tile) ++jn;
                if (jn != j) {
                    j = jn;
                    gp = t.grads + (uint64_t)j * p.R;
                    params = t.params[j];
                    t0 = t.offs[j];
                    bb = t.offs[j + 1] & ~7ull;
                    tfirst = t.tiles[j];
                }
                e0 = t0 + (tile - tfirst) * kTile;
            } else {
                e0 = va + tile * kTile;
            }
            n = (uint32_t)((bb - e0) < (uint64_t)kTile ? (bb - e0) : (uint64_t)kTile);
        }
        const uint32_t stages = have ? C : 1u;  // past the last tile: one end marker
        for (uint32_t c = 0; c < stages; ++c, ++k) {
            const uint32_t st = k % D;
            if (k >= D && !mbar_wait_bounded(&empty[st], ((k / D) - 1u) & 1u)) {
                ok = false;
                break;
            }
            if (!have) {
                desc[st] = ChunkDesc{0ull, 0ull, nullptr, 0u, 0u};
                mbar_arrive(&full[st]);
            } else {
                const uint32_t r0 = c * kChunkRanks;
                const uint32_t rn = p.R - r0 < kChunkRanks ? p.R - r0 : kChunkRanks;
                desc[st] = ChunkDesc{e0, t0, params, n, c};
                chunk_issue<G>(io, gp, r0, rn, c + 1u == C, ring + st * Sh::kStage, &full[st], e0, e0 - t0, n);
            }
        }
        if (!ok || !have) break;
        tile = next;
    }
    if (!ok) {
        // Do not leave while copies of this CTA may still land in its shared
        // memory: wait (bounded) for the last chunk of every stage.
        note_timeout();
        for (uint32_t i = k > D ? k - D : 0u; i < k; ++i) (void)mbar_wait_bounded(&full[i % D], (i / D) & 1u);
    }
}

// The producer thread of the chunked kernel for a list call for one owner:
// CTA b walks its own contiguous range [a, b) of the concatenation, tile by
// tile through the vector bodies of its tensors (TileWalk), each tile taking
// ceil(R/8) stages as above.
template <class G>
__device__ __forceinline__ void chunk_produce_static(const StepParams& p, uint64_t a, uint64_t b, uint64_t* full,
                                                     uint64_t* empty, ChunkDesc* desc, unsigned char* ring) {
    using Sh = ChunkShape<G>;
    constexpr uint32_t D = (uint32_t)Sh::kStages;
    const StateIO io = state_io(p);
    const uint32_t C = (p.R + kChunkRanks - 1u) / kChunkRanks;
    TileWalk<G, 1, true, false> pw;
    pw.start(p, a, b);
    uint32_t k = 0;
    bool ok = true;
    for (;;) {
        uint64_t e0 = 0;
        uint32_t n = 0;
        const bool have = pw.next(p, e0, n);
        // the walk has just moved past the tile's tensor: its index is j - 1
        const void* const* gp = have ? p.tab.grads + (uint64_t)(pw.j - 1u) * p.R : nullptr;
        const uint32_t stages = have ? C : 1u;  // past the last tile: one end marker
        for (uint32_t c = 0; c < stages; ++c, ++k) {
            const uint32_t st = k % D;
            if (k >= D && !mbar_wait_bounded(&empty[st], ((k / D) - 1u) & 1u)) {
                ok = false;
                break;
            }
            if (!have) {
                desc[st] = ChunkDesc{0ull, 0ull, nullptr, 0u, 0u};
                mbar_arrive(&full[st]);
            } else {
                const uint32_t r0 = c * kChunkRanks;
                const uint32_t rn = p.R - r0 < kChunkRanks ? p.R - r0 : kChunkRanks;
                desc[st] = ChunkDesc{e0, pw.toff, pw.params, n, c};
                chunk_issue<G>(io, gp, r0, rn, c + 1u == C, ring + st * Sh::kStage, &full[st], e0, e0 - pw.toff, n);
            }
        }
        if (!ok || !have) break;
    }
    if (!ok) {
        note_timeout();
        for (uint32_t i = k > D ? k - D : 0u; i < k; ++i) (void)mbar_wait_bounded(&full[i % D], (i / D) & 1u);
    }
}

// Adam on the four elements of a consumer thread after a tile's last chunk
// (`st`: the stage's state part), and the stores: the arithmetic of
// bulk_group after its reduction.
template <class Pm, bool PUSH>
__device__ __forceinline__ void chunk_update(const StepParams& p, const Scal& s, const double (&acc)[4],
                                             const unsigned char* st, uint32_t q, uint64_t e, uint64_t le,
                                             const StateIO& io, Pm* pp) {
    const float4 w4 = *reinterpret_cast<const float4*>(st + q * 4u);
    const float4 m4 = *reinterpret_cast<const float4*>(st + kTile * 4u + q * 4u);
    const float4 v4 = *reinterpret_cast<const float4*>(st + 2u * kTile * 4u + q * 4u);
    float w[4] = {w4.x, w4.y, w4.z, w4.w};
    float m[4] = {m4.x, m4.y, m4.z, m4.w};
    float v[4] = {v4.x, v4.y, v4.z, v4.w};
    float g[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        g[k] = (float)(acc[k] * s.inv_ws);
        adam1(g[k], w[k], m[k], v[k], s);
    }
    __stcs(reinterpret_cast<float4*>(io.wo + e), make_float4(w[0], w[1], w[2], w[3]));
    __stcs(reinterpret_cast<float4*>(io.mo + e), make_float4(m[0], m[1], m[2], m[3]));
    __stcs(reinterpret_cast<float4*>(io.vo + e), make_float4(v[0], v[1], v[2], v[3]));
    uint2 o;
    o.x = pack2<Pm>(w[0], w[1]);
    o.y = pack2<Pm>(w[2], w[3]);
    __stcs(reinterpret_cast<uint2*>(pp + le), o);
    if constexpr (PUSH)
        for (uint32_t i = 0; i < p.npush; ++i) __stcs(reinterpret_cast<uint2*>(static_cast<Pm*>(p.push[i]) + le), o);
    if (p.reduced != nullptr) __stcs(reinterpret_cast<float4*>(p.reduced + e), make_float4(g[0], g[1], g[2], g[3]));
}

// The consumer warps of the chunked kernel.
template <class G, class Pm, bool PUSH>
__device__ __forceinline__ void chunk_consume(const StepParams& p, uint64_t* full, uint64_t* empty,
                                              const ChunkDesc* desc, const unsigned char* ring, bool& bad) {
    using Sh = ChunkShape<G>;
    constexpr uint32_t D = (uint32_t)Sh::kStages;
    const StateIO io = state_io(p);
    const Scal s = make_scal(p.h, p.ctrl->step + 1ull, p.ctrl->loss_scale, p.wsum);
    const uint32_t C = (p.R + kChunkRanks - 1u) / kChunkRanks;
    const uint32_t q = 4u * threadIdx.x;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (uint32_t k = 0;; ++k) {
        const uint32_t st = k % D;
        if (!mbar_wait_bounded(&full[st], (k / D) & 1u)) {
            note_timeout();
            break;
        }
        const ChunkDesc d = desc[st];
        if (d.n == 0u) break;
        const unsigned char* stage = ring + st * Sh::kStage;
        if (d.chunk == 0u) {
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = 0.0;
        }
        if (q < d.n) {
            const uint32_t r0 = d.chunk * kChunkRanks;
            const uint32_t rn = p.R - r0 < kChunkRanks ? p.R - r0 : kChunkRanks;
            for (uint32_t r = 0; r < rn; ++r) {
                const Raw4<G> raw = lds4<G>(stage + r * Sh::kGradSlice + q * sizeof(G));
                if (p.check == 1) bad |= bad4(raw);
                float f[4];
                unpack4(raw, f);
                const double c = p.wt[r0 + r];
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] = fma(c, (double)f[i], acc[i]);
            }
            if (d.chunk + 1u == C)
                chunk_update<Pm, PUSH>(p, s, acc, stage + kChunkRanks * Sh::kGradSlice, q, d.e0 + q,
                                       d.e0 - d.toff + q, io, static_cast<Pm*>(d.params));
        }
        __syncwarp();
        if ((threadIdx.x & 31u) == 0u) mbar_arrive(&empty[st]);
    }
}

// Flat calls (PUSH as in step_bulk_kernel) and list calls, over the whole
// vector or for one owner, any number of gradient buffers.
template <class G, class Pm, bool LIST, bool PUSH = false>
__global__ void __launch_bounds__(kBulkThreads, 1) step_chunked_kernel(const __grid_constant__ StepParams p) {
    static_assert(!(LIST && PUSH), "parameter push is for flat calls");
    using Sh = ChunkShape<G>;
    constexpr int D = Sh::kStages;
    constexpr uint32_t kConsumerWarps = kConsumers / 32;
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + 64);
    ChunkDesc* desc = reinterpret_cast<ChunkDesc*>(smem + 128);
    unsigned char* ring = smem + kBarBytes + kGpBytes;
    __shared__ const void* s_gp[LIST ? ZERO_MAX_RANKS : 1];  // a tensor's gradient bases (scalar pass)
    __shared__ StepStart s_start;

    uint64_t a = p.base + (uint64_t)blockIdx.x * p.chunk;  // this CTA's range (list calls)
    uint64_t b = a + p.chunk;
    if (a < p.lo) a = p.lo;
    if (b > p.hi) b = p.hi;
    const bool work = (LIST && !p.whole) ? a < b : p.lo < p.hi;
    if (threadIdx.x == 0) {
        s_timed_out = 0u;
        if (work) {
            for (int i = 0; i < D; ++i) {
                mbar_init(&full[i], 1u);
                mbar_init(&empty[i], kConsumerWarps);
            }
            fence_mbar_init();
        }
    }
    grid_dependency_wait();
    allow_dependents();
    bool skip = false;
    if (p.check == 2) skip = *reinterpret_cast<volatile const unsigned*>(&p.ws->found) != 0u;
    bool bad = false;
    if (!skip && work) {
        __syncthreads();
        if (threadIdx.x == 0) s_start = StepStart{*p.ctrl, p.ws->found};
        const uint64_t va = (p.lo + 7) & ~7ull, vb = p.hi & ~7ull;
        if (threadIdx.x == kConsumers) {
            if (LIST && !p.whole) chunk_produce_static<G>(p, a, b, full, empty, desc, ring);
            else chunk_produce<G, LIST>(p, va, vb, full, empty, desc, ring);
        } else if (threadIdx.x < kConsumers) {
            chunk_consume<G, Pm, PUSH>(p, full, empty, desc, ring, bad);
        } else if (!LIST && blockIdx.x == gridDim.x - 1) {
            const StateIO io = state_io(p);
            const Scal s = make_scal(p.h, p.ctrl->step + 1ull, p.ctrl->loss_scale, p.wsum);
            flat_ends<G, Pm, 0, PUSH>(p, s, io, threadIdx.x - kConsumers - 1u, bad);
        }
        if constexpr (LIST) {
            // Ragged heads and tails, and tensors that cannot take the vector path.
            __syncthreads();
            const StateIO io = state_io(p);
            const Scal s = make_scal(p.h, p.ctrl->step + 1ull, p.ctrl->loss_scale, p.wsum);
            if (a < b) {
                if (p.whole) list_scalar_whole<G, Pm, 0>(p, s, a, b, io, bad, s_gp);
                else bulk_scalar_pass<G, Pm, 0, true>(p, s, a, b, io, bad, s_gp);
            }
        }
    } else if (threadIdx.x == 0) {
        s_start = StepStart{*p.ctrl, p.ws->found};
    }
    finish_step<PUSH>(p, bad, s_timed_out != 0u, &s_start);
}

// ------------------------------------------------------------ micro-step accumulation

// Stage of the accumulation kernel: [R gradient slices][acc slice]; the acc
// slice is loaded only when the window continues (first == 0).
template <class G, int RC>
struct AccumShape {
    static constexpr uint32_t kGradSlice = kTile * sizeof(G);
    static constexpr uint32_t kStage = RC * kGradSlice + kTile * 4u;
    static constexpr int kBudget = 200 * 1024;
    static constexpr int kStages = (kBudget / kStage) > 8 ? 8 : (kBudget / kStage);
    static constexpr uint32_t kSmem = kBarBytes + kGpBytes + kStages * kStage;
    static_assert(kStages >= 2, "stage too large for the ring");
    static_assert(kStage % 1024 == 0, "stages must stay 1024-byte aligned");
};

// Four consecutive elements at flat index e (offset q in the stage): the
// arithmetic of accum_vec, element for element, so the register and the
// bulk kernels give bitwise identical sums.
template <class G, int RC>
__device__ __forceinline__ void accum_group(const AccumParams& p, const unsigned char* stage, uint32_t q,
                                            uint64_t e) {
    using Sh = AccumShape<G, RC>;
    Raw4<G> raw[RC];
#pragma unroll
    for (int r = 0; r < RC; ++r) raw[r] = lds4<G>(stage + r * Sh::kGradSlice + q * sizeof(G));
    float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!p.first) a4 = *reinterpret_cast<const float4*>(stage + RC * Sh::kGradSlice + q * 4u);
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int r = 0; r < RC; ++r) {
        float f[4];
        unpack4(raw[r], f);
        const double c = p.wt[r];
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = fma(c, (double)f[k], acc[k]);
    }
    const float prev[4] = {a4.x, a4.y, a4.z, a4.w};
    float out[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) out[k] = (float)((double)prev[k] + p.scale * (acc[k] * p.inv_wsum));
    __stcs(reinterpret_cast<float4*>(p.acc + e), make_float4(out[0], out[1], out[2], out[3]));
}

// Last CTA to finish: record a wait timeout in ctrl->device_error and leave
// the workspace ready for the next launch (the packed arrival of
// finish_step, without the found field).
__device__ __forceinline__ void finish_accum(const AccumParams& p) {
    __syncthreads();
    if (threadIdx.x == 0) {
        Workspace* ws = p.ws;
        const unsigned long long mine = Arrival::mine(false, s_timed_out != 0u);
        const unsigned long long all = atomicAdd(&ws->arrive, mine) + mine;
        if (Arrival::count(all) == gridDim.x) {
            if (Arrival::any_timeout(all)) p.ctrl->device_error = 1u;
            ws->next_tile = 0u;
            ws->arrive = 0ull;
        }
    }
}

// acc[lo, hi) = (first ? 0 : acc) + scale * (sum_r w_r g_r) / sum(w), with
// the tiles of the vector body streamed through the shared-memory ring and
// handed out dynamically, as in the flat step; CTA 0 takes the ragged ends.
template <class G, int RC>
__global__ void __launch_bounds__(kBulkThreads, 1) accum_bulk_kernel(const __grid_constant__ AccumParams p) {
    using Sh = AccumShape<G, RC>;
    constexpr int D = Sh::kStages;
    constexpr uint32_t kConsumerWarps = kConsumers / 32;
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + 64);
    uint32_t* slot = reinterpret_cast<uint32_t*>(smem + 128);
    unsigned char* ring = smem + kBarBytes + kGpBytes;
    if (threadIdx.x == 0) {
        s_timed_out = 0u;
        for (int i = 0; i < D; ++i) {
            mbar_init(&full[i], 1u);
            mbar_init(&empty[i], kConsumerWarps);
        }
        fence_mbar_init();
    }
    grid_dependency_wait();
    allow_dependents();
    __syncthreads();
    const uint64_t va = (p.lo + 7) & ~7ull;
    const uint64_t vb = p.hi & ~7ull;
    if (threadIdx.x == kConsumers) {
        const G* gb[RC];
#pragma unroll
        for (int r = 0; r < RC; ++r) gb[r] = static_cast<const G*>(p.grads[r]);
        const bool load_acc = !p.first;
        flat_produce<D>(p.ws, va, vb, full, empty, slot, [&](int st, uint64_t e0, uint32_t n) {
            unsigned char* stage = ring + st * Sh::kStage;
            const uint32_t gbytes = n * (uint32_t)sizeof(G);
            mbar_expect_tx(&full[st], RC * gbytes + (load_acc ? n * 4u : 0u));
#pragma unroll
            for (int r = 0; r < RC; ++r) bulk_g2s(stage + r * Sh::kGradSlice, gb[r] + e0, gbytes, &full[st]);
            if (load_acc) bulk_g2s(stage + RC * Sh::kGradSlice, p.acc + e0, n * 4u, &full[st]);
        });
    } else if (threadIdx.x < kConsumers) {
        flat_consume<D>(p.ws, va, vb, full, empty, slot, [&](int st, uint64_t e0, uint32_t n) {
            const unsigned char* stage = ring + st * Sh::kStage;
            for (uint32_t q = 4u * threadIdx.x; q < n; q += 4u * kConsumers) accum_group<G, RC>(p, stage, q, e0 + q);
        });
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        const GradPtrs<G, RC> gp(&p.grads[0]);
        uint64_t ha = va > p.hi ? p.hi : va;
        uint64_t tb = vb < ha ? ha : vb;
        for (uint64_t e = p.lo + threadIdx.x; e < ha; e += kBulkThreads) accum_elem<G, RC>(p, gp, e);
        for (uint64_t e = tb + threadIdx.x; e < p.hi; e += kBulkThreads) accum_elem<G, RC>(p, gp, e);
    }
    finish_accum(p);
}

// Accumulation for rank counts without a staged instance: the tiles of the
// vector body as in accum_bulk_kernel, each passed through the ring as
// ceil(R/8) stages of up to eight ranks' gradient slices, the last stage also
// holding the accumulator slice when the window continues.  The float64
// sums stay in registers across a tile's chunks, so the result is bitwise
// accum_vec's.
template <class G>
using AccumChunkShape = AccumShape<G, (int)kChunkRanks>;

template <class G>
__global__ void __launch_bounds__(kBulkThreads, 1) accum_chunked_kernel(const __grid_constant__ AccumParams p) {
    using Sh = AccumChunkShape<G>;
    constexpr uint32_t D = (uint32_t)Sh::kStages;
    constexpr uint32_t kConsumerWarps = kConsumers / 32;
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + 64);
    ChunkDesc* desc = reinterpret_cast<ChunkDesc*>(smem + 128);
    unsigned char* ring = smem + kBarBytes + kGpBytes;
    // the rank weights, read from shared memory (a parameter array indexed at
    // run time would be a memory load on the critical path of every stage)
    __shared__ double s_wt[ZERO_MAX_RANKS];
    for (uint32_t r = threadIdx.x; r < p.R; r += kBulkThreads) s_wt[r] = p.wt[r];
    if (threadIdx.x == 0) {
        s_timed_out = 0u;
        for (uint32_t i = 0; i < D; ++i) {
            mbar_init(&full[i], 1u);
            mbar_init(&empty[i], kConsumerWarps);
        }
        fence_mbar_init();
    }
    grid_dependency_wait();
    allow_dependents();
    __syncthreads();
    const uint64_t va = (p.lo + 7) & ~7ull;
    const uint64_t vb = p.hi & ~7ull;
    const uint32_t C = (p.R + kChunkRanks - 1u) / kChunkRanks;
    if (threadIdx.x == kConsumers) {
        const G* gb1[kChunkRanks];  // R <= 8: the rank pointers, once
#pragma unroll
        for (uint32_t r = 0; r < kChunkRanks; ++r) gb1[r] = r < p.R ? static_cast<const G*>(p.grads[r]) : nullptr;
        const uint64_t ntiles = flat_tile_count(va, vb);
        uint64_t tile = blockIdx.x;
        uint32_t k = 0;
        bool ok = true;
        for (;;) {
            const bool have = tile < ntiles;
            uint64_t next = 0, e0 = 0;
            uint32_t n = 0;
            if (have) {
                next = (uint64_t)gridDim.x + atomicAdd(&p.ws->next_tile, 1u);  // one claim ahead
                e0 = va + tile * kTile;
                n = (uint32_t)((vb - e0) < (uint64_t)kTile ? (vb - e0) : (uint64_t)kTile);
            }
            const uint32_t stages = have ? C : 1u;  // past the last tile: one end marker
            for (uint32_t c = 0; c < stages; ++c, ++k) {
                const uint32_t st = k % D;
                if (k >= D && !mbar_wait_bounded(&empty[st], ((k / D) - 1u) & 1u)) {
                    ok = false;
                    break;
                }
                if (!have) {
                    desc[st] = ChunkDesc{0ull, 0ull, nullptr, 0u, 0u};
                    mbar_arrive(&full[st]);
                } else {
                    const uint32_t r0 = c * kChunkRanks;
                    const uint32_t rn = p.R - r0 < kChunkRanks ? p.R - r0 : kChunkRanks;
                    const bool load_acc = c + 1u == C && !p.first;
                    desc[st] = ChunkDesc{e0, 0ull, nullptr, n, c};
                    unsigned char* stage = ring + st * Sh::kStage;
                    const uint32_t gbytes = n * (uint32_t)sizeof(G);
                    mbar_expect_tx(&full[st], rn * gbytes + (load_acc ? n * 4u : 0u));
                    if (C == 1u) {
#pragma unroll
                        for (uint32_t r = 0; r < kChunkRanks; ++r)
                            if (r < rn) bulk_g2s(stage + r * Sh::kGradSlice, gb1[r] + e0, gbytes, &full[st]);
                    } else {
                        for (uint32_t r = 0; r < rn; ++r)
                            bulk_g2s(stage + r * Sh::kGradSlice, static_cast<const G*>(p.grads[r0 + r]) + e0,
                                     gbytes, &full[st]);
                    }
                    if (load_acc) bulk_g2s(stage + kChunkRanks * Sh::kGradSlice, p.acc + e0, n * 4u, &full[st]);
                }
            }
            if (!ok || !have) break;
            tile = next;
        }
        if (!ok) {
            // Do not leave while copies of this CTA may still land in its
            // shared memory: wait (bounded) for the last use of every stage.
            note_timeout();
            for (uint32_t i = k > D ? k - D : 0u; i < k; ++i) (void)mbar_wait_bounded(&full[i % D], (i / D) & 1u);
        }
    } else if (threadIdx.x < kConsumers) {
        const uint32_t q = 4u * threadIdx.x;
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        double w1[kChunkRanks];  // R <= 8: the weights, once
#pragma unroll
        for (uint32_t r = 0; r < kChunkRanks; ++r) w1[r] = r < p.R ? s_wt[r] : 0.0;
        for (uint32_t k = 0;; ++k) {
            const uint32_t st = k % D;
            if (!mbar_wait_bounded(&full[st], (k / D) & 1u)) {
                note_timeout();
                break;
            }
            const ChunkDesc d = desc[st];
            if (d.n == 0u) break;
            const unsigned char* stage = ring + st * Sh::kStage;
            if (d.chunk == 0u) {
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[i] = 0.0;
            }
            if (q < d.n) {
                const uint32_t r0 = d.chunk * kChunkRanks;
                const uint32_t rn = p.R - r0 < kChunkRanks ? p.R - r0 : kChunkRanks;
                // all of the chunk's loads first, then the sums in rank order
                Raw4<G> raw[kChunkRanks];
                double wc[kChunkRanks];
#pragma unroll
                for (uint32_t r = 0; r < kChunkRanks; ++r) {
                    if (r < rn) {
                        raw[r] = lds4<G>(stage + r * Sh::kGradSlice + q * sizeof(G));
                        wc[r] = C == 1u ? w1[r] : s_wt[r0 + r];
                    }
                }
#pragma unroll
                for (uint32_t r = 0; r < kChunkRanks; ++r) {
                    if (r < rn) {
                        float f[4];
                        unpack4(raw[r], f);
                        const double c = wc[r];
#pragma unroll
                        for (int i = 0; i < 4; ++i) acc[i] = fma(c, (double)f[i], acc[i]);
                    }
                }
                if (d.chunk + 1u == C) {
                    float4 a4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (!p.first) a4 = *reinterpret_cast<const float4*>(stage + kChunkRanks * Sh::kGradSlice + q * 4u);
                    const float prev[4] = {a4.x, a4.y, a4.z, a4.w};
                    float out[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) out[i] = (float)((double)prev[i] + p.scale * (acc[i] * p.inv_wsum));
                    __stcs(reinterpret_cast<float4*>(p.acc + d.e0 + q), make_float4(out[0], out[1], out[2], out[3]));
                }
            }
            __syncwarp();
            if ((threadIdx.x & 31u) == 0u) mbar_arrive(&empty[st]);
        }
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        const GradPtrs<G, 0> gp(&p.grads[0]);
        uint64_t ha = va > p.hi ? p.hi : va;
        uint64_t tb = vb < ha ? ha : vb;
        for (uint64_t e = p.lo + threadIdx.x; e < ha; e += kBulkThreads) accum_elem<G, 0>(p, gp, e);
        for (uint64_t e = tb + threadIdx.x; e < p.hi; e += kBulkThreads) accum_elem<G, 0>(p, gp, e);
    }
    finish_accum(p);
}

// ------------------------------------------------------------ timeout health check

// One thread waits on a barrier that nothing arrives at; the bounded wait
// gives up and the kernel records the outcome through the step epilogue's
// control-block update, as a two-set step with the overflow check on whose
// wait gave up: device_error set, the step not applied.
__global__ void wait_timeout_probe_kernel(zero_ctrl* c) {
    __shared__ __align__(8) uint64_t bar;
    grid_dependency_wait();
    allow_dependents();
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1u);
        fence_mbar_init();
        // growth_interval 1: a step wrongly counted as applied would also
        // double the loss scale, which the health check's caller can see.
        if (!mbar_wait_bounded(&bar, 0u)) {
            const zero_ctrl c0 = *c;
            ctrl_after_step(c0, c, false, true, true, 1, 1u);
        }
    }
}

}  // namespace zadam
