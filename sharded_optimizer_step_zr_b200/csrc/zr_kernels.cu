// Fused sharded optimizer step kernels for B200 (sm_100a).
//
// The step is a pure stream over the owned slice: per owned element it reads
// W bf16 gradients (2W bytes), fp32 master, m and v (12 bytes), writes them
// back (12 bytes) and writes one bf16 parameter (2 bytes).  Nothing here is
// a contraction, so there is no tensor-core work; the roofline is HBM
// bandwidth and the design goal is keeping enough bytes in flight:
//   * one 128-thread CTA per tile of up to 2048 owned elements (tiles never
//     cross a bucket; the hardware block scheduler balances them across the
//     148 SMs, five CTAs per SM);
//   * each thread owns 8 consecutive elements per iteration and issues the
//     16-byte gradient loads of a group of up to 8 replicas back to back,
//     plus the 32-byte master / m / v loads, before consuming any of them;
//   * the fold is a strict left fold in rank order in fp32, exactly the
//     reduce of the definition; the AdamW arithmetic uses round-to-nearest
//     intrinsics without contraction, so results equal the definition's
//     fp32 evaluation order bit for bit.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "zr_internal.hpp"

namespace zr {
namespace {

template <int CAP>
struct GradPtrs {
    const uint16_t* p[CAP];
};

// ---------------------------------------------------------------------------
// memory helpers
// ---------------------------------------------------------------------------

// Read-only streaming 16-byte load (gradients are never written by the step).
__device__ __forceinline__ uint4 ld_grad16(const uint16_t* p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

__device__ __forceinline__ uint16_t ld_grad2(const uint16_t* p) {
    unsigned short r;
    asm("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ float4 ld_state16(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ void st_state16(float* p, float4 x) { __stcs(reinterpret_cast<float4*>(p), x); }

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_1(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

__device__ __forceinline__ void unpack8(const uint4 q, float s[8]) {
    s[0] = bf16_lo(q.x); s[1] = bf16_hi(q.x);
    s[2] = bf16_lo(q.y); s[3] = bf16_hi(q.y);
    s[4] = bf16_lo(q.z); s[5] = bf16_hi(q.z);
    s[6] = bf16_lo(q.w); s[7] = bf16_hi(q.w);
}

__device__ __forceinline__ void add8(const uint4 q, float s[8]) {
    s[0] = __fadd_rn(s[0], bf16_lo(q.x)); s[1] = __fadd_rn(s[1], bf16_hi(q.x));
    s[2] = __fadd_rn(s[2], bf16_lo(q.y)); s[3] = __fadd_rn(s[3], bf16_hi(q.y));
    s[4] = __fadd_rn(s[4], bf16_lo(q.z)); s[5] = __fadd_rn(s[5], bf16_hi(q.z));
    s[6] = __fadd_rn(s[6], bf16_lo(q.w)); s[7] = __fadd_rn(s[7], bf16_hi(q.w));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);   // RNE on both halves
    uint32_t u;
    memcpy(&u, &h, 4);
    return u;
}

// ---------------------------------------------------------------------------
// element arithmetic
// ---------------------------------------------------------------------------

__device__ __forceinline__ float average(float s, const LaunchArgs& a) {
    // Division by a power of two is exact scaling: multiplying by 1/W gives
    // the same correctly rounded value as the division (zr_debug_average_check
    // compares the two on every fp32 input).
    return a.w_is_pow2 ? __fmul_rn(s, a.inv_w) : __fdiv_rn(s, static_cast<float>(a.world_size));
}

// Decoupled weight decay on the pre-update weight, then the bias-corrected
// Adam step; one rounding per operation, no fused multiply-add.
__device__ __forceinline__ void adamw(const AdamScalars& c, float g, float& p, float& m, float& v) {
    const float m_new = __fadd_rn(__fmul_rn(c.beta1, m), __fmul_rn(c.one_minus_beta1, g));
    const float v_new = __fadd_rn(__fmul_rn(c.beta2, v), __fmul_rn(c.one_minus_beta2, __fmul_rn(g, g)));
    const float p_dec = __fmul_rn(p, c.decay);
    const float denom = __fadd_rn(__fdiv_rn(__fsqrt_rn(v_new), c.bc2_sqrt), c.eps);
    const float update = __fdiv_rn(__fmul_rn(c.step_size, m_new), denom);
    p = __fsub_rn(p_dec, update);
    m = m_new;
    v = v_new;
}

// The bf16 results go to this rank's parameter buffer, or (GATHER) to every
// rank's: the all-gather done by peer stores in the same pass that computes
// the values.  A compile-time choice, so that the single-buffer kernels keep
// their register allocation.
template <bool GATHER>
__device__ __forceinline__ void store_params8(const LaunchArgs& a, int64_t go, uint4 q) {
    if constexpr (!GATHER) {
        __stcs(reinterpret_cast<uint4*>(a.param_out + go), q);
    } else {
#pragma unroll 1
        for (int d = 0; d < a.n_targets; ++d) __stcs(reinterpret_cast<uint4*>(a.targets[d] + go), q);
    }
}

template <bool GATHER>
__device__ __forceinline__ void store_param1(const LaunchArgs& a, int64_t go, uint16_t u) {
    if constexpr (!GATHER) {
        a.param_out[go] = u;
    } else {
#pragma unroll 1
        for (int d = 0; d < a.n_targets; ++d) a.targets[d][go] = u;
    }
}

// Left fold of W replicas for 8 consecutive owned elements at `off`.  The
// loads of one group of G replicas are all issued before the first add.
template <int CAP, int G>
__device__ __forceinline__ void fold8(const GradPtrs<CAP>& gp, int W, int64_t off, float s[8]) {
    uint4 q[G];
#pragma unroll
    for (int j = 0; j < G; ++j)
        if (j < W) q[j] = ld_grad16(gp.p[j] + off);
    unpack8(q[0], s);
#pragma unroll
    for (int j = 1; j < G; ++j)
        if (j < W) add8(q[j], s);
    if constexpr (CAP > G && CAP <= 2 * G) {
        // At most one more group (W = 9 .. 16): its replica indices are
        // compile-time constants, so the pointer array stays in the
        // parameter bank (a runtime index made the compiler copy it to
        // local memory, 128 bytes per thread) and the loads of both groups
        // can be issued together.
        if (W > G) {
#pragma unroll
            for (int j = 0; j < G; ++j)
                if (G + j < W) q[j] = ld_grad16(gp.p[G + j] + off);
#pragma unroll
            for (int j = 0; j < G; ++j)
                if (G + j < W) add8(q[j], s);
        }
    } else if constexpr (CAP > G) {
        for (int w0 = G; w0 < W; w0 += G) {
#pragma unroll
            for (int j = 0; j < G; ++j)
                if (w0 + j < W) q[j] = ld_grad16(gp.p[w0 + j] + off);
#pragma unroll
            for (int j = 0; j < G; ++j)
                if (w0 + j < W) add8(q[j], s);
        }
    }
}

template <int CAP>
__device__ __forceinline__ float fold1(const GradPtrs<CAP>& gp, int W, int64_t off) {
    float s = bf16_1(ld_grad2(gp.p[0] + off));
    if constexpr (CAP <= 16) {
#pragma unroll
        for (int w = 1; w < CAP; ++w)
            if (w < W) s = __fadd_rn(s, bf16_1(ld_grad2(gp.p[w] + off)));
    } else {
        for (int w = 1; w < W; ++w) s = __fadd_rn(s, bf16_1(ld_grad2(gp.p[w] + off)));
    }
    return s;
}

// Deterministic block sum of one double per thread (fixed shuffle tree, then
// warp partials in order).
__device__ double block_sum(double x) {
    __shared__ double warp_part[kThreads / 32];
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) x += __shfl_down_sync(0xFFFFFFFFu, x, d);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) warp_part[warp] = x;
    __syncthreads();
    double total = 0.0;
    if (threadIdx.x == 0) {
        for (int w = 0; w < kThreads / 32; ++w) total += warp_part[w];
    }
    return total;   // valid in thread 0
}

// ---------------------------------------------------------------------------
// the clip's sum of squares, in a fixed order
// ---------------------------------------------------------------------------

// Sum of count doubles at p by one 128-thread CTA, in a fixed order: thread
// t adds p[t], p[t + 128], p[t + 256], ... in turn (loads of eight issued
// before their additions), then block_sum.  L2 loads: the values were
// written by other CTAs of this or an earlier launch.  Valid in thread 0.
__device__ double fixed_sum128(const double* p, int32_t count) {
    double x = 0.0;
    for (int32_t i0 = threadIdx.x; i0 < count; i0 += 8 * kThreads) {
        double v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = (i0 + k * kThreads < count) ? __ldcg(p + i0 + k * kThreads) : 0.0;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (i0 + k * kThreads < count) x += v[k];
    }
    return block_sum(x);
}

// This rank's S_r is final: store it, and from all ranks' entries (summed in
// rank order) the clip coefficient min(1, max_norm / (sqrt(S) + 1e-6)).
__device__ void clip_coefficient(const ClipArgs& c, double own) {
    if (c.sumsq_out) *c.sumsq_out = own;
    if (c.partials_all) {
        c.partials_all[c.rank] = own;
        double S = c.partials_all[0];
        for (int32_t w = 1; w < c.world_size; ++w) S += c.partials_all[w];
        const double coef = static_cast<double>(c.max_norm) / (sqrt(S) + 1e-6);
        *c.coef_out = static_cast<float>(coef < 1.0 ? coef : 1.0);
    }
}

// CTA g of the combine: group g's total to group_sums[g]; the CTA that
// finishes last then sums the groups and forms the coefficient.  "Last" is
// decided by an atomic ticket after a memory fence (publish, then count);
// no CTA ever waits for another, and the last one resets the counter for
// the next launch.
__device__ void clip_group_done(const ClipArgs& c, int32_t g) {
    __shared__ int s_last;
    const int32_t n_groups = clip_groups(c.n_tiles);
    const int32_t first = g * kClipGroupTiles;
    const double T = fixed_sum128(c.tile_partials + first, min(kClipGroupTiles, c.n_tiles - first));
    if (threadIdx.x == 0) {
        c.group_sums[g] = T;
        __threadfence();
        const uint32_t prev = atomicAdd(c.ticket, 1u);
        s_last = prev == static_cast<uint32_t>(n_groups - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const double own = fixed_sum128(c.group_sums, n_groups);
    if (threadIdx.x == 0) {
        *c.ticket = 0u;
        clip_coefficient(c, own);
    }
}

// ---------------------------------------------------------------------------
// the tile kernel
// ---------------------------------------------------------------------------

template <int CAP, int G, Pass PASS, bool G_FROM_SCRATCH, bool WRITE_G, bool DEV_SCALARS, bool GATHER>
__global__ void __launch_bounds__(kThreads)
zr_tile_kernel(const GradPtrs<CAP> gp, const LaunchArgs a) {
    // Launched as a programmatic dependent of the previous kernel on the
    // stream (see launch_one): this grid may be scheduled while that one
    // drains, and waits here until it has completed and its writes are
    // visible -- before touching any memory (the previous kernel may be the
    // last step, which wrote master / m / v, or checked mode's table check).
    // Then it lets the next launch be scheduled as its own last CTAs run.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int32_t tix = a.reverse ? a.n_tiles - 1 - static_cast<int32_t>(blockIdx.x)
                                  : static_cast<int32_t>(blockIdx.x);
    const Tile tile = a.tiles[tix];
    const int W = a.world_size;
    AdamScalars sc = a.s;
    if constexpr (DEV_SCALARS) sc = *a.dev_scalars;   // computed on the device for this step
    float coef = 1.0f;
    if constexpr (PASS == Pass::kStepClip) coef = *a.clip_coef;
    double sq = 0.0;

    if (tile.flags & kTileVector) {
        for (int e = threadIdx.x * 8; e < tile.len; e += kThreads * 8) {
            const int64_t o = tile.owned + e;
            float g[8];
            float4 p0, p1, m0, m1, v0, v1;
            constexpr bool kUpdate = PASS == Pass::kStep || PASS == Pass::kStepClip;
            // Small W: state loads go out with the gradient loads.  Large W:
            // the fold alone keeps enough bytes in flight, and deferring the
            // state loads frees 24 registers across it.
            constexpr bool kEarlyState = kUpdate && (CAP <= 16 || G_FROM_SCRATCH);
            if constexpr (kEarlyState) {
                p0 = ld_state16(a.master + o); p1 = ld_state16(a.master + o + 4);
                m0 = ld_state16(a.m + o);      m1 = ld_state16(a.m + o + 4);
                v0 = ld_state16(a.v + o);      v1 = ld_state16(a.v + o + 4);
            }
            if constexpr (G_FROM_SCRATCH) {
                const float4 g0 = ld_state16(a.g_buf + o), g1 = ld_state16(a.g_buf + o + 4);
                g[0] = g0.x; g[1] = g0.y; g[2] = g0.z; g[3] = g0.w;
                g[4] = g1.x; g[5] = g1.y; g[6] = g1.z; g[7] = g1.w;
            } else {
                fold8<CAP, G>(gp, W, o, g);
#pragma unroll
                for (int k = 0; k < 8; ++k) g[k] = average(g[k], a);
            }
            if constexpr (PASS == Pass::kReduceOnly || WRITE_G) {
                st_state16(a.g_buf + o, make_float4(g[0], g[1], g[2], g[3]));
                st_state16(a.g_buf + o + 4, make_float4(g[4], g[5], g[6], g[7]));
            }
            if constexpr (PASS == Pass::kSumsq) {
#pragma unroll
                for (int k = 0; k < 8; ++k) sq += static_cast<double>(g[k]) * static_cast<double>(g[k]);
            }
            if constexpr (kUpdate) {
                if constexpr (!kEarlyState) {
                    p0 = ld_state16(a.master + o); p1 = ld_state16(a.master + o + 4);
                    m0 = ld_state16(a.m + o);      m1 = ld_state16(a.m + o + 4);
                    v0 = ld_state16(a.v + o);      v1 = ld_state16(a.v + o + 4);
                }
                if constexpr (PASS == Pass::kStepClip) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) g[k] = __fmul_rn(g[k], coef);
                }
                float p[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                float mm[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
                float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
                for (int k = 0; k < 8; ++k) adamw(sc, g[k], p[k], mm[k], vv[k]);
                st_state16(a.master + o, make_float4(p[0], p[1], p[2], p[3]));
                st_state16(a.master + o + 4, make_float4(p[4], p[5], p[6], p[7]));
                st_state16(a.m + o, make_float4(mm[0], mm[1], mm[2], mm[3]));
                st_state16(a.m + o + 4, make_float4(mm[4], mm[5], mm[6], mm[7]));
                st_state16(a.v + o, make_float4(vv[0], vv[1], vv[2], vv[3]));
                st_state16(a.v + o + 4, make_float4(vv[4], vv[5], vv[6], vv[7]));
                const int64_t go = tile.global + e;
                if (tile.flags & kTileStoreVector) {
                    uint4 q;
                    q.x = pack_bf16x2(p[0], p[1]);
                    q.y = pack_bf16x2(p[2], p[3]);
                    q.z = pack_bf16x2(p[4], p[5]);
                    q.w = pack_bf16x2(p[6], p[7]);
                    store_params8<GATHER>(a, go, q);
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        __nv_bfloat16 h = __float2bfloat16_rn(p[k]);
                        uint16_t u;
                        memcpy(&u, &h, 2);
                        store_param1<GATHER>(a, go + k, u);
                    }
                }
            }
        }
    } else {
        // Ragged tile: one element per thread.
        for (int e = threadIdx.x; e < tile.len; e += kThreads) {
            const int64_t o = tile.owned + e;
            float g;
            if constexpr (G_FROM_SCRATCH) g = a.g_buf[o];
            else g = average(fold1<CAP>(gp, W, o), a);
            if constexpr (PASS == Pass::kReduceOnly || WRITE_G) a.g_buf[o] = g;
            if constexpr (PASS == Pass::kSumsq) sq += static_cast<double>(g) * static_cast<double>(g);
            if constexpr (PASS == Pass::kStep || PASS == Pass::kStepClip) {
                if constexpr (PASS == Pass::kStepClip) g = __fmul_rn(g, coef);
                float p = a.master[o], mm = a.m[o], vv = a.v[o];
                adamw(sc, g, p, mm, vv);
                a.master[o] = p;
                a.m[o] = mm;
                a.v[o] = vv;
                __nv_bfloat16 h = __float2bfloat16_rn(p);
                uint16_t u;
                memcpy(&u, &h, 2);
                store_param1<GATHER>(a, tile.global + e, u);
            }
        }
    }
    if constexpr (PASS == Pass::kSumsq) {
        const double total = block_sum(sq);
        if (threadIdx.x == 0) a.tile_partials[tile.index] = total;
    }
}

// S_r and the coefficient from the per-tile partials of pass 1: CTA g sums
// group g, the last to finish sums the groups (clip_group_done).  Launched
// as a programmatic dependent of pass 1 (it waits for it here) and lets
// pass 2 be scheduled while it runs.
__global__ void __launch_bounds__(kThreads) zr_clip_combine_kernel(const ClipArgs c) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    clip_group_done(c, static_cast<int32_t>(blockIdx.x));
}

// The same sums for a plan of at most kSmallCombineGroups groups, in one CTA
// of 128 threads per group: threads 128g .. 128g + 127 sum group g exactly as
// fixed_sum128 does (a named barrier per group in place of the block-wide
// one), the group totals meet in shared memory, and the first 128 threads
// sum them in the same fixed order -- the same additions in the same order
// as the grid, without the fence, the ticket and the second trip to L2.
constexpr int kSmallCombineGroups = 8;

__device__ __forceinline__ void group_bar(int g) {
    asm volatile("bar.sync %0, %1;" :: "r"(g + 1), "r"(kThreads) : "memory");
}

__global__ void __launch_bounds__(kThreads * kSmallCombineGroups) zr_clip_combine_small_kernel(const ClipArgs c) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    __shared__ double warp_part[kSmallCombineGroups * (kThreads / 32)];
    __shared__ double group_total[kSmallCombineGroups];
    const int g = static_cast<int>(threadIdx.x) / kThreads;
    const int t = static_cast<int>(threadIdx.x) % kThreads;
    const int lane = t & 31, warp = t >> 5;
    const int32_t n_groups = clip_groups(c.n_tiles);
    // Group g's partials: thread t adds p[t], p[t + 128], ... (eight loads in
    // flight), then the shuffle tree and the four warp totals in order.
    const int32_t first = g * kClipGroupTiles;
    const int32_t count = min(kClipGroupTiles, c.n_tiles - first);
    double x = 0.0;
    for (int32_t i0 = t; i0 < count; i0 += 8 * kThreads) {
        double v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            v[k] = (i0 + k * kThreads < count) ? __ldcg(c.tile_partials + first + i0 + k * kThreads) : 0.0;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (i0 + k * kThreads < count) x += v[k];
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) x += __shfl_down_sync(0xFFFFFFFFu, x, d);
    if (lane == 0) warp_part[g * (kThreads / 32) + warp] = x;
    group_bar(g);
    if (t == 0) {
        double total = 0.0;
        for (int w = 0; w < kThreads / 32; ++w) total += warp_part[g * (kThreads / 32) + w];
        group_total[g] = total;
    }
    __syncthreads();
    if (g != 0) return;
    // The group totals, by threads 0..127 in the same fixed order.
    double y = t < n_groups ? 0.0 + group_total[t] : 0.0;
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) y += __shfl_down_sync(0xFFFFFFFFu, y, d);
    if (lane == 0) warp_part[warp] = y;
    group_bar(0);
    if (t == 0) {
        double own = 0.0;
        for (int w = 0; w < kThreads / 32; ++w) own += warp_part[w];
        clip_coefficient(c, own);
    }
}

// Every fp32 bit pattern s through average() for one W, against IEEE
// division: the count of results whose bits differ (NaN against NaN counts
// as equal).
__global__ void __launch_bounds__(kThreads) zr_average_check_kernel(const LaunchArgs a,
                                                                   unsigned long long* mismatches) {
    const float w = static_cast<float>(a.world_size);
    unsigned long long bad = 0;
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * kThreads;
    for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * kThreads + threadIdx.x; i < (1ull << 32); i += stride) {
        const float s = __uint_as_float(static_cast<uint32_t>(i));
        const float got = average(s, a);
        const float want = __fdiv_rn(s, w);
        if (__float_as_uint(got) != __float_as_uint(want) && !(got != got && want != want)) ++bad;
    }
    if (bad) atomicAdd(mismatches, bad);
}

// Launch configuration for a programmatic dependent launch: the grid may be
// scheduled while the previous kernel on the stream drains (the kernel's
// first instruction, griddepcontrol.wait, holds it until that kernel has
// completed and its writes are visible).  Copies, memsets and event waits
// before it keep their full ordering.
struct PdlLaunch {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    PdlLaunch(unsigned grid, cudaStream_t stream) {
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = stream;
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
};

template <int CAP, int G, Pass PASS, bool FROM, bool WRITE, bool DEVSC, bool GATHER>
cudaError_t launch_one(const LaunchArgs& a, const void* const* grad_ptrs, cudaStream_t stream) {
    // grad_ptrs may be NULL for the pass that reads the g scratch instead.
    GradPtrs<CAP> gp;
    for (int w = 0; w < CAP; ++w)
        gp.p[w] = (grad_ptrs != nullptr && w < a.world_size) ? static_cast<const uint16_t*>(grad_ptrs[w]) : nullptr;
    // Programmatic dependent launch: back-to-back steps lose less to the
    // launch gap.
    PdlLaunch l(static_cast<unsigned>(a.n_tiles), stream);
    return cudaLaunchKernelEx(&l.cfg, zr_tile_kernel<CAP, G, PASS, FROM, WRITE, DEVSC, GATHER>, gp, a);
}

template <Pass PASS, bool FROM, bool WRITE, bool DEVSC = false, bool GATHER = false>
cudaError_t dispatch_w(const LaunchArgs& a, const void* const* grad_ptrs, cudaStream_t stream) {
    if constexpr (FROM) {
        return launch_one<1, 1, PASS, FROM, WRITE, DEVSC, GATHER>(a, grad_ptrs, stream);
    } else {
        const int W = a.world_size;
        if (W <= 2) return launch_one<2, 2, PASS, FROM, WRITE, DEVSC, GATHER>(a, grad_ptrs, stream);
        if (W <= 4) return launch_one<4, 4, PASS, FROM, WRITE, DEVSC, GATHER>(a, grad_ptrs, stream);
        if (W <= 8) return launch_one<8, 8, PASS, FROM, WRITE, DEVSC, GATHER>(a, grad_ptrs, stream);
        if (W <= 16) return launch_one<16, 8, PASS, FROM, WRITE, DEVSC, GATHER>(a, grad_ptrs, stream);
        if (W <= 64) return launch_one<64, 8, PASS, FROM, WRITE, DEVSC, GATHER>(a, grad_ptrs, stream);
        return launch_one<ZR_MAX_WORLD_SIZE, 8, PASS, FROM, WRITE, DEVSC, GATHER>(a, grad_ptrs, stream);
    }
}

// The passes that write parameters, with the device-scalar and gather-target
// variants chosen from the launch arguments.
template <Pass PASS, bool FROM>
cudaError_t dispatch_update(const LaunchArgs& a, const void* const* grad_ptrs, cudaStream_t s) {
    const bool dev = a.dev_scalars != nullptr, gather = a.n_targets > 0;
    if (dev && gather) return dispatch_w<PASS, FROM, false, true, true>(a, grad_ptrs, s);
    if (dev) return dispatch_w<PASS, FROM, false, true, false>(a, grad_ptrs, s);
    if (gather) return dispatch_w<PASS, FROM, false, false, true>(a, grad_ptrs, s);
    return dispatch_w<PASS, FROM, false, false, false>(a, grad_ptrs, s);
}

}  // namespace

int launch_tiles(Pass pass, const LaunchArgs& a, const void* const* grad_ptrs, bool g_from_scratch,
                 bool write_g_scratch, void* stream_v) {
    if (a.n_tiles == 0) return cudaSuccess;
    cudaStream_t s = static_cast<cudaStream_t>(stream_v);
    switch (pass) {
        case Pass::kStep: return dispatch_update<Pass::kStep, false>(a, grad_ptrs, s);
        case Pass::kReduceOnly: return dispatch_w<Pass::kReduceOnly, false, false>(a, grad_ptrs, s);
        case Pass::kSumsq:
            return write_g_scratch ? dispatch_w<Pass::kSumsq, false, true>(a, grad_ptrs, s)
                                   : dispatch_w<Pass::kSumsq, false, false>(a, grad_ptrs, s);
        case Pass::kStepClip:
            return g_from_scratch ? dispatch_update<Pass::kStepClip, true>(a, grad_ptrs, s)
                                  : dispatch_update<Pass::kStepClip, false>(a, grad_ptrs, s);
    }
    return cudaErrorInvalidValue;
}

int launch_clip_combine(const ClipArgs& c, void* stream_v) {
    if (c.n_tiles <= 0) return cudaSuccess;
    const int32_t n_groups = clip_groups(c.n_tiles);
    if (n_groups <= kSmallCombineGroups) {
        PdlLaunch l(1u, static_cast<cudaStream_t>(stream_v));
        l.cfg.blockDim = dim3(static_cast<unsigned>(kThreads * n_groups));
        return cudaLaunchKernelEx(&l.cfg, zr_clip_combine_small_kernel, c);
    }
    PdlLaunch l(static_cast<unsigned>(n_groups), static_cast<cudaStream_t>(stream_v));
    return cudaLaunchKernelEx(&l.cfg, zr_clip_combine_kernel, c);
}

int launch_average_check(int32_t w_first, int32_t w_last, unsigned long long* mismatches, void* stream_v) {
    cudaStream_t s = static_cast<cudaStream_t>(stream_v);
    const int n = w_last - w_first + 1;
    cudaError_t e = cudaMemsetAsync(mismatches, 0, sizeof(unsigned long long) * n, s);
    if (e != cudaSuccess) return e;
    for (int32_t W = w_first; W <= w_last; ++W) {
        LaunchArgs a{};
        set_world_size(a, W);
        zr_average_check_kernel<<<148 * 32, kThreads, 0, s>>>(a, mismatches + (W - w_first));
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace zr
