// ZeRO-3 parameter gather: whole tensors assembled from every rank's bf16
// shard ("Scaling training to thousands of GPUs", talk summary, section
// 11:24 ZeRO; "CS336 lecture 8", section "ZeRO levels": stage 3 all-gathers
// a layer's parameters just before the layer runs).
//
// A pure copy, so the roofline is memory bandwidth: 2 bytes read from the
// owner's shard and 2 written per element -- over NVLink for the elements
// other GPUs own, when the shard pointers are peer mappings.  One CTA per
// piece (at most 16384 elements of one tensor from one owner, a 32 KB run):
// enough CTAs for one transformer layer to cover the 148 SMs several times,
// and each CTA fetches its own data with plain loads (no TMA, no multicast).
// A caller prefetching under compute may cap the grid so the gather runs
// beside the compute on a few SMs instead of taking all of them.
#include <cuda_runtime.h>

#include <cstdint>

#include "zr_internal.hpp"

namespace zr {
namespace {

template <int CAP>
struct ShardPtrs {
    const uint16_t* p[CAP];
};

constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 8;   // 16-byte vectors in flight per thread (4: 0.97, 16: 0.96 of the copy peak)

// One piece: source and destination share their offset modulo 16 bytes --
// a scalar head brings both to a 16-byte boundary, then 16-byte vectors
// (the loads of kGatherUnroll of them issued before their stores), then a
// scalar tail; otherwise element by element.  Loads and stores carry the
// streaming (evict-first) hint: the gathered bytes are used once, by the
// layer that runs next, and should not push that layer's working set out
// of L2 while a prefetch overlaps it.
__device__ __forceinline__ void copy_piece(const uint16_t* src, uint16_t* out, int32_t len) {
    const uintptr_t sa = reinterpret_cast<uintptr_t>(src), da = reinterpret_cast<uintptr_t>(out);
    if (((sa ^ da) & 15u) != 0) {
        for (int32_t i = threadIdx.x; i < len; i += kGatherThreads) __stcs(out + i, __ldcs(src + i));
        return;
    }
    int32_t head = static_cast<int32_t>(((16u - (da & 15u)) & 15u) >> 1);   // 0..7 elements
    if (head > len) head = len;
    if (static_cast<int32_t>(threadIdx.x) < head) __stcs(out + threadIdx.x, __ldcs(src + threadIdx.x));
    const int32_t nvec = (len - head) >> 3;
    const uint4* s4 = reinterpret_cast<const uint4*>(src + head);
    uint4* d4 = reinterpret_cast<uint4*>(out + head);
    for (int32_t v0 = threadIdx.x; v0 < nvec; v0 += kGatherThreads * kGatherUnroll) {
        uint4 q[kGatherUnroll];
#pragma unroll
        for (int k = 0; k < kGatherUnroll; ++k) {
            const int32_t v = v0 + k * kGatherThreads;
            if (v < nvec) q[k] = __ldcs(s4 + v);
        }
#pragma unroll
        for (int k = 0; k < kGatherUnroll; ++k) {
            const int32_t v = v0 + k * kGatherThreads;
            if (v < nvec) __stcs(d4 + v, q[k]);
        }
    }
    for (int32_t i = head + (nvec << 3) + threadIdx.x; i < len; i += kGatherThreads)
        __stcs(out + i, __ldcs(src + i));
}

// CTA b copies pieces b, b + gridDim.x, ...: one CTA per piece at full
// speed, or a capped grid that leaves the other SMs to concurrent work.
template <int CAP>
__global__ void __launch_bounds__(kGatherThreads)
zr_gather_kernel(const ShardPtrs<CAP> sp, const GatherPiece* __restrict__ pieces, int32_t first, int32_t n,
                 uint16_t* dst, int64_t dst_base) {
    // Launched as a programmatic dependent of the previous kernel on the
    // stream: scheduled while that kernel drains, it waits here until that
    // kernel has completed and its writes are visible (it may be the step
    // that wrote the shards, or the layer that read the slot about to be
    // overwritten), then lets the next launch be scheduled.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    for (int32_t k = blockIdx.x; k < n; k += gridDim.x) {
        const GatherPiece pc = pieces[first + k];
        copy_piece(sp.p[pc.owner] + pc.src, dst + (pc.dst - dst_base), pc.len);
    }
}

template <int CAP>
cudaError_t launch_gather_cap(const GatherPiece* pieces, int32_t first, int32_t n, int32_t ctas, int32_t world_size,
                              const void* const* shard_ptrs, uint16_t* dst, int64_t dst_base, cudaStream_t s) {
    ShardPtrs<CAP> sp;
    for (int w = 0; w < CAP; ++w)
        sp.p[w] = w < world_size ? static_cast<const uint16_t*>(shard_ptrs[w]) : nullptr;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3(static_cast<unsigned>(ctas));
    cfg.blockDim = dim3(kGatherThreads);
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, zr_gather_kernel<CAP>, sp, pieces, first, n, dst, dst_base);
}

}  // namespace

int launch_gather(const GatherPiece* pieces, int32_t first, int32_t n, int32_t max_ctas, int32_t world_size,
                  const void* const* shard_ptrs, uint16_t* dst, int64_t dst_base, void* stream_v) {
    if (n == 0) return cudaSuccess;
    cudaStream_t s = static_cast<cudaStream_t>(stream_v);
    const int32_t ctas = (max_ctas > 0 && max_ctas < n) ? max_ctas : n;
    if (world_size <= 8)
        return launch_gather_cap<8>(pieces, first, n, ctas, world_size, shard_ptrs, dst, dst_base, s);
    if (world_size <= 64)
        return launch_gather_cap<64>(pieces, first, n, ctas, world_size, shard_ptrs, dst, dst_base, s);
    return launch_gather_cap<ZR_MAX_WORLD_SIZE>(pieces, first, n, ctas, world_size, shard_ptrs, dst, dst_base, s);
}

}  // namespace zr
