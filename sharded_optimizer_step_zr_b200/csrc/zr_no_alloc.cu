// zr_step_no_alloc: the optimizer step for callers that cannot allocate
// device memory.
//
// zr_step needs a caller-allocated workspace for its tile table and, when
// clipping, its per-tile sums of squares.  Some callers cannot provide one:
// a plug-in running inside a host framework whose allocator owns all of the
// GPU's memory (a caching allocator that has reserved it, or a framework
// that forbids outside cudaMalloc calls), or a latency-critical loop that
// must not call cudaMalloc because it can synchronise the device.  They have
// their inputs and outputs, but nowhere to put scratch.  For them this entry
// point keeps its scratch in a fixed-size array that is part of the library
// image: every GPU that loads libzr.so holds ZR_NO_ALLOC_SCRATCH_BYTES of it
// until the process exits.  The kernels it runs are zr_step's own; with
// clipping, the second pass re-reads the gradients instead of keeping an
// fp32 copy of the averaged gradient (results are identical, as the fold is
// deterministic).
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "zr_internal.hpp"

namespace {

// The scratch shared by every call on a device.  In host code this name is
// only a host-side stand-in for the device array; kernels receive the
// device address obtained with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char zr_no_alloc_scratch[ZR_NO_ALLOC_SCRATCH_BYTES];

// Per device: the array's device address (looked up once), and which plan's
// tile table the array holds now (that plan's uid and table generation), so
// a loop stepping one plan uploads its table once, not on every call.
struct DeviceScratch {
    void* address = nullptr;
    uint64_t plan_uid = 0;          // 0: no table uploaded yet
    uint64_t table_generation = 0;
};
constexpr int kMaxDevices = 256;
DeviceScratch g_device[kMaxDevices];
std::mutex g_mutex;

struct ScratchLayout {
    uint64_t tiles, tile_partials, ticket, group_sums, clip_coef, own_sumsq, total;
};

uint64_t up256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

ScratchLayout scratch_layout(uint64_t n_tiles, bool clip) {
    const uint64_t groups = clip ? static_cast<uint64_t>(zr::clip_groups(static_cast<int32_t>(n_tiles))) : 0;
    ScratchLayout L{};
    uint64_t off = 0;
    L.tiles = off;
    off = up256(off + sizeof(zr::Tile) * n_tiles);
    L.tile_partials = off;
    off = up256(off + (clip ? sizeof(double) * n_tiles : 0));
    L.ticket = off;
    off = up256(off + (clip ? sizeof(uint32_t) : 0));
    L.group_sums = off;
    off = up256(off + sizeof(double) * groups);
    L.clip_coef = off;
    off = up256(off + sizeof(float));
    L.own_sumsq = off;
    off = up256(off + sizeof(double));
    L.total = off;
    return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" zr_status zr_step_no_alloc(const zr_plan* p, const void* const* grad_ptrs, float* master,
                                      float* m, float* v, void* param_out, double* d_sumsq_partials,
                                      int64_t step, zr_stream_t stream) {
    if (!p || step < 1) return ZR_ERR_INVALID_ARG;
    if (p->owned_numel() == 0) return ZR_OK;
    if (!grad_ptrs || !master || !m || !v || !param_out) return ZR_ERR_INVALID_ARG;
    for (int32_t w = 0; w < p->world_size; ++w) {
        if (!grad_ptrs[w]) return ZR_ERR_INVALID_ARG;
        if (!aligned16(grad_ptrs[w])) return ZR_ERR_ALIGNMENT;
    }
    if (!aligned16(master) || !aligned16(m) || !aligned16(v) || !aligned16(param_out)) return ZR_ERR_ALIGNMENT;
    const bool clip = p->clip_enabled();
    if (clip) {
        if (!d_sumsq_partials) return ZR_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(d_sumsq_partials) & 7u) != 0) return ZR_ERR_ALIGNMENT;
    }
    // Size check before any CUDA call: the plan's tables must fit the array.
    const ScratchLayout L = scratch_layout(p->tiles.size(), clip);
    if (L.total > ZR_NO_ALLOC_SCRATCH_BYTES) return ZR_ERR_UNSUPPORTED;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ZR_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ZR_ERR_UNSUPPORTED;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return ZR_ERR_CUDA;
    if (major != 10) return ZR_ERR_UNSUPPORTED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    char* base = nullptr;
    zr::Tile* d_tiles = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        DeviceScratch& ds = g_device[dev];
        if (ds.address == nullptr) {
            // Set-up on this device's first call: the array's device address.
            void* addr = nullptr;
            const cudaError_t e = cudaGetSymbolAddress(&addr, zr_no_alloc_scratch);
            if (e != cudaSuccess || addr == nullptr) return ZR_ERR_CUDA;
            ds.address = addr;
        }
        base = static_cast<char*>(ds.address);
        d_tiles = reinterpret_cast<zr::Tile*>(base + L.tiles);
        // The tile table, unless this plan's current table is the one the
        // array already holds (the host-to-device copy from the plan's host
        // memory happens once per plan and table, not once per step).
        if (ds.plan_uid != p->uid || ds.table_generation != p->table_generation) {
            ds.plan_uid = 0;   // stays unset if the copy cannot be enqueued
            if (cudaMemcpyAsync(d_tiles, p->tiles.data(), sizeof(zr::Tile) * p->tiles.size(),
                                cudaMemcpyHostToDevice, s) != cudaSuccess)
                return ZR_ERR_CUDA;
            ds.plan_uid = p->uid;
            ds.table_generation = p->table_generation;
        }
    }

    zr::LaunchArgs a{};
    a.tiles = d_tiles;
    a.n_tiles = static_cast<int32_t>(p->tiles.size());
    zr::set_world_size(a, p->world_size);
    a.master = master;
    a.m = m;
    a.v = v;
    a.param_out = static_cast<uint16_t*>(param_out);
    a.s = zr::adam_scalars(p->hp, step);
    if (!clip)
        return zr::launch_tiles(zr::Pass::kStep, a, grad_ptrs, false, false, s) == cudaSuccess ? ZR_OK : ZR_ERR_CUDA;

    // The combine's completion counter must start at zero: cleared on every
    // call (a device-side memset, no host copy).  Every other scratch word
    // the kernels read is written earlier in this call (one partial per
    // tile, the group totals, the coefficient).
    uint32_t* d_ticket = reinterpret_cast<uint32_t*>(base + L.ticket);
    if (cudaMemsetAsync(d_ticket, 0, sizeof(uint32_t), s) != cudaSuccess) return ZR_ERR_CUDA;
    float* d_coef = reinterpret_cast<float*>(base + L.clip_coef);
    a.tile_partials = reinterpret_cast<double*>(base + L.tile_partials);
    if (zr::launch_tiles(zr::Pass::kSumsq, a, grad_ptrs, false, false, s) != cudaSuccess) return ZR_ERR_CUDA;
    zr::ClipArgs c{};
    c.tile_partials = a.tile_partials;
    c.n_tiles = a.n_tiles;
    c.world_size = p->world_size;
    c.ticket = d_ticket;
    c.group_sums = reinterpret_cast<double*>(base + L.group_sums);
    c.partials_all = d_sumsq_partials;
    c.sumsq_out = reinterpret_cast<double*>(base + L.own_sumsq);
    c.coef_out = d_coef;
    c.rank = p->rank;
    c.max_norm = p->hp.max_grad_norm;
    if (zr::launch_clip_combine(c, s) != cudaSuccess) return ZR_ERR_CUDA;
    a.clip_coef = d_coef;
    a.reverse = 1;
    return zr::launch_tiles(zr::Pass::kStepClip, a, grad_ptrs, false, false, s) == cudaSuccess ? ZR_OK : ZR_ERR_CUDA;
}
