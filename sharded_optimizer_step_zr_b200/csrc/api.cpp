// C ABI of the fused sharded optimizer step (declared in include/zr.h).
//
// This layer validates arguments, holds the host-side plan, binds the
// caller's device workspace and enqueues the kernels.  It never allocates
// device memory, and the step, gather and check calls never synchronise;
// zr_plan_set_gather_targets and zr_plan_check_result synchronise their
// stream (documented in the header), and zr_step_host creates its two copy
// streams and events on first use.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <new>

#include "zr_internal.hpp"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

zr_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ZR_OK : ZR_ERR_CUDA; }

zr_status check_grads(const zr_plan* p, const void* const* grad_ptrs) {
    if (!grad_ptrs) return ZR_ERR_INVALID_ARG;
    for (int32_t w = 0; w < p->world_size; ++w) {
        if (!grad_ptrs[w]) return ZR_ERR_INVALID_ARG;
        if (!aligned16(grad_ptrs[w])) return ZR_ERR_ALIGNMENT;
    }
    return ZR_OK;
}

zr::LaunchArgs base_args(const zr_plan* p) {
    zr::LaunchArgs a{};
    a.tiles = p->d_tiles;
    a.n_tiles = static_cast<int32_t>(p->tiles.size());
    zr::set_world_size(a, p->world_size);
    a.n_targets = p->n_gather_targets;
    a.targets = p->d_gather_targets;
    return a;
}

// The clip's S_r / coefficient arguments over every tile of the plan.
zr::ClipArgs clip_args(const zr_plan* p, double* partials_all, double* sumsq_out) {
    zr::ClipArgs c{};
    c.tile_partials = p->d_tile_partials;
    c.n_tiles = static_cast<int32_t>(p->tiles.size());
    c.world_size = p->world_size;
    c.ticket = p->d_clip_ticket;
    c.group_sums = p->d_clip_group_sums;
    c.partials_all = partials_all;
    c.sumsq_out = sumsq_out;
    c.coef_out = p->d_clip_coef;
    c.rank = p->rank;
    c.max_norm = p->hp.max_grad_norm;
    return c;
}

// The bf16 destination: param_out, or the plan's gather targets (then
// param_out may be NULL).
zr_status check_param_out(const zr_plan* p, const void* param_out) {
    if (p->n_gather_targets > 0) return (param_out && !aligned16(param_out)) ? ZR_ERR_ALIGNMENT : ZR_OK;
    if (!param_out) return ZR_ERR_INVALID_ARG;
    return aligned16(param_out) ? ZR_OK : ZR_ERR_ALIGNMENT;
}

// Kernels launch on the current device; the plan's buffers belong to the
// device that was current when its workspace was bound.
zr_status check_device(const zr_plan* p) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ZR_ERR_CUDA;
    return dev == p->device ? ZR_OK : ZR_ERR_INVALID_ARG;
}

// Checked mode: verify the device tile tables before a launch that reads
// them (one kernel on the caller's stream).
zr_status verify_tables(const zr_plan* p, zr_stream_t stream) {
    zr::VerifyArgs a{};
    a.tiles = p->d_tiles;
    a.tiles_by_owned = p->d_tiles_by_owned;
    a.n_tiles = static_cast<int32_t>(p->tiles.size());
    a.n_buckets = p->n_buckets;
    a.n_owned = p->owned_numel();
    a.n_out = p->param_layout == ZR_PARAMS_OWNED ? p->owned_numel() : p->padded_numel;
    a.pieces = p->d_gather_pieces;
    a.n_pieces = static_cast<int32_t>(p->gather_pieces.size());
    a.world_size = p->world_size;
    a.total_numel = p->total_numel;
    a.n_tensors = p->n_tensors;
    a.hash_tiles = p->hash_tiles;
    a.hash_by_owned = p->hash_tiles_by_owned;
    a.hash_pieces = p->hash_gather_pieces;
    a.check = p->d_check;
    return cuda_status(static_cast<cudaError_t>(zr::launch_verify_tables(a, stream)));
}

zr_status verify_if_checked(const zr_plan* p, zr_stream_t stream) {
    return p->checked ? verify_tables(p, stream) : ZR_OK;
}

// The tile tables and the gather piece table to the workspace on `stream`,
// with checked mode's reference hashes and fresh status words (no failure,
// smallest failing position all ones).
zr_status upload_tables(zr_plan* p, zr_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!p->tiles.empty()) {
        const size_t bytes_tiles = sizeof(zr::Tile) * p->tiles.size();
        if (cudaMemcpyAsync(p->d_tiles, p->tiles.data(), bytes_tiles, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(p->d_tiles_by_owned, p->tiles_by_owned.data(), bytes_tiles, cudaMemcpyHostToDevice, s) !=
                cudaSuccess)
            return ZR_ERR_CUDA;
    }
    if (!p->gather_pieces.empty() &&
        cudaMemcpyAsync(p->d_gather_pieces, p->gather_pieces.data(), sizeof(zr::GatherPiece) * p->gather_pieces.size(),
                        cudaMemcpyHostToDevice, s) != cudaSuccess)
        return ZR_ERR_CUDA;
    p->hash_tiles = zr::table_hash(p->tiles);
    p->hash_tiles_by_owned = zr::table_hash(p->tiles_by_owned);
    p->hash_gather_pieces = zr::table_hash(p->gather_pieces);
    if (cudaMemsetAsync(p->d_check, 0, sizeof(uint64_t) * zr::kCheckWords, s) != cudaSuccess ||
        cudaMemsetAsync(p->d_check + 1, 0xFF, sizeof(uint64_t), s) != cudaSuccess)
        return ZR_ERR_CUDA;
    // The clip's completion counter starts at zero (each combine leaves it
    // at zero again).
    if (p->d_clip_ticket && cudaMemsetAsync(p->d_clip_ticket, 0, sizeof(uint32_t), s) != cudaSuccess)
        return ZR_ERR_CUDA;
    return ZR_OK;
}

zr_status check_state(const float* master, const float* m, const float* v) {
    if (!master || !m || !v) return ZR_ERR_INVALID_ARG;
    if (!aligned16(master) || !aligned16(m) || !aligned16(v)) return ZR_ERR_ALIGNMENT;
    return ZR_OK;
}

void release_host_pipeline(const zr_plan* p) {
    for (cudaEvent_t& e : p->host_events) {
        if (e) cudaEventDestroy(e);
        e = nullptr;
    }
    if (p->h2d_stream) cudaStreamDestroy(p->h2d_stream);
    if (p->d2h_stream) cudaStreamDestroy(p->d2h_stream);
    p->h2d_stream = p->d2h_stream = nullptr;
    p->host_pipeline_ready = false;
}

// The copy streams and events of zr_step_host, created on first use; a
// failure part way releases what was created, so a later call starts over.
zr_status ensure_host_pipeline(const zr_plan* p) {
    if (p->host_pipeline_ready) return ZR_OK;
    bool ok = cudaStreamCreateWithFlags(&p->h2d_stream, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p->d2h_stream, cudaStreamNonBlocking) == cudaSuccess;
    for (cudaEvent_t& e : p->host_events)
        ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        release_host_pipeline(p);
        return ZR_ERR_CUDA;
    }
    p->host_pipeline_ready = true;
    return ZR_OK;
}

}  // namespace

zr_plan::~zr_plan() { release_host_pipeline(this); }

extern "C" {

const char* zr_status_string(zr_status s) {
    switch (s) {
        case ZR_OK: return "ZR_OK";
        case ZR_ERR_INVALID_ARG: return "ZR_ERR_INVALID_ARG: invalid argument";
        case ZR_ERR_ALIGNMENT: return "ZR_ERR_ALIGNMENT: device pointer not 16-byte aligned";
        case ZR_ERR_NO_WORKSPACE: return "ZR_ERR_NO_WORKSPACE: workspace (or clip partials) not bound or too small";
        case ZR_ERR_CUDA: return "ZR_ERR_CUDA: a CUDA runtime call failed";
        case ZR_ERR_UNSUPPORTED: return "ZR_ERR_UNSUPPORTED: unsupported configuration or device";
        case ZR_ERR_BUFFER_TOO_SMALL: return "ZR_ERR_BUFFER_TOO_SMALL: output array too small";
        case ZR_ERR_IO: return "ZR_ERR_IO: checkpoint file could not be read or written";
        case ZR_ERR_MISMATCH: return "ZR_ERR_MISMATCH: checkpoint of another partition, rank or step, or corrupt";
    }
    return "unknown zr_status";
}

static zr_status create_plan(int32_t n_tensors, const int32_t* ndims, const int64_t* const* shapes,
                             const int32_t* tensor_group, int32_t world_size, int32_t rank, zr_partition mode,
                             uint64_t bucket_cap_bytes, const zr_adamw* hp, zr_plan** out);

zr_status zr_plan_create(int32_t n_tensors, const int32_t* ndims, const int64_t* const* shapes,
                         int32_t world_size, int32_t rank, zr_partition mode,
                         uint64_t bucket_cap_bytes, const zr_adamw* hp, zr_plan** out) {
    return create_plan(n_tensors, ndims, shapes, nullptr, world_size, rank, mode, bucket_cap_bytes, hp, out);
}

zr_status zr_plan_create_grouped(int32_t n_tensors, const int32_t* ndims, const int64_t* const* shapes,
                                 const int32_t* tensor_group, int32_t world_size, int32_t rank,
                                 zr_partition mode, const zr_adamw* hp, zr_plan** out) {
    if (out) *out = nullptr;
    if (n_tensors > 0 && !tensor_group) return ZR_ERR_INVALID_ARG;
    for (int32_t t = 1; t < n_tensors; ++t)
        if (tensor_group[t] < tensor_group[t - 1]) return ZR_ERR_INVALID_ARG;
    // (an empty set has no buckets either way)
    return create_plan(n_tensors, ndims, shapes, tensor_group, world_size, rank, mode, 0, hp, out);
}

static zr_status create_plan(int32_t n_tensors, const int32_t* ndims, const int64_t* const* shapes,
                             const int32_t* tensor_group, int32_t world_size, int32_t rank, zr_partition mode,
                             uint64_t bucket_cap_bytes, const zr_adamw* hp, zr_plan** out) {
    if (!out) return ZR_ERR_INVALID_ARG;
    *out = nullptr;
    if (n_tensors < 0 || (n_tensors > 0 && (!ndims || !shapes)) || !hp) return ZR_ERR_INVALID_ARG;
    if (world_size < 1 || rank < 0 || rank >= world_size) return ZR_ERR_INVALID_ARG;
    if (world_size > ZR_MAX_WORLD_SIZE) return ZR_ERR_UNSUPPORTED;
    if (mode != ZR_PARTITION_FLAT && mode != ZR_PARTITION_WHOLE_TENSOR) return ZR_ERR_INVALID_ARG;
    zr_plan* p = new (std::nothrow) zr_plan();
    if (!p) return ZR_ERR_INVALID_ARG;
    static std::atomic<uint64_t> next_uid{1};
    p->uid = next_uid.fetch_add(1);
    p->world_size = world_size;
    p->rank = rank;
    p->mode = mode;
    p->cap_bytes = bucket_cap_bytes;
    p->hp = *hp;
    if (tensor_group && n_tensors > 0) p->tensor_group.assign(tensor_group, tensor_group + n_tensors);
    zr_status st;
    try {
        st = zr::build_plan(*p, n_tensors, ndims, shapes);
    } catch (...) {
        st = ZR_ERR_INVALID_ARG;
    }
    if (st != ZR_OK) {
        delete p;
        return st;
    }
    // A tile index must fit the grid's x dimension.
    if (p->tiles.size() > 0x7FFFFFFFull) {
        delete p;
        return ZR_ERR_UNSUPPORTED;
    }
    *out = p;
    return ZR_OK;
}

void zr_plan_destroy(zr_plan* plan) { delete plan; }

zr_status zr_plan_query(const zr_plan* p, int64_t* total_numel, int64_t* padded_numel,
                        int64_t* owned_numel, int32_t* n_buckets, int64_t* n_segments) {
    if (!p) return ZR_ERR_INVALID_ARG;
    if (total_numel) *total_numel = p->total_numel;
    if (padded_numel) *padded_numel = p->padded_numel;
    if (owned_numel) *owned_numel = p->owned_numel();
    if (n_buckets) *n_buckets = p->n_buckets;
    if (n_segments) *n_segments = static_cast<int64_t>(p->segments.size());
    return ZR_OK;
}

zr_status zr_plan_segments(const zr_plan* p, zr_segment* out, int64_t cap, int64_t* n) {
    if (!p || !n || cap < 0 || (cap > 0 && !out)) return ZR_ERR_INVALID_ARG;
    *n = static_cast<int64_t>(p->segments.size());
    if (*n > cap) return ZR_ERR_BUFFER_TOO_SMALL;
    if (*n) std::memcpy(out, p->segments.data(), sizeof(zr_segment) * p->segments.size());
    return ZR_OK;
}

zr_status zr_plan_workspace_bytes(const zr_plan* p, uint64_t* bytes) {
    if (!p || !bytes) return ZR_ERR_INVALID_ARG;
    *bytes = zr::workspace_layout(*p).total;
    return ZR_OK;
}

zr_status zr_plan_set_workspace(zr_plan* p, void* d_ws, uint64_t bytes, zr_stream_t stream) {
    if (!p || !d_ws) return ZR_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_ws) & 255u) != 0) return ZR_ERR_ALIGNMENT;
    const zr::WorkspaceLayout L = zr::workspace_layout(*p);
    if (bytes < L.total) return ZR_ERR_NO_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ZR_ERR_CUDA;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return ZR_ERR_CUDA;
    if (major != 10) return ZR_ERR_UNSUPPORTED;
    char* base = static_cast<char*>(d_ws);
    p->device = dev;
    p->d_workspace = d_ws;
    p->workspace_bytes = bytes;
    p->d_tiles = reinterpret_cast<zr::Tile*>(base + L.tiles);
    p->d_tiles_by_owned = reinterpret_cast<zr::Tile*>(base + L.tiles_by_owned);
    p->d_tile_partials = p->clip_enabled() ? reinterpret_cast<double*>(base + L.tile_partials) : nullptr;
    p->d_clip_ticket = p->clip_enabled() ? reinterpret_cast<uint32_t*>(base + L.clip_ticket) : nullptr;
    p->d_clip_group_sums = p->clip_enabled() ? reinterpret_cast<double*>(base + L.clip_group_sums) : nullptr;
    p->d_clip_coef = reinterpret_cast<float*>(base + L.clip_coef);
    p->d_own_sumsq = reinterpret_cast<double*>(base + L.own_sumsq);
    p->d_gather_targets = reinterpret_cast<uint16_t**>(base + L.gather_targets);
    p->d_scalars = reinterpret_cast<zr::AdamScalars*>(base + L.dev_scalars);
    p->d_check = reinterpret_cast<uint64_t*>(base + L.check);
    p->n_gather_targets = 0;
    p->d_g_scratch = p->clip_uses_scratch() ? reinterpret_cast<float*>(base + L.g_scratch) : nullptr;
    p->d_gather_pieces = reinterpret_cast<zr::GatherPiece*>(base + L.gather_pieces);
    return upload_tables(p, stream);
}

zr_status zr_plan_set_param_layout(zr_plan* p, int32_t layout, zr_stream_t stream) {
    if (!p || (layout != ZR_PARAMS_GLOBAL && layout != ZR_PARAMS_OWNED)) return ZR_ERR_INVALID_ARG;
    if (layout == ZR_PARAMS_OWNED && p->n_gather_targets > 0) return ZR_ERR_UNSUPPORTED;
    if (layout == p->param_layout) return ZR_OK;
    if (p->d_workspace) {
        const zr_status dst = check_device(p);
        if (dst != ZR_OK) return dst;
    }
    p->param_layout = layout;
    try {
        zr::build_tiles_for_layout(*p);
    } catch (...) {
        return ZR_ERR_INVALID_ARG;
    }
    return p->d_workspace ? upload_tables(p, stream) : ZR_OK;
}

zr_status zr_gather_params(const zr_plan* p, int32_t first_tensor, int32_t n_tensors, const void* const* shard_ptrs,
                           void* dst, int32_t max_ctas, zr_stream_t stream) {
    if (!p || !shard_ptrs || first_tensor < 0 || n_tensors < 0 || first_tensor > p->n_tensors - n_tensors)
        return ZR_ERR_INVALID_ARG;
    if (!p->d_workspace) return ZR_ERR_NO_WORKSPACE;
    const zr_status dst_st = check_device(p);
    if (dst_st != ZR_OK) return dst_st;
    const int32_t a = p->tensor_first_piece[first_tensor], b = p->tensor_first_piece[first_tensor + n_tensors];
    if (a == b) return ZR_OK;   // only zero-element tensors
    {
        const zr_status cs = verify_if_checked(p, stream);
        if (cs != ZR_OK) return cs;
    }
    if (!dst) return ZR_ERR_INVALID_ARG;
    if (!aligned16(dst)) return ZR_ERR_ALIGNMENT;
    for (int32_t w = 0; w < p->world_size; ++w) {
        if (p->rank_numel[w] == 0) continue;
        if (!shard_ptrs[w]) return ZR_ERR_INVALID_ARG;
        if (!aligned16(shard_ptrs[w])) return ZR_ERR_ALIGNMENT;
    }
    return cuda_status(static_cast<cudaError_t>(zr::launch_gather(p->d_gather_pieces, a, b - a, max_ctas,
                                                                  p->world_size, shard_ptrs,
                                                                  static_cast<uint16_t*>(dst), p->goff[first_tensor],
                                                                  stream)));
}

zr_status zr_plan_set_checked(zr_plan* p, int32_t enable) {
    if (!p) return ZR_ERR_INVALID_ARG;
    p->checked = enable != 0;
    return ZR_OK;
}

zr_status zr_plan_verify(const zr_plan* p, zr_stream_t stream) {
    if (!p) return ZR_ERR_INVALID_ARG;
    if (!p->d_workspace) return ZR_ERR_NO_WORKSPACE;
    const zr_status dst = check_device(p);
    if (dst != ZR_OK) return dst;
    return verify_tables(p, stream);
}

zr_status zr_plan_check_result(const zr_plan* p, zr_check_result* out, zr_stream_t stream) {
    if (!p || !out) return ZR_ERR_INVALID_ARG;
    if (!p->d_workspace) return ZR_ERR_NO_WORKSPACE;
    const zr_status dst = check_device(p);
    if (dst != ZR_OK) return dst;
    uint64_t w[zr::kCheckWords];
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(w, p->d_check, sizeof w, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return ZR_ERR_CUDA;
    out->bad_tiles = w[0];
    out->first_bad = w[1] == ~0ull ? -1 : static_cast<int64_t>(w[1]);
    out->hash_mismatch = static_cast<uint32_t>(w[2]);
    out->tables_emptied = (w[0] != 0 || w[2] != 0) ? 1u : 0u;
    return ZR_OK;
}

zr_status zr_plan_set_adamw(zr_plan* p, const zr_adamw* hp) {
    if (!p || !hp) return ZR_ERR_INVALID_ARG;
    // Clipping on or off changes what the workspace must hold.
    if ((hp->max_grad_norm > 0.0f) != p->clip_enabled()) return ZR_ERR_UNSUPPORTED;
    p->hp = *hp;
    return ZR_OK;
}

zr_status zr_plan_set_device_lr(zr_plan* p, const float* d_lr) {
    if (!p) return ZR_ERR_INVALID_ARG;
    if (d_lr && (reinterpret_cast<uintptr_t>(d_lr) & 3u) != 0) return ZR_ERR_ALIGNMENT;
    p->d_lr = d_lr;
    return ZR_OK;
}

zr_status zr_plan_set_sumsq_partials(zr_plan* p, double* d_partials) {
    if (!p || !d_partials) return ZR_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_partials) & 7u) != 0) return ZR_ERR_ALIGNMENT;
    p->d_sumsq_partials = d_partials;
    return ZR_OK;
}

zr_status zr_plan_owner_offsets(const zr_plan* p, int64_t* offsets) {
    if (!p || !offsets) return ZR_ERR_INVALID_ARG;
    // Each rank's region starts on a 16-byte boundary (8 bf16 elements), as
    // the step's vector loads need.
    int64_t at = 0;
    for (int32_t r = 0; r < p->world_size; ++r) {
        offsets[r] = at;
        at += (p->rank_numel[r] + 7) / 8 * 8;
    }
    offsets[p->world_size] = at;
    return ZR_OK;
}

zr_status zr_plan_set_gather_targets(zr_plan* p, void* const* targets, zr_stream_t stream) {
    if (!p) return ZR_ERR_INVALID_ARG;
    if (!p->d_workspace) return ZR_ERR_NO_WORKSPACE;
    if (!targets) {
        p->n_gather_targets = 0;
        return ZR_OK;
    }
    if (p->param_layout == ZR_PARAMS_OWNED) return ZR_ERR_UNSUPPORTED;   // a shard is not gathered by the step
    for (int32_t w = 0; w < p->world_size; ++w) {
        if (!targets[w]) return ZR_ERR_INVALID_ARG;
        if (!aligned16(targets[w])) return ZR_ERR_ALIGNMENT;
    }
    if (cudaMemcpyAsync(p->d_gather_targets, targets, sizeof(void*) * p->world_size, cudaMemcpyHostToDevice,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess ||
        cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return ZR_ERR_CUDA;
    p->n_gather_targets = p->world_size;
    return ZR_OK;
}

static zr_status step_impl(const zr_plan* p, const void* const* grad_ptrs, float* master, float* m, float* v,
                           void* param_out, int64_t step, int64_t* d_step, zr_stream_t stream);

zr_status zr_step(const zr_plan* p, const void* const* grad_ptrs, float* master, float* m, float* v,
                  void* param_out, int64_t step, zr_stream_t stream) {
    return step_impl(p, grad_ptrs, master, m, v, param_out, step, nullptr, stream);
}

zr_status zr_step_device_count(const zr_plan* p, const void* const* grad_ptrs, float* master, float* m, float* v,
                               void* param_out, int64_t* d_step, zr_stream_t stream) {
    if (!d_step) return ZR_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_step) & 7u) != 0) return ZR_ERR_ALIGNMENT;
    return step_impl(p, grad_ptrs, master, m, v, param_out, 1, d_step, stream);
}

static zr_status step_impl(const zr_plan* p, const void* const* grad_ptrs, float* master, float* m, float* v,
                           void* param_out, int64_t step, int64_t* d_step, zr_stream_t stream) {
    if (!p || step < 1) return ZR_ERR_INVALID_ARG;
    if (!p->d_workspace) return ZR_ERR_NO_WORKSPACE;
    {
        const zr_status dst = check_device(p);
        if (dst != ZR_OK) return dst;
    }
    if (p->owned_numel() == 0) {
        // Nothing to update, but a device step count still advances, so it
        // stays equal on every rank.
        if (d_step)
            return cuda_status(static_cast<cudaError_t>(zr::launch_device_scalars(d_step, p->hp, p->d_lr, p->d_scalars, stream)));
        return ZR_OK;
    }
    zr_status st = check_grads(p, grad_ptrs);
    if (st != ZR_OK) return st;
    if ((st = check_state(master, m, v)) != ZR_OK || (st = check_param_out(p, param_out)) != ZR_OK) return st;
    if (p->clip_enabled() && !p->d_sumsq_partials) return ZR_ERR_NO_WORKSPACE;

    {
        const zr_status cs = verify_if_checked(p, stream);
        if (cs != ZR_OK) return cs;
    }
    zr::LaunchArgs a = base_args(p);
    a.master = master;
    a.m = m;
    a.v = v;
    a.param_out = static_cast<uint16_t*>(param_out);
    a.s = zr::adam_scalars(p->hp, step);
    void* s = stream;
    if (d_step) {
        // The count and the scalars live in device memory, so a captured
        // graph of this call replays as the next step each time.
        if (zr::launch_device_scalars(d_step, p->hp, p->d_lr, p->d_scalars, s) != cudaSuccess) return ZR_ERR_CUDA;
        a.dev_scalars = p->d_scalars;
    }
    if (!p->clip_enabled())
        return cuda_status(static_cast<cudaError_t>(zr::launch_tiles(zr::Pass::kStep, a, grad_ptrs, false, false, s)));

    // Pass 1: reduce, per-tile sums of squares (and the fp32 g scratch for W > 4).
    const bool scratch = p->clip_uses_scratch();
    a.g_buf = p->d_g_scratch;
    a.tile_partials = p->d_tile_partials;
    int e = zr::launch_tiles(zr::Pass::kSumsq, a, grad_ptrs, false, scratch, s);
    if (e != cudaSuccess) return ZR_ERR_CUDA;
    // This rank's S_r (groups of tiles in parallel, then the groups), all
    // ranks' S in rank order, the coefficient.
    e = zr::launch_clip_combine(clip_args(p, p->d_sumsq_partials, p->d_own_sumsq), s);
    if (e != cudaSuccess) return ZR_ERR_CUDA;
    // Pass 2: scale by the coefficient, AdamW, cast.  Tiles in reverse
    // order: the first CTAs then read the g scratch that pass 1's last CTAs
    // wrote, while it is still in L2.
    a.clip_coef = p->d_clip_coef;
    a.reverse = 1;
    e = zr::launch_tiles(zr::Pass::kStepClip, a, grad_ptrs, scratch, false, s);
    return cuda_status(static_cast<cudaError_t>(e));
}

zr_status zr_step_bucket(const zr_plan* p, int32_t bucket, const void* const* grad_ptrs, float* master, float* m,
                         float* v, void* param_out, int64_t step, zr_stream_t stream) {
    if (!p || step < 1) return ZR_ERR_INVALID_ARG;
    if (bucket < 0 || bucket >= p->n_buckets) return ZR_ERR_INVALID_ARG;
    if (!p->d_workspace) return ZR_ERR_NO_WORKSPACE;
    {
        const zr_status dst = check_device(p);
        if (dst != ZR_OK) return dst;
    }
    const int32_t first = p->bucket_first_tile[bucket];
    const int32_t count = p->bucket_first_tile[bucket + 1] - first;
    if (count == 0) return ZR_OK;   // this rank owns nothing in the bucket
    zr_status st = check_grads(p, grad_ptrs);
    if (st != ZR_OK) return st;
    {
        const zr_status cs = verify_if_checked(p, stream);
        if (cs != ZR_OK) return cs;
    }
    zr::LaunchArgs a = base_args(p);
    a.tiles = p->d_tiles + first;
    a.n_tiles = count;
    void* s = stream;
    if (!p->clip_enabled()) {
        if ((st = check_state(master, m, v)) != ZR_OK || (st = check_param_out(p, param_out)) != ZR_OK) return st;
        a.master = master;
        a.m = m;
        a.v = v;
        a.param_out = static_cast<uint16_t*>(param_out);
        a.s = zr::adam_scalars(p->hp, step);
        return cuda_status(static_cast<cudaError_t>(zr::launch_tiles(zr::Pass::kStep, a, grad_ptrs, false, false, s)));
    }
    // Clipping: the bucket's share of pass 1 (reduce, per-tile sums of
    // squares, the fp32 g scratch when W > 4); zr_step_finish does the rest.
    const bool scratch = p->clip_uses_scratch();
    a.g_buf = p->d_g_scratch;
    a.tile_partials = p->d_tile_partials;
    return cuda_status(static_cast<cudaError_t>(zr::launch_tiles(zr::Pass::kSumsq, a, grad_ptrs, false, scratch, s)));
}

zr_status zr_step_finish(const zr_plan* p, const void* const* grad_ptrs, float* master, float* m, float* v,
                         void* param_out, int64_t step, zr_stream_t stream) {
    if (!p || step < 1) return ZR_ERR_INVALID_ARG;
    if (!p->d_workspace) return ZR_ERR_NO_WORKSPACE;
    {
        const zr_status dst = check_device(p);
        if (dst != ZR_OK) return dst;
    }
    if (!p->clip_enabled() || p->owned_numel() == 0) return ZR_OK;
    if (!p->d_sumsq_partials) return ZR_ERR_NO_WORKSPACE;
    const bool scratch = p->clip_uses_scratch();
    if (!scratch) {
        zr_status st = check_grads(p, grad_ptrs);   // pass 2 reads the gradients again
        if (st != ZR_OK) return st;
    } else {
        grad_ptrs = nullptr;                         // pass 2 reads the g scratch only
    }
    zr_status st2 = check_state(master, m, v);
    if (st2 != ZR_OK || (st2 = check_param_out(p, param_out)) != ZR_OK) return st2;
    {
        const zr_status cs = verify_if_checked(p, stream);
        if (cs != ZR_OK) return cs;
    }
    zr::LaunchArgs a = base_args(p);
    a.master = master;
    a.m = m;
    a.v = v;
    a.param_out = static_cast<uint16_t*>(param_out);
    a.s = zr::adam_scalars(p->hp, step);
    a.g_buf = p->d_g_scratch;
    void* s = stream;
    int e = zr::launch_clip_combine(clip_args(p, p->d_sumsq_partials, p->d_own_sumsq), s);
    if (e != cudaSuccess) return ZR_ERR_CUDA;
    a.clip_coef = p->d_clip_coef;
    a.reverse = 1;
    e = zr::launch_tiles(zr::Pass::kStepClip, a, grad_ptrs, scratch, false, s);
    return cuda_status(static_cast<cudaError_t>(e));
}

zr_status zr_bucket_sumsq(const zr_plan* p, double* d_out, zr_stream_t stream) {
    if (!p || !d_out) return ZR_ERR_INVALID_ARG;
    if (!p->d_workspace) return ZR_ERR_NO_WORKSPACE;
    {
        const zr_status dst = check_device(p);
        if (dst != ZR_OK) return dst;
    }
    if (!p->clip_enabled()) return ZR_ERR_INVALID_ARG;   // tile partials live in the clip workspace
    if ((reinterpret_cast<uintptr_t>(d_out) & 7u) != 0) return ZR_ERR_ALIGNMENT;
    if (p->owned_numel() == 0)
        return cuda_status(cudaMemsetAsync(d_out, 0, sizeof(double), reinterpret_cast<cudaStream_t>(stream)));
    return cuda_status(static_cast<cudaError_t>(zr::launch_clip_combine(clip_args(p, nullptr, d_out), stream)));
}

zr_status zr_grad_sumsq(const zr_plan* p, const void* const* grad_ptrs, double* d_out, zr_stream_t stream) {
    if (!p || !d_out) return ZR_ERR_INVALID_ARG;
    if (!p->d_workspace) return ZR_ERR_NO_WORKSPACE;
    {
        const zr_status dst = check_device(p);
        if (dst != ZR_OK) return dst;
    }
    if (!p->clip_enabled()) return ZR_ERR_INVALID_ARG;   // tile partials live in the clip workspace
    if ((reinterpret_cast<uintptr_t>(d_out) & 7u) != 0) return ZR_ERR_ALIGNMENT;
    void* s = stream;
    if (p->owned_numel() == 0) {
        return cuda_status(cudaMemsetAsync(d_out, 0, sizeof(double), static_cast<cudaStream_t>(s)));
    }
    zr_status st = check_grads(p, grad_ptrs);
    if (st != ZR_OK) return st;
    {
        const zr_status cs = verify_if_checked(p, stream);
        if (cs != ZR_OK) return cs;
    }
    zr::LaunchArgs a = base_args(p);
    a.tile_partials = p->d_tile_partials;
    int e = zr::launch_tiles(zr::Pass::kSumsq, a, grad_ptrs, false, false, s);
    if (e != cudaSuccess) return ZR_ERR_CUDA;
    return cuda_status(static_cast<cudaError_t>(zr::launch_clip_combine(clip_args(p, nullptr, d_out), s)));
}

zr_status zr_debug_average_check(int32_t w_first, int32_t w_last, uint64_t* d_mismatches, zr_stream_t stream) {
    if (w_first < 1 || w_last < w_first || w_last > ZR_MAX_WORLD_SIZE || !d_mismatches) return ZR_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_mismatches) & 7u) != 0) return ZR_ERR_ALIGNMENT;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ZR_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return ZR_ERR_CUDA;
    if (major != 10) return ZR_ERR_UNSUPPORTED;
    return cuda_status(static_cast<cudaError_t>(zr::launch_average_check(
        w_first, w_last, reinterpret_cast<unsigned long long*>(d_mismatches), stream)));
}

zr_status zr_debug_reduce(const zr_plan* p, const void* const* grad_ptrs, float* g_out, zr_stream_t stream) {
    if (!p || !g_out) return ZR_ERR_INVALID_ARG;
    if (!p->d_workspace) return ZR_ERR_NO_WORKSPACE;
    {
        const zr_status dst = check_device(p);
        if (dst != ZR_OK) return dst;
    }
    if (p->owned_numel() == 0) return ZR_OK;
    zr_status st = check_grads(p, grad_ptrs);
    if (st != ZR_OK) return st;
    if (!aligned16(g_out)) return ZR_ERR_ALIGNMENT;
    {
        const zr_status cs = verify_if_checked(p, stream);
        if (cs != ZR_OK) return cs;
    }
    zr::LaunchArgs a = base_args(p);
    a.g_buf = g_out;
    return cuda_status(static_cast<cudaError_t>(
        zr::launch_tiles(zr::Pass::kReduceOnly, a, grad_ptrs, false, false, stream)));
}

zr_status zr_step_host(const zr_plan* p, const void* const* host_grad_ptrs, void* const* dev_grad_ptrs,
                       float* master, float* m, float* v, void* param_out, void* host_param_out,
                       int64_t step, zr_stream_t stream) {
    if (!p || !host_grad_ptrs || !dev_grad_ptrs || !host_param_out || step < 1) return ZR_ERR_INVALID_ARG;
    if (!p->d_workspace) return ZR_ERR_NO_WORKSPACE;
    {
        const zr_status dst = check_device(p);
        if (dst != ZR_OK) return dst;
    }
    if (p->n_gather_targets > 0) return ZR_ERR_UNSUPPORTED;   // copies back this rank's buffer only
    const int64_t n = p->owned_numel();
    if (n == 0) return ZR_OK;
    for (int32_t w = 0; w < p->world_size; ++w)
        if (!host_grad_ptrs[w]) return ZR_ERR_INVALID_ARG;
    const void* const* dev_grads = const_cast<const void* const*>(dev_grad_ptrs);
    zr_status st = check_grads(p, dev_grads);
    if (st != ZR_OK) return st;
    if (!master || !m || !v || !param_out) return ZR_ERR_INVALID_ARG;
    if (!aligned16(master) || !aligned16(m) || !aligned16(v) || !aligned16(param_out)) return ZR_ERR_ALIGNMENT;
    const bool clip = p->clip_enabled();
    if (clip && !p->d_sumsq_partials) return ZR_ERR_NO_WORKSPACE;
    st = ensure_host_pipeline(p);
    if (st != ZR_OK) return st;

    // Chunks of the owned range, cut at tile boundaries (tiles in owned
    // order), halving in size: 1/2, 1/4, 1/8, 1/8.  Each chunk's copy-back
    // overlaps the next chunk's copy-in, so only the last eighth of the
    // copy-back is exposed, and the copy-in stays in few large transfers
    // (small host-to-device copies lose PCIe throughput).
    const int32_t n_tiles = static_cast<int32_t>(p->tiles_by_owned.size());
    const int K = static_cast<int>(std::min<int32_t>(zr_plan::kHostChunks, n_tiles));
    int32_t bounds[zr_plan::kHostChunks + 1];
    bounds[0] = 0;
    {
        int64_t seen = 0;
        int k = 1;
        for (int32_t i = 0; i < n_tiles && k < K; ++i) {
            seen += p->tiles_by_owned[i].len;
            const int64_t target = n - (n >> k);   // n/2, 3n/4, 7n/8, ...
            if (seen >= target) bounds[k++] = i + 1;
        }
        for (; k <= K; ++k) bounds[k] = n_tiles;
    }
    cudaStream_t S = reinterpret_cast<cudaStream_t>(stream);
    cudaStream_t C = p->h2d_stream, D = p->d2h_stream;
    cudaEvent_t* ev_in = p->host_events;                       // K: chunk k's gradients on the device
    cudaEvent_t* ev_done = p->host_events + zr_plan::kHostChunks;   // K: chunk k's parameters written
    cudaEvent_t ev_start = p->host_events[2 * zr_plan::kHostChunks];
    cudaEvent_t ev_end = p->host_events[2 * zr_plan::kHostChunks + 1];
    st = verify_if_checked(p, stream);
    if (st != ZR_OK) return st;
    // The copies may overwrite the device gradient buffers only after the
    // work already queued on the caller's stream.
    if (cudaEventRecord(ev_start, S) != cudaSuccess || cudaStreamWaitEvent(C, ev_start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(D, ev_start, 0) != cudaSuccess)
        return ZR_ERR_CUDA;

    zr::LaunchArgs a = base_args(p);
    a.master = master;
    a.m = m;
    a.v = v;
    a.param_out = static_cast<uint16_t*>(param_out);
    a.s = zr::adam_scalars(p->hp, step);
    const bool scratch = p->clip_uses_scratch();
    a.g_buf = p->d_g_scratch;
    a.tile_partials = p->d_tile_partials;
    const uint16_t* out_dev = static_cast<const uint16_t*>(param_out);
    uint16_t* out_host = static_cast<uint16_t*>(host_param_out);

    auto chunk_args = [&](int k) {
        zr::LaunchArgs c = a;
        c.tiles = p->d_tiles_by_owned + bounds[k];
        c.n_tiles = bounds[k + 1] - bounds[k];
        return c;
    };
    auto copy_out = [&](int k) -> bool {
        if (cudaStreamWaitEvent(D, ev_done[k], 0) != cudaSuccess) return false;
        int64_t run_start = -1, run_len = 0;
        for (int32_t i = bounds[k]; i <= bounds[k + 1]; ++i) {
            const bool more = i < bounds[k + 1];
            if (more && run_len > 0 && run_start + run_len == p->tiles_by_owned[i].global) {
                run_len += p->tiles_by_owned[i].len;
                continue;
            }
            if (run_len > 0 &&
                cudaMemcpyAsync(out_host + run_start, out_dev + run_start, sizeof(uint16_t) * run_len,
                                cudaMemcpyDeviceToHost, D) != cudaSuccess)
                return false;
            if (more) {
                run_start = p->tiles_by_owned[i].global;
                run_len = p->tiles_by_owned[i].len;
            }
        }
        return true;
    };

    for (int k = 0; k < K; ++k) {
        if (bounds[k + 1] == bounds[k]) continue;
        const zr::Tile& first = p->tiles_by_owned[bounds[k]];
        const zr::Tile& last = p->tiles_by_owned[bounds[k + 1] - 1];
        const int64_t o0 = first.owned, len = last.owned + last.len - first.owned;
        for (int32_t w = 0; w < p->world_size; ++w) {
            if (cudaMemcpyAsync(static_cast<uint16_t*>(dev_grad_ptrs[w]) + o0,
                                static_cast<const uint16_t*>(host_grad_ptrs[w]) + o0, sizeof(uint16_t) * len,
                                cudaMemcpyHostToDevice, C) != cudaSuccess)
                return ZR_ERR_CUDA;
        }
        if (cudaEventRecord(ev_in[k], C) != cudaSuccess || cudaStreamWaitEvent(S, ev_in[k], 0) != cudaSuccess)
            return ZR_ERR_CUDA;
        const zr::LaunchArgs c = chunk_args(k);
        if (!clip) {
            if (zr::launch_tiles(zr::Pass::kStep, c, dev_grads, false, false, S) != cudaSuccess) return ZR_ERR_CUDA;
            if (cudaEventRecord(ev_done[k], S) != cudaSuccess || !copy_out(k)) return ZR_ERR_CUDA;
        } else if (zr::launch_tiles(zr::Pass::kSumsq, c, dev_grads, false, scratch, S) != cudaSuccess) {
            return ZR_ERR_CUDA;
        }
    }
    if (clip) {
        if (zr::launch_clip_combine(clip_args(p, p->d_sumsq_partials, p->d_own_sumsq), S) != cudaSuccess)
            return ZR_ERR_CUDA;
        a.clip_coef = p->d_clip_coef;
        for (int k = 0; k < K; ++k) {
            if (bounds[k + 1] == bounds[k]) continue;
            const zr::LaunchArgs c = chunk_args(k);
            if (zr::launch_tiles(zr::Pass::kStepClip, c, dev_grads, scratch, false, S) != cudaSuccess)
                return ZR_ERR_CUDA;
            if (cudaEventRecord(ev_done[k], S) != cudaSuccess || !copy_out(k)) return ZR_ERR_CUDA;
        }
    }
    // The caller's stream reaches this point only when every copy is done.
    if (cudaEventRecord(ev_end, D) != cudaSuccess || cudaStreamWaitEvent(S, ev_end, 0) != cudaSuccess)
        return ZR_ERR_CUDA;
    return ZR_OK;
}

}  // extern "C"
