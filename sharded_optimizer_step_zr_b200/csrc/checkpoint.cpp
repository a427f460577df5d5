// Sharded optimizer-state checkpoints (host side).
//
// ZeRO keeps the fp32 master weights and Adam moments only on their owner,
// so a checkpoint is one file per rank ("DDP -> ZeRO" blog, section 3.3: a
// sharded model must be gathered before it is saved as a whole; the bf16
// parameters are whole after the step's all-gather, the fp32 state is not).
// Shard file layout (little-endian):
//   header (256 bytes, ShardHeader below), then master, m and v of the
//   owner's elements in owned order (fp32, owned_numel each).
// The header names the partition (a hash of the tensor shapes, W and the
// mode), the rank, the step and the hyperparameters, and carries a 64-bit
// FNV-1a checksum of the payload.  zr_state_reshard rebuilds any rank's
// shard of another partition of the same tensors from a complete set of
// shards, which is how a job resumes on a different number of ranks; a
// W = 1 flat target is the consolidated fp32 state in declaration order.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstddef>
#include <cstdio>
#include <cstring>
#include <memory>
#include <new>
#include <string>
#include <vector>

#include "zr_internal.hpp"

namespace {

constexpr char kMagic[8] = {'Z', 'R', 'S', 'H', 'A', 'R', 'D', '1'};
constexpr uint32_t kVersion = 1;

struct ShardHeader {
    char magic[8];
    uint32_t version;
    int32_t world_size;
    int32_t rank;
    int32_t mode;
    int64_t total_numel;
    int64_t padded_numel;
    int64_t owned_numel;
    uint64_t shapes_hash;      // the tensors alone
    uint64_t partition_hash;   // the tensors, W and the mode
    int64_t step;
    zr_adamw hp;
    uint64_t payload_checksum;
    uint8_t reserved[256 - 104];
};
static_assert(sizeof(ShardHeader) == 256, "shard header is 256 bytes");
static_assert(offsetof(ShardHeader, payload_checksum) == 96, "header layout");

constexpr uint64_t kFnvOffset = 0xcbf29ce484222325ull;
constexpr uint64_t kFnvPrime = 0x100000001b3ull;

uint64_t fnv_words(uint64_t h, const void* data, size_t bytes) {
    // FNV-1a over little-endian 64-bit words; a trailing partial word is
    // zero-padded.
    const unsigned char* p = static_cast<const unsigned char*>(data);
    size_t i = 0;
    for (; i + 8 <= bytes; i += 8) {
        uint64_t w;
        std::memcpy(&w, p + i, 8);
        h ^= w;
        h *= kFnvPrime;
    }
    if (i < bytes) {
        uint64_t w = 0;
        std::memcpy(&w, p + i, bytes - i);
        h ^= w;
        h *= kFnvPrime;
    }
    return h;
}

uint64_t shapes_hash(const zr_plan& p) {
    uint64_t h = kFnvOffset;
    const int64_t n = p.n_tensors;
    h = fnv_words(h, &n, 8);
    for (int32_t t = 0; t < p.n_tensors; ++t) h = fnv_words(h, &p.numel[t], 8);
    return h;
}

uint64_t partition_hash(const zr_plan& p) {
    uint64_t h = shapes_hash(p);
    const int64_t wm[2] = {p.world_size, p.mode};
    return fnv_words(h, wm, 16);
}

struct File {
    FILE* f = nullptr;
    File() = default;
    File(const File&) = delete;
    File& operator=(const File&) = delete;
    ~File() {
        if (f) std::fclose(f);
    }
};

bool read_header(const char* path, ShardHeader* h, File* file) {
    file->f = std::fopen(path, "rb");
    if (!file->f) return false;
    if (std::fread(h, sizeof(*h), 1, file->f) != 1) return false;
    return std::memcmp(h->magic, kMagic, 8) == 0 && h->version == kVersion;
}

// A complete set of shards of one partition, read and checked: the headers,
// each rank's payload (master, m, v) and the partition's segments sorted by
// global offset.
struct ShardSet {
    std::vector<ShardHeader> hs;
    std::vector<std::vector<float>> payload;
    std::vector<zr_segment> segs;
};

zr_status read_shard_set(const zr_plan& like, const char* const* src_paths, int32_t n_src, ShardSet* set) {
    if (!src_paths || n_src < 1) return ZR_ERR_INVALID_ARG;
    // Every source header: one complete partition of `like`'s tensors,
    // ranks 0..n_src-1 in order, one step.
    std::vector<ShardHeader>& hs = set->hs;
    hs.resize(n_src);
    for (int32_t r = 0; r < n_src; ++r) {
        if (!src_paths[r]) return ZR_ERR_INVALID_ARG;
        File f;
        if (!read_header(src_paths[r], &hs[r], &f)) return f.f ? ZR_ERR_MISMATCH : ZR_ERR_IO;
        if (hs[r].shapes_hash != shapes_hash(like) || hs[r].world_size != n_src || hs[r].rank != r ||
            hs[r].mode != hs[0].mode || hs[r].partition_hash != hs[0].partition_hash || hs[r].step != hs[0].step ||
            hs[r].total_numel != like.total_numel)
            return ZR_ERR_MISMATCH;
    }
    // The source partition's segments, from a plan of the same tensors.
    std::vector<int32_t> ndims(like.n_tensors, 1);
    std::vector<const int64_t*> shape_ptrs(like.n_tensors);
    for (int32_t t = 0; t < like.n_tensors; ++t) shape_ptrs[t] = &like.numel[t];
    zr_plan* src_plan = nullptr;
    zr_status st = zr_plan_create(like.n_tensors, ndims.data(), shape_ptrs.data(), n_src, 0,
                                  static_cast<zr_partition>(hs[0].mode), 1ull << 62, &like.hp, &src_plan);
    if (st != ZR_OK) return st;
    std::unique_ptr<zr_plan, void (*)(zr_plan*)> guard(src_plan, zr_plan_destroy);
    for (int32_t r = 0; r < n_src; ++r)
        if (hs[r].owned_numel != src_plan->rank_numel[r] || hs[r].partition_hash != partition_hash(*src_plan))
            return ZR_ERR_MISMATCH;
    set->segs = src_plan->segments;
    std::sort(set->segs.begin(), set->segs.end(),
              [](const zr_segment& a, const zr_segment& b) { return a.global_offset < b.global_offset; });
    // Each source payload is read once, whole, and its checksum verified.
    set->payload.assign(n_src, {});
    for (int32_t r = 0; r < n_src; ++r) {
        const int64_t k = hs[r].owned_numel;
        try {
            set->payload[r].resize(static_cast<size_t>(3 * k));
        } catch (...) {
            return ZR_ERR_INVALID_ARG;
        }
        File f;
        f.f = std::fopen(src_paths[r], "rb");
        if (!f.f) return ZR_ERR_IO;
        if (std::fseek(f.f, sizeof(ShardHeader), SEEK_SET) != 0) return ZR_ERR_IO;
        const size_t bytes = sizeof(float) * static_cast<size_t>(3 * k);
        if (k > 0 && std::fread(set->payload[r].data(), 1, bytes, f.f) != bytes) return ZR_ERR_IO;
        if (fnv_words(kFnvOffset, set->payload[r].data(), bytes) != hs[r].payload_checksum) return ZR_ERR_MISMATCH;
    }
    return ZR_OK;
}

// Round to nearest, ties to even; a NaN stays a (quiet) NaN, overflow
// rounds to infinity through the carry into the exponent.
uint16_t bf16_rne(float x) {
    uint32_t b;
    std::memcpy(&b, &x, 4);
    if ((b & 0x7fffffffu) > 0x7f800000u) return static_cast<uint16_t>((b >> 16) | 0x0040u);
    b += 0x7fffu + ((b >> 16) & 1u);
    return static_cast<uint16_t>(b >> 16);
}

}  // namespace

extern "C" {

zr_status zr_state_save(const zr_plan* p, const char* path, const float* master, const float* m, const float* v,
                        int64_t step, zr_stream_t stream) {
    if (!p || !path || step < 0) return ZR_ERR_INVALID_ARG;
    const int64_t n = p->owned_numel();
    if (n > 0 && (!master || !m || !v)) return ZR_ERR_INVALID_ARG;
    std::vector<float> host;
    try {
        host.resize(static_cast<size_t>(3 * n));
    } catch (...) {
        return ZR_ERR_INVALID_ARG;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t bytes = sizeof(float) * static_cast<size_t>(n);
    if (n > 0) {
        if (cudaMemcpyAsync(host.data(), master, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaMemcpyAsync(host.data() + n, m, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaMemcpyAsync(host.data() + 2 * n, v, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return ZR_ERR_CUDA;
    }
    ShardHeader h;
    std::memset(&h, 0, sizeof h);
    std::memcpy(h.magic, kMagic, 8);
    h.version = kVersion;
    h.world_size = p->world_size;
    h.rank = p->rank;
    h.mode = p->mode;
    h.total_numel = p->total_numel;
    h.padded_numel = p->padded_numel;
    h.owned_numel = n;
    h.shapes_hash = shapes_hash(*p);
    h.partition_hash = partition_hash(*p);
    h.step = step;
    h.hp = p->hp;
    h.payload_checksum = fnv_words(kFnvOffset, host.data(), 3 * bytes);
    // Write to a temporary name, then rename: a crash mid-write never leaves
    // a truncated file under the final name.
    const std::string tmp = std::string(path) + ".tmp";
    {
        File out;
        out.f = std::fopen(tmp.c_str(), "wb");
        if (!out.f) return ZR_ERR_IO;
        if (std::fwrite(&h, sizeof h, 1, out.f) != 1) return ZR_ERR_IO;
        if (n > 0 && std::fwrite(host.data(), 1, 3 * bytes, out.f) != 3 * bytes) return ZR_ERR_IO;
        if (std::fflush(out.f) != 0) return ZR_ERR_IO;
    }
    if (std::rename(tmp.c_str(), path) != 0) return ZR_ERR_IO;
    return ZR_OK;
}

zr_status zr_state_load(const zr_plan* p, const char* path, float* master, float* m, float* v, int64_t* step,
                        zr_stream_t stream) {
    if (!p || !path) return ZR_ERR_INVALID_ARG;
    const int64_t n = p->owned_numel();
    if (n > 0 && (!master || !m || !v)) return ZR_ERR_INVALID_ARG;
    ShardHeader h;
    File in;
    if (!read_header(path, &h, &in)) return in.f ? ZR_ERR_MISMATCH : ZR_ERR_IO;
    if (h.partition_hash != partition_hash(*p) || h.world_size != p->world_size || h.rank != p->rank ||
        h.mode != p->mode || h.owned_numel != n || h.total_numel != p->total_numel ||
        h.padded_numel != p->padded_numel)
        return ZR_ERR_MISMATCH;
    std::vector<float> host;
    try {
        host.resize(static_cast<size_t>(3 * n));
    } catch (...) {
        return ZR_ERR_INVALID_ARG;
    }
    const size_t bytes = sizeof(float) * static_cast<size_t>(n);
    if (n > 0 && std::fread(host.data(), 1, 3 * bytes, in.f) != 3 * bytes) return ZR_ERR_IO;
    if (fnv_words(kFnvOffset, host.data(), 3 * bytes) != h.payload_checksum) return ZR_ERR_MISMATCH;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (n > 0) {
        if (cudaMemcpyAsync(master, host.data(), bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(m, host.data() + n, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(v, host.data() + 2 * n, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return ZR_ERR_CUDA;
    }
    if (step) *step = h.step;
    return ZR_OK;
}

zr_status zr_state_reshard(const zr_plan* target, const char* const* src_paths, int32_t n_src,
                           const char* dst_path) {
    if (!target || !src_paths || n_src < 1 || !dst_path) return ZR_ERR_INVALID_ARG;
    ShardSet set;
    zr_status st = read_shard_set(*target, src_paths, n_src, &set);
    if (st != ZR_OK) return st;
    const std::vector<ShardHeader>& hs = set.hs;
    const std::vector<zr_segment>& src_segs = set.segs;
    const std::vector<std::vector<float>>& payload = set.payload;

    // Global position -> (source rank, owned offset) for the target's owned
    // elements: walk the target's segments and, inside each, the source
    // segments that overlap it.  Pad elements are 0 in every state.
    const int64_t n = target->owned_numel();
    std::vector<float> out;
    try {
        out.assign(static_cast<size_t>(3 * n), 0.0f);
    } catch (...) {
        return ZR_ERR_INVALID_ARG;
    }
    for (const zr_segment& t : target->segments) {
        if (t.owner != target->rank || t.tensor < 0) continue;   // the target's own pad stays 0
        int64_t g = t.global_offset;
        const int64_t g_end = t.global_offset + t.length;
        auto it = std::upper_bound(src_segs.begin(), src_segs.end(), g,
                                   [](int64_t x, const zr_segment& s) { return x < s.global_offset; });
        if (it == src_segs.begin()) return ZR_ERR_MISMATCH;
        --it;
        while (g < g_end) {
            if (it == src_segs.end() || g < it->global_offset || g >= it->global_offset + it->length)
                return ZR_ERR_MISMATCH;
            const int64_t take = std::min(g_end, it->global_offset + it->length) - g;
            const int32_t r = it->owner;
            const int64_t so = it->owned_offset + (g - it->global_offset);
            const int64_t to = t.owned_offset + (g - t.global_offset);
            const int64_t k = hs[r].owned_numel;
            for (int part = 0; part < 3; ++part)
                std::memcpy(&out[part * n + to], &payload[r][part * k + so], sizeof(float) * take);
            g += take;
            ++it;
        }
    }
    ShardHeader h;
    std::memset(&h, 0, sizeof h);
    std::memcpy(h.magic, kMagic, 8);
    h.version = kVersion;
    h.world_size = target->world_size;
    h.rank = target->rank;
    h.mode = target->mode;
    h.total_numel = target->total_numel;
    h.padded_numel = target->padded_numel;
    h.owned_numel = n;
    h.shapes_hash = shapes_hash(*target);
    h.partition_hash = partition_hash(*target);
    h.step = hs[0].step;
    h.hp = hs[0].hp;
    const size_t bytes = sizeof(float) * static_cast<size_t>(3 * n);
    h.payload_checksum = fnv_words(kFnvOffset, out.data(), bytes);
    const std::string tmp = std::string(dst_path) + ".tmp";
    {
        File o;
        o.f = std::fopen(tmp.c_str(), "wb");
        if (!o.f) return ZR_ERR_IO;
        if (std::fwrite(&h, sizeof h, 1, o.f) != 1) return ZR_ERR_IO;
        if (n > 0 && std::fwrite(out.data(), 1, bytes, o.f) != bytes) return ZR_ERR_IO;
        if (std::fflush(o.f) != 0) return ZR_ERR_IO;
    }
    if (std::rename(tmp.c_str(), dst_path) != 0) return ZR_ERR_IO;
    return ZR_OK;
}

zr_status zr_state_export_params(const zr_plan* plan, const char* const* src_paths, int32_t n_src, int32_t dtype,
                                 const char* out_path, int64_t* n_written) {
    if (!plan || !src_paths || n_src < 1 || !out_path) return ZR_ERR_INVALID_ARG;
    if (dtype != ZR_EXPORT_F32 && dtype != ZR_EXPORT_BF16) return ZR_ERR_INVALID_ARG;
    ShardSet set;
    zr_status st = read_shard_set(*plan, src_paths, n_src, &set);
    if (st != ZR_OK) return st;
    // Every tensor element has exactly one source segment; the pad (tensor
    // -1) is not a parameter and is left out.
    const int64_t N = plan->total_numel;
    const size_t elem = dtype == ZR_EXPORT_BF16 ? 2 : 4;
    std::vector<unsigned char> out;
    try {
        out.assign(static_cast<size_t>(N) * elem, 0);
    } catch (...) {
        return ZR_ERR_INVALID_ARG;
    }
    int64_t covered = 0;
    for (const zr_segment& sg : set.segs) {
        if (sg.tensor < 0) continue;
        if (sg.global_offset < 0 || sg.global_offset + sg.length > N) return ZR_ERR_MISMATCH;
        const float* src = set.payload[sg.owner].data() + sg.owned_offset;   // master: the first third
        if (dtype == ZR_EXPORT_F32) {
            std::memcpy(out.data() + 4 * sg.global_offset, src, 4 * static_cast<size_t>(sg.length));
        } else {
            uint16_t* dst = reinterpret_cast<uint16_t*>(out.data()) + sg.global_offset;
            for (int64_t j = 0; j < sg.length; ++j) dst[j] = bf16_rne(src[j]);
        }
        covered += sg.length;
    }
    if (covered != N) return ZR_ERR_MISMATCH;
    const std::string tmp = std::string(out_path) + ".tmp";
    {
        File o;
        o.f = std::fopen(tmp.c_str(), "wb");
        if (!o.f) return ZR_ERR_IO;
        if (N > 0 && std::fwrite(out.data(), 1, out.size(), o.f) != out.size()) return ZR_ERR_IO;
        if (std::fflush(o.f) != 0) return ZR_ERR_IO;
    }
    if (std::rename(tmp.c_str(), out_path) != 0) return ZR_ERR_IO;
    if (n_written) *n_written = N;
    return ZR_OK;
}

}  // extern "C"
