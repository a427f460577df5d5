// Internal types shared by the planner, the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "zr.h"

namespace zr {

// A unit of GPU work: a run of consecutive owned elements that is also
// consecutive in the global layout and lies inside one bucket.
struct Tile {
    int64_t owned;     // first element in owned order
    int64_t global;    // first element in the global layout
    int32_t len;       // element count, 1..kTileElems
    int32_t flags;     // kTileVector | kTileStoreVector
    int32_t bucket;
    int32_t index;     // position in the plan's tile list (bucket order):
                       // where the tile's clip partial is stored
};
static_assert(sizeof(Tile) == 32, "Tile is 32 bytes");

constexpr int32_t kTileVector = 1;       // owned % 8 == 0 and len % 8 == 0
constexpr int32_t kTileStoreVector = 2;  // global % 8 == 0 as well: 16-byte bf16 stores

// 128-thread CTAs over 2048-element tiles (two 8-element vectors per
// thread): at ~94 registers five CTAs fit per SM, which measured faster on
// B200 than 256-thread CTAs over 4096 elements (two CTAs per SM).
constexpr int kThreads = 128;                  // threads per CTA
constexpr int kElemsPerThreadIter = 8;         // one 16-byte bf16 vector
constexpr int kTileElems = kThreads * kElemsPerThreadIter * 2;  // 2048

#if defined(__CUDACC__)
#define ZR_HOST_DEVICE __host__ __device__
#else
#define ZR_HOST_DEVICE
#endif

// Order-independent 64-bit hash of a tile table, for checked mode: the sum
// (mod 2^64) over the table's 64-bit words w_k (k = word position) of
// f(w_k + k * 0x9E3779B97F4A7C15), f the splitmix64 output function (Steele,
// Lea & Flood 2014).  Any change of one word changes the sum except with
// probability about 2^-64, and the sum can be formed in any order.
ZR_HOST_DEVICE inline uint64_t tile_word_hash(uint64_t w, uint64_t k) {
    uint64_t z = w + k * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}
constexpr int kTileWords = static_cast<int>(sizeof(Tile) / sizeof(uint64_t));   // 4

// Checked mode's status words in the workspace: [0] entries failing a
// check (all three tables, cumulative), [1] the smallest failing position
// (bucket-order tile table i, owned-order tile table n_tiles + i, gather
// pieces 2 n_tiles + i; all ones when none), [2] hash mismatch bits (1:
// bucket-order tiles, 2: owned-order tiles, 4: gather pieces), [3], [4] the
// tile tables' hash sums while a check runs, [5] the count of its finished
// blocks, [6] the gather pieces' hash sum (words 3-6 are 0 between checks).
constexpr int kCheckWords = 7;

// A piece of the ZeRO-3 parameter gather: `len` consecutive elements of one
// tensor that one rank owns, copied from that rank's bf16 shard (owned
// order, offset `src`) to the global position `dst`.  Pieces never cross a
// tensor or an owner boundary and hold at most kGatherPieceElems elements.
struct GatherPiece {
    int64_t src;
    int64_t dst;
    int32_t len;
    int32_t owner;
    int32_t tensor;
    int32_t reserved;
};
static_assert(sizeof(GatherPiece) == 32, "GatherPiece is 32 bytes");
constexpr int32_t kGatherPieceElems = 16384;   // 32 KB of bf16: one CTA's share

// AdamW scalars for one step, fp64 on the host rounded once to fp32.
struct AdamScalars {
    float beta1, beta2, one_minus_beta1, one_minus_beta2;
    float step_size;   // lr / (1 - beta1^t)
    float bc2_sqrt;    // sqrt(1 - beta2^t)
    float decay;       // 1 - lr * weight_decay
    float eps;
};

enum class Pass : int {
    kStep = 0,         // reduce -> AdamW -> cast (no clipping)
    kReduceOnly = 1,   // reduce -> fp32 g to an output buffer
    kSumsq = 2,        // reduce -> per-tile fp64 sum of squares (+ optional g scratch)
    kStepClip = 3,     // (reduce | read g scratch) -> * clip coef -> AdamW -> cast
};

// The clip's sum of squares S_r of a rank's averaged gradient, in a fixed
// order: the per-tile partials (by tile index) in groups of
// kClipGroupTiles; each group's total by fixed_sum128, then the groups'
// totals by fixed_sum128 again (zr_kernels.cu: one CTA per group, the last
// to finish sums the groups).  Every path that forms S_r uses that kernel,
// so S_r and the coefficient are the same bits on every call and every rank.
constexpr int32_t kClipGroupTiles = 1024;
ZR_HOST_DEVICE inline int32_t clip_groups(int32_t n_tiles) { return (n_tiles + kClipGroupTiles - 1) / kClipGroupTiles; }

struct ClipArgs {
    const double* tile_partials;  // one per tile of the plan (tile index)
    int32_t n_tiles;               // every tile of the plan
    int32_t world_size;
    uint32_t* ticket;              // completion counter of the groups, zero between launches
    double* group_sums;            // clip_groups(n_tiles) group totals
    double* partials_all;          // world_size entries: this rank's S_r written, all summed (or null)
    double* sumsq_out;             // this rank's S_r alone (or null)
    float* coef_out;               // the clip coefficient (when partials_all is set)
    int32_t rank;
    float max_norm;
};

struct LaunchArgs {
    const Tile* tiles;
    int32_t n_tiles;
    int32_t world_size;
    int32_t w_is_pow2;
    float inv_w;               // 1/W rounded to nearest (exact, and used, for powers of two)
    int32_t reverse;           // CTA b takes tile n_tiles - 1 - b (see the clip pass 2)
    int32_t n_targets;         // 0: bf16 results to param_out; else to each of targets[0..n)
    uint16_t* const* targets;  // device array of parameter buffers (every rank's, for the
                               // all-gather by peer stores)
    float* master;
    float* m;
    float* v;
    uint16_t* param_out;
    float* g_buf;              // kReduceOnly: output; kSumsq/kStepClip: scratch (may be null)
    double* tile_partials;     // kSumsq: one double per tile
    const float* clip_coef;    // kStepClip: device scalar
    AdamScalars s;
    const AdamScalars* dev_scalars;   // when set, the step's scalars are read from here instead of s
};

// Kernel launchers (zr_kernels.cu).  grad_ptrs: host array of W device
// pointers.  Return cudaError_t as int.
int launch_tiles(Pass pass, const LaunchArgs& a, const void* const* grad_ptrs, bool g_from_scratch,
                 bool write_g_scratch, void* stream);
int launch_device_scalars(int64_t* d_step, const zr_adamw& hp, const float* d_lr, AdamScalars* out, void* stream);
// S_r and the coefficient from the per-tile partials of pass 1: one
// 128-thread CTA per group of tiles, the last to finish sums the groups.
int launch_clip_combine(const ClipArgs& c, void* stream);

// W's scalars in the launch arguments: the count, whether it is a power of
// two, and 1/W rounded to nearest (IEEE single division on the host).
inline void set_world_size(LaunchArgs& a, int32_t W) {
    a.world_size = W;
    a.w_is_pow2 = (W & (W - 1)) == 0 ? 1 : 0;
    a.inv_w = 1.0f / static_cast<float>(W);
}

// For every W in [w_first, w_last]: how many of the 2^32 fp32 values s
// the step's averaging (s / W) maps to other bits than IEEE division does;
// mismatches[W - w_first] receives the count (a verification hook).
int launch_average_check(int32_t w_first, int32_t w_last, unsigned long long* mismatches, void* stream);
// ZeRO-3 gather: copy pieces [first, first + n) from the W shards to dst,
// where dst holds the global range starting at dst_base, on at most
// max_ctas CTAs (<= 0: one per piece).  shard_ptrs: host
// array of W device pointers (any may be NULL for a rank owning nothing).
int launch_gather(const GatherPiece* pieces, int32_t first, int32_t n, int32_t max_ctas, int32_t world_size,
                  const void* const* shard_ptrs, uint16_t* dst, int64_t dst_base, void* stream);

// Checked mode: verify both device tile tables and the gather piece table
// against their invariants and the hashes taken on the host at upload,
// then, if anything failed (now or before), overwrite all three with empty
// entries.  One launch; `check` holds kCheckWords words, zeroed (word 1 all
// ones) when the workspace is bound.
struct VerifyArgs {
    Tile* tiles;
    Tile* tiles_by_owned;
    int32_t n_tiles;
    int32_t n_buckets;
    int64_t n_owned;       // this rank's owned elements
    int64_t n_out;         // elements of the buffer the step writes
    GatherPiece* pieces;
    int32_t n_pieces;
    int32_t world_size;
    int64_t total_numel;
    int32_t n_tensors;
    uint64_t hash_tiles, hash_by_owned, hash_pieces;
    uint64_t* check;
};
int launch_verify_tables(const VerifyArgs& args, void* stream);

}  // namespace zr

// The opaque plan.
struct zr_plan {
    int32_t n_tensors = 0;
    int32_t world_size = 1;
    int32_t rank = 0;
    int32_t mode = 0;
    uint64_t cap_bytes = 0;
    zr_adamw hp{};

    std::vector<int64_t> numel;          // per tensor
    std::vector<int64_t> goff;           // per tensor, global layout
    std::vector<int32_t> tensor_owner;   // whole-tensor mode
    std::vector<int32_t> tensor_bucket;
    std::vector<int32_t> tensor_group;   // empty: buckets by cap_bytes; else one bucket per group
    std::vector<int64_t> rank_numel;     // owned element count per rank
    int64_t total_numel = 0;
    int64_t padded_numel = 0;
    int64_t chunk = 0;
    int32_t n_buckets = 0;

    std::vector<zr_segment> segments;    // all ranks
    std::vector<zr::Tile> tiles;         // this rank, bucket by bucket
    std::vector<int32_t> bucket_first_tile;  // n_buckets + 1 entries
    std::vector<zr::Tile> tiles_by_owned;    // the same tiles sorted by owned offset

    // device binding
    int device = -1;
    void* d_workspace = nullptr;
    uint64_t workspace_bytes = 0;
    zr::Tile* d_tiles = nullptr;
    zr::Tile* d_tiles_by_owned = nullptr;
    double* d_tile_partials = nullptr;
    uint32_t* d_clip_ticket = nullptr;    // workspace: the combine's completion counter (zeroed at upload)
    double* d_clip_group_sums = nullptr;  // workspace: clip_groups(n_tiles) group totals
    float* d_clip_coef = nullptr;
    double* d_own_sumsq = nullptr;
    float* d_g_scratch = nullptr;
    double* d_sumsq_partials = nullptr;   // caller-owned, world_size doubles
    uint16_t** d_gather_targets = nullptr; // workspace: world_size parameter buffers
    zr::AdamScalars* d_scalars = nullptr;  // workspace: scalars computed on the device
    const float* d_lr = nullptr;           // caller-owned learning rate for zr_step_device_count
    int32_t n_gather_targets = 0;          // 0 until zr_plan_set_gather_targets
    uint64_t* d_check = nullptr;           // workspace: checked mode's status words
    int32_t param_layout = ZR_PARAMS_GLOBAL;   // where zr_step writes the bf16 parameters
    std::vector<zr::GatherPiece> gather_pieces;     // all ranks, tensor by tensor
    std::vector<int32_t> tensor_first_piece;        // n_tensors + 1 entries
    zr::GatherPiece* d_gather_pieces = nullptr;     // workspace copy
    bool checked = false;                  // verify the tables before every launch
    uint64_t uid = 0;                      // unique per plan in this process (never reused)
    uint64_t table_generation = 0;         // bumped whenever the tile tables are rebuilt
    uint64_t hash_tiles = 0;               // tile_word_hash sums of the host tables
    uint64_t hash_tiles_by_owned = 0;
    uint64_t hash_gather_pieces = 0;

    // zr_step_host's copy streams and events, created on its first call
    // (host-side resources, not part of the plan's observable state).
    static constexpr int kHostChunks = 4;
    mutable cudaStream_t h2d_stream = nullptr;
    mutable cudaStream_t d2h_stream = nullptr;
    mutable cudaEvent_t host_events[2 * kHostChunks + 2] = {};
    mutable bool host_pipeline_ready = false;

    ~zr_plan();

    bool clip_enabled() const { return hp.max_grad_norm > 0.0f; }
    // Clipping keeps the fp32 averaged gradient for pass 2 when re-reading W
    // replicas would cost more than writing and reading 8 bytes (W > 4), and
    // always for grouped plans, whose per-layer gradients are released
    // before the norm is known.
    bool clip_uses_scratch() const { return clip_enabled() && (world_size > 4 || !tensor_group.empty()); }
    int64_t owned_numel() const { return rank_numel[rank]; }
};

namespace zr {
// planner.cpp
zr_status build_plan(zr_plan& p, int32_t n_tensors, const int32_t* ndims,
                     const int64_t* const* shapes);
// Workspace layout: offsets of each region, total bytes.
struct WorkspaceLayout {
    uint64_t tiles, tiles_by_owned, tile_partials, clip_ticket, clip_group_sums, clip_coef, own_sumsq,
        gather_targets, dev_scalars, check, gather_pieces, g_scratch, total;
};
WorkspaceLayout workspace_layout(const zr_plan& p);
// Rebuilds this rank's tile tables for the plan's parameter layout: the
// global layout as planned, or (ZR_PARAMS_OWNED) with every tile's output
// offset moved to its owned offset, so the same kernels write the rank's
// bf16 shard in owned order.
void build_tiles_for_layout(zr_plan& p);
uint64_t table_hash(const std::vector<Tile>& tiles);
uint64_t table_hash(const std::vector<GatherPiece>& pieces);
AdamScalars adam_scalars(const zr_adamw& hp, int64_t step);
}  // namespace zr
