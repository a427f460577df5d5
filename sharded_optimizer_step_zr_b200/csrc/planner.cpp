// Partition / bucket / segment planner and the GPU tile list (host only).
//
// Partition ("Scaling training to thousands of GPUs", 11:24 ZeRO): flat
// (FSDP1: concatenate, zero pad to W equal chunks) or whole-tensor ownership
// (FSDP2 / Muon: each tensor stays whole on one rank, balanced greedily by
// element count, largest first).  Buckets ("Scaling training ...", 03:41 DP;
// "DDP -> ZeRO" blog section 2.1): whole tensors in the order the backward
// pass produces their gradients (reverse declaration order), capped by
// bucket_cap_bytes of bf16 gradient -- or one bucket per group of tensors
// (a layer: the FSDP unit of "CS336 lecture 8", FSDP sketch).
#include <algorithm>
#include <cstring>
#include <cmath>
#include <limits>
#include <queue>
#include <tuple>

#include "zr_internal.hpp"

namespace zr {
namespace {

bool mul_overflows(int64_t a, int64_t b, int64_t* out) {
    if (a != 0 && b > std::numeric_limits<int64_t>::max() / a) return true;
    *out = a * b;
    return false;
}

// Greedy longest-processing-time assignment with a min-heap of ranks keyed
// by (load, rank).
void assign_whole_tensors(zr_plan& p) {
    const int32_t T = p.n_tensors;
    std::vector<int32_t> by_size(T);
    for (int32_t t = 0; t < T; ++t) by_size[t] = t;
    std::stable_sort(by_size.begin(), by_size.end(),
                     [&](int32_t a, int32_t b) { return p.numel[a] > p.numel[b]; });
    using Entry = std::pair<int64_t, int32_t>;  // (load, rank)
    std::priority_queue<Entry, std::vector<Entry>, std::greater<Entry>> heap;
    for (int32_t r = 0; r < p.world_size; ++r) heap.push({0, r});
    p.tensor_owner.assign(T, 0);
    p.rank_numel.assign(p.world_size, 0);
    for (int32_t t : by_size) {
        Entry e = heap.top();
        heap.pop();
        p.tensor_owner[t] = e.second;
        e.first += p.numel[t];
        p.rank_numel[e.second] = e.first;
        heap.push(e);
    }
}

void pack_buckets(zr_plan& p) {
    p.tensor_bucket.assign(p.n_tensors, 0);
    std::vector<std::vector<int32_t>> members;
    uint64_t bytes_in_open = 0;
    for (int32_t t = p.n_tensors - 1; t >= 0; --t) {
        const uint64_t b = 2ull * static_cast<uint64_t>(p.numel[t]);
        // grouped plans: a new bucket wherever the (next in backward order) tensor changes group
        const bool open_new = members.empty() ||
                              (p.tensor_group.empty()
                                   ? (!members.back().empty() && bytes_in_open + b > p.cap_bytes)
                                   : p.tensor_group[t] != p.tensor_group[t + 1]);
        if (open_new) {
            members.emplace_back();
            bytes_in_open = 0;
        }
        members.back().push_back(t);
        bytes_in_open += b;
        p.tensor_bucket[t] = static_cast<int32_t>(members.size()) - 1;
    }
    p.n_buckets = static_cast<int32_t>(members.size());
}

void cut_segments(zr_plan& p) {
    p.segments.clear();
    // owned offset of each tensor inside its owner's owned order (whole-tensor)
    std::vector<int64_t> owned_at(p.n_tensors, 0);
    if (p.mode == ZR_PARTITION_WHOLE_TENSOR) {
        std::vector<int64_t> next(p.world_size, 0);
        for (int32_t t = 0; t < p.n_tensors; ++t) {
            owned_at[t] = next[p.tensor_owner[t]];
            next[p.tensor_owner[t]] += p.numel[t];
        }
    }
    auto add = [&](int32_t bucket, int32_t tensor, int32_t owner, int64_t off, int64_t len,
                   int64_t glob, int64_t owned) {
        zr_segment s;
        s.bucket = bucket;
        s.tensor = tensor;
        s.owner = owner;
        s.reserved = 0;
        s.offset_in_tensor = off;
        s.length = len;
        s.global_offset = glob;
        s.owned_offset = owned;
        p.segments.push_back(s);
    };
    // Cut the global range [lo, hi) at multiples of the chunk.
    auto cut_flat = [&](int32_t bucket, int32_t tensor, int64_t base, int64_t lo, int64_t hi) {
        const int64_t C = p.chunk;
        for (int64_t r = lo / C; r * C < hi; ++r) {
            const int64_t a = std::max(lo, r * C);
            const int64_t b = std::min(hi, (r + 1) * C);
            add(bucket, tensor, static_cast<int32_t>(r), a - base, b - a, a, a - r * C);
        }
    };
    // Tensors of a bucket are consecutive in declaration order, packed from
    // the highest index down.
    int32_t t = p.n_tensors - 1;
    for (int32_t b = 0; b < p.n_buckets; ++b) {
        for (; t >= 0 && p.tensor_bucket[t] == b; --t) {
            if (p.numel[t] == 0) continue;
            if (p.mode == ZR_PARTITION_FLAT)
                cut_flat(b, t, p.goff[t], p.goff[t], p.goff[t] + p.numel[t]);
            else
                add(b, t, p.tensor_owner[t], 0, p.numel[t], p.goff[t], owned_at[t]);
        }
        if (b == 0 && p.mode == ZR_PARTITION_FLAT && p.padded_numel > p.total_numel)
            cut_flat(0, -1, p.total_numel, p.total_numel, p.padded_numel);
    }
}

// This rank's tiles, bucket by bucket.  Inside a bucket, the rank's pieces
// are merged where they are contiguous in both owned order and the global
// layout, then cut into tiles: a scalar head up to the next multiple of 8
// owned elements, vector tiles of kTileElems, a scalar tail.
void build_tiles(zr_plan& p) {
    ++p.table_generation;
    p.tiles.clear();
    p.bucket_first_tile.assign(p.n_buckets + 1, 0);
    struct Run { int64_t owned, global, len; };
    size_t k = 0;
    for (int32_t b = 0; b < p.n_buckets; ++b) {
        p.bucket_first_tile[b] = static_cast<int32_t>(p.tiles.size());
        std::vector<Run> runs;
        for (; k < p.segments.size() && p.segments[k].bucket == b; ++k) {
            const zr_segment& s = p.segments[k];
            if (s.owner == p.rank) runs.push_back({s.owned_offset, s.global_offset, s.length});
        }
        std::sort(runs.begin(), runs.end(),
                  [](const Run& x, const Run& y) { return x.owned < y.owned; });
        std::vector<Run> merged;
        for (const Run& r : runs) {
            if (!merged.empty() && merged.back().owned + merged.back().len == r.owned &&
                merged.back().global + merged.back().len == r.global)
                merged.back().len += r.len;
            else
                merged.push_back(r);
        }
        auto emit = [&](int64_t owned, int64_t global, int64_t len) {
            Tile tile{};
            tile.owned = owned;
            tile.global = global;
            tile.len = static_cast<int32_t>(len);
            tile.bucket = b;
            tile.index = static_cast<int32_t>(p.tiles.size());
            const bool vec = (owned % 8 == 0) && (len % 8 == 0);
            tile.flags = (vec ? kTileVector : 0) | ((vec && global % 8 == 0) ? kTileStoreVector : 0);
            p.tiles.push_back(tile);
        };
        for (const Run& r : merged) {
            int64_t o = r.owned, g = r.global, left = r.len;
            const int64_t head = std::min<int64_t>(left, (8 - o % 8) % 8);
            if (head > 0) { emit(o, g, head); o += head; g += head; left -= head; }
            const int64_t body = left - left % 8;
            for (int64_t done = 0; done < body; done += kTileElems) {
                const int64_t n = std::min<int64_t>(kTileElems, body - done);
                emit(o + done, g + done, n);
            }
            o += body; g += body; left -= body;
            if (left > 0) emit(o, g, left);
        }
    }
    p.bucket_first_tile[p.n_buckets] = static_cast<int32_t>(p.tiles.size());
    p.tiles_by_owned = p.tiles;
    std::sort(p.tiles_by_owned.begin(), p.tiles_by_owned.end(),
              [](const Tile& x, const Tile& y) { return x.owned < y.owned; });
}

// The ZeRO-3 gather's pieces: every tensor's segments (all owners) in order
// of their offset in the tensor, each cut into pieces of at most
// kGatherPieceElems elements.
void build_gather_pieces(zr_plan& p) {
    p.gather_pieces.clear();
    p.tensor_first_piece.assign(p.n_tensors + 1, 0);
    std::vector<std::vector<const zr_segment*>> by_tensor(p.n_tensors);
    for (const zr_segment& s : p.segments)
        if (s.tensor >= 0) by_tensor[s.tensor].push_back(&s);
    for (int32_t t = 0; t < p.n_tensors; ++t) {
        p.tensor_first_piece[t] = static_cast<int32_t>(p.gather_pieces.size());
        std::sort(by_tensor[t].begin(), by_tensor[t].end(),
                  [](const zr_segment* a, const zr_segment* b) { return a->offset_in_tensor < b->offset_in_tensor; });
        for (const zr_segment* s : by_tensor[t]) {
            for (int64_t done = 0; done < s->length; done += kGatherPieceElems) {
                GatherPiece g{};
                g.src = s->owned_offset + done;
                g.dst = s->global_offset + done;
                g.len = static_cast<int32_t>(std::min<int64_t>(kGatherPieceElems, s->length - done));
                g.owner = s->owner;
                g.tensor = t;
                p.gather_pieces.push_back(g);
            }
        }
    }
    p.tensor_first_piece[p.n_tensors] = static_cast<int32_t>(p.gather_pieces.size());
}

// Self-check of the tile list before anything reaches a kernel: the tiles
// cover this rank's owned range [0, owned) exactly once, each maps owned
// offsets to the same global offsets as the segment it came from, stays
// inside [0, padded), and carries vector flags only where the 8-element
// alignment holds.
bool tiles_are_consistent(const zr_plan& p) {
    const int64_t owned = p.rank_numel[p.rank];
    std::vector<std::pair<int64_t, int64_t>> span;   // (owned start, global start - owned start)
    for (const zr_segment& s : p.segments)
        if (s.owner == p.rank) span.push_back({s.owned_offset, s.global_offset - s.owned_offset});
    std::sort(span.begin(), span.end());
    std::vector<std::pair<int64_t, int64_t>> cover;
    for (const Tile& t : p.tiles) {
        if (t.len <= 0 || t.len > kTileElems || t.owned < 0 || t.owned + t.len > owned) return false;
        if (t.global < 0 || t.global + t.len > p.padded_numel) return false;
        auto it = std::upper_bound(span.begin(), span.end(), std::make_pair(t.owned, std::numeric_limits<int64_t>::max()));
        if (it == span.begin()) return false;
        --it;
        if (t.global - t.owned != it->second) return false;
        const bool vec = (t.owned % 8 == 0) && (t.len % 8 == 0);
        if ((t.flags & kTileVector) && !vec) return false;
        if ((t.flags & kTileStoreVector) && !(vec && t.global % 8 == 0)) return false;
        cover.push_back({t.owned, t.len});
    }
    std::sort(cover.begin(), cover.end());
    int64_t next = 0;
    for (const auto& c : cover) {
        if (c.first != next) return false;
        next += c.second;
    }
    return next == owned;
}

}  // namespace

zr_status build_plan(zr_plan& p, int32_t n_tensors, const int32_t* ndims,
                     const int64_t* const* shapes) {
    p.n_tensors = n_tensors;
    p.numel.assign(n_tensors, 0);
    p.goff.assign(n_tensors, 0);
    int64_t total = 0;
    for (int32_t t = 0; t < n_tensors; ++t) {
        if (ndims[t] < 0 || (ndims[t] > 0 && shapes[t] == nullptr)) return ZR_ERR_INVALID_ARG;
        int64_t n = 1;
        for (int32_t d = 0; d < ndims[t]; ++d) {
            if (shapes[t][d] < 0) return ZR_ERR_INVALID_ARG;
            if (mul_overflows(n, shapes[t][d], &n)) return ZR_ERR_INVALID_ARG;
        }
        p.numel[t] = n;
        p.goff[t] = total;
        if (n > std::numeric_limits<int64_t>::max() - total) return ZR_ERR_INVALID_ARG;
        total += n;
    }
    p.total_numel = total;
    if (p.mode == ZR_PARTITION_FLAT) {
        p.chunk = total / p.world_size + (total % p.world_size != 0 ? 1 : 0);
        int64_t padded;
        if (mul_overflows(p.chunk, p.world_size, &padded)) return ZR_ERR_INVALID_ARG;
        p.padded_numel = padded;
        p.rank_numel.assign(p.world_size, p.chunk);
        p.tensor_owner.assign(n_tensors, -1);
    } else {
        p.chunk = 0;
        p.padded_numel = total;
        assign_whole_tensors(p);
    }
    // One tile's length fits int32 by construction; owned counts must fit
    // the kernels' int64 offsets (always true).
    pack_buckets(p);
    cut_segments(p);
    build_tiles(p);
    if (!tiles_are_consistent(p)) return ZR_ERR_INVALID_ARG;
    build_gather_pieces(p);
    if (p.gather_pieces.size() > 0x7FFFFFFFull) return ZR_ERR_UNSUPPORTED;
    return ZR_OK;
}

void build_tiles_for_layout(zr_plan& p) {
    build_tiles(p);
    if (p.param_layout != ZR_PARAMS_OWNED) return;
    for (std::vector<Tile>* table : {&p.tiles, &p.tiles_by_owned}) {
        for (Tile& t : *table) {
            t.global = t.owned;
            if (t.flags & kTileVector) t.flags |= kTileStoreVector;   // owned offsets of vector tiles are 8-aligned
        }
    }
}

static uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

WorkspaceLayout workspace_layout(const zr_plan& p) {
    WorkspaceLayout L{};
    uint64_t off = 0;
    L.tiles = off;
    off = align256(off + sizeof(Tile) * std::max<size_t>(1, p.tiles.size()));
    L.tiles_by_owned = off;
    off = align256(off + sizeof(Tile) * std::max<size_t>(1, p.tiles.size()));
    L.tile_partials = off;
    off = align256(off + (p.clip_enabled() ? sizeof(double) * std::max<size_t>(1, p.tiles.size()) : 0));
    const uint64_t groups = static_cast<uint64_t>(clip_groups(static_cast<int32_t>(std::max<size_t>(1, p.tiles.size()))));
    L.clip_ticket = off;
    off = align256(off + (p.clip_enabled() ? sizeof(uint32_t) : 0));
    L.clip_group_sums = off;
    off = align256(off + (p.clip_enabled() ? sizeof(double) * groups : 0));
    L.clip_coef = off;
    off = align256(off + sizeof(float));
    L.own_sumsq = off;
    off = align256(off + sizeof(double));
    L.gather_targets = off;
    off = align256(off + sizeof(void*) * static_cast<uint64_t>(p.world_size));
    L.dev_scalars = off;
    off = align256(off + sizeof(AdamScalars));
    L.check = off;
    off = align256(off + sizeof(uint64_t) * kCheckWords);
    L.gather_pieces = off;
    off = align256(off + sizeof(GatherPiece) * std::max<size_t>(1, p.gather_pieces.size()));
    L.g_scratch = off;
    off = align256(off + (p.clip_uses_scratch() ? sizeof(float) * static_cast<uint64_t>(p.owned_numel()) : 0));
    L.total = off;
    return L;
}

template <typename Entry>
static uint64_t hash_entries(const std::vector<Entry>& table) {
    static_assert(sizeof(Entry) == sizeof(uint64_t) * kTileWords, "4-word entries");
    uint64_t h = 0;
    for (size_t i = 0; i < table.size(); ++i) {
        uint64_t w[kTileWords];
        std::memcpy(w, &table[i], sizeof(Entry));
        for (int j = 0; j < kTileWords; ++j) h += tile_word_hash(w[j], kTileWords * i + j);
    }
    return h;
}

uint64_t table_hash(const std::vector<Tile>& tiles) { return hash_entries(tiles); }
uint64_t table_hash(const std::vector<GatherPiece>& pieces) { return hash_entries(pieces); }

AdamScalars adam_scalars(const zr_adamw& hp, int64_t step) {
    const double b1 = hp.beta1, b2 = hp.beta2, lr = hp.lr, t = static_cast<double>(step);
    AdamScalars s;
    s.beta1 = hp.beta1;
    s.beta2 = hp.beta2;
    s.one_minus_beta1 = static_cast<float>(1.0 - b1);
    s.one_minus_beta2 = static_cast<float>(1.0 - b2);
    s.step_size = static_cast<float>(lr / (1.0 - std::pow(b1, t)));
    s.bc2_sqrt = static_cast<float>(std::sqrt(1.0 - std::pow(b2, t)));
    s.decay = static_cast<float>(1.0 - lr * static_cast<double>(hp.weight_decay));
    s.eps = hp.eps;
    return s;
}

}  // namespace zr
