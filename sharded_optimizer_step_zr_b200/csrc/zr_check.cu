// Checked mode's kernels: verification of a plan's device tile tables.
//
// The tables live in the caller's workspace, so another kernel that writes
// there by mistake (a race, a stray pointer) would send the next step to
// wrong or out-of-bounds addresses.  With checked mode on, every launching
// call first runs this kernel: it tests every tile and gather piece against
// the invariants the planner guarantees, hashes the three tables, compares
// the hashes with the ones the host took when it uploaded them and, if
// anything failed, empties the tables so that the step or gather that
// follows touches no parameter memory.  Nothing waits on anything.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "zr_internal.hpp"

namespace zr {
namespace {

// The invariants every tile of a plan satisfies (the planner's own
// self-check establishes them on the host): a length of 1..kTileElems, an
// owned range inside [0, n_owned), a global range inside [0, n_out), only
// the two known flags and only where their 8-element alignment holds, a
// bucket and an index inside their ranges.
__device__ __forceinline__ bool tile_ok(const Tile& t, int64_t n_owned, int64_t n_out, int32_t n_buckets,
                                        int32_t n_tiles) {
    if (t.len < 1 || t.len > kTileElems) return false;
    if (t.owned < 0 || t.owned > n_owned - t.len) return false;
    if (t.global < 0 || t.global > n_out - t.len) return false;
    if ((t.flags & ~(kTileVector | kTileStoreVector)) != 0) return false;
    const bool vec = (t.owned % 8 == 0) && (t.len % 8 == 0);
    if ((t.flags & kTileVector) && !vec) return false;
    if ((t.flags & kTileStoreVector) && !((t.flags & kTileVector) && t.global % 8 == 0)) return false;
    return t.bucket >= 0 && t.bucket < n_buckets && t.index >= 0 && t.index < n_tiles;
}

// A gather piece: a length of 1..kGatherPieceElems, an owner and a tensor
// in range, a destination inside [0, total_numel).  (Its source offset is
// bounded by the owner's shard, which only the host knows; the hash covers
// it.)
__device__ __forceinline__ bool piece_ok(const GatherPiece& g, int32_t world_size, int64_t total_numel,
                                         int32_t n_tensors) {
    if (g.len < 1 || g.len > kGatherPieceElems) return false;
    if (g.owner < 0 || g.owner >= world_size || g.tensor < 0 || g.tensor >= n_tensors) return false;
    if (g.src < 0 || g.dst < 0 || g.dst > total_numel - g.len) return false;
    return g.reserved == 0;
}

template <typename Entry>
__device__ __forceinline__ uint64_t entry_hash(const Entry* table, int32_t i) {
    const uint64_t* w = reinterpret_cast<const uint64_t*>(table + i);
    uint64_t h = 0;
#pragma unroll
    for (int j = 0; j < kTileWords; ++j) h += tile_word_hash(w[j], static_cast<uint64_t>(kTileWords) * i + j);
    return h;
}

// One launch.  Grid-stride over the three tables: count the entries that
// break an invariant (a bucket-order tile must also sit at its own index),
// keep the smallest failing position, and add every entry's words into the
// tables' hash sums.  The last block to finish (a counter of finished
// blocks; nothing waits) compares the sums with the host's, records
// mismatches, resets the sums and the counter for the next check and, if
// anything has failed (now or at an earlier check since the workspace was
// bound), empties every table -- tiles get length 0 and their own position
// as index, gather pieces length 0 -- so that the kernels queued after this
// one touch no parameter memory.
__global__ void __launch_bounds__(256) zr_verify_tables_kernel(const VerifyArgs a) {
    unsigned long long* check = reinterpret_cast<unsigned long long*>(a.check);
    unsigned long long h0 = 0, h1 = 0, h2 = 0;
    const int32_t n = a.n_tiles > a.n_pieces ? a.n_tiles : a.n_pieces;
    for (int32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        if (i < a.n_tiles) {
            const Tile t = a.tiles[i], b = a.tiles_by_owned[i];
            if (!tile_ok(t, a.n_owned, a.n_out, a.n_buckets, a.n_tiles) || t.index != i) {
                atomicAdd(&check[0], 1ull);
                atomicMin(&check[1], static_cast<unsigned long long>(i));
            }
            if (!tile_ok(b, a.n_owned, a.n_out, a.n_buckets, a.n_tiles)) {
                atomicAdd(&check[0], 1ull);
                atomicMin(&check[1], static_cast<unsigned long long>(a.n_tiles) + i);
            }
            h0 += entry_hash(a.tiles, i);
            h1 += entry_hash(a.tiles_by_owned, i);
        }
        if (i < a.n_pieces) {
            if (!piece_ok(a.pieces[i], a.world_size, a.total_numel, a.n_tensors)) {
                atomicAdd(&check[0], 1ull);
                atomicMin(&check[1], 2ull * static_cast<unsigned long long>(a.n_tiles) + i);
            }
            h2 += entry_hash(a.pieces, i);
        }
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
        h0 += __shfl_down_sync(0xFFFFFFFFu, h0, d);
        h1 += __shfl_down_sync(0xFFFFFFFFu, h1, d);
        h2 += __shfl_down_sync(0xFFFFFFFFu, h2, d);
    }
    if ((threadIdx.x & 31) == 0) {
        atomicAdd(&check[3], h0);
        atomicAdd(&check[4], h1);
        atomicAdd(&check[6], h2);
    }
    __shared__ int last, failed;
    __syncthreads();                      // every warp of the block has added its sums
    if (threadIdx.x == 0) {
        __threadfence();
        last = atomicAdd(&check[5], 1ull) == gridDim.x - 1ull;
    }
    __syncthreads();
    if (!last) return;
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned long long s0 = atomicExch(&check[3], 0ull), s1 = atomicExch(&check[4], 0ull),
                                 s2 = atomicExch(&check[6], 0ull);
        atomicExch(&check[5], 0ull);
        const unsigned long long bits = (s0 != a.hash_tiles ? 1ull : 0ull) | (s1 != a.hash_by_owned ? 2ull : 0ull) |
                                        (s2 != a.hash_pieces ? 4ull : 0ull);
        const unsigned long long mismatch = atomicOr(&check[2], bits) | bits;
        failed = (mismatch != 0 || atomicAdd(&check[0], 0ull) != 0) ? 1 : 0;
    }
    __syncthreads();
    if (!failed) return;
    for (int32_t i = threadIdx.x; i < a.n_tiles; i += blockDim.x) {
        Tile empty{};
        empty.index = i;
        a.tiles[i] = empty;
        a.tiles_by_owned[i] = empty;
    }
    for (int32_t i = threadIdx.x; i < a.n_pieces; i += blockDim.x) a.pieces[i] = GatherPiece{};
}

}  // namespace

int launch_verify_tables(const VerifyArgs& args, void* stream_v) {
    const int32_t n = args.n_tiles > args.n_pieces ? args.n_tiles : args.n_pieces;
    if (n == 0) return cudaSuccess;
    const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, 148 * 4));
    zr_verify_tables_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream_v)>>>(args);
    return cudaGetLastError();
}

}  // namespace zr
