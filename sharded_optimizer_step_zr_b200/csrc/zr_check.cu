// Checked mode's kernels: verification of a plan's device tile tables.
//
// The tables live in the caller's workspace, so another kernel that writes
// there by mistake (a race, a stray pointer) would send the next step to
// wrong or out-of-bounds addresses.  With checked mode on, every launching
// call first runs this kernel: it tests every tile against the invariants
// the planner guarantees, hashes both tables, compares the hashes with the
// ones the host took when it uploaded the tables and, if anything failed,
// empties the tables so that the step that
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

__device__ __forceinline__ uint64_t tile_hash(const Tile* table, int32_t i) {
    const uint64_t* w = reinterpret_cast<const uint64_t*>(table + i);
    uint64_t h = 0;
#pragma unroll
    for (int j = 0; j < kTileWords; ++j) h += tile_word_hash(w[j], static_cast<uint64_t>(kTileWords) * i + j);
    return h;
}

// One launch.  Grid-stride over both tables: count the tiles that break an
// invariant (a bucket-order tile must also sit at its own index), keep the
// smallest failing position, and add every tile's words into the two hash
// sums.  The last block to finish (a counter of finished blocks; nothing
// waits) compares the sums with the host's, records mismatches, resets the
// sums and the counter for the next check and, if anything has failed (now
// or at an earlier check since the workspace was bound), empties both tables
// -- every tile gets length 0 and its own position as index -- so that the
// kernels queued after this one touch no parameter memory.
__global__ void __launch_bounds__(256)
zr_verify_tables_kernel(Tile* tiles, Tile* by_owned, int32_t n_tiles, int64_t n_owned, int64_t n_out,
                        int32_t n_buckets, unsigned long long hash_tiles, unsigned long long hash_by_owned,
                        unsigned long long* check) {
    unsigned long long h0 = 0, h1 = 0;
    for (int32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n_tiles; i += gridDim.x * blockDim.x) {
        const Tile a = tiles[i], b = by_owned[i];
        if (!tile_ok(a, n_owned, n_out, n_buckets, n_tiles) || a.index != i) {
            atomicAdd(&check[0], 1ull);
            atomicMin(&check[1], static_cast<unsigned long long>(i));
        }
        if (!tile_ok(b, n_owned, n_out, n_buckets, n_tiles)) {
            atomicAdd(&check[0], 1ull);
            atomicMin(&check[1], static_cast<unsigned long long>(n_tiles) + i);
        }
        h0 += tile_hash(tiles, i);
        h1 += tile_hash(by_owned, i);
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
        h0 += __shfl_down_sync(0xFFFFFFFFu, h0, d);
        h1 += __shfl_down_sync(0xFFFFFFFFu, h1, d);
    }
    if ((threadIdx.x & 31) == 0) {
        atomicAdd(&check[3], h0);
        atomicAdd(&check[4], h1);
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
        const unsigned long long s0 = atomicExch(&check[3], 0ull), s1 = atomicExch(&check[4], 0ull);
        atomicExch(&check[5], 0ull);
        const unsigned long long bits = (s0 != hash_tiles ? 1ull : 0ull) | (s1 != hash_by_owned ? 2ull : 0ull);
        const unsigned long long mismatch = atomicOr(&check[2], bits) | bits;
        failed = (mismatch != 0 || atomicAdd(&check[0], 0ull) != 0) ? 1 : 0;
    }
    __syncthreads();
    if (!failed) return;
    for (int32_t i = threadIdx.x; i < n_tiles; i += blockDim.x) {
        Tile empty{};
        empty.index = i;
        tiles[i] = empty;
        by_owned[i] = empty;
    }
}

}  // namespace

int launch_verify_tables(Tile* tiles, Tile* tiles_by_owned, int32_t n_tiles, int64_t n_owned, int64_t n_out,
                         int32_t n_buckets, uint64_t hash_tiles, uint64_t hash_by_owned, uint64_t* check,
                         void* stream_v) {
    if (n_tiles == 0) return cudaSuccess;
    const int blocks = static_cast<int>(std::min<int64_t>((n_tiles + 255) / 256, 148 * 4));
    zr_verify_tables_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream_v)>>>(
        tiles, tiles_by_owned, n_tiles, n_owned, n_out, n_buckets, hash_tiles, hash_by_owned,
        reinterpret_cast<unsigned long long*>(check));
    return cudaGetLastError();
}

}  // namespace zr
