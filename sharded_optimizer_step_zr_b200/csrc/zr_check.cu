// Checked mode's kernels: verification of a plan's device tile tables.
//
// The tables live in the caller's workspace, so another kernel that writes
// there by mistake (a race, a stray pointer) would send the next step to
// wrong or out-of-bounds addresses.  With checked mode on, every launching
// call first runs these two kernels: the first tests every tile against the
// invariants the planner guarantees and hashes both tables; the second
// compares the hashes with the ones the host took when it uploaded the
// tables and, if anything failed, empties the tables so that the step that
// follows touches no parameter memory.  Neither waits on anything.
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

// Grid-stride over both tables: count the tiles that break an invariant
// (a bucket-order tile must also sit at its own index), keep the smallest
// failing position, and add every tile's words into the two hash sums.
__global__ void __launch_bounds__(256)
zr_verify_tables_kernel(const Tile* tiles, const Tile* by_owned, int32_t n_tiles, int64_t n_owned, int64_t n_out,
                        int32_t n_buckets, unsigned long long* check) {
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
}

// After the verification: compare the hashes with the host's, record the
// mismatches, and if anything has failed (now or at an earlier check since
// the workspace was bound) empty both tables -- every tile gets length 0 and
// its own position as index -- so that kernels queued after this touch no
// parameter memory.  Every block decides from the same words; block 0
// records the mismatch bits.
__global__ void __launch_bounds__(256)
zr_neutralise_tables_kernel(Tile* tiles, Tile* by_owned, int32_t n_tiles, unsigned long long hash_tiles,
                            unsigned long long hash_by_owned, unsigned long long* check) {
    const unsigned long long bits = (check[3] != hash_tiles ? 1ull : 0ull) | (check[4] != hash_by_owned ? 2ull : 0ull);
    if (blockIdx.x == 0 && threadIdx.x == 0 && bits) atomicOr(&check[2], bits);
    if (bits == 0 && check[0] == 0 && check[2] == 0) return;
    for (int32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n_tiles; i += gridDim.x * blockDim.x) {
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
    cudaStream_t s = static_cast<cudaStream_t>(stream_v);
    const int blocks = static_cast<int>(std::min<int64_t>((n_tiles + 255) / 256, 148 * 4));
    unsigned long long* c = reinterpret_cast<unsigned long long*>(check);
    zr_verify_tables_kernel<<<blocks, 256, 0, s>>>(tiles, tiles_by_owned, n_tiles, n_owned, n_out, n_buckets, c);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    zr_neutralise_tables_kernel<<<blocks, 256, 0, s>>>(tiles, tiles_by_owned, n_tiles, hash_tiles, hash_by_owned, c);
    return cudaGetLastError();
}

}  // namespace zr
