// prefix_hash: hashes of every full KV block of every sequence, for finding
// cached prefix blocks again.
//
// What it computes ("Infra: PagedAttention", section 共享前缀，分叉时
// Copy-on-write, the paragraphs on Automatic Prefix Caching): only full
// blocks are hashed, and a block's hash covers the hash of the block before
// it, the block's tokens and a per-sequence context key (a LoRA id, say), so
// equal hashes mean the whole prefix matches.  Definitions (the pages name no
// function): FNV-1a 64 (Fowler, Noll, Vo): h = 0xcbf29ce484222325, per byte
// h = (h ^ byte) * 0x100000001b3.  Block digest c_b = FNV-1a over the block's
// tokens (int32, little-endian bytes) then the key (uint64, little-endian);
// hash h_b = FNV-1a over h_{b-1} then c_b (uint64 LE each), h_{-1} = 0.
//
// One warp per sequence: the lanes hash the contents of 32 consecutive blocks
// side by side, then every lane walks the short parent chain over those 32
// digests (uniformly, from shuffles) and keeps its own block's hash.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

constexpr uint64_t FNV64_OFFSET = 0xCBF29CE484222325ull;
constexpr uint64_t FNV64_PRIME = 0x100000001B3ull;

// One FNV-1a step, (h ^ b) * FNV64_PRIME mod 2^64, on 32-bit halves: the
// prime is 2^40 + 0x1b3, so with x = h ^ b = (hi, lo)
//   x * prime = lo * 0x1b3 + ((hi * 0x1b3 + (lo << 8)) mod 2^32) * 2^32,
// one wide multiply and one short one instead of a general 64-bit product.
__device__ __forceinline__ uint64_t fnv_byte(uint64_t h, uint32_t b) {
    const uint32_t lo = (uint32_t)h ^ b;
    const uint32_t hi = (uint32_t)(h >> 32);
    const uint64_t t = (uint64_t)lo * 0x1b3u;
    const uint32_t nhi = (uint32_t)(t >> 32) + hi * 0x1b3u + (lo << 8);
    return ((uint64_t)nhi << 32) | (uint32_t)t;
}

__device__ __forceinline__ uint64_t fnv_u32(uint64_t h, uint32_t v) {
#pragma unroll
    for (int i = 0; i < 4; ++i) h = fnv_byte(h, (v >> (8 * i)) & 0xFFu);
    return h;
}

__device__ __forceinline__ uint64_t fnv_u64(uint64_t h, uint64_t v) {
    h = fnv_u32(h, (uint32_t)v);
    return fnv_u32(h, (uint32_t)(v >> 32));
}

__global__ void __launch_bounds__(256)
prefix_hash_kernel(const int32_t* __restrict__ tokens, long long row_stride,
                   const int32_t* __restrict__ seq_lens, const uint64_t* __restrict__ extra_keys,
                   const int32_t* __restrict__ first_block,      // null: 0
                   const uint64_t* __restrict__ parent_hashes,   // null: 0
                   int num_seqs, int block_size, uint64_t* __restrict__ hashes, int max_blocks) {
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int s = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); s < num_seqs; s += warps) {
        long long len = __ldg(seq_lens + s);
        if (len > row_stride) {
            if (lane == 0) raise_status(PKV_DEV_LENGTH);
            len = row_stride;
        }
        long long full = len > 0 ? len / block_size : 0;
        if (full > max_blocks) {
            if (lane == 0) raise_status(PKV_DEV_LENGTH);
            full = max_blocks;
        }
        const uint64_t key = extra_keys ? __ldg(extra_keys + s) : 0ull;
        const int32_t* row = tokens + (size_t)s * row_stride;
        // resume: blocks before `start` are hashed already; parent is the hash
        // of block start - 1 (ignored at start 0)
        long long start = first_block ? __ldg(first_block + s) : 0;
        if (start < 0) start = 0;
        uint64_t parent = (start > 0 && parent_hashes) ? __ldg(parent_hashes + s) : 0ull;
        for (long long b0 = start; b0 < full; b0 += 32) {
            const long long b = b0 + lane;
            uint64_t c = 0;
            if (b < full) {
                // tokens loaded 8 at a time ahead of the hashing, so a block
                // costs a round trip per 8 tokens, not one per token
                uint64_t h = FNV64_OFFSET;
                const int32_t* t = row + b * block_size;
                int i = 0;
                for (; i + 8 <= block_size; i += 8) {
                    uint32_t v[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) v[k] = (uint32_t)__ldg(t + i + k);
#pragma unroll
                    for (int k = 0; k < 8; ++k) h = fnv_u32(h, v[k]);
                }
                for (; i < block_size; ++i) h = fnv_u32(h, (uint32_t)__ldg(t + i));
                c = fnv_u64(h, key);
            }
            const int n = full - b0 < 32 ? (int)(full - b0) : 32;
            uint64_t mine = 0;
            for (int j = 0; j < n; ++j) {
                const uint64_t cj = __shfl_sync(0xFFFFFFFFu, c, j);
                parent = fnv_u64(fnv_u64(FNV64_OFFSET, parent), cj);
                if (lane == j) mine = parent;
            }
            if (b < full) hashes[(size_t)s * max_blocks + b] = mine;
        }
    }
}

}  // namespace pkv
