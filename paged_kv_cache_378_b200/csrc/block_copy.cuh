// block_copy: copy-on-write of whole physical blocks, every layer, K and V.
//
// "Infra: PagedAttention", section 共享前缀，分叉时 Copy-on-write: the shared,
// partially filled tail is copied before a writer appends; full blocks stay
// shared.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

// Work unit = (pair, layer, K|V): one block of all heads, contiguous
// (num_kv_heads * block_size * head_dim bf16).  Each CTA walks units with a
// grid stride; its threads copy the unit's 16-byte chunks.
__global__ void __launch_bounds__(256)
block_copy_kernel(uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                  const int32_t* __restrict__ pairs, int num_pairs, int num_layers,
                  int num_blocks, long long chunks_per_block) {
    const long long units = (long long)num_pairs * num_layers * 2;
    for (long long u = blockIdx.x; u < units; u += gridDim.x) {
        const int which = (int)(u & 1);
        const long long pl = u >> 1;
        const int pair = (int)(pl / num_layers);
        const int layer = (int)(pl - (long long)pair * num_layers);
        const int src = pairs[2 * pair];
        const int dst = pairs[2 * pair + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            if (threadIdx.x == 0) raise_status(PKV_DEV_RANGE);
            continue;
        }
        uint4* pool = which ? v_pool : k_pool;
        const size_t layer_base = (size_t)layer * num_blocks * chunks_per_block;
        const uint4* s = pool + layer_base + (size_t)src * chunks_per_block;
        uint4* d = pool + layer_base + (size_t)dst * chunks_per_block;
        for (long long i = threadIdx.x; i < chunks_per_block; i += blockDim.x) d[i] = s[i];
    }
}

}  // namespace pkv
