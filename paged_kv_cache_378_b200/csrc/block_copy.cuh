// block_copy: copy-on-write of whole physical blocks, every layer, K and V.
//
// "Infra: PagedAttention", section 共享前缀，分叉时 Copy-on-write: the shared,
// partially filled tail is copied before a writer appends; full blocks stay
// shared.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

// Work: for every (pair, layer, K|V) one block of all heads, contiguous
// (num_kv_heads * block_size * head_dim bf16 = chunks_per_block 16-byte
// chunks).  The flattened (unit, chunk) space is walked with a grid stride;
// four independent chunk copies per thread per step keep loads in flight.
// Source and destination pools may differ (block swap between the device
// pool and a pinned host pool): each has its own block count.
__global__ void __launch_bounds__(256)
block_copy_kernel(uint4* __restrict__ dst_k, uint4* __restrict__ dst_v,
                  const uint4* __restrict__ src_k, const uint4* __restrict__ src_v,
                  const int32_t* __restrict__ pairs, int num_pairs, int num_layers,
                  int src_blocks, int dst_blocks, long long chunks_per_block,
                  const int32_t* __restrict__ d_num_pairs) {   // null: num_pairs is the count
    pdl_launch_dependents();
    pdl_wait();                                          // earlier writes to the pools land first
    if (d_num_pairs) {
        const int n = *d_num_pairs;
        num_pairs = n < 0 ? 0 : (n < num_pairs ? n : num_pairs);
    }
    const long long units = (long long)num_pairs * num_layers * 2;
    const long long total = units * chunks_per_block;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long base = blockIdx.x * (long long)blockDim.x + threadIdx.x; base < total;
         base += 4 * stride) {
        uint4 v[4];
        uint4* dptr[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            dptr[k] = nullptr;
            const long long i = base + k * stride;
            if (i >= total) continue;
            const long long u = i / chunks_per_block;
            const long long c = i - u * chunks_per_block;
            const int which = (int)(u & 1);
            const long long pl = u >> 1;
            const int pair = (int)(pl / num_layers);
            const int layer = (int)(pl - (long long)pair * num_layers);
            const int src = __ldg(pairs + 2 * pair);
            const int dst = __ldg(pairs + 2 * pair + 1);
            if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
                if (c == 0) raise_status(PKV_DEV_RANGE);
                continue;
            }
            const uint4* sp = which ? src_v : src_k;
            uint4* dp = which ? dst_v : dst_k;
            v[k] = sp[((size_t)layer * src_blocks + src) * chunks_per_block + c];
            dptr[k] = dp + ((size_t)layer * dst_blocks + dst) * chunks_per_block + c;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (dptr[k]) *dptr[k] = v[k];
    }
}

}  // namespace pkv
