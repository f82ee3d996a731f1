// kv_append: scatter each new token's K and V (all kv heads) into its slot.
//
// "Infra: PagedAttention", section 按 Block 分配: a new token fills the tail
// block's next slot; slot s is row s % B of physical block s / B.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

// One thread moves one 16-byte chunk (8 bf16) of one token's K or V row for
// one kv head.  Chunks of one token are adjacent threads, so a warp reads
// contiguous bytes of k_new/v_new and writes whole 16-byte pieces of rows.
__global__ void __launch_bounds__(256)
kv_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                 uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,  // layer base
                 const int64_t* __restrict__ slot_mapping, int num_tokens,
                 int num_kv_heads, int block_size, int head_dim, int num_blocks) {
    pdl_launch_dependents();
    pdl_wait();                                          // earlier writes to the pool land first
    const int chunks_per_row = head_dim / 8;            // uint4 per head row
    const int chunks_per_tok = num_kv_heads * chunks_per_row;
    const long long total = (long long)num_tokens * chunks_per_tok * 2;
    const long long slot_limit = (long long)num_blocks * block_size;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int which = (int)(i / ((long long)num_tokens * chunks_per_tok));   // 0 = K, 1 = V
        const long long r = i - (long long)which * num_tokens * chunks_per_tok;
        const int t = (int)(r / chunks_per_tok);
        const int c = (int)(r - (long long)t * chunks_per_tok);
        const int h = c / chunks_per_row;
        const int j = c - h * chunks_per_row;
        const long long slot = slot_mapping[t];
        if (slot < 0) continue;                          // padding token
        if (slot >= slot_limit) {
            raise_status(PKV_DEV_RANGE);
            continue;
        }
        const long long blk = slot / block_size;
        const int row = (int)(slot - blk * block_size);
        const size_t dst = (((size_t)blk * num_kv_heads + h) * block_size + row) * chunks_per_row + j;
        const size_t src = (size_t)t * chunks_per_tok + c;
        if (which == 0)
            k_pool[dst] = __ldg(k_new + src);
        else
            v_pool[dst] = __ldg(v_new + src);
    }
}

}  // namespace pkv
