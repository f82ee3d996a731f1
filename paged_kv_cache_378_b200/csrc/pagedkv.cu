// Host side of the C ABI declared in include/pagedkv.h: argument checks,
// launch shapes and template dispatch.  Every entry point launches on the
// caller's stream and never synchronises (except pkv_get_device_status).
#include <cmath>
#include <cstdint>
#include <cstring>

#include <cuda_runtime.h>

#include "pagedkv.h"
#include "pkv_device.cuh"
#include "kv_append.cuh"
#include "block_copy.cuh"
#include "paged_attention.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kAttnWarps = 4;

int device_sm_count() {
    static int cached[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_head_dim(int d) { return d == 64 || d == 128; }
bool supported_block_size(int b) { return b == 8 || b == 16 || b == 32; }

int check_cache(const pkv_cache_t* c) {
    if (!c || !c->k_pool || !c->v_pool) return PKV_ERR_NULL;
    if (c->num_layers <= 0 || c->num_blocks <= 0 || c->num_kv_heads <= 0 || c->block_size <= 0 ||
        c->head_dim <= 0)
        return PKV_ERR_SHAPE;
    if (!supported_head_dim(c->head_dim) || !supported_block_size(c->block_size))
        return PKV_ERR_UNSUPPORTED;
    if (!aligned16(c->k_pool) || !aligned16(c->v_pool)) return PKV_ERR_ALIGN;
    return PKV_OK;
}

size_t layer_elems(const pkv_cache_t* c) {
    return (size_t)c->num_blocks * c->num_kv_heads * c->block_size * c->head_dim;
}

int launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int tile_tokens(int block_size) { return block_size < 16 ? 16 : block_size; }

// KV partition length.  Default: 256 tokens, grown while a launch would
// still have more than 16 CTAs per SM at full length, so long sequences are
// split across SMs while short-sequence batches keep few partitions.
int resolve_partition(int num_seqs, int num_kv_heads, int max_blocks, int block_size,
                      int requested) {
    if (num_seqs < 0 || num_kv_heads <= 0 || max_blocks <= 0 || !supported_block_size(block_size))
        return -1;
    const int tile = tile_tokens(block_size);
    long long pt;
    if (requested > 0) {
        pt = requested;
    } else {
        const long long max_len = (long long)max_blocks * block_size;
        const long long units = (long long)num_seqs * num_kv_heads;
        const long long sms = device_sm_count();
        pt = 256;
        while (pt < 4096 && units * ((max_len + pt - 1) / pt) > 16 * sms) pt *= 2;
    }
    pt = (pt + tile - 1) / tile * tile;
    if (pt > (1LL << 30)) return -1;
    return (int)pt;
}

struct WorkspaceLayout {
    size_t o_off, mz_off, cnt_off, total;
    int partitions;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool workspace_layout(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                      int max_blocks, int block_size, int partition_tokens, WorkspaceLayout* w) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads ||
        !supported_head_dim(head_dim) || max_blocks <= 0 || !supported_block_size(block_size))
        return false;
    const int pt = resolve_partition(num_seqs, num_kv_heads, max_blocks, block_size, partition_tokens);
    if (pt <= 0) return false;
    const long long max_len = (long long)max_blocks * block_size;
    const int parts = (int)((max_len + pt - 1) / pt);
    const size_t units = (size_t)num_seqs * num_kv_heads;
    const size_t G = (size_t)(num_q_heads / num_kv_heads);
    w->partitions = parts;
    w->o_off = 0;
    w->mz_off = align_up(units * parts * G * head_dim * sizeof(float), 256);
    w->cnt_off = w->mz_off + align_up(units * parts * G * sizeof(float2), 256);
    w->total = w->cnt_off + align_up(units * sizeof(unsigned int), 256);
    return true;
}

template <int D, int G, int BS>
int launch_attention(const pkv::AttnArgs& args, int num_seqs, cudaStream_t s) {
    using C = pkv::AttnCfg<D, G, BS, kAttnWarps>;
    auto kern = pkv::paged_attention_kernel<D, G, BS, kAttnWarps>;
    static bool configured[kMaxDevices] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < kMaxDevices && !configured[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
            cudaSuccess)
            return PKV_ERR_CUDA;
        configured[dev] = true;
    }
    const dim3 grid(args.num_partitions, args.num_kv_heads, num_seqs);
    kern<<<grid, kAttnWarps * 32, C::SMEM_BYTES, s>>>(args);
    return launch_status();
}

template <int D, int G>
int dispatch_block(int bs, const pkv::AttnArgs& a, int n, cudaStream_t s) {
    switch (bs) {
        case 8: return launch_attention<D, G, 8>(a, n, s);
        case 16: return launch_attention<D, G, 16>(a, n, s);
        case 32: return launch_attention<D, G, 32>(a, n, s);
    }
    return PKV_ERR_UNSUPPORTED;
}

template <int D>
int dispatch_group(int g, int bs, const pkv::AttnArgs& a, int n, cudaStream_t s) {
    switch (g) {
        case 1: return dispatch_block<D, 1>(bs, a, n, s);
        case 2: return dispatch_block<D, 2>(bs, a, n, s);
        case 4: return dispatch_block<D, 4>(bs, a, n, s);
        case 8: return dispatch_block<D, 8>(bs, a, n, s);
    }
    return PKV_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

int pkv_abi_version(void) { return PKV_ABI_VERSION; }

const char* pkv_strerror(int code) {
    switch (code) {
        case PKV_OK: return "ok";
        case PKV_ERR_NULL: return "a required pointer is NULL";
        case PKV_ERR_SHAPE: return "a size is negative or inconsistent";
        case PKV_ERR_ALIGN: return "a bf16 buffer is not 16-byte aligned";
        case PKV_ERR_WORKSPACE: return "workspace missing or too small";
        case PKV_ERR_UNSUPPORTED: return "head_dim / block_size / group size not supported";
        case PKV_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
        case PKV_ERR_LAYER: return "layer index outside the cache";
    }
    return "unknown pagedkv status";
}

int pkv_kv_append(const pkv_cache_t* cache, int layer, const void* k_new, const void* v_new,
                  const int64_t* slot_mapping, int num_tokens, void* stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (num_tokens < 0) return PKV_ERR_SHAPE;
    if (layer < 0 || layer >= cache->num_layers) return PKV_ERR_LAYER;
    if (num_tokens == 0) return PKV_OK;
    if (!k_new || !v_new || !slot_mapping) return PKV_ERR_NULL;
    if (!aligned16(k_new) || !aligned16(v_new)) return PKV_ERR_ALIGN;
    const size_t base = (size_t)layer * layer_elems(cache);
    const long long total = (long long)num_tokens * cache->num_kv_heads * (cache->head_dim / 8) * 2;
    const int threads = 256;
    long long blocks = (total + threads - 1) / threads;
    const long long cap = (long long)device_sm_count() * 16;
    if (blocks > cap) blocks = cap;
    pkv::kv_append_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const uint4*>(k_new), reinterpret_cast<const uint4*>(v_new),
        reinterpret_cast<uint4*>(static_cast<uint16_t*>(cache->k_pool) + base),
        reinterpret_cast<uint4*>(static_cast<uint16_t*>(cache->v_pool) + base), slot_mapping,
        num_tokens, cache->num_kv_heads, cache->block_size, cache->head_dim, cache->num_blocks);
    return launch_status();
}

int pkv_block_copy(const pkv_cache_t* cache, const int32_t* src_dst_pairs, int num_pairs,
                   void* stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (num_pairs < 0) return PKV_ERR_SHAPE;
    if (num_pairs == 0) return PKV_OK;
    if (!src_dst_pairs) return PKV_ERR_NULL;
    const long long chunks = (long long)cache->num_kv_heads * cache->block_size * cache->head_dim / 8;
    long long units = (long long)num_pairs * cache->num_layers * 2;
    const long long cap = (long long)device_sm_count() * 8;
    const unsigned grid = (unsigned)(units < cap ? units : cap);
    pkv::block_copy_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<uint4*>(cache->k_pool), reinterpret_cast<uint4*>(cache->v_pool),
        src_dst_pairs, num_pairs, cache->num_layers, cache->num_blocks, chunks);
    return launch_status();
}

int pkv_partition_tokens(int num_seqs, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                         int block_size, int requested) {
    if (!supported_head_dim(head_dim) || requested < 0) return -1;
    return resolve_partition(num_seqs, num_kv_heads, max_blocks_per_seq, block_size, requested);
}

size_t pkv_attention_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                     int max_blocks_per_seq, int block_size, int partition_tokens) {
    if (partition_tokens < 0) return 0;
    WorkspaceLayout w;
    if (!workspace_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                          block_size, partition_tokens, &w))
        return 0;
    return w.total;
}

int pkv_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
    if (workspace_bytes == 0) return PKV_OK;
    if (!workspace) return PKV_ERR_NULL;
    if (cudaMemsetAsync(workspace, 0, workspace_bytes, (cudaStream_t)stream) != cudaSuccess)
        return PKV_ERR_CUDA;
    return PKV_OK;
}

int pkv_paged_decode_attention(const pkv_cache_t* cache, int layer, const void* q, int num_seqs,
                               int num_q_heads, const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* seq_lens, float scale, void* out, void* workspace,
                               size_t workspace_bytes, int partition_tokens, void* stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (layer < 0 || layer >= cache->num_layers) return PKV_ERR_LAYER;
    if (num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0 || partition_tokens < 0)
        return PKV_ERR_SHAPE;
    if (num_q_heads % cache->num_kv_heads) return PKV_ERR_SHAPE;
    if (!std::isfinite(scale)) return PKV_ERR_SHAPE;
    const int G = num_q_heads / cache->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return PKV_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PKV_OK;
    if (num_seqs > 65535 || cache->num_kv_heads > 65535) return PKV_ERR_SHAPE;
    if (!q || !block_tables || !seq_lens || !out) return PKV_ERR_NULL;
    if (!aligned16(q) || !aligned16(out)) return PKV_ERR_ALIGN;
    WorkspaceLayout w;
    if (!workspace_layout(num_seqs, num_q_heads, cache->num_kv_heads, cache->head_dim,
                          max_blocks_per_seq, cache->block_size, partition_tokens, &w))
        return PKV_ERR_SHAPE;
    if (w.partitions > 1) {
        if (!workspace) return PKV_ERR_WORKSPACE;
        if (workspace_bytes < w.total || !aligned16(workspace)) return PKV_ERR_WORKSPACE;
    }
    pkv::AttnArgs a;
    const size_t base = (size_t)layer * layer_elems(cache);
    a.q = static_cast<const uint16_t*>(q);
    a.k_pool = static_cast<const uint16_t*>(cache->k_pool) + base;
    a.v_pool = static_cast<const uint16_t*>(cache->v_pool) + base;
    a.out = static_cast<uint16_t*>(out);
    a.block_tables = block_tables;
    a.seq_lens = seq_lens;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    a.part_o = ws ? reinterpret_cast<float*>(ws + w.o_off) : nullptr;
    a.part_mz = ws ? reinterpret_cast<float2*>(ws + w.mz_off) : nullptr;
    a.counters = ws ? reinterpret_cast<unsigned int*>(ws + w.cnt_off) : nullptr;
    a.num_kv_heads = cache->num_kv_heads;
    a.num_blocks = cache->num_blocks;
    a.max_blocks = max_blocks_per_seq;
    a.partition_tokens = resolve_partition(num_seqs, cache->num_kv_heads, max_blocks_per_seq,
                                           cache->block_size, partition_tokens);
    a.num_partitions = w.partitions;
    a.qscale = (float)((double)scale * 1.4426950408889634074);   // scale * log2(e)
    cudaStream_t s = (cudaStream_t)stream;
    if (cache->head_dim == 64) return dispatch_group<64>(G, cache->block_size, a, num_seqs, s);
    return dispatch_group<128>(G, cache->block_size, a, num_seqs, s);
}

int pkv_get_device_status(unsigned int* status_out, int reset) {
    if (!status_out) return PKV_ERR_NULL;
    if (cudaDeviceSynchronize() != cudaSuccess) return PKV_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, pkv::g_status, sizeof(v)) != cudaSuccess) return PKV_ERR_CUDA;
    *status_out = v;
    if (reset) {
        const unsigned int z = 0;
        if (cudaMemcpyToSymbol(pkv::g_status, &z, sizeof(z)) != cudaSuccess) return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

}  // extern "C"
