// Host side of the C ABI declared in include/pagedkv.h: argument checks,
// launch shapes and template dispatch.  Every entry point launches on the
// caller's stream and never synchronises (except pkv_get_device_status).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "pagedkv.h"
#include "pkv_device.cuh"
#include "kv_append.cuh"
#include "block_copy.cuh"
#include "block_manager.cuh"
#include "prefix_hash.cuh"
#include "attn_paged.cuh"

namespace {

constexpr int kMaxDevices = 64;
// Attention CTA shape: warps per CTA and pipeline stages per warp (build-time
// tunables; the stage count is per head_dim / block size, see attn_stages).
#ifndef PKV_ATTN_WARPS
#define PKV_ATTN_WARPS 4
#endif
#ifndef PKV_ATTN_STAGE_BUDGET
#define PKV_ATTN_STAGE_BUDGET 8192    // bytes of K+V tiles per warp ring
#endif
constexpr int kAttnWarps = PKV_ATTN_WARPS;
constexpr int kMaxCtasPerSm = 16;

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
bool supported_block_size(int b) { return b == 4 || b == 8 || b == 16 || b == 32; }

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

// tokens per pipeline stage of the attention kernel (TileSmem::TILE)
int tile_tokens(int head_dim, int block_size) {
    return block_size >= 32 ? block_size : ((head_dim == 64 && block_size >= 8) ? 32 : 16);
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream finishes; every kernel here waits
// (griddepcontrol.wait) before it reads or writes data.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
               Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) {
        cudaGetLastError();
        return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

// Longest work range, in tokens, rounded up to the tile; 0 = no cap (ranges
// are as long as an even split of the whole batch over the grid's warps).
int resolve_partition(int head_dim, int block_size, int requested) {
    if (!supported_block_size(block_size) || !supported_head_dim(head_dim) || requested < 0) return -1;
    if (requested == 0) return 0;
    const long long tile = tile_tokens(head_dim, block_size);
    const long long pt = ((long long)requested + tile - 1) / tile * tile;
    return pt > (1LL << 30) ? -1 : (int)pt;
}

template <int D, int BS>
constexpr int attn_stages() {
    return PKV_ATTN_STAGE_BUDGET / (2 * pkv::TileSmem<D, BS>::KT_BYTES) < 2
               ? 2
               : PKV_ATTN_STAGE_BUDGET / (2 * pkv::TileSmem<D, BS>::KT_BYTES);
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WorkspaceLayout {
    size_t prefix_off, mz_off, o_off, tickets_off, gtickets_off, total;
    int R_max;
    int cap_tiles;
};

// Regions of a workspace holding r_max ranges.
bool fill_layout(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, long long r_max,
                 int cap_tiles, WorkspaceLayout* w) {
    if (r_max > (1LL << 30)) return false;
    const size_t G = (size_t)(num_q_heads / num_kv_heads);
    const size_t N = (size_t)num_seqs;
    w->R_max = (int)r_max;
    w->cap_tiles = cap_tiles;
    w->prefix_off = 0;
    w->mz_off = N > (size_t)pkv::PREFIX_SMEM ? align_up((N + 1) * sizeof(long long), 256) : 0;
    w->o_off = w->mz_off + align_up((size_t)r_max * 2 * G * sizeof(float2), 256);
    w->tickets_off = w->o_off + align_up((size_t)r_max * 2 * G * head_dim * sizeof(float), 256);
    w->gtickets_off = w->tickets_off + align_up(N * num_kv_heads * sizeof(unsigned int), 256);
    w->total = w->gtickets_off + align_up((size_t)r_max * 2 * sizeof(unsigned int), 256);
    return true;
}

// Upper bound on the ranges of one launch over a grid of K warps (see the
// planning in the attention kernel): K ranges, or at most ceil(T / cap) + K
// under a cap of cap_tiles, for T <= max_tiles_total.
long long ranges_bound(long long K, long long max_tiles_total, int cap_tiles) {
    long long r = K;
    if (cap_tiles > 0) r += (max_tiles_total + cap_tiles - 1) / cap_tiles + 1;
    return r;
}

int grid_warps_for(int D, int G, int BS);

// The tile prefix of large batches, two partials per range (one range per
// warp of the grid this instance runs on this device; a cap adds one range
// per cap-length piece of the longest possible batch), one ticket per
// (sequence, kv head).
bool workspace_layout(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                      int max_blocks, int block_size, int partition_tokens, WorkspaceLayout* w) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads ||
        !supported_head_dim(head_dim) || max_blocks <= 0 || !supported_block_size(block_size))
        return false;
    const int pt = resolve_partition(head_dim, block_size, partition_tokens);
    if (pt < 0) return false;
    const int tile = tile_tokens(head_dim, block_size);
    const long long max_tiles = ((long long)max_blocks * block_size + tile - 1) / tile;
    const long long K = grid_warps_for(head_dim, num_q_heads / num_kv_heads, block_size);
    const int cap_tiles = pt / tile;
    const long long r_max = ranges_bound(K, (long long)num_seqs * num_kv_heads * max_tiles, cap_tiles);
    return fill_layout(num_seqs, num_q_heads, num_kv_heads, head_dim, r_max, cap_tiles, w);
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (no link-time dependency on libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D view of a whole pool (all layers): rows of head_dim bf16, one TMA box =
// one (block, kv head) tile's block_size rows x 64 dims, 128-byte swizzle.
bool encode_pool_map(CUtensorMap* map, void* pool, const pkv_cache_t* c) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const unsigned long long rows =
        (unsigned long long)c->num_layers * c->num_blocks * c->num_kv_heads * c->block_size;
    if (rows > (1ull << 31)) return false;   // row coordinates are 32-bit signed
    const cuuint64_t dims[2] = {(cuuint64_t)c->head_dim, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)c->head_dim * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)c->block_size};
    const cuuint32_t estr[2] = {1u, 1u};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pool, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// One template instance of the attention kernel: configuration, occupancy and launch.
template <int D, int G, int BS>
struct Attn {
    static constexpr int STAGES = attn_stages<D, BS>();
    using C = pkv::AttnCfg<D, G, BS, kAttnWarps, STAGES>;

    static int ctas_per_sm() {
        static int cached[kMaxDevices] = {0};
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
        if (cached[dev] == 0) {
            auto kern = pkv::paged_attention_kernel<D, G, BS, kAttnWarps, STAGES>;
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
                cudaSuccess)
                return -1;
            int n = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kAttnWarps * 32, C::SMEM_BYTES) !=
                    cudaSuccess || n <= 0)
                return -1;
            cached[dev] = n < kMaxCtasPerSm ? n : kMaxCtasPerSm;
        }
        return cached[dev];
    }

    static int launch(const CUtensorMap& mk, const CUtensorMap& mv, const pkv::AttnArgs& a, int grid,
                      cudaStream_t s) {
        return launch_pdl(pkv::paged_attention_kernel<D, G, BS, kAttnWarps, STAGES>, dim3(grid),
                          dim3(kAttnWarps * 32), C::SMEM_BYTES, s, mk, mv, a);
    }
};

// Dispatch on (head_dim, group, block size); op(Attn<...>{}) for the instance.
template <typename Op>
int with_instance(int D, int G, int BS, Op&& op) {
#define PKV_BS(DD, GG)                                             \
    switch (BS) {                                                  \
        case 4: return op(Attn<DD, GG, 4>{});                      \
        case 8: return op(Attn<DD, GG, 8>{});                      \
        case 16: return op(Attn<DD, GG, 16>{});                    \
        case 32: return op(Attn<DD, GG, 32>{});                    \
    }                                                              \
    return PKV_ERR_UNSUPPORTED;
#define PKV_G(DD)                                                  \
    switch (G) {                                                   \
        case 1: { PKV_BS(DD, 1) }                                  \
        case 2: { PKV_BS(DD, 2) }                                  \
        case 4: { PKV_BS(DD, 4) }                                  \
        case 8: { PKV_BS(DD, 8) }                                  \
    }                                                              \
    return PKV_ERR_UNSUPPORTED;
    if (D == 64) { PKV_G(64) }
    if (D == 128) { PKV_G(128) }
    return PKV_ERR_UNSUPPORTED;
#undef PKV_G
#undef PKV_BS
}

// Warps of the attention grid for this instance on the current device.
int grid_warps_for(int D, int G, int BS) {
    const int n = with_instance(D, G, BS, [](auto inst) { return decltype(inst)::ctas_per_sm(); });
    const int per_sm = n > 0 ? n : kMaxCtasPerSm;
    return device_sm_count() * per_sm * kAttnWarps;
}

// ---- attention without allocation ------------------------------------------
//
// Scratch for pkv_paged_decode_attention_noalloc: one fixed array per device
// that loads this library, kept for the life of the process.  Host code must
// not pass the array's name to a kernel (on the host it is only a stand-in
// symbol); the device address comes from cudaGetSymbolAddress, taken once per
// device on that device's first call.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

// Layout of the scratch for one call: the same regions as a caller-provided
// workspace, sized for the grid this call launches rather than the largest
// grid the device could run.
bool noalloc_layout(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int max_blocks,
                    int block_size, int partition_tokens, int grid_warps, WorkspaceLayout* w) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads ||
        !supported_head_dim(head_dim) || max_blocks <= 0 || !supported_block_size(block_size) ||
        grid_warps <= 0)
        return false;
    const int pt = resolve_partition(head_dim, block_size, partition_tokens);
    if (pt < 0) return false;
    const int tile = tile_tokens(head_dim, block_size);
    const long long max_tiles = ((long long)max_blocks * block_size + tile - 1) / tile;
    const long long tiles = (long long)num_seqs * num_kv_heads * max_tiles;
    const int cap_tiles = pt / tile;
    return fill_layout(num_seqs, num_q_heads, num_kv_heads, head_dim,
                       ranges_bound(grid_warps, tiles, cap_tiles), cap_tiles, w);
}

// Device address of the scratch on the current device (set up on first use).
unsigned char* noalloc_scratch_ptr() {
    static unsigned char* ptrs[kMaxDevices] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (!ptrs[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
        ptrs[dev] = static_cast<unsigned char*>(p);
    }
    return ptrs[dev];
}

// Shared body of the attention entry points that take a workspace; k_new and
// v_new non-null = fused append of each sequence's newest token.
int attention_with_workspace(const pkv_cache_t* cache, int layer, const void* k_new,
                                    const void* v_new, const int32_t* cow_src, const void* q,
                                    int num_seqs, int num_q_heads,
                                    const int32_t* block_tables, int max_blocks_per_seq,
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
    if ((long long)max_blocks_per_seq * cache->block_size > (1LL << 30)) return PKV_ERR_SHAPE;
    if (!q || !block_tables || !seq_lens || !out) return PKV_ERR_NULL;
    if (!aligned16(q) || !aligned16(out)) return PKV_ERR_ALIGN;
    if ((k_new == nullptr) != (v_new == nullptr)) return PKV_ERR_NULL;
    if (k_new && (!aligned16(k_new) || !aligned16(v_new))) return PKV_ERR_ALIGN;
    const int D = cache->head_dim, BS = cache->block_size;
    const int grid_warps = grid_warps_for(D, G, BS);
    WorkspaceLayout w;
    if (!workspace_layout(num_seqs, num_q_heads, cache->num_kv_heads, D, max_blocks_per_seq, BS,
                          partition_tokens, &w))
        return PKV_ERR_SHAPE;
    if (!workspace || workspace_bytes < w.total || !aligned16(workspace)) return PKV_ERR_WORKSPACE;
    if (grid_warps > w.R_max) return PKV_ERR_WORKSPACE;

    CUtensorMap mk, mv;
    if (!encode_pool_map(&mk, cache->k_pool, cache) || !encode_pool_map(&mv, cache->v_pool, cache))
        return PKV_ERR_CUDA;
    pkv::AttnArgs a;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    a.q = static_cast<const uint16_t*>(q);
    a.out = static_cast<uint16_t*>(out);
    a.block_tables = block_tables;
    a.seq_lens = seq_lens;
    a.num_seqs = num_seqs;
    a.num_kv_heads = cache->num_kv_heads;
    a.num_blocks = cache->num_blocks;
    a.max_blocks = max_blocks_per_seq;
    a.qscale = (float)((double)scale * 1.4426950408889634074);   // scale * log2(e)
    a.row_base = (long long)layer * cache->num_blocks * cache->num_kv_heads * cache->block_size;
    a.part_mz = reinterpret_cast<float2*>(ws + w.mz_off);
    a.part_o = reinterpret_cast<float*>(ws + w.o_off);
    a.tickets = reinterpret_cast<unsigned int*>(ws + w.tickets_off);
    a.group_tickets = reinterpret_cast<unsigned int*>(ws + w.gtickets_off);
    a.prefix_g = reinterpret_cast<long long*>(ws + w.prefix_off);
    a.R_max = w.R_max;
    a.k_new = static_cast<const uint4*>(k_new);
    a.v_new = static_cast<const uint4*>(v_new);
    a.cow_src = k_new ? cow_src : nullptr;
    a.k_pool = static_cast<uint16_t*>(cache->k_pool);
    a.v_pool = static_cast<uint16_t*>(cache->v_pool);
    a.cap_tiles = w.cap_tiles;
    a.K = grid_warps;
    cudaStream_t s = (cudaStream_t)stream;
    return with_instance(D, G, BS, [&](auto inst) {
        return decltype(inst)::launch(mk, mv, a, grid_warps / kAttnWarps, s);
    });
}

// Copy whole blocks from pool `src` to pool `dst` (the same cache for a
// copy-on-write copy); d_num_pairs non-null: the count is read on the device
// and num_pairs is its upper bound.
int block_copy_launch(const pkv_cache_t* dst, const pkv_cache_t* src, const void* dst_k,
                      const void* dst_v, const void* src_k, const void* src_v,
                      const int32_t* src_dst_pairs, int num_pairs, const int32_t* d_num_pairs,
                      void* stream) {
    if (num_pairs < 0) return PKV_ERR_SHAPE;
    if (num_pairs == 0) return PKV_OK;
    if (!src_dst_pairs) return PKV_ERR_NULL;
    const long long chunks = (long long)dst->num_kv_heads * dst->block_size * dst->head_dim / 8;
    const long long total = (long long)num_pairs * dst->num_layers * 2 * chunks;
    const long long want = (total + 256 * 4 - 1) / (256 * 4);   // four chunks per thread
    const long long cap = (long long)device_sm_count() * 8;
    const unsigned grid = (unsigned)(want < cap ? want : cap);
    return launch_pdl(pkv::block_copy_kernel, dim3(grid), dim3(256), 0, (cudaStream_t)stream,
                      (uint4*)dst_k, (uint4*)dst_v, (const uint4*)src_k, (const uint4*)src_v,
                      src_dst_pairs, num_pairs, dst->num_layers, src->num_blocks, dst->num_blocks,
                      chunks, d_num_pairs);
}

// Device address of a host pool pointer: pinned (page-locked, mapped) host
// memory only; null for pageable or device memory.
const void* host_pool_device_ptr(const void* p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (at.type != cudaMemoryTypeHost || !at.devicePointer) return nullptr;
    return at.devicePointer;
}

}  // namespace

#ifndef PKV_BUILD_HASH
#define PKV_BUILD_HASH "0000000000000000"
#endif
// The build's source hash, after a tag the loader finds in the file itself.
__attribute__((used)) static const char kBuildTag[] = "PKV_BUILD_HASH:" PKV_BUILD_HASH;

extern "C" {

int pkv_abi_version(void) { return PKV_ABI_VERSION; }

const char* pkv_build_hash(void) { return kBuildTag + sizeof("PKV_BUILD_HASH:") - 1; }

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
        case PKV_ERR_MEMORY: return "a host pool is not pinned, mapped host memory";
        case PKV_ERR_SCRATCH:
            return "request needs more scratch than the no-allocation buffer holds "
                   "(PKV_NOALLOC_SCRATCH_BYTES); use pkv_paged_decode_attention with a workspace";
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
    return launch_pdl(pkv::kv_append_kernel, dim3((unsigned)blocks), dim3(threads), 0,
                      (cudaStream_t)stream, reinterpret_cast<const uint4*>(k_new),
                      reinterpret_cast<const uint4*>(v_new),
                      reinterpret_cast<uint4*>(static_cast<uint16_t*>(cache->k_pool) + base),
                      reinterpret_cast<uint4*>(static_cast<uint16_t*>(cache->v_pool) + base),
                      slot_mapping, num_tokens, cache->num_kv_heads, cache->block_size,
                      cache->head_dim, cache->num_blocks);
}

int pkv_block_copy(const pkv_cache_t* cache, const int32_t* src_dst_pairs, int num_pairs,
                   void* stream) {
    const int rc = check_cache(cache);
    if (rc) return rc;
    return block_copy_launch(cache, cache, cache->k_pool, cache->v_pool, cache->k_pool,
                             cache->v_pool, src_dst_pairs, num_pairs, nullptr, stream);
}

int pkv_block_copy_device_count(const pkv_cache_t* cache, const int32_t* src_dst_pairs,
                                int max_pairs, const int32_t* num_pairs, void* stream) {
    const int rc = check_cache(cache);
    if (rc) return rc;
    if (!num_pairs && max_pairs > 0) return PKV_ERR_NULL;
    return block_copy_launch(cache, cache, cache->k_pool, cache->v_pool, cache->k_pool,
                             cache->v_pool, src_dst_pairs, max_pairs, num_pairs, stream);
}

int pkv_swap_blocks(const pkv_cache_t* device_cache, const pkv_cache_t* host_cache,
                    const int32_t* src_dst_pairs, int num_pairs, int direction, void* stream) {
    int rc = check_cache(device_cache);
    if (rc) return rc;
    rc = check_cache(host_cache);
    if (rc) return rc;
    if (direction != PKV_SWAP_OUT && direction != PKV_SWAP_IN) return PKV_ERR_SHAPE;
    if (host_cache->num_layers != device_cache->num_layers ||
        host_cache->num_kv_heads != device_cache->num_kv_heads ||
        host_cache->block_size != device_cache->block_size ||
        host_cache->head_dim != device_cache->head_dim)
        return PKV_ERR_SHAPE;
    if (num_pairs < 0) return PKV_ERR_SHAPE;
    if (num_pairs == 0) return PKV_OK;
    if (!src_dst_pairs) return PKV_ERR_NULL;
    const void* hk = host_pool_device_ptr(host_cache->k_pool);
    const void* hv = host_pool_device_ptr(host_cache->v_pool);
    if (!hk || !hv) return PKV_ERR_MEMORY;
    if (direction == PKV_SWAP_OUT)
        return block_copy_launch(host_cache, device_cache, hk, hv, device_cache->k_pool,
                                 device_cache->v_pool, src_dst_pairs, num_pairs, nullptr, stream);
    return block_copy_launch(device_cache, host_cache, device_cache->k_pool, device_cache->v_pool,
                             hk, hv, src_dst_pairs, num_pairs, nullptr, stream);
}

int pkv_prefix_block_hashes(const int32_t* tokens, int max_tokens, const int32_t* seq_lens,
                            const uint64_t* extra_keys, const int32_t* first_block,
                            const uint64_t* parent_hashes, int num_seqs, int block_size,
                            uint64_t* hashes, int max_blocks, void* stream) {
    if (num_seqs < 0 || max_tokens < 0 || max_blocks < 0 || block_size <= 0) return PKV_ERR_SHAPE;
    // resuming needs the stored hash of the block before: without it the
    // chain would restart from 0 and match another sequence's first blocks
    if (first_block && !parent_hashes) return PKV_ERR_NULL;
    if (num_seqs == 0 || max_blocks == 0) return PKV_OK;
    if (!tokens || !seq_lens || !hashes) return PKV_ERR_NULL;
    const int per_cta = 8;                                  // warps (sequences) per CTA
    long long grid = ((long long)num_seqs + per_cta - 1) / per_cta;
    const long long cap = (long long)device_sm_count() * 8;
    if (grid > cap) grid = cap;
    return launch_pdl(pkv::prefix_hash_kernel, dim3((unsigned)grid), dim3(per_cta * 32), 0,
                      (cudaStream_t)stream, tokens, (long long)max_tokens, seq_lens, extra_keys,
                      first_block, parent_hashes, num_seqs, block_size, hashes, max_blocks);
}

int pkv_block_manager_step(const pkv_block_state_t* st, int num_seqs, int max_blocks_per_seq,
                           int num_blocks, int block_size, const int32_t* order,
                           int64_t* slot_mapping, int32_t* copy_pairs, int32_t* num_pairs,
                           int32_t* cow_src, void* stream) {
    if (!st) return PKV_ERR_NULL;
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 || block_size <= 0)
        return PKV_ERR_SHAPE;
    if (num_seqs > pkv::BM_MAX_SEQS) return PKV_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PKV_OK;
    if (!st->block_tables || !st->seq_lens || !st->refcount || !st->free_ring || !st->free_state ||
        !slot_mapping || !copy_pairs || !num_pairs)
        return PKV_ERR_NULL;
    pkv::BmArgs a;
    a.block_tables = st->block_tables;
    a.seq_lens = st->seq_lens;
    a.refcount = st->refcount;
    a.free_ring = st->free_ring;
    a.free_state = st->free_state;
    a.order = order;
    a.slot_mapping = slot_mapping;
    a.copy_pairs = copy_pairs;
    a.num_pairs = num_pairs;
    a.cow_src = cow_src;
    a.num_seqs = num_seqs;
    a.max_blocks = max_blocks_per_seq;
    a.num_blocks = num_blocks;
    a.block_size = block_size;
    return launch_pdl(pkv::block_manager_kernel, dim3(1), dim3(pkv::BM_THREADS), 0,
                      (cudaStream_t)stream, a);
}

int pkv_block_manager_release(const pkv_block_state_t* st, int num_seqs, int max_blocks_per_seq,
                              int num_blocks, int block_size, const int32_t* seqs, int num_release,
                              void* stream) {
    if (!st) return PKV_ERR_NULL;
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 || block_size <= 0 ||
        num_release < 0 || num_release > num_seqs)
        return PKV_ERR_SHAPE;
    if (num_seqs > pkv::BM_MAX_SEQS) return PKV_ERR_UNSUPPORTED;
    if (num_release == 0) return PKV_OK;
    if (!st->block_tables || !st->seq_lens || !st->refcount || !st->free_ring || !st->free_state ||
        !seqs)
        return PKV_ERR_NULL;
    static bool configured[kMaxDevices] = {false};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(pkv::block_release_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(pkv::BrShared)) != cudaSuccess)
            return PKV_ERR_CUDA;
        configured[dev] = true;
    }
    pkv::BrArgs a;
    a.block_tables = st->block_tables;
    a.seq_lens = st->seq_lens;
    a.refcount = st->refcount;
    a.free_ring = st->free_ring;
    a.free_state = st->free_state;
    a.seqs = seqs;
    a.num_seqs = num_seqs;
    a.num_release = num_release;
    a.max_blocks = max_blocks_per_seq;
    a.num_blocks = num_blocks;
    a.block_size = block_size;
    return launch_pdl(pkv::block_release_kernel, dim3(1), dim3(pkv::BM_THREADS), sizeof(pkv::BrShared),
                      (cudaStream_t)stream, a);
}

int pkv_partition_tokens(int num_seqs, int num_kv_heads, int head_dim, int max_blocks_per_seq,
                         int block_size, int requested) {
    if (!supported_head_dim(head_dim) || num_seqs < 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0)
        return -1;
    return resolve_partition(head_dim, block_size, requested);
}

size_t pkv_attention_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                     int max_blocks_per_seq, int block_size, int partition_tokens) {
    if (num_kv_heads <= 0 || num_q_heads <= 0 || num_q_heads % num_kv_heads) return 0;
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
    return attention_with_workspace(cache, layer, nullptr, nullptr, nullptr, q, num_seqs, num_q_heads,
                                    block_tables, max_blocks_per_seq, seq_lens, scale, out, workspace,
                                    workspace_bytes, partition_tokens, stream);
}

int pkv_append_paged_decode_attention(const pkv_cache_t* cache, int layer, const void* k_new,
                                      const void* v_new, const int32_t* cow_src, const void* q,
                                      int num_seqs,
                                      int num_q_heads, const int32_t* block_tables,
                                      int max_blocks_per_seq, const int32_t* seq_lens, float scale,
                                      void* out, void* workspace, size_t workspace_bytes,
                                      int partition_tokens, void* stream) {
    if (!k_new || !v_new) return PKV_ERR_NULL;
    return attention_with_workspace(cache, layer, k_new, v_new, cow_src, q, num_seqs, num_q_heads,
                                    block_tables, max_blocks_per_seq, seq_lens, scale, out, workspace,
                                    workspace_bytes, partition_tokens, stream);
}

int pkv_paged_decode_attention_noalloc(const pkv_cache_t* cache, int layer, const void* q,
                                       int num_seqs, int num_q_heads, const int32_t* block_tables,
                                       int max_blocks_per_seq, const int32_t* seq_lens, float scale,
                                       void* out, int partition_tokens, void* stream) {
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
    if ((long long)max_blocks_per_seq * cache->block_size > (1LL << 30)) return PKV_ERR_SHAPE;
    if (!q || !block_tables || !seq_lens || !out) return PKV_ERR_NULL;
    if (!aligned16(q) || !aligned16(out)) return PKV_ERR_ALIGN;
    const int D = cache->head_dim, BS = cache->block_size;
    const int grid_warps = grid_warps_for(D, G, BS);
    WorkspaceLayout w;
    if (!noalloc_layout(num_seqs, num_q_heads, cache->num_kv_heads, D, max_blocks_per_seq, BS,
                        partition_tokens, grid_warps, &w))
        return PKV_ERR_SHAPE;
    if (w.total > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_ERR_SCRATCH;
    unsigned char* ws = noalloc_scratch_ptr();
    if (!ws) return PKV_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    // the tickets must start at zero; the scratch keeps whatever the last call left
    if (cudaMemsetAsync(ws + w.tickets_off, 0, w.total - w.tickets_off, s) != cudaSuccess)
        return PKV_ERR_CUDA;

    CUtensorMap mk, mv;
    if (!encode_pool_map(&mk, cache->k_pool, cache) || !encode_pool_map(&mv, cache->v_pool, cache))
        return PKV_ERR_CUDA;
    pkv::AttnArgs a;
    a.q = static_cast<const uint16_t*>(q);
    a.out = static_cast<uint16_t*>(out);
    a.block_tables = block_tables;
    a.seq_lens = seq_lens;
    a.num_seqs = num_seqs;
    a.num_kv_heads = cache->num_kv_heads;
    a.num_blocks = cache->num_blocks;
    a.max_blocks = max_blocks_per_seq;
    a.qscale = (float)((double)scale * 1.4426950408889634074);   // scale * log2(e)
    a.row_base = (long long)layer * cache->num_blocks * cache->num_kv_heads * cache->block_size;
    a.part_mz = reinterpret_cast<float2*>(ws + w.mz_off);
    a.part_o = reinterpret_cast<float*>(ws + w.o_off);
    a.tickets = reinterpret_cast<unsigned int*>(ws + w.tickets_off);
    a.group_tickets = reinterpret_cast<unsigned int*>(ws + w.gtickets_off);
    a.prefix_g = reinterpret_cast<long long*>(ws + w.prefix_off);
    a.k_new = nullptr;                                // no fused append here
    a.v_new = nullptr;
    a.cow_src = nullptr;
    a.k_pool = static_cast<uint16_t*>(cache->k_pool);
    a.v_pool = static_cast<uint16_t*>(cache->v_pool);
    a.R_max = w.R_max;
    a.cap_tiles = w.cap_tiles;
    a.K = grid_warps;
    return with_instance(D, G, BS, [&](auto inst) {
        return decltype(inst)::launch(mk, mv, a, grid_warps / kAttnWarps, s);
    });
}

int pkv_set_wait_limit_ns(unsigned long long limit_ns) {
    const unsigned long long v = limit_ns ? limit_ns : pkv::WAIT_LIMIT_NS;
    if (cudaMemcpyToSymbol(pkv::g_wait_limit_ns, &v, sizeof(v)) != cudaSuccess) return PKV_ERR_CUDA;
    return PKV_OK;
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
