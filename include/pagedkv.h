/*
 * pagedkv.h -- C ABI of the paged KV-cache decode path (sm_100a).
 *
 * Three operations, each one asynchronous launch sequence on the caller's
 * CUDA stream:
 *
 *   pkv_block_copy              copy-on-write of shared tail blocks
 *   pkv_kv_append               store each new token's K and V in its slot
 *   pkv_paged_decode_attention  decode attention read through block tables
 *
 * Sources: "Infra: PagedAttention" (Fanyi Pu), sections "按 Block 分配" and
 * "共享前缀，分叉时 Copy-on-write"; ithelp.ithome.com.tw article 10405755,
 * sections "PagedAttention 的核心想法" and "手動畫一次 block table".
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every pointer argument except `cache` (host) and `status_out` (host) is
 *    a DEVICE pointer on the current device, owned by the caller.  The
 *    library never allocates, frees or keeps a pointer past the call.
 *  - bf16 buffers (pools, q, k_new, v_new, out) must be 16-byte aligned;
 *    the pools, q and out are dense row-major as documented per argument.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls return before the GPU work finishes; nothing inside a
 *    call synchronises the host.
 *  - Kernels are launched with programmatic stream serialization: each one
 *    may start while the kernel before it on the stream finishes, and waits
 *    for that kernel to complete before it reads or writes the pools, q,
 *    k_new, v_new, the tables, the workspace or out.  The one exception:
 *    the attention kernels read seq_lens and block_tables before that wait
 *    (to plan their work), so those two must be written by copies or by
 *    kernels that do not release their dependents early
 *    (cudaTriggerProgrammaticLaunchCompletion): such a writer could still
 *    be running when the attention kernel starts.  The one kernel of this
 *    library that writes them, pkv_block_manager_step, does not release
 *    early.
 *  - Return value: PKV_OK, or a negative PKV_ERR_* code when an argument
 *    check fails on the host (nothing is launched) or a launch fails.
 *  - Faults found by the kernels themselves (a block id or slot outside the
 *    pool, a sequence longer than its table, a bounded wait that gave up)
 *    never trap: the kernel skips the access and ORs a PKV_DEV_* bit into a
 *    per-device status word read by pkv_get_device_status().  Outputs of a
 *    launch that raised a device bit are undefined.
 *
 * KV cache layout (the pages fix none; this is the library's contract)
 * ------------------------------------------------------------------
 *   k_pool, v_pool : bf16 [num_layers][num_blocks][num_kv_heads][block_size][head_dim]
 * The tile of one (physical block, kv head) is contiguous
 * (block_size * head_dim * 2 bytes).  Slot s (flat numbering) is token row
 * s % block_size of physical block s / block_size, as in the page's example:
 * with table [3, 0, 4] and B = 4, position 8 is logical block 2 -> P4, row 0.
 *
 * Supported shapes: head_dim in {64, 128}; block_size in {4, 8, 16, 32};
 * num_q_heads = G * num_kv_heads with G in {1, 2, 4, 8}.  Query head h
 * reads kv head h / G (contiguous GQA groups).
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PKV_ABI_VERSION 1

/* host-side status codes */
#define PKV_OK                0
#define PKV_ERR_NULL         -1  /* a required pointer is NULL */
#define PKV_ERR_SHAPE        -2  /* a size is negative or inconsistent */
#define PKV_ERR_ALIGN        -3  /* a bf16 buffer is not 16-byte aligned */
#define PKV_ERR_WORKSPACE    -4  /* workspace missing or too small */
#define PKV_ERR_UNSUPPORTED  -5  /* head_dim / block_size / group size not built */
#define PKV_ERR_CUDA         -6  /* a CUDA runtime call or launch failed */
#define PKV_ERR_LAYER        -7  /* layer index outside [0, num_layers) */
#define PKV_ERR_SCRATCH      -8  /* request too large for the no-allocation scratch */
#define PKV_ERR_MEMORY       -9  /* a host pool is not pinned (page-locked, mapped) memory */

/* size of the device buffer behind pkv_paged_decode_attention_noalloc */
#define PKV_NOALLOC_SCRATCH_BYTES (16u << 20)

/* cow_src value: this sequence appends nothing in this step (written by an
 * aborted pkv_block_manager_step; see pkv_append_paged_decode_attention) */
#define PKV_COW_NO_APPEND (-2)

/* device-side status bits (pkv_get_device_status) */
#define PKV_DEV_RANGE    0x1u  /* block id or slot outside the pool: access skipped */
#define PKV_DEV_LENGTH   0x2u  /* seq_len above max_blocks_per_seq * block_size: clamped */
#define PKV_DEV_TIMEOUT  0x4u  /* a bounded wait for staged KV gave up */
#define PKV_DEV_NOBLOCKS 0x8u  /* block manager step: not enough free blocks, nothing changed */

typedef struct pkv_cache {
    void*   k_pool;        /* bf16 [num_layers][num_blocks][num_kv_heads][block_size][head_dim] */
    void*   v_pool;        /* same shape as k_pool */
    int32_t num_layers;
    int32_t num_blocks;
    int32_t num_kv_heads;
    int32_t block_size;
    int32_t head_dim;
} pkv_cache_t;

/*
 * pkv_kv_append -- write the K and V of `num_tokens` new tokens into their slots.
 *
 * Defines: a new token fills the next free slot of its sequence's tail block
 * (the caller's block manager picks the slot: a fresh block only once the
 * tail is full) -- ithelp article 10405755, "手動畫一次 block table";
 * "Infra: PagedAttention", "按 Block 分配".
 *
 *   layer         layer of the pools to write, 0 <= layer < num_layers
 *   k_new, v_new  bf16 [num_tokens][num_kv_heads][head_dim]
 *   slot_mapping  int64 [num_tokens]; slot < 0 means padding (skipped);
 *                 slot >= num_blocks*block_size sets PKV_DEV_RANGE (skipped)
 *   num_tokens    >= 0; 0 launches nothing
 * The bf16 bit patterns are moved unchanged (NaN payloads and -0 survive).
 * Precondition: no slot appears twice (the later write would race).
 */
int pkv_kv_append(const pkv_cache_t* cache, int layer,
                  const void* k_new, const void* v_new,
                  const int64_t* slot_mapping, int num_tokens, void* stream);

/*
 * pkv_block_copy -- copy whole physical blocks, every layer, K and V.
 *
 * Defines: copy-on-write of a shared, partially filled tail block: before a
 * writer appends to a block whose reference count is above one, the block is
 * copied and the writer remapped to the copy; full prefix blocks stay shared
 * -- "Infra: PagedAttention", "共享前缀，分叉时 Copy-on-write" and its figure
 * (A copies P0 -> P4, B keeps P0, P3 stays shared).
 *
 *   src_dst_pairs  int32 [num_pairs][2] = (src block, dst block)
 *   num_pairs      >= 0; 0 launches nothing
 * For every pair and every layer l: pool[l][dst] = pool[l][src] (all heads,
 * all rows, K and V), bit exact.  A block id outside [0, num_blocks) sets
 * PKV_DEV_RANGE and that pair is skipped.  Precondition: dst ids are
 * distinct and none is also a src (otherwise the copies race).
 */
int pkv_block_copy(const pkv_cache_t* cache, const int32_t* src_dst_pairs,
                   int num_pairs, void* stream);

/*
 * pkv_block_copy_device_count -- pkv_block_copy with the pair count read on
 * the device: copies the first *num_pairs (at most max_pairs) pairs.  For a
 * step whose copy pairs come from pkv_block_manager_step, so the host never
 * waits for the count.
 *
 *   num_pairs   device int32 [1]
 *   max_pairs   >= 0, capacity of src_dst_pairs; 0 launches nothing
 */
int pkv_block_copy_device_count(const pkv_cache_t* cache, const int32_t* src_dst_pairs,
                                int max_pairs, const int32_t* num_pairs, void* stream);

/*
 * pkv_swap_blocks -- move whole blocks between the device pool and a pool in
 * pinned host memory, every layer, K and V, in one launch.
 *
 * Defines: under memory pressure, blocks can be swapped out to CPU memory and
 * brought back later ("只用了 8 格，為什麼占了 12 格？", 故事沒有說完的部分).
 *
 *   device_cache   the device pool (as for the other calls)
 *   host_cache     a pool of the same layers, kv heads, block size and
 *                  head_dim in page-locked host memory that the device can
 *                  address (cudaHostAlloc, or cudaHostRegister with the
 *                  mapped flag; torch's pin_memory qualifies); its own
 *                  num_blocks.  Pageable memory gives PKV_ERR_MEMORY.
 *   src_dst_pairs  device int32 [num_pairs][2]
 *   direction      PKV_SWAP_OUT: host[l][dst] = device[l][src];
 *                  PKV_SWAP_IN:  device[l][dst] = host[l][src]
 * Bit exact.  A block id outside its pool sets PKV_DEV_RANGE and that pair is
 * skipped.  The copy runs over PCIe inside the kernel (no per-block memcpy).
 */
#define PKV_SWAP_OUT 0
#define PKV_SWAP_IN  1
int pkv_swap_blocks(const pkv_cache_t* device_cache, const pkv_cache_t* host_cache,
                    const int32_t* src_dst_pairs, int num_pairs, int direction, void* stream);

/*
 * pkv_prefix_block_hashes -- hash every full block of every sequence, for
 * finding cached prefix blocks again (automatic prefix caching).
 *
 * Defines ("Infra: PagedAttention", "共享前缀，分叉时 Copy-on-write", the
 * paragraphs on Automatic Prefix Caching): only full blocks are cached; a
 * block is reusable only when the whole prefix before it matches, so its
 * hash covers the previous block's hash, the block's tokens and context
 * identifiers such as a LoRA id.  The pages name no hash function; this one
 * is FNV-1a 64 (h = 0xcbf29ce484222325, per byte h = (h ^ byte) *
 * 0x100000001b3 mod 2^64):
 *   digest c_b = FNV-1a(tokens of block b as int32 LE, extra key as uint64 LE)
 *   hash   h_b = FNV-1a(h_{b-1} as uint64 LE, c_b as uint64 LE),  h_{-1} = 0
 *
 *   tokens       device int32 [num_seqs][max_tokens], token ids by position
 *   seq_lens     device int32 [num_seqs]; blocks 0 .. seq_lens/B - 1 are hashed
 *   extra_keys   device uint64 [num_seqs], or NULL for 0
 *   first_block  device int32 [num_seqs], or NULL for 0: hash only blocks
 *                first_block[s] .. seq_lens/B - 1 (resuming, e.g. in decode
 *                only the block that just became full)
 *   parent_hashes device uint64 [num_seqs]: hash of block first_block[s] - 1
 *                (unused where first_block[s] is 0).  Required whenever
 *                first_block is given (PKV_ERR_NULL otherwise: a chain
 *                restarted from 0 would give block k the hash of a first
 *                block with the same tokens, a false prefix match); may be
 *                NULL when first_block is NULL.
 *   hashes       device uint64 [num_seqs][max_blocks] out; entries outside
 *                [first_block, full blocks) are not written
 * A length above max_tokens, or more full blocks than max_blocks, sets
 * PKV_DEV_LENGTH and is clamped.
 */
int pkv_prefix_block_hashes(const int32_t* tokens, int max_tokens, const int32_t* seq_lens,
                            const uint64_t* extra_keys, const int32_t* first_block,
                            const uint64_t* parent_hashes, int num_seqs, int block_size,
                            uint64_t* hashes, int max_blocks, void* stream);

/*
 * Block manager state on the device, for pkv_block_manager_step.  All device
 * pointers, owned by the caller.
 */
typedef struct pkv_block_state {
    int32_t* block_tables;  /* [num_seqs][max_blocks_per_seq]; entries past a
                               sequence's blocks are ignored */
    int32_t* seq_lens;      /* [num_seqs] tokens cached per sequence */
    int32_t* refcount;      /* [num_blocks] users of each physical block */
    int32_t* free_ring;     /* [num_blocks] ring of free block ids */
    int32_t* free_state;    /* [2]: ring index of the next free id, number of free ids */
} pkv_block_state_t;

/*
 * pkv_block_manager_step -- one decode step of the block manager, on the
 * device: every sequence appends one token.
 *
 * Defines ("Infra: PagedAttention", "按 Block 分配" and "共享前缀，分叉时
 * Copy-on-write"; ithelp article 10405755, "手動畫一次 block table"): a new
 * token fills the tail block; a full tail (or no block) takes the next free
 * block; a tail with room whose reference count is above one is copied first
 * (take a free block, record the copy pair, remap, drop one reference on the
 * old tail).  Writers are served in `order`; each writer that still sees a
 * count above one copies, so the last of k sharers that all write keeps the
 * block.  Free blocks are handed out from the ring in order.
 *
 *   order          device int32 [num_seqs], a permutation of 0..num_seqs-1
 *                  (writer order), or NULL for 0..num_seqs-1
 *   slot_mapping   device int64 [num_seqs] out: slot of each sequence's new
 *                  token (block * block_size + offset)
 *   copy_pairs     device int32 [num_seqs][2] out, (src, dst) in writer order
 *   num_pairs      device int32 [1] out
 *   cow_src        device int32 [num_seqs] out, or NULL: per sequence the
 *                  source block of its copy (-1 if it does not copy), the
 *                  form pkv_append_paged_decode_attention takes
 * On return the tables, lengths (+1), counts and free state are updated.
 * num_seqs <= 4096 (PKV_ERR_UNSUPPORTED above).  If the free blocks do not
 * suffice, or an order entry, a length, a tail block id or a free-ring entry
 * is out of range, the kernel sets PKV_DEV_NOBLOCKS / PKV_DEV_RANGE /
 * PKV_DEV_LENGTH and changes no state (tables, lengths, counts, free state).
 * It still writes its outputs, so that work already queued behind it on the
 * stream does no harm before the host sees the status: every slot_mapping
 * entry -1 (pkv_kv_append skips it), *num_pairs = 0 (no copy), and, when
 * cow_src is given, cow_src[s] = PKV_COW_NO_APPEND for every sequence (the
 * fused pkv_append_paged_decode_attention then appends and copies nothing).
 * The kernel reads all of its state (order, lengths, tables, counts, free
 * ring and state) and makes every decision before its wait on the previous
 * kernel, and writes only after it; so that state, like the attention
 * calls' lengths and tables, must be written by copies or by kernels that
 * do not release their dependents early (in this library only this kernel
 * writes it).  It does not release its own dependents early, so an attention
 * launch that follows on the stream reads the new lengths.
 */
int pkv_block_manager_step(const pkv_block_state_t* state, int num_seqs,
                           int max_blocks_per_seq, int num_blocks, int block_size,
                           const int32_t* order, int64_t* slot_mapping,
                           int32_t* copy_pairs, int32_t* num_pairs, int32_t* cow_src,
                           void* stream);

/*
 * pkv_block_manager_release -- finished requests give their blocks back, on
 * the device.
 *
 * Defines ("Infra: PagedAttention", "按 Block 分配": a finished request drops
 * its references; ithelp article 10405755, "手動畫一次 block table": when the
 * request ends its blocks return to the pool): for each row of `seqs`, in the
 * given order, each block of the row's table, in table order, loses one
 * reference; a block whose count reaches zero is appended to the free ring
 * after the blocks already free, in that order of drops (head unchanged,
 * count grows).  The row's length becomes 0 and its table entries -1, so the
 * row can serve a new request: the next pkv_block_manager_step gives it a
 * fresh block for its first token.
 *
 *   state        as for pkv_block_manager_step, num_seqs rows
 *   seqs         device int32 [num_release]: the rows to release, distinct
 *   num_release  0..num_seqs
 * The state must be consistent (each count equal to the number of table
 * entries, over all rows, that name the block).  Errors: PKV_ERR_SHAPE,
 * PKV_ERR_NULL, PKV_ERR_UNSUPPORTED (num_seqs > 4096), PKV_ERR_CUDA.  On the
 * device, a row out of range or named twice, a length above the table, a
 * block id out of range, more drops on a block than its count, or more than
 * 8192 drops on shared blocks in one call set PKV_DEV_RANGE / PKV_DEV_LENGTH
 * and change nothing.  The kernel waits for the kernel before it on the
 * stream before reading anything and does not release its dependents early.
 */
int pkv_block_manager_release(const pkv_block_state_t* state, int num_seqs,
                              int max_blocks_per_seq, int num_blocks, int block_size,
                              const int32_t* seqs, int num_release, void* stream);

/*
 * pkv_attention_workspace_bytes -- bytes of workspace pkv_paged_decode_attention
 * needs for these sizes on the current device: the tile prefix per sequence
 * (batches over 768 sequences; smaller ones keep it in shared memory), the
 * partial results of sequences split across ranges, one ticket per (sequence,
 * kv head) and one per group of ranges.  `partition_tokens` as passed to the
 * attention call.  Returns 0 for invalid sizes.
 */
size_t pkv_attention_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads,
                                     int head_dim, int max_blocks_per_seq, int block_size,
                                     int partition_tokens);

/*
 * pkv_partition_tokens -- the longest work range (tokens) the attention call
 * uses: `requested` rounded up to the kernel's tile (32 tokens at head_dim 64,
 * 16 at head_dim 128 or with 4-token blocks, never less than one block), or 0
 * when `requested` is 0 (no cap).  Returns < 0 for invalid sizes.
 */
int pkv_partition_tokens(int num_seqs, int num_kv_heads, int head_dim,
                         int max_blocks_per_seq, int block_size, int requested);

/*
 * pkv_workspace_init -- zero a workspace before its first use (asynchronous
 * memset on `stream`).  The attention kernel leaves every counter back at
 * zero when it finishes, so a workspace is initialised once, not per call.
 */
int pkv_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * pkv_paged_decode_attention -- one decode step of attention for `num_seqs`
 * sequences, reading K and V through block tables.
 *
 * Defines: the attention formula is unchanged by paging; the kernel looks up
 * the block table and reads the physical blocks in place, without copying
 * them into one contiguous range (ithelp article 10405755, "PagedAttention
 * 的核心想法"; "Infra: PagedAttention", "按 Block 分配").  Score
 * s_i = scale * q . k_i, softmax over every visible token.  The work over all
 * (sequence, kv head) pairs is cut into equal ranges of tiles, one per warp
 * of the grid (more under a partition cap); a sequence that spans several
 * ranges is computed in pieces, each keeping (max score
 * m_r, Z_r = sum e^{s_i - m_r}, unnormalised output), and the pieces are
 * merged with o = sum_r e^{m_r - M} Z_r o_r / sum_r e^{m_r - M} Z_r,
 * M = max_r m_r ("Infra: PagedAttention", "按 Block 分配", the merge
 * equation and the paragraph on max rescaling).  One kernel launch.
 *
 *   layer              layer of the pools to read
 *   q                  bf16 [num_seqs][num_q_heads][head_dim]
 *   block_tables       int32 [num_seqs][max_blocks_per_seq]; entry j of
 *                      sequence s is the physical block of positions
 *                      [j*B, (j+1)*B); entries past ceil(len/B) are never read
 *   seq_lens           int32 [num_seqs], tokens to attend to (including a
 *                      token appended this step); 0 gives a zero output;
 *                      values above max_blocks_per_seq*B set PKV_DEV_LENGTH
 *                      and are clamped
 *   scale              score scale, usually 1/sqrt(head_dim)
 *   out                bf16 [num_seqs][num_q_heads][head_dim], round to
 *                      nearest even from fp32
 *   workspace          device buffer of at least
 *                      pkv_attention_workspace_bytes(...) bytes (same sizes,
 *                      same device), 16-byte aligned, zeroed once
 *                      (pkv_workspace_init) before its first use; the call
 *                      leaves it ready for the next call.  After a launch
 *                      that raised PKV_DEV_TIMEOUT, zero it again.
 *   partition_tokens   0 = no cap on the ranges; > 0 = no range longer than
 *                      this many tokens (rounded up to the tile)
 * Concurrent calls must not share a workspace.
 */
int pkv_paged_decode_attention(const pkv_cache_t* cache, int layer,
                               const void* q, int num_seqs, int num_q_heads,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* seq_lens, float scale, void* out,
                               void* workspace, size_t workspace_bytes,
                               int partition_tokens, void* stream);

/*
 * pkv_append_paged_decode_attention -- one decode step of one layer in one
 * launch: pkv_kv_append of every sequence's newest token followed by
 * pkv_paged_decode_attention, for the decode case where sequence s appends
 * exactly one token, at position seq_lens[s] - 1.  The pages ask for the
 * block-table lookup, the K/V read and the attention math to be organised
 * together ("Infra: PagedAttention", "按 Block 分配", the paragraph on what a
 * PagedAttention kernel has to do); this entry goes one step further and
 * folds the append into the same kernel.
 *
 *   k_new, v_new   bf16 [num_seqs][num_kv_heads][head_dim], 16-byte aligned:
 *                  the newest token of each sequence.  Its slot is the one
 *                  the table gives for position seq_lens[s] - 1, i.e. block
 *                  block_tables[s][(seq_lens[s]-1)/B], row (seq_lens[s]-1)%B;
 *                  sequences with seq_lens[s] == 0 append nothing.
 *   cow_src        device int32 [num_seqs], or NULL: the copy-on-write of
 *                  the step folded into this launch.  cow_src[s] >= 0 means
 *                  the sequence's tail block (the table's block for position
 *                  seq_lens[s] - 1) is a fresh copy of block cow_src[s]: this
 *                  launch reads the tail from cow_src[s] and writes the whole
 *                  block, this layer, every kv head, K and V, to the tail
 *                  block with the new token in place -- what pkv_block_copy
 *                  of (cow_src[s], tail) for this layer followed by
 *                  pkv_kv_append would leave.  -1: no copy.
 *                  PKV_COW_NO_APPEND (-2): sequence s appends nothing and
 *                  copies nothing in this launch (its attention reads the
 *                  pool as it is); an aborted pkv_block_manager_step writes
 *                  this for every sequence, so a device-only step chained
 *                  behind it leaves the pools untouched.  Read, like
 *                  seq_lens and the tables, before the wait on the previous
 *                  kernel.
 *   other arguments as pkv_paged_decode_attention.
 *
 * Result: the pools hold exactly what pkv_kv_append with that slot mapping
 * would store, and out is what pkv_paged_decode_attention computes over the
 * updated pools.  The attention reads the new token from k_new/v_new, not
 * back from the pool.  Precondition (as for any decode step): the block
 * holding the new slot belongs to this sequence alone (copy-on-write done).
 * Errors: as pkv_paged_decode_attention; PKV_ERR_NULL if k_new or v_new is
 * NULL, PKV_ERR_ALIGN if either is not 16-byte aligned.
 */
int pkv_append_paged_decode_attention(const pkv_cache_t* cache, int layer,
                                      const void* k_new, const void* v_new,
                                      const int32_t* cow_src,
                                      const void* q, int num_seqs, int num_q_heads,
                                      const int32_t* block_tables, int max_blocks_per_seq,
                                      const int32_t* seq_lens, float scale, void* out,
                                      void* workspace, size_t workspace_bytes,
                                      int partition_tokens, void* stream);

/*
 * pkv_paged_decode_attention_noalloc -- pkv_paged_decode_attention for callers
 * that cannot allocate device memory.  The pages describe no such call.  It is
 * for code that has no way to get a workspace: a plugin inside a host
 * framework that owns all device memory and hands the plugin only its input
 * and output buffers, or a real-time serving loop that must never call the
 * allocator (an allocation can fail, or synchronise the device, at the worst
 * moment).
 *
 * Same arguments and result as pkv_paged_decode_attention, without a
 * workspace: the scratch (partial results of split sequences, their tickets,
 * the tile prefix of batches over 768 sequences) lives
 * in one fixed device array of PKV_NOALLOC_SCRATCH_BYTES (16 MiB) inside this
 * library.  Every GPU that loads the library holds that array until the
 * process exits.  The call itself allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 *
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and keeps it; make that
 *     first call before any stream capture.
 *   - Each call zeroes the tickets it uses (an asynchronous memset on
 *     `stream`), then launches the attention kernel on `stream`.
 *   - All calls share the one array and it keeps the last call's contents:
 *     calls whose GPU work can overlap (different streams without ordering
 *     between them, or concurrent host threads on different streams) race
 *     and give wrong results.  Order them on one stream.
 *   - A request whose scratch would exceed PKV_NOALLOC_SCRATCH_BYTES returns
 *     PKV_ERR_SCRATCH before launching anything (the size grows with the
 *     number of warps the device runs, the group size G, head_dim, and with
 *     a partition cap, the batch's total length).
 */
int pkv_paged_decode_attention_noalloc(const pkv_cache_t* cache, int layer,
                                       const void* q, int num_seqs, int num_q_heads,
                                       const int32_t* block_tables, int max_blocks_per_seq,
                                       const int32_t* seq_lens, float scale, void* out,
                                       int partition_tokens, void* stream);

/*
 * pkv_set_wait_limit_ns -- how long the attention kernel's bounded wait for a
 * staged tile may last on the current device before it gives up with
 * PKV_DEV_TIMEOUT (0 = the default, 2 seconds).  A timed-out warp still
 * waits (up to half a second, a fixed limit) for the copies it has in
 * flight before it exits, so no copy outlives the launch.  A short limit
 * turns a stuck launch into an error status sooner; tests use a limit of a
 * few nanoseconds to drive the timeout path without any fault.  Synchronous
 * (a copy to a device variable); affects launches made after it returns.
 * After a timeout, zero the workspace again (pkv_workspace_init).
 */
int pkv_set_wait_limit_ns(unsigned long long limit_ns);

/*
 * pkv_get_device_status -- read (and with reset != 0, clear) the device status
 * word of the current device.  Synchronises the device first.
 */
int pkv_get_device_status(unsigned int* status_out, int reset);

/* pkv_strerror -- static text for a PKV_ERR_* code. */
const char* pkv_strerror(int code);

/* pkv_abi_version -- PKV_ABI_VERSION of the loaded library. */
int pkv_abi_version(void);

/* pkv_build_hash -- 16 hex digits identifying the sources, header and
 * compiler flags this library was built from (static string).  The Python
 * loader rebuilds the library when it differs from the checkout's. */
const char* pkv_build_hash(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
