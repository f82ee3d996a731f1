// block_manager_step: one decode step of the block manager on the device.
//
// What it computes ("Infra: PagedAttention", sections 按 Block 分配 and 共享前缀，
// 分叉时 Copy-on-write; ithelp article 10405755, section 手動畫一次 block table):
// every sequence appends one token.  Writers are served in the given order.
// A writer whose tail block is full (or who has no block) takes the next free
// block.  A writer whose tail has room but is shared (reference count above
// one) copies it: it takes a free block, records (tail, new) as a copy pair,
// remaps its table and drops one reference on the old tail.  Otherwise it
// writes in place.  The new token's slot is table[pos / B] * B + pos % B.
//
// The order-dependent choices are made without a serial walk:
//   - a writer on shared tail b sees count c_b - r, where r is the number of
//     earlier writers on b (each of them copied and dropped one reference),
//     so it copies exactly when r < c_b - 1;
//   - the k-th block taken, in writer order, is the free ring's entry at
//     head + k (an exclusive scan of "takes a block" over the writers);
//   - copy pairs are numbered by an exclusive scan of "copies".
// One CTA of 1024 threads; writer i is handled by thread i mod 1024.  All
// reads and decisions come before the wait on the previous kernel, all writes
// after it.
//
// An abort (free blocks short, an index out of range) changes no state and
// leaves outputs that make a step queued behind it harmless: every slot -1,
// no copy pair, and cow_src = PKV_COW_NO_APPEND for every sequence.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

constexpr int BM_THREADS = 1024;
constexpr int BM_PER_THREAD = 4;
constexpr int BM_MAX_SEQS = BM_THREADS * BM_PER_THREAD;

struct BmArgs {
    int32_t* block_tables;      // [N][max_blocks], updated in place
    int32_t* seq_lens;          // [N] lengths before the step; + 1 on return
    int32_t* refcount;          // [num_blocks]
    const int32_t* free_ring;   // [num_blocks] free block ids, in hand-out order from head
    int32_t* free_state;        // [2] head (ring index of the next free id), count
    const int32_t* order;       // [N] writer order (sequence ids), or null: 0..N-1
    int64_t* slot_mapping;      // [N] out, by sequence
    int32_t* copy_pairs;        // [N][2] out, (src, dst) in writer order
    int32_t* num_pairs;         // [1] out
    int32_t* cow_src;           // [N] out (may be null): copy source per sequence, -1 if none
    int num_seqs;
    int max_blocks;
    int num_blocks;
    int block_size;
};

// Block-wide exclusive scan of one int per thread (BM_THREADS threads).
__device__ __forceinline__ int bm_scan(int v, int* s_warp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = s_warp[lane];                           // BM_THREADS / 32 == 32 warps
        int incl = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (lane >= off) incl += y;
        }
        s_warp[lane] = incl - w;                        // exclusive prefix of warp sums
        if (lane == 31) s_warp[32] = incl;
    }
    __syncthreads();
    const int before = s_warp[warp] + x - v;
    *total = s_warp[32];
    __syncthreads();
    return before;
}

__global__ void __launch_bounds__(BM_THREADS, 1) block_manager_kernel(const BmArgs a) {
    // Reads first, writes after the wait.  What this kernel reads (order,
    // lengths, tables, counts, free ring and state) is written only by this
    // kernel, which never releases its dependents early (so an earlier step
    // has completed before this one starts), and by copies; so every read and
    // decision runs before the wait, overlapping the tail of the kernel before
    // it on the stream (an attention launch that still reads the tables), and
    // every write comes after.  Not releasing early also lets the next
    // attention launch read the new lengths before its own wait.
    __shared__ int s_tail[BM_MAX_SEQS];                 // tail block of writer i, -1: takes a new one
    __shared__ int s_list[BM_MAX_SEQS];                 // writers whose tail is shared (any order)
    __shared__ int s_warp[33];
    __shared__ int s_abort, s_nlist;
    const int N = a.num_seqs, B = a.block_size;
    const int tid = threadIdx.x;
    if (tid == 0) { s_abort = 0; s_nlist = 0; }
    const int head = a.free_state[0], avail = a.free_state[1];
    __syncthreads();

    // writer i = k * BM_THREADS + tid: one per thread for up to 1024 sequences
    int seq[BM_PER_THREAD], pos[BM_PER_THREAD], cnt[BM_PER_THREAD];
#pragma unroll
    for (int k = 0; k < BM_PER_THREAD; ++k) {
        const int i = k * BM_THREADS + tid;
        seq[k] = -1; pos[k] = 0; cnt[k] = 0;
        if (i >= N) continue;
        s_tail[i] = -1;
        const int s = a.order ? a.order[i] : i;
        if (s < 0 || s >= N) { raise_status(PKV_DEV_RANGE); atomicExch(&s_abort, 1); continue; }
        seq[k] = s;
        pos[k] = a.seq_lens[s];
        const int lb = pos[k] / B;
        if (pos[k] < 0 || lb >= a.max_blocks) { raise_status(PKV_DEV_LENGTH); atomicExch(&s_abort, 1); continue; }
        if (pos[k] % B != 0) {
            const int tail = a.block_tables[(size_t)s * a.max_blocks + lb];
            if (tail < 0 || tail >= a.num_blocks) { raise_status(PKV_DEV_RANGE); atomicExch(&s_abort, 1); continue; }
            s_tail[i] = tail;
            cnt[k] = a.refcount[tail];
            if (cnt[k] > 1) s_list[atomicAdd(&s_nlist, 1)] = i;
        }
    }
    __syncthreads();

    // which writers take a block, which of them copy: a writer on a shared
    // tail needs its rank among earlier writers of the same block, counted
    // over the (usually short) list of writers on shared tails
    int v[BM_PER_THREAD];                               // takes | copies << 16
    const int nlist = s_nlist;
#pragma unroll
    for (int k = 0; k < BM_PER_THREAD; ++k) {
        const int i = k * BM_THREADS + tid;
        v[k] = 0;
        if (seq[k] < 0) continue;
        const int tail = s_tail[i];
        if (tail < 0) {
            v[k] = 1;
        } else if (cnt[k] > 1) {
            int r = 0;                                  // earlier writers on the same tail
            for (int j = 0; j < nlist; ++j) {
                const int w = s_list[j];
                r += (w < i && s_tail[w] == tail);
            }
            if (cnt[k] - r > 1) v[k] = 1 | (1 << 16);
        }
    }
    // one exclusive scan in writer order of both counts (each below 2^16),
    // one round of BM_THREADS writers at a time
    int take_base[BM_PER_THREAD], copy_base[BM_PER_THREAD];
    int total_takes = 0, total_copies = 0;
#pragma unroll
    for (int k = 0; k < BM_PER_THREAD; ++k) {
        if (k * BM_THREADS >= N) { take_base[k] = copy_base[k] = 0; continue; }   // uniform
        int t;
        const int before = bm_scan(v[k], s_warp, &t);
        take_base[k] = total_takes + (before & 0xFFFF);
        copy_base[k] = total_copies + (before >> 16);
        total_takes += t & 0xFFFF;
        total_copies += t >> 16;
    }
    // the blocks the takers will get, checked before anything changes
    int newb[BM_PER_THREAD];
#pragma unroll
    for (int k = 0; k < BM_PER_THREAD; ++k) newb[k] = -1;
    if (total_takes <= avail) {
#pragma unroll
        for (int k = 0; k < BM_PER_THREAD; ++k) {
            if (seq[k] < 0 || !(v[k] & 1)) continue;
            newb[k] = a.free_ring[(head + take_base[k]) % a.num_blocks];
            if (newb[k] < 0 || newb[k] >= a.num_blocks) { raise_status(PKV_DEV_RANGE); atomicExch(&s_abort, 1); }
        }
    }
    __syncthreads();
    const bool abort = s_abort || total_takes > avail;

    pdl_wait();                                         // the kernel before this one has finished
    if (abort) {
        // Change nothing, and say so to whatever is queued behind this step:
        // no slot (kv_append skips slot -1), no copy pair, and per sequence
        // the marker that makes the fused append + attention append nothing.
        if (tid == 0 && total_takes > avail) raise_status(PKV_DEV_NOBLOCKS);
        for (int i = tid; i < N; i += BM_THREADS) {
            a.slot_mapping[i] = -1;
            if (a.cow_src) a.cow_src[i] = PKV_COW_NO_APPEND;
        }
        if (tid == 0) *a.num_pairs = 0;
        return;
    }

#pragma unroll
    for (int k = 0; k < BM_PER_THREAD; ++k) {
        if (seq[k] < 0) continue;
        const int s = seq[k], p = pos[k];
        const int tail = s_tail[k * BM_THREADS + tid];
        const bool copies = (v[k] >> 16) != 0;
        int32_t* entry = a.block_tables + (size_t)s * a.max_blocks + p / B;
        int blk = tail;
        if (v[k] & 1) {
            blk = newb[k];
            a.refcount[blk] = 1;
            if (copies) {
                a.copy_pairs[2 * copy_base[k]] = tail;
                a.copy_pairs[2 * copy_base[k] + 1] = blk;
                atomicSub(a.refcount + tail, 1);
            }
            *entry = blk;
        }
        if (a.cow_src) a.cow_src[s] = copies ? tail : -1;
        a.slot_mapping[s] = (int64_t)blk * B + p % B;
        a.seq_lens[s] = p + 1;
    }
    if (tid == 0) {
        a.free_state[0] = (head + total_takes) % a.num_blocks;
        a.free_state[1] = avail - total_takes;
        *a.num_pairs = total_copies;
    }
}

// ---- release: finished requests give their blocks back ---------------------------
//
// What it computes ("Infra: PagedAttention", section 按 Block 分配: a finished
// request drops its references; ithelp article 10405755, section 手動畫一次
// block table: when the request ends its blocks return to the pool): for each
// released sequence in the given order, each block of its table in table
// order loses one reference, and a block whose count reaches zero is appended
// to the free ring, after the blocks already free, in that order of drops.
// The sequence's length becomes 0 and its table row -1.
//
// The order of drops is made without a serial walk: drop e (release r, table
// entry j, numbered by a scan of the released sequences' block counts) on a
// block of count c frees it exactly when it is the c-th drop on that block,
// i.e. when r_e = c - 1 earlier drops hit the same block.  Unshared blocks
// (c = 1) are freed by their one drop; drops on shared blocks list themselves
// in shared memory and count the earlier ones there.  Ring positions are an
// exclusive scan of "frees" in drop order.  Every check comes before any
// write, so an invalid request changes nothing.
constexpr int BR_MAX_SHARED = 8192;                  // drops on shared blocks one call can take

struct BrArgs {
    int32_t* block_tables;      // [N][max_blocks]
    int32_t* seq_lens;          // [N]
    int32_t* refcount;          // [num_blocks]
    int32_t* free_ring;         // [num_blocks]
    int32_t* free_state;        // [2] head, count
    const int32_t* seqs;        // [num_release] rows to release, distinct
    int num_seqs;
    int num_release;
    int max_blocks;
    int num_blocks;
    int block_size;
};

struct BrShared {
    int off[BM_MAX_SEQS + 1];                        // first drop of release r; off[n] = drops
    unsigned seen[BM_MAX_SEQS / 32];                 // rows named so far (duplicates abort)
    int nlist;
    int abort;
    int warp[33];
    int list_e[BR_MAX_SHARED], list_b[BR_MAX_SHARED], list_c[BR_MAX_SHARED];
};

__global__ void __launch_bounds__(BM_THREADS, 1) block_release_kernel(const BrArgs a) {
    extern __shared__ unsigned char br_smem_raw[];
    BrShared& sh = *reinterpret_cast<BrShared*>(br_smem_raw);
    const int tid = threadIdx.x;
    const int n = a.num_release, B = a.block_size;
    pdl_wait();                                       // earlier steps' writes have landed
    for (int i = tid; i < BM_MAX_SEQS / 32; i += BM_THREADS) sh.seen[i] = 0u;
    if (tid == 0) { sh.nlist = 0; sh.abort = 0; }
    __syncthreads();

    // the released rows, their block counts and the drop numbering
    int carry = 0;
    for (int base = 0; base < n; base += BM_THREADS) {   // uniform trip count
        const int r = base + tid;
        int nb = 0;
        if (r < n) {
            const int s = a.seqs[r];
            if (s < 0 || s >= a.num_seqs) {
                raise_status(PKV_DEV_RANGE); atomicExch(&sh.abort, 1);
            } else if (atomicOr(&sh.seen[s >> 5], 1u << (s & 31)) & (1u << (s & 31))) {
                raise_status(PKV_DEV_RANGE); atomicExch(&sh.abort, 1);   // named twice
            } else {
                const int len = a.seq_lens[s];
                nb = len > 0 ? (len + B - 1) / B : 0;
                if (len < 0 || nb > a.max_blocks) {
                    raise_status(PKV_DEV_LENGTH); atomicExch(&sh.abort, 1); nb = 0;
                }
            }
        }
        int tot;
        const int before = bm_scan(nb, sh.warp, &tot);
        if (r < n) sh.off[r] = carry + before;
        carry += tot;
    }
    if (tid == 0) sh.off[n] = carry;
    __syncthreads();
    const int E = carry;
    // drop e -> (release r, table entry j): the last r with off[r] <= e
    auto locate = [&](int e, int& r, int& j) {
        int lo = 0, hi = n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sh.off[mid] <= e) lo = mid; else hi = mid - 1;
        }
        r = lo;
        j = e - sh.off[lo];
    };
    auto block_of = [&](int e, int& blk) -> bool {
        int r, j;
        locate(e, r, j);
        blk = a.block_tables[(size_t)a.seqs[r] * a.max_blocks + j];
        return blk >= 0 && blk < a.num_blocks;
    };

    // checks, and the list of drops on shared blocks
    if (!sh.abort) {
        for (int e = tid; e < E; e += BM_THREADS) {
            int blk;
            if (!block_of(e, blk)) { raise_status(PKV_DEV_RANGE); atomicExch(&sh.abort, 1); continue; }
            const int c = a.refcount[blk];
            if (c <= 0) { raise_status(PKV_DEV_RANGE); atomicExch(&sh.abort, 1); continue; }
            if (c > 1) {
                const int k = atomicAdd(&sh.nlist, 1);
                if (k < BR_MAX_SHARED) { sh.list_e[k] = e; sh.list_b[k] = blk; sh.list_c[k] = c; }
                else { raise_status(PKV_DEV_RANGE); atomicExch(&sh.abort, 1); }
            }
        }
    }
    __syncthreads();
    if (sh.abort) return;                             // nothing written
    const int nlist = sh.nlist;
    // drops on a block beyond its count: a count that would fall below zero
    for (int k = tid; k < nlist; k += BM_THREADS) {
        int r = 0;
        for (int q = 0; q < nlist; ++q) r += (sh.list_b[q] == sh.list_b[k] && sh.list_e[q] < sh.list_e[k]);
        if (r >= sh.list_c[k]) { raise_status(PKV_DEV_RANGE); atomicExch(&sh.abort, 1); }
    }
    __syncthreads();
    if (sh.abort) return;

    // which drops free their block, and where it goes in the ring (counts not yet changed)
    const int head = a.free_state[0], avail = a.free_state[1];
    int freed = 0;
    for (int base = 0; base < E; base += BM_THREADS) {   // uniform trip count
        const int e = base + tid;
        int frees = 0, blk = -1;
        if (e < E) {
            block_of(e, blk);
            const int c = a.refcount[blk];
            if (c == 1) {
                frees = 1;
            } else {
                int r = 0;
                for (int q = 0; q < nlist; ++q) r += (sh.list_b[q] == blk && sh.list_e[q] < e);
                frees = r == c - 1;
            }
        }
        int tot;
        const int before = bm_scan(frees, sh.warp, &tot);
        if (frees) a.free_ring[(head + avail + freed + before) % a.num_blocks] = blk;
        freed += tot;
    }
    __syncthreads();                                  // every count read before any changes
    for (int e = tid; e < E; e += BM_THREADS) {
        int blk;
        block_of(e, blk);
        atomicSub(a.refcount + blk, 1);
    }
    __syncthreads();                                  // every table entry read before any is reset
    for (int r = 0; r < n; ++r) {
        const int s = a.seqs[r];
        for (int j = tid; j < a.max_blocks; j += BM_THREADS) a.block_tables[(size_t)s * a.max_blocks + j] = -1;
        if (tid == 0) a.seq_lens[s] = 0;
    }
    if (tid == 0) a.free_state[1] = avail + freed;
}

}  // namespace pkv
