// Paged decode attention: one persistent grid, work split evenly per warp.
//
// What is computed ("Infra: PagedAttention", section 按 Block 分配; ithelp
// article 10405755, section PagedAttention 的核心想法): per (sequence, kv
// head) and each of its G query heads, softmax(scale * q . k_i) over all the
// sequence's tokens, read in place through the block table, times V.  Work
// computed in pieces is merged with the page's max-rescaled rule
//     o = sum_r e^{m_r - M} o_r / sum_r e^{m_r - M} Z_r,   M = max_r m_r.
//
// Decomposition.  Every (sequence, kv head) is a unit of ceil(len/TILE)
// tiles; units are laid end to end (sequence-major, kv head minor) into one
// flat space of positions, cut into R ranges of equal length.  A tile takes
// tc positions and a unit adds a gap after its last tile for its fixed
// costs (see the layout in the planning below), so equal ranges take about
// equal time whatever the length mix.  Without a partition cap R is the
// number of warps in the grid (one range each); with a cap of C tiles
// (positions are then tiles), each warp takes ceil(ceil(T/C)/K) consecutive
// ranges.  A warp streams its tiles with one continuous bulk-copy pipeline
// that runs across unit and range boundaries, so it never drains between
// sequences.  A unit inside one range is finished by its warp; a unit cut by
// range boundaries leaves one partial per range.  Pieces count themselves on a
// ticket; the last one merges them in range order into its own registers
// (a piece that finds every other piece already counted merges without
// publishing itself).  Units of more than 8 pieces merge in two levels:
// groups of 8 ranges, then the groups.  The fold order is fixed, so the
// result does not depend on which piece finishes last.
//
// Planning.  Every CTA reads the sequence lengths once and scans them into
// a prefix of positions per sequence, kept in shared memory (in global
// memory, written identically by every CTA, for batches of more than
// PREFIX_SMEM sequences); a warp finds its first tile by binary search and
// loads its first block ids.  All of this reads only the lengths and the
// tables and runs before the wait on the previous kernel (programmatic
// dependent launch); the rest of the kernel runs after it.  A warp that has
// no tile left to issue lets the next kernel on the stream start launching.
//
// Data movement.  Each warp owns a ring of STAGES shared-memory stages.  One
// lane issues, per stage, TMA tensor loads (cp.async.bulk.tensor, 2-D tensor
// map over all pool rows, 128-byte swizzle, no multicast) of the tile's
// physical blocks for K and V, plus a bulk copy of the unit's q when the unit
// starts; all complete on the stage's mbarrier.  The swizzle makes the
// ldmatrix reads of K and V conflict-free.  Rows of a tail block past the
// sequence's length are loaded with the block but masked: their scores are
// -inf and their V rows are zeroed in shared memory before the P V product.
//
// Fused append and copy-on-write (k_new set).  The unit's last tile also
// brings the new token's K and V rows (bulk copies into a staging area); they
// replace the stale row in shared memory and are stored in their slot.  With
// cow_src, the tail block is fetched from its copy source and written whole
// (this layer, this kv head, K and V, new row included) to the fresh block.
//
// Compute.  Tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate) with
// the G query heads as the MMA rows; see attn_common.cuh.
//
// Faults never trap: waits are bounded (pkv_set_wait_limit_ns; a timeout
// sets PKV_DEV_TIMEOUT, drains this warp's copies in flight and returns),
// block ids outside the pool set PKV_DEV_RANGE and are not fetched, lengths
// above the table's capacity set PKV_DEV_LENGTH and are clamped.
#pragma once

#include <cuda.h>

#include "attn_common.cuh"

namespace pkv {

struct AttnArgs {
    const uint16_t* q;             // [N][Hq][D]
    uint16_t* out;                 // [N][Hq][D]
    const int32_t* block_tables;   // [N][max_blocks]
    const int32_t* seq_lens;       // [N]
    int num_seqs;
    int num_kv_heads;
    int num_blocks;
    int max_blocks;
    float qscale;                  // scale * log2(e)
    long long row_base;            // pool row of (layer, block 0, head 0, row 0) in the tensor maps
    // workspace
    float2* part_mz;               // [R_max][2][G]    (m, Z) of a partial, base 2
    float* part_o;                 // [R_max][2][G][D] unnormalised partial output
    unsigned int* tickets;         // [N*Hkv] zero at rest
    unsigned int* group_tickets;   // [R_max][2] zero at rest: a group's first range and slot
    long long* prefix_g;           // [N+1] tile prefix, used when N > PREFIX_SMEM
    int R_max;                     // ranges the workspace holds
    // fused append (k_new != nullptr): the new token of sequence s, at
    // position seq_lens[s] - 1, is stored in its slot and used in place
    const uint4* k_new;            // [N][Hkv][D] bf16
    const uint4* v_new;
    uint16_t* k_pool;              // pool bases (all layers)
    uint16_t* v_pool;
    // fused copy-on-write (with the fused append; may be null): sequence s's
    // tail block is a fresh copy of block cow_src[s] (>= 0), made here for
    // this layer: the tile reads the source and writes the copy
    const int32_t* cow_src;        // [N]
    int cap_tiles;                 // > 0: no range longer than this many tiles
    int K;                         // warps in the grid
};

constexpr int PREFIX_SMEM = 768;       // sequences whose tile prefix fits in shared memory

// Weights of the position layout: a tile, a unit's start and end, and the
// expected cost of the unit's end being a piece published mid-stream.
#ifndef PKV_W_TILE
#define PKV_W_TILE 8
#endif
#ifndef PKV_W_UNIT
#define PKV_W_UNIT 10
#endif
#ifndef PKV_W_PIECE
#define PKV_W_PIECE 18
#endif

// R equal ranges over the flat space of T tiles (R <= T, so none is empty).
struct Sched {
    long long T, R;                    // positions in the flat space, ranges
    __device__ __forceinline__ long long begin(long long r) const { return r * T / R; }
    // the range holding flat tile t: the largest r with begin(r) <= t
    __device__ __forceinline__ long long range_of(long long t) const { return ((t + 1) * R - 1) / T; }
};

__device__ __forceinline__ int clamp_len(int len, int cap) { return len > cap ? cap : (len < 0 ? 0 : len); }

// Weights of the position layout (see the planning in the kernel).
struct Weights {
    long long tc, uc, pc, lr;          // tile, unit, expected piece; static range length
};

// Positions taken by one unit of n tiles: its tiles, then a gap for the
// unit's fixed cost and its expected piece cost.  0 for an empty unit.
__device__ __forceinline__ long long unit_cost(const Weights& w, long long n) {
    if (n <= 0) return 0;
    long long c = n * w.tc + w.uc;
    if (w.pc) {
        const long long span = n * w.tc;
        c += w.pc * (span < w.lr ? span : w.lr) / w.lr;
    }
    return c;
}

template <int D, int G, int BS, int NW, int STAGES>
struct AttnCfg {
    using TS = TileSmem<D, BS>;
    static constexpr int TILE = TS::TILE;
    static constexpr int BPT = TS::BPT;
    static constexpr int KT_BYTES = TS::KT_BYTES;
    static constexpr int STAGE_BYTES = 2 * KT_BYTES;            // K tile, V tile
    static constexpr int Q_BYTES = G * D * 2;                   // q of a unit
    static constexpr int META_BYTES = 32;
    static constexpr int RING_BYTES = NW * STAGES * STAGE_BYTES;
    static constexpr int Q_OFF = RING_BYTES;
    static constexpr int META_OFF = Q_OFF + NW * STAGES * Q_BYTES;
    static constexpr int BAR_OFF = META_OFF + NW * STAGES * META_BYTES;
    // fused append: per stage, the new token's physical block (16-byte
    // header) and its K and V rows, brought by bulk copies with the tile
    // header: new-row destinations (K, V), copy-on-write block destinations (K, V)
    static constexpr int NEW_HDR = 32;
    static constexpr int NEW_BYTES = NEW_HDR + 4 * D;
    static constexpr int NEW_OFF = BAR_OFF + NW * STAGES * 8;
    static constexpr int PREFIX_OFF = NEW_OFF + NW * STAGES * NEW_BYTES;
    static constexpr int SMEM_BYTES = PREFIX_OFF + (PREFIX_SMEM + 1) * 4 + 1024;   // + alignment slack
    static constexpr int BOX_BYTES = BS * 128;                  // one TMA box: BS rows x 64 dims
    static constexpr int NT = NW * 32;
};

struct StageMeta {
    int s, h, t, len;
    long long f;      // flat tile index
    int flags;
    int r;            // range
};
static_assert(sizeof(StageMeta) == 32, "meta layout");

constexpr int F_FIRST = 1;        // first tile of a unit within this range: q staged, state reset
constexpr int F_LAST = 2;         // last tile of a unit within this range: finish the unit
constexpr int F_UNIT_START = 4;   // tile 0 of the unit
constexpr int F_UNIT_END = 8;     // last tile of the unit

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Block-wide exclusive scan of one value per thread (NT threads); returns
// the thread's exclusive prefix and writes the block total to *total.
template <int NT>
__device__ __forceinline__ long long block_scan(long long v, long long* s_red, long long* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const long long y = __shfl_up_sync(FULL, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) s_red[warp] = x;
    __syncthreads();
    long long before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        const long long sw = s_red[w];
        if (w < warp) before += sw;
        all += sw;
    }
    __syncthreads();
    *total = all;
    return before + x - v;
}

// register budgets: at least this many warps resident per SM (head_dim 64 / 128)
#ifndef PKV_ATTN_MIN_WARPS_PER_SM
#define PKV_ATTN_MIN_WARPS_PER_SM 12
#endif
#ifndef PKV_ATTN_MIN_WARPS_PER_SM_128
#define PKV_ATTN_MIN_WARPS_PER_SM_128 8
#endif

template <int D, int G, int BS, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32, (D == 64 ? PKV_ATTN_MIN_WARPS_PER_SM : PKV_ATTN_MIN_WARPS_PER_SM_128) / NW)
paged_attention_kernel(const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const AttnArgs a) {
    using C = AttnCfg<D, G, BS, NW, STAGES>;
    using TS = typename C::TS;
    constexpr int TILE = C::TILE;
    constexpr int NT = C::NT;
    extern __shared__ unsigned char smem_raw[];
    __shared__ long long s_red[NW];
    __shared__ Weights s_w;                               // the launch's position weights
    __shared__ unsigned long long s_wait_limit;           // bounded wait on a stage (ns)

    // 1024-byte aligned base (swizzled TMA destinations)
    const uint32_t raw_addr = smem_addr(smem_raw);
    unsigned char* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tid = threadIdx.x;
    unsigned char* ring = smem + (size_t)warp * STAGES * C::STAGE_BYTES;
    unsigned char* qslots = smem + C::Q_OFF + (size_t)warp * STAGES * C::Q_BYTES;
    StageMeta* meta = reinterpret_cast<StageMeta*>(smem + C::META_OFF) + warp * STAGES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF) + warp * STAGES;
    unsigned char* newrows = smem + C::NEW_OFF + (size_t)warp * STAGES * C::NEW_BYTES;
    const bool fused_append = a.k_new != nullptr;
    constexpr int CH = D / 8;                             // 16-byte chunks of a K or V row

    if (lane == 0) {
        if (warp == 0) {
            prefetch_tensormap(&tmap_k);
            prefetch_tensormap(&tmap_v);
        }
#pragma unroll
        for (int st = 0; st < STAGES; ++st) mbar_init(smem_addr(&bars[st]), 1);
        fence_mbar_init();
    }

    const int N = a.num_seqs;
    const int Hkv = a.num_kv_heads;
    const int Hq = Hkv * G;
    const int cap = a.max_blocks * BS;
    const bool pre_smem = N <= PREFIX_SMEM;
    int* s_prefix = reinterpret_cast<int*>(smem + C::PREFIX_OFF);

    // ---- plan: prefix of tiles per sequence, T, the schedule -------------------------
    // For up to PREFIX_SMEM / 2 - 1 sequences the clamped lengths are kept in
    // the upper half of the prefix array, so no later length read leaves the SM.
    const bool lens_smem = N < PREFIX_SMEM / 2;
    int* s_len = s_prefix + PREFIX_SMEM / 2;
    long long T = 0;
    auto scan_chunk = [&](int base, int raw) {
        const int s = base + tid;
        long long v = 0;
        if (s < N) {
            const int len = clamp_len(raw, cap);
            v = (long long)Hkv * ((len + TILE - 1) / TILE);
            if (lens_smem) s_len[s] = len;
            if (blockIdx.x == 0 && raw > cap) raise_status(PKV_DEV_LENGTH);
        }
        long long tot;
        const long long incl = T + block_scan<NT>(v, s_red, &tot) + v;
        if (s < N && pre_smem) s_prefix[s + 1] = (int)incl;   // (global prefix: positions only, below)
        T += tot;
    };
    // clamped length of sequence s (planning and cursor)
    auto seq_len_raw = [&](int s) -> long long {
        return lens_smem ? s_len[s] : clamp_len(__ldg(a.seq_lens + s), cap);
    };
    if (pre_smem) {
        // every length this thread scans, loaded before the first scan: one round trip
        constexpr int MAXC = (PREFIX_SMEM + NT - 1) / NT;
        int raw[MAXC];
#pragma unroll
        for (int c = 0; c < MAXC; ++c) {
            const int s = c * NT + tid;
            raw[c] = s < N ? __ldg(a.seq_lens + s) : 0;
        }
#pragma unroll
        for (int c = 0; c < MAXC; ++c)
            if (c * NT < N) scan_chunk(c * NT, raw[c]);
    } else {
        for (int base = 0; base < N; base += NT) {
            const int s = base + tid;
            scan_chunk(base, s < N ? __ldg(a.seq_lens + s) : 0);
        }
    }
    if (tid == 0) {
        if (pre_smem) s_prefix[0] = 0;
        else a.prefix_g[0] = 0;
    }
    const long long K = a.K;
    // The position layout.  Units lie in flat order; a tile takes tc
    // positions and a unit adds uc + its expected piece cost after its last
    // tile, so ranges of equal length in positions take about equal time.
    // Timed per warp: a unit's fixed costs (its query load, state reset and
    // finish) come to about one tile, and a piece of a split unit (published,
    // counted, possibly merged) about two more.  A unit of n tiles is cut by a
    // range boundary with probability about min(1, n tc / lr), lr the range
    // length, which weights its piece cost.  The weights (tile 8, unit 10,
    // piece 18) are the best of a sweep timed on the length mixes of the
    // benchmark workloads.  Under a partition cap (whose ranges count tiles),
    // and for sizes whose positions would not fit 32 bits, positions are tiles.
    Weights wt;
    wt.tc = 1; wt.uc = 0; wt.pc = 0; wt.lr = 1;
    if (PKV_W_TILE > 1 && a.cap_tiles == 0 && T > 0 &&
        T * (PKV_W_TILE + PKV_W_UNIT + PKV_W_PIECE) < (1LL << 30)) {
        wt.tc = PKV_W_TILE;
        wt.uc = PKV_W_UNIT;
        wt.pc = PKV_W_PIECE;
        wt.lr = T * PKV_W_TILE / K > 1 ? T * PKV_W_TILE / K : 1;
    }
    // Prefix of positions per sequence.  In shared memory the tile prefix
    // already is it when tc = 1; the global prefix (large batches) is written
    // here only, every CTA writing the same values.
    if (wt.tc != 1 || !pre_smem) {
        T = 0;
        for (int base = 0; base < N; base += NT) {
            const int s_ = base + tid;
            const long long n = s_ < N ? (seq_len_raw(s_) + TILE - 1) / TILE : 0;
            const long long v = (long long)Hkv * unit_cost(wt, n);
            long long tot;
            const long long incl = T + block_scan<NT>(v, s_red, &tot) + v;
            if (s_ < N) {
                if (pre_smem) s_prefix[s_ + 1] = (int)incl;
                else a.prefix_g[s_ + 1] = incl;
            }
            T += tot;
        }
    }
    Sched sc;
    sc.T = T;
    long long rpw = 1;                                    // ranges per warp
    if (a.cap_tiles > 0 && T > 0) {
        const long long need = (T + a.cap_tiles - 1) / a.cap_tiles;
        rpw = (need + K - 1) / K;
    }
    // every range at least one tile long, so each range a unit spans holds
    // one of its tiles
    sc.R = K * rpw;
    if (sc.R > T / wt.tc) sc.R = T / wt.tc;
    if (sc.R > a.R_max) {                                 // cannot happen with a workspace of the queried size
        if (tid == 0 && blockIdx.x == 0) raise_status(PKV_DEV_RANGE);
        sc.R = a.R_max;
    }
    if (tid == 0) {
        s_w = wt;
        s_wait_limit = *(volatile unsigned long long*)&g_wait_limit_ns;
    }
    __syncthreads();
    const int tc = (int)wt.tc;
    const long long wg = (long long)blockIdx.x * NW + warp;
    const long long r_first = wg * rpw;
    const long long r_stop = r_first + rpw < sc.R ? r_first + rpw : sc.R;   // this warp's ranges

    // The first tile at or after position `pos`: its (sequence, kv head,
    // tile) and position, or -1 when there is none.
    auto locate = [&](long long pos, int& s_out, int& h_out, int& t_out) -> long long {
#pragma unroll 1
        for (int it = 0; it < 2; ++it) {
            if (pos >= sc.T) return -1;
            int lo = 0, hi = N - 1;                       // largest s with prefix[s] <= pos
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                const long long pm = pre_smem ? (long long)s_prefix[mid] : a.prefix_g[mid];
                if (pm <= pos) lo = mid; else hi = mid - 1;
            }
            const long long p0 = pre_smem ? (long long)s_prefix[lo] : a.prefix_g[lo];
            const long long n = (seq_len_raw(lo) + TILE - 1) / TILE;
            const long long ucs = unit_cost(s_w, n);
            const long long off = pos - p0;
            long long h = off / ucs;
            const long long t = (off - h * ucs + tc - 1) / tc;
            if (t < n) {
                s_out = lo; h_out = (int)h; t_out = (int)t;
                return p0 + h * ucs + t * tc;
            }
            if (++h < Hkv) {                              // in the unit's end gap: the next unit
                s_out = lo; h_out = (int)h; t_out = 0;
                return p0 + h * ucs;
            }
            pos = pre_smem ? (long long)s_prefix[lo + 1] : a.prefix_g[lo + 1];   // the next sequence
        }
        return -1;
    };

    const uint64_t pol_stream = policy_evict_first();

    // ---- producer cursor (every lane keeps an identical copy) ------------------
    long long r = r_first;                                // range of the next tile to issue
    long long f = 0, f_end = 0, f_stop = 0;             // positions: next tile, range end, warp's end
    long long pnext = 0;                                  // position of the next unit's tile 0
    int puc = 1;                                          // positions a unit of this sequence takes
    int ps = 0, ph = 0, pt = 0, plen = 0, pnt = 0, next_len = 0;
    int pcow = -1, next_cow = -1;                         // copy-on-write source of ps, ps + 1
    bool range_first = true;
    int ids = -1, ids_seq = -1, ids_base = 0;
    int pre = -1, pre_seq = -1, pre_base = 0;

    auto load_batch = [&](int s, int base, int len) -> int {
        const int lb = base + lane;
        return (lb * BS < len) ? __ldg(a.block_tables + (size_t)s * a.max_blocks + lb) : -1;
    };
    auto seq_len = [&](int s) -> int {
        if (s >= N) return 0;
        return lens_smem ? s_len[s] : clamp_len(__ldg(a.seq_lens + s), cap);
    };
    auto cow_of = [&](int s) -> int { return (a.cow_src && s < N) ? __ldg(a.cow_src + s) : -1; };
    auto advance_unit = [&]() {
        pt = 0;
        f = pnext;                                        // (empty sequences take no positions)
        if (++ph < Hkv) {
            pnext += puc;
            return;
        }
        ph = 0;
        ++ps;
        plen = next_len;
        pcow = next_cow;
        pnt = (plen + TILE - 1) / TILE;
        while (pnt == 0 && ps + 1 < N) {   // skip empty sequences (rare, synchronous)
            ++ps;
            plen = seq_len(ps);
            pcow = cow_of(ps);
            pnt = (plen + TILE - 1) / TILE;
        }
        next_len = seq_len(ps + 1);
        next_cow = cow_of(ps + 1);
        puc = (int)unit_cost(s_w, pnt);
        pnext = f + puc;
    };
    // Block ids of the current tile's batch of 32 logical blocks (one per
    // lane), taken from the prefetched batch when it holds them; then the
    // batch needed after this one is prefetched: the rest of this table row,
    // else the row's start again for the next kv head, else the next
    // sequence's row.
    auto fetch_ids = [&](int lb0) {
        if (ids_seq == ps && lb0 >= ids_base && lb0 + C::BPT <= ids_base + 32) return;
        if (pre_seq == ps && lb0 >= pre_base && lb0 + C::BPT <= pre_base + 32) {
            ids = pre; ids_seq = pre_seq; ids_base = pre_base;
        } else {
            ids = load_batch(ps, lb0, plen); ids_seq = ps; ids_base = lb0;
        }
        if ((ids_base + 32) * BS < plen) {
            pre_seq = ps; pre_base = ids_base + 32; pre = load_batch(ps, pre_base, plen);
        } else if (ph + 1 < Hkv && ids_base != 0) {
            pre_seq = ps; pre_base = 0; pre = load_batch(ps, 0, plen);
        } else if (ps + 1 < N) {
            pre_seq = ps + 1; pre_base = 0; pre = load_batch(ps + 1, 0, next_len);
        }
    };
    bool have_work = false;
    if (r_first < r_stop) {
        f_end = sc.begin(r_first + 1);
        f_stop = sc.begin(r_stop);
        const long long fpos = locate(sc.begin(r_first), ps, ph, pt);
        if (fpos >= 0 && fpos < f_stop) {                 // (a range in a unit's end gap has no tile)
            have_work = true;
            f = fpos;
            plen = seq_len(ps);
            pnt = (plen + TILE - 1) / TILE;
            puc = (int)unit_cost(s_w, pnt);
            pnext = fpos - (long long)pt * tc + puc;
            next_len = seq_len(ps + 1);
            pcow = cow_of(ps);
            next_cow = cow_of(ps + 1);
            fetch_ids(pt * C::BPT);                       // the first tile's block ids
        }
    }

    // Everything so far read only the lengths and the block tables, which no
    // kernel of this library writes; from here on the pools, q and the
    // outputs are touched, so the kernel before this one on the stream must
    // have finished.
    pdl_wait();
    if (blockIdx.x == 0) {                                // nothing to attend to: zero output
        for (int s = tid; s < N; s += NT) {
            if (clamp_len(__ldg(a.seq_lens + s), cap) == 0) {
                uint4* o4 = reinterpret_cast<uint4*>(a.out + (size_t)s * Hq * D);
                for (int c = 0; c < Hq * D / 8; ++c) o4[c] = make_uint4(0, 0, 0, 0);
            }
        }
    }

    // Stage the next tile into stage `st`; false when this warp has no more tiles.
    auto issue = [&](int st) -> bool {
        if (f >= f_stop) return false;
        if (f >= f_end) {                                 // next range of this warp (contiguous)
            ++r;
            f_end = sc.begin(r + 1);
            range_first = true;
        }
        // position of the tile after this one
        const long long f_next = pt + 1 < pnt ? f + tc : pnext;
        const int nv = min(TILE, plen - pt * TILE);
        int flags = 0;
        if (pt == 0) flags |= F_UNIT_START;
        if (pt == pnt - 1) flags |= F_UNIT_END;
        if (range_first || pt == 0) flags |= F_FIRST;
        if (f_next >= f_end || pt == pnt - 1) flags |= F_LAST;
        range_first = false;
        const int lb0 = pt * C::BPT;
        fetch_ids(lb0);
        int bid[C::BPT];
#pragma unroll
        for (int j = 0; j < C::BPT; ++j) bid[j] = __shfl_sync(FULL, ids, lb0 - ids_base + j);
        // physical block of the new token (fused append, unit's last tile)
        const int nblk = __shfl_sync(FULL, ids, ((plen - 1) / BS - ids_base) & 31);
        if (lane == 0) {
            StageMeta m;
            m.s = ps; m.h = ph; m.t = pt; m.len = plen; m.f = f; m.flags = flags; m.r = (int)r;
            meta[st] = m;
            if (fused_append && (flags & F_UNIT_END)) {
                // where the new token's K and V rows go, and (copy-on-write) the
                // copied tail block's rows of this head (null: none, or an id
                // out of range)
                uint16_t* dk = nullptr;
                uint16_t* dv = nullptr;
                uint16_t* ck = nullptr;
                uint16_t* cv = nullptr;
                if (nblk >= 0 && nblk < a.num_blocks && pcow != PKV_COW_NO_APPEND) {
                    const size_t brow = (size_t)(a.row_base + ((long long)nblk * Hkv + ph) * BS);
                    dk = a.k_pool + (brow + (plen - 1) % BS) * D;
                    dv = a.v_pool + (brow + (plen - 1) % BS) * D;
                    if (pcow >= 0 && pcow < a.num_blocks) {
                        ck = a.k_pool + brow * D;
                        cv = a.v_pool + brow * D;
                    } else if (pcow >= a.num_blocks) {
                        raise_status(PKV_DEV_RANGE);
                    }
                }
                uint16_t** hdr = reinterpret_cast<uint16_t**>(newrows + (size_t)st * C::NEW_BYTES);
                hdr[0] = dk;
                hdr[1] = dv;
                hdr[2] = ck;
                hdr[3] = cv;
            }
            const uint32_t bar = smem_addr(&bars[st]);
            const uint32_t dK = smem_addr(ring + (size_t)st * C::STAGE_BYTES);
            const uint32_t dV = dK + C::KT_BYTES;
            uint32_t bytes = (flags & F_FIRST) ? C::Q_BYTES : 0u;
            // fused append: the unit's last tile also brings the new token's rows
            const bool app = fused_append && (flags & F_UNIT_END) && pcow != PKV_COW_NO_APPEND;
            if (app) bytes += 4u * D;
            bool bad = false;
#pragma unroll
            for (int j = 0; j < C::BPT; ++j) {
                if (j * BS >= nv) continue;
                if (bid[j] < 0 || bid[j] >= a.num_blocks) { bad = true; continue; }
                bytes += 2u * TS::HALVES * C::BOX_BYTES;
            }
            if (bad) raise_status(PKV_DEV_RANGE);
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(bar, bytes);
            if (flags & F_FIRST)
                bulk_g2s(smem_addr(qslots + (size_t)st * C::Q_BYTES),
                         a.q + ((size_t)ps * Hq + (size_t)ph * G) * D, C::Q_BYTES, bar, pol_stream);
            if (app) {
                unsigned char* nb = newrows + (size_t)st * C::NEW_BYTES;
                const size_t row = ((size_t)ps * Hkv + ph) * CH;       // in 16-byte chunks
                bulk_g2s(smem_addr(nb + C::NEW_HDR), a.k_new + row, 2u * D, bar, pol_stream);
                bulk_g2s(smem_addr(nb + C::NEW_HDR + 2 * D), a.v_new + row, 2u * D, bar, pol_stream);
            }
#pragma unroll
            for (int j = 0; j < C::BPT; ++j) {
                if (j * BS >= nv || bid[j] < 0 || bid[j] >= a.num_blocks) continue;
                // copy-on-write: the tail block is read from its source
                const int blk = (app && pcow >= 0 && pcow < a.num_blocks &&
                                 lb0 + j == (plen - 1) / BS) ? pcow : bid[j];
                // pool row of (layer, block, head, row 0); the layer is in row_base
                const int y = (int)(a.row_base + ((long long)blk * Hkv + ph) * BS);
                const uint32_t off = (uint32_t)(j * TS::RPB * 128);
#pragma unroll
                for (int hf = 0; hf < TS::HALVES; ++hf) {
                    tma_load_2d(dK + hf * TS::HALF_BYTES + off, &tmap_k, 64 * hf, y, bar, pol_stream);
                    tma_load_2d(dV + hf * TS::HALF_BYTES + off, &tmap_v, 64 * hf, y, bar, pol_stream);
                }
            }
        }
        if (++pt == pnt) advance_unit();
        else f += tc;
        return true;
    };

    // ---- finishing a unit --------------------------------------------------------
    MmaState<D> ws;
    ws.reset();
    uint32_t qa[D / 16][4];
    bool began = false;
    const int g_row = lane >> 2;    // query head of this lane's fragment row
    const int c4 = lane & 3;

    // Finish this warp's share of unit (m.s, m.h).  A unit computed entirely
    // here is normalised and written.  A piece of a split unit is stored as a
    // partial of its range; the piece that completes the unit's ticket merges
    // every partial of the unit in range order (max rescaled) and writes bf16.
    auto finish_unit = [&](const StageMeta& m) {
        // full row sums: the 4 lanes of a row own disjoint columns
        float l = ws.l;
        l += __shfl_xor_sync(FULL, l, 1);
        l += __shfl_xor_sync(FULL, l, 2);
        const bool complete = began && (m.flags & F_UNIT_END);
        const size_t unit = (size_t)m.s * Hkv + m.h;
        uint16_t* out_row = a.out + ((size_t)m.s * Hq + (size_t)m.h * G + g_row) * D + 2 * c4;
        if (complete) {
            if (g_row < G) {
                const float inv = 1.0f / l;
#pragma unroll
                for (int n = 0; n < D / 8; ++n)
                    *reinterpret_cast<uint32_t*>(out_row + 8 * n) =
                        pack_bf16x2(ws.o[n][0] * inv, ws.o[n][1] * inv);
            }
            return;
        }
        const long long nt = (m.len + TILE - 1) / TILE;
        const long long au = m.f - (long long)m.t * tc;   // position of the unit's tile 0
        const long long r_lo = sc.range_of(au);
        const long long r_hi = sc.range_of(au + (nt - 1) * tc);
        // partial slot of range j: 0 if the unit began in an earlier range
        auto piece_row = [&](long long j) -> size_t {
            return ((size_t)j * 2 + ((au < sc.begin(j)) ? 0 : 1)) * G + g_row;
        };
        // Two levels when a unit has many pieces: groups of GR consecutive
        // ranges merge first (their result goes to the slot of the group's
        // first range), then the groups merge.  A warp folds at most GR + the
        // number of groups pieces one after another instead of every piece.
        constexpr int GR = 8;
        const long long P = r_hi - r_lo + 1;
        const long long NG = (P + GR - 1) / GR;
        const long long kg = (m.r - r_lo) / GR;             // this piece's group
        float M = ws.m, Z = l;                              // this piece's state (row of the lane)
        auto store_state = [&](size_t pr) {
            if (g_row < G) {
                float* po = a.part_o + pr * D + 2 * c4;
#pragma unroll
                for (int n = 0; n < D / 8; ++n)
                    st_cg(reinterpret_cast<float2*>(po + 8 * n), make_float2(ws.o[n][0], ws.o[n][1]));
                if (c4 == 0) st_cg(a.part_mz + pr, make_float2(M, Z));
            }
        };
        // head_dim 64: the next element's loads are issued before this one is
        // folded in; head_dim 128 has no registers to spare for that
        constexpr bool PREFETCH = D == 64;
        // One merge level over elements first..last (slot_of(e): the element's
        // partial row), this warp holding element `mine` in registers.  Every
        // other element already counted on the ticket: this warp is the last
        // and merges without publishing its own.  Otherwise publish, count,
        // and merge only if the count makes it the last.  The fold runs in
        // element order from the first element, so the result does not depend
        // on which warp merges:
        //   (M, Z, o) <- (M', e^{M-M'} Z + e^{m_e-M'} Z_e, e^{M-M'} o + e^{m_e-M'} o_e),
        //   M' = max(M, m_e).
        // Returns false when another warp will merge.
        // element e's partial row: range e, or (groups) the first range of group e
        auto slot_of_level = [&](long long e, bool groups) -> size_t {
            return piece_row(groups ? r_lo + e * GR : e);
        };
        auto merge_level = [&](long long first, long long last, long long mine, unsigned* ticket,
                               bool groups) -> bool {
            auto slot_of = [&](long long e) -> size_t { return slot_of_level(e, groups); };
            const unsigned others = (unsigned)(last - first);
            unsigned seen = 0;
            if (lane == 0) seen = ld_acquire(ticket);
            seen = __shfl_sync(FULL, seen, 0);
            bool stored = false;
            if (seen != others) {
                store_state(slot_of(mine));
                __threadfence();
                __syncwarp();
                unsigned prev = 0;
                if (lane == 0) prev = atomicAdd(ticket, 1u);
                prev = __shfl_sync(FULL, prev, 0);
                if (prev != others) return false;           // not the last
                __threadfence();
                stored = true;
            }
            if (lane == 0) st_cg(reinterpret_cast<int*>(ticket), 0);   // ready for the next launch
            if (G < 8 && D == 64) {
                // Fetch rounds: every lane loads, not only the lanes of the G
                // rows; lane row g_row takes element e0 + g_row / G, row
                // g_row % G, so one round trip brings 8 / G elements.  The fold
                // takes them in element order through shuffles: the same
                // arithmetic, in the same order, as the path below.  (At head_dim
                // 128 the extra registers spill and cost more than they save.)
                constexpr int S = 8 / G;
                const int k_lane = g_row / G, r_lane = g_row % G;
                if (mine != first && !stored) store_state(slot_of(mine));
                __syncwarp();
                bool acc = mine == first;                   // the state holds element `first`
                float2 v[D / 8], mz = make_float2(0.f, 0.f);
                for (long long e0 = acc ? first + 1 : first; e0 <= last; e0 += S) {
                    const long long el = e0 + k_lane;
                    if (el <= last) {
                        const size_t pr = slot_of(el) - g_row + r_lane;
                        const float* po = a.part_o + pr * D + 2 * c4;
#pragma unroll
                        for (int n = 0; n < D / 8; ++n) v[n] = ld_cg(reinterpret_cast<const float2*>(po + 8 * n));
                        mz = ld_cg(a.part_mz + pr);
                    }
#pragma unroll
                    for (int k = 0; k < S; ++k) {
                        if (e0 + k > last) break;
                        const int src = lane + 4 * G * k;       // the lane holding this row of element e0 + k
                        auto take = [&](float2 x) -> float2 {
                            return k == 0 ? x : make_float2(__shfl_sync(FULL, x.x, src), __shfl_sync(FULL, x.y, src));
                        };
                        const float2 wz = take(mz);
                        if (!acc) {
#pragma unroll
                            for (int n = 0; n < D / 8; ++n) {
                                const float2 w = take(v[n]);
                                ws.o[n][0] = w.x;
                                ws.o[n][1] = w.y;
                            }
                            M = wz.x;
                            Z = wz.y;
                            acc = true;
                            continue;
                        }
                        const float mx = fmaxf(M, wz.x);
                        const float ca = fast_exp2(M - mx), cb = fast_exp2(wz.x - mx);
                        if (g_row < G) {
                            Z = fmaf(cb, wz.y, Z * ca);
                            M = mx;
                        }
#pragma unroll
                        for (int n = 0; n < D / 8; ++n) {
                            const float2 w = take(v[n]);
                            if (g_row < G) {
                                ws.o[n][0] = fmaf(cb, w.x, ws.o[n][0] * ca);
                                ws.o[n][1] = fmaf(cb, w.y, ws.o[n][1] * ca);
                            }
                        }
                    }
                }
                return true;
            }
            if (mine != first) {                            // the fold starts from the first element
                if (!stored) store_state(slot_of(mine));
                __syncwarp();
                if (g_row < G) {
                    const size_t pr = slot_of(first);
                    const float* po = a.part_o + pr * D + 2 * c4;
#pragma unroll
                    for (int n = 0; n < D / 8; ++n) {
                        const float2 v = ld_cg(reinterpret_cast<const float2*>(po + 8 * n));
                        ws.o[n][0] = v.x;
                        ws.o[n][1] = v.y;
                    }
                    const float2 mz = ld_cg(a.part_mz + pr);
                    M = mz.x;
                    Z = mz.y;
                }
            }
            float2 v[D / 8], mz = make_float2(0.f, 0.f);
            auto fetch = [&](long long e) {
                if (g_row < G) {
                    const size_t pr = slot_of(e);
                    const float* po = a.part_o + pr * D + 2 * c4;
#pragma unroll
                    for (int n = 0; n < D / 8; ++n) v[n] = ld_cg(reinterpret_cast<const float2*>(po + 8 * n));
                    mz = ld_cg(a.part_mz + pr);
                }
            };
            if (PREFETCH && first < last) fetch(first + 1);
            for (long long e = first + 1; e <= last; ++e) {
                float2 w[D / 8], wz;
                if (PREFETCH) {
#pragma unroll
                    for (int n = 0; n < D / 8; ++n) w[n] = v[n];
                    wz = mz;
                    if (e < last) fetch(e + 1);
                } else {
                    fetch(e);
#pragma unroll
                    for (int n = 0; n < D / 8; ++n) w[n] = v[n];
                    wz = mz;
                }
                if (g_row < G) {
                    const float mx = fmaxf(M, wz.x);
                    const float ca = fast_exp2(M - mx), cb = fast_exp2(wz.x - mx);
                    Z = fmaf(cb, wz.y, Z * ca);
                    M = mx;
#pragma unroll
                    for (int n = 0; n < D / 8; ++n) {
                        ws.o[n][0] = fmaf(cb, w[n].x, ws.o[n][0] * ca);
                        ws.o[n][1] = fmaf(cb, w[n].y, ws.o[n][1] * ca);
                    }
                }
            }
            return true;
        };
        // level 1: the pieces of this piece's group (all pieces when there is
        // one group); level 2: the groups, whose results sit in the slots of
        // their first ranges.  One call site, so the merge is inlined once.
        long long first = r_lo + kg * GR;
        long long last = first + GR - 1 < r_hi ? first + GR - 1 : r_hi;
        long long mine = m.r;
        // a group is named by its first range and this unit's slot in it (a
        // range starts groups of at most two units: the one it continues and
        // the one it starts)
        unsigned* ticket = NG == 1 ? a.tickets + unit
                                   : a.group_tickets + first * 2 + ((au < sc.begin(first)) ? 0 : 1);
        bool groups = false;
        for (int level = 0;; ++level) {
            if (!merge_level(first, last, mine, ticket, groups)) return;
            if (NG == 1 || level == 1) break;
            first = 0;
            last = NG - 1;
            mine = kg;
            ticket = a.tickets + unit;
            groups = true;
        }
        if (g_row < G) {
            const float inv = 1.0f / Z;
#pragma unroll
            for (int n = 0; n < D / 8; ++n)
                *reinterpret_cast<uint32_t*>(out_row + 8 * n) =
                    pack_bf16x2(ws.o[n][0] * inv, ws.o[n][1] * inv);
        }
    };

    // ---- main loop ------------------------------------------------------------------
    // The next kernel on the stream may start launching once every warp has no
    // tile left to issue: its CTAs become resident as this grid's CTAs exit
    // and plan while the last tiles here finish; they touch no data before
    // their wait on this grid's completion.
    bool released = false;
    auto release = [&]() {
        if (!released) {
            pdl_launch_dependents();
            released = true;
        }
    };
    int issued = 0;
    bool more = have_work;
    while (issued < STAGES && more) {
        more = issue(issued);
        if (more) ++issued;
    }
    if (!more) release();
    int failed_at = -1;
    for (int i = 0; i < issued; ++i) {
        const int st = i % STAGES;
        const bool ok = mbar_wait_bounded(smem_addr(&bars[st]), (uint32_t)(i / STAGES) & 1u,
                                          s_wait_limit);
        if (__any_sync(FULL, !ok)) { failed_at = i; break; }
        const StageMeta m = meta[st];
        unsigned char* sKp = ring + (size_t)st * C::STAGE_BYTES;
        const uint32_t sK = smem_addr(sKp);
        const uint32_t sV = sK + C::KT_BYTES;
        if (fused_append && (m.flags & F_UNIT_END)) {
            // Fused append: the unit's last tile holds the new token.  Its rows
            // came with the stage; they replace the stale row the tile copy
            // brought and are stored in their slot (one 16-byte chunk a lane).
            const unsigned char* nb = newrows + (size_t)st * C::NEW_BYTES;
            if (lane < 2 * CH) {
                const int c = lane % CH;
                uint4* dst = reinterpret_cast<uint4* const*>(nb)[lane < CH ? 0 : 1];
                if (dst) {
                    const uint4 v = reinterpret_cast<const uint4*>(nb + C::NEW_HDR)[lane];   // K row, then V row
                    *reinterpret_cast<uint4*>(sKp + (lane < CH ? 0 : C::KT_BYTES) +
                                              TS::offset(m.len - 1 - m.t * TILE, c)) = v;
                    dst[c] = v;
                }
            }
            __syncwarp();
            // Copy-on-write: the tail block came from its source; with the new
            // row in place, all of its rows (this head, this layer, K and V)
            // go to the fresh block, before V rows past the length are zeroed.
            uint4* ck = reinterpret_cast<uint4* const*>(nb)[2];
            if (ck) {
                uint4* cv = reinterpret_cast<uint4* const*>(nb)[3];
                const int t0 = ((m.len - 1) / BS) * BS - m.t * TILE;   // tail block's first token in the tile
                for (int e = lane; e < 2 * BS * CH; e += 32) {
                    const int kv = e / (BS * CH);
                    const int rc = e - kv * BS * CH;
                    const int row = rc / CH, c = rc - row * CH;
                    const uint4 v = *reinterpret_cast<const uint4*>(sKp + (kv ? C::KT_BYTES : 0) +
                                                                    TS::offset(t0 + row, c));
                    (kv ? cv : ck)[row * CH + c] = v;
                }
                __syncwarp();                                 // before V rows are zeroed
            }
        }
        if (m.flags & F_FIRST) {
            load_q_frags<D, G>(qa, reinterpret_cast<const uint16_t*>(qslots + (size_t)st * C::Q_BYTES),
                               lane);
            ws.reset();
            began = (m.flags & F_UNIT_START) != 0;
        }
        const int nv = min(TILE, m.len - m.t * TILE);
        if (nv < TILE) {
            // zero the V rows past the sequence's end (0 * NaN would poison P V)
            unsigned char* vbase = sKp + C::KT_BYTES;
            for (int e = lane; e < (TILE - nv) * TS::HALVES * 8; e += 32) {
                const int row = nv + e / (TS::HALVES * 8);
                const int rest = e % (TS::HALVES * 8);
                *reinterpret_cast<uint4*>(vbase + TS::row_offset(row, rest >> 3) + ((rest & 7) << 4)) =
                    make_uint4(0, 0, 0, 0);
            }
            __syncwarp();
            mma_tile<D, BS, true>(ws, qa, sK, sV, nv, a.qscale, lane);
        } else {
            mma_tile<D, BS, false>(ws, qa, sK, sV, nv, a.qscale, lane);
        }
        if (m.flags & F_LAST) finish_unit(m);
        __syncwarp();
        if (more) {
            more = issue(st);
            if (more) ++issued;
            else release();
        }
    }
    release();                                            // (a warp that stopped early)
    if (failed_at >= 0) {
        if (lane == 0) raise_status(PKV_DEV_TIMEOUT);
        for (int i = failed_at; i < issued; ++i)
            mbar_wait_bounded(smem_addr(&bars[i % STAGES]), (uint32_t)(i / STAGES) & 1u,
                              DRAIN_LIMIT_NS);
    }
}

}  // namespace pkv
