// Paged decode attention: one CTA per (KV partition, kv head, sequence).
//
// What is computed ("Infra: PagedAttention", section 按 Block 分配; ithelp
// article 10405755, section PagedAttention 的核心想法): for each query head h
// of the kv head's GQA group, s_i = scale * q_h . k_i over the sequence's
// tokens, read in place through the block table, softmax over all of them,
// output sum_i p_i v_i.  A partition keeps (m_r, Z_r, unnormalised o_r);
// partitions merge with the max-rescaled rule
//     o = sum_r e^{m_r - M} o_r / sum_r e^{m_r - M} Z_r,   M = max_r m_r.
//
// B200 design (the pages' kernel advice -- fuse lookup, KV read and
// attention; neighbouring threads read neighbouring data; little merge
// synchronisation -- kept, the rest chosen for sm_100a):
//  * Each warp owns a private ring of STAGES shared-memory stages and streams
//    its own tiles (TILE tokens = one or two physical blocks) with bulk
//    copies (cp.async.bulk, no tensor map) that complete on a per-stage
//    mbarrier.  The whole (block, kv head) tile is contiguous in the pool, so
//    a tile is one or two 1-4 KiB copies for K and the same for V; only the
//    valid rows of a sequence's tail block are fetched.  Streaming data gets
//    an L2 evict-first policy.
//  * The G query heads of a kv head live in every lane's registers (8 dims
//    per lane), so each K/V byte is read from HBM once and used G times.
//    Lane layout: LG = D/8 lanes per token, 32/LG tokens per pass; q.k uses
//    packed fp32 FMAs (FFMA2) on bf16 widened by shift/mask; the G partial
//    dot products are reduce-scattered over the LG lanes so each lane ends
//    with one head's full score; p_h is gathered back with shuffles for the
//    V accumulation.
//  * Online softmax per warp in the base-2 domain (q pre-scaled by
//    scale*log2 e); warps merge in shared memory; partitions of one
//    (sequence, kv head) merge in the last CTA to finish (an atomic ticket
//    per (sequence, kv head), reset by that CTA), so no second kernel runs.
//  * Waits on staged data are bounded (about 2 s); a timeout records
//    PKV_DEV_TIMEOUT, drains this warp's copies still in flight (bounded
//    again) and finishes without trapping.  Block ids outside the pool record
//    PKV_DEV_RANGE and are not fetched.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

struct AttnArgs {
    const uint16_t* q;             // [N][Hq][D]
    const uint16_t* k_pool;        // layer base: [NB][Hkv][BS][D]
    const uint16_t* v_pool;
    uint16_t* out;                 // [N][Hq][D]
    const int32_t* block_tables;   // [N][max_blocks]
    const int32_t* seq_lens;       // [N]
    float* part_o;                 // [N*Hkv][P][G][D]   unnormalised partial outputs
    float2* part_mz;               // [N*Hkv][P][G]      (m_r, Z_r), base 2
    unsigned int* counters;        // [N*Hkv]            split-K tickets, zero at rest
    int num_kv_heads;
    int num_blocks;
    int max_blocks;
    int partition_tokens;          // multiple of the tile
    int num_partitions;            // P (workspace stride)
    float qscale;                  // scale * log2(e)
};

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // bounded wait on a stage
constexpr uint64_t DRAIN_LIMIT_NS = 500000000ull;   // bounded drain after a timeout

template <int D, int G, int BS, int NW>
struct AttnCfg {
    static constexpr int LG = D / 8;                 // lanes per token row
    static constexpr int TPP = 32 / LG;              // tokens per pass
    static constexpr int TILE = BS < 16 ? 16 : BS;   // tokens per stage
    static constexpr int BPT = TILE / BS;            // physical blocks per stage
    static constexpr int PASSES = TILE / TPP;
    static constexpr int DUP = LG / G;               // lanes holding the same head's score
    static constexpr int TILE_BYTES = TILE * D * 2;  // K (or V) bytes per stage
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    static constexpr int STAGES = (16384 / STAGE_BYTES) < 2 ? 2 : (16384 / STAGE_BYTES);
    static constexpr int RING_BYTES = NW * STAGES * STAGE_BYTES;
    static constexpr int BAR_BYTES = NW * STAGES * 8;
    static constexpr int MERGE_STRIDE = D + 2;       // per (warp, head): m, z, o[D]
    static constexpr int SMEM_BYTES = RING_BYTES + BAR_BYTES + NW * G * MERGE_STRIDE * 4;
    static_assert(G <= LG, "group larger than lanes per row");
    static_assert(TILE % TPP == 0, "tile must be whole passes");
};

// Reduce-scatter G partial sums over the LG lanes of one token: afterwards
// each lane holds the full sum of head (sub / (LG/G)).
template <int G, int LG>
__device__ __forceinline__ float reduce_scatter(float (&v)[G], int sub) {
#pragma unroll
    for (int off = LG / 2, cnt = G; off >= 1; off >>= 1) {
        if (cnt > 1) {
            const bool upper = (sub & off) != 0;
            const int half = cnt / 2;
#pragma unroll
            for (int i = 0; i < G / 2; ++i) {
                if (i < half) {
                    const float send = upper ? v[i] : v[i + half];
                    const float keep = upper ? v[i + half] : v[i];
                    v[i] = keep + __shfl_xor_sync(FULL, send, off);
                }
            }
            cnt = half;
        } else {
            v[0] += __shfl_xor_sync(FULL, v[0], off);
        }
    }
    return v[0];
}

template <int G>
__device__ __forceinline__ float pick(const float (&v)[G], int idx) {
    float r = v[0];
#pragma unroll
    for (int g = 1; g < G; ++g) r = (idx == g) ? v[g] : r;
    return r;
}

// Softmax state of one warp: running max per head (same in every lane),
// this lane's partial Z for its own head, and 8 output dims x G heads.
template <int G>
struct WarpState {
    float m[G];
    float2 acc[G][4];
    float z;
};

template <int D, int G, int BS, int NW, bool MASKED>
__device__ __forceinline__ void consume_tile(WarpState<G>& ws, const float2 (&qf)[G][4],
                                             const unsigned char* sK, const unsigned char* sV,
                                             int nv, int grp, int sub, int hsel) {
    using C = AttnCfg<D, G, BS, NW>;
    float sc[C::PASSES];
#pragma unroll
    for (int j = 0; j < C::PASSES; ++j) {
        const int t = j * C::TPP + grp;
        const uint4 kw = lds128(sK + (size_t)(t * D + sub * 8) * 2);
        const float2 k0 = bf16x2_to_float2(kw.x), k1 = bf16x2_to_float2(kw.y);
        const float2 k2 = bf16x2_to_float2(kw.z), k3 = bf16x2_to_float2(kw.w);
        float pd[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float2 a = __fmul2_rn(qf[g][0], k0);
            a = __ffma2_rn(qf[g][1], k1, a);
            a = __ffma2_rn(qf[g][2], k2, a);
            a = __ffma2_rn(qf[g][3], k3, a);
            pd[g] = a.x + a.y;
        }
        float s = reduce_scatter<G, C::LG>(pd, sub);
        if (MASKED && t >= nv) s = -INFINITY;
        sc[j] = s;
    }
    // tile max of this lane's head, then across the token groups of the warp
    float mt = sc[0];
#pragma unroll
    for (int j = 1; j < C::PASSES; ++j) mt = fmaxf(mt, sc[j]);
#pragma unroll
    for (int off = C::LG; off < 32; off <<= 1) mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, off));
    float alpha[G];
    bool changed = false;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const float mg = __shfl_sync(FULL, mt, g * C::DUP);
        const float mn = fmaxf(ws.m[g], mg);
        alpha[g] = fast_exp2(ws.m[g] - mn);
        changed |= (alpha[g] != 1.0f);
        ws.m[g] = mn;
    }
    if (changed) {   // uniform across the warp: every lane holds the same alpha[]
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float2 a2 = make_float2(alpha[g], alpha[g]);
#pragma unroll
            for (int k = 0; k < 4; ++k) ws.acc[g][k] = __fmul2_rn(ws.acc[g][k], a2);
        }
        ws.z *= pick<G>(alpha, hsel);
    }
    const float m_mine = pick<G>(ws.m, hsel);
    float p[C::PASSES];
#pragma unroll
    for (int j = 0; j < C::PASSES; ++j) {
        p[j] = fast_exp2(sc[j] - m_mine);
        ws.z += p[j];
    }
#pragma unroll
    for (int j = 0; j < C::PASSES; ++j) {
        const int t = j * C::TPP + grp;
        const uint4 vw = lds128(sV + (size_t)(t * D + sub * 8) * 2);
        float2 v0 = bf16x2_to_float2(vw.x), v1 = bf16x2_to_float2(vw.y);
        float2 v2 = bf16x2_to_float2(vw.z), v3 = bf16x2_to_float2(vw.w);
        if (MASKED && t >= nv) {
            v0 = v1 = v2 = v3 = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float pg = __shfl_sync(FULL, p[j], grp * C::LG + g * C::DUP);
            const float2 pp = make_float2(pg, pg);
            ws.acc[g][0] = __ffma2_rn(pp, v0, ws.acc[g][0]);
            ws.acc[g][1] = __ffma2_rn(pp, v1, ws.acc[g][1]);
            ws.acc[g][2] = __ffma2_rn(pp, v2, ws.acc[g][2]);
            ws.acc[g][3] = __ffma2_rn(pp, v3, ws.acc[g][3]);
        }
    }
}

template <int D, int G, int BS, int NW>
__global__ void __launch_bounds__(NW * 32)
paged_attention_kernel(const AttnArgs a) {
    using C = AttnCfg<D, G, BS, NW>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int s_last;

    const int part = blockIdx.x;
    const int kvh = blockIdx.y;
    const int seq = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int Hkv = a.num_kv_heads;
    const int PT = a.partition_tokens;
    const size_t unit = (size_t)seq * Hkv + kvh;

    int len = __ldg(a.seq_lens + seq);
    const int cap = a.max_blocks * BS;
    if (len > cap) {
        if (threadIdx.x == 0 && part == 0 && kvh == 0) raise_status(PKV_DEV_LENGTH);
        len = cap;
    }
    uint16_t* out = a.out + ((size_t)seq * Hkv * G + (size_t)kvh * G) * D;
    if (len <= 0) {   // nothing to attend to: zero output
        if (part == 0)
            for (int e = threadIdx.x; e < G * D; e += NW * 32) out[e] = 0;
        return;
    }
    const int nparts = (len + PT - 1) / PT;
    if (part >= nparts) return;
    const int t0 = part * PT;
    const int t1 = min(len, t0 + PT);
    const int ntiles = (t1 - t0 + C::TILE - 1) / C::TILE;
    const int my_n = warp < ntiles ? (ntiles - 1 - warp) / NW + 1 : 0;

    unsigned char* ring = smem + (size_t)warp * STAGES * C::STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::RING_BYTES) + warp * STAGES;
    float* mscratch = reinterpret_cast<float*>(smem + C::RING_BYTES + C::BAR_BYTES);

    const int grp = lane / C::LG;
    const int sub = lane % C::LG;
    const int hsel = sub / C::DUP;

    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < STAGES; ++st) mbar_init(smem_addr(&bars[st]), 1);
        fence_mbar_init();
    }
    __syncwarp();

    const uint64_t pol = policy_evict_first();
    const int32_t* table = a.block_tables + (size_t)seq * a.max_blocks;
    const size_t head_stride = (size_t)BS * D;                // elements of one (block, head) tile
    const size_t block_stride = (size_t)Hkv * head_stride;
    const uint16_t* kbase = a.k_pool + (size_t)kvh * head_stride;
    const uint16_t* vbase = a.v_pool + (size_t)kvh * head_stride;

    // Physical ids for a batch of this warp's tiles: lane l holds block
    // (l % BPT) of tile (batch + l / BPT).  -1 marks "past the partition".
    constexpr int TPB = 32 / C::BPT;
    int id_base = -TPB;
    int ids = -1;
    auto load_ids = [&](int base) {
        const int i = base + lane / C::BPT;
        int v = -1;
        if (i < my_n) {
            const int tok0 = t0 + (warp + i * NW) * C::TILE;
            const int lb = tok0 / BS + lane % C::BPT;
            if (lb * BS < t1) v = __ldg(table + lb);
        }
        ids = v;
        id_base = base;
    };
    // Stage my tile i (warp-uniform call).
    auto issue = [&](int i) {
        if (i >= id_base + TPB) load_ids((i / TPB) * TPB);
        const int tok0 = t0 + (warp + i * NW) * C::TILE;
        const int nv = min(C::TILE, t1 - tok0);
        int bid[C::BPT];
#pragma unroll
        for (int j = 0; j < C::BPT; ++j) bid[j] = __shfl_sync(FULL, ids, (i - id_base) * C::BPT + j);
        if (lane == 0) {
            const int st = i % STAGES;
            const uint32_t bar = smem_addr(&bars[st]);
            const uint32_t dK = smem_addr(ring + (size_t)st * C::STAGE_BYTES);
            const uint32_t dV = dK + C::TILE_BYTES;
            uint32_t bytes = 0;
            bool bad = false;
#pragma unroll
            for (int j = 0; j < C::BPT; ++j) {
                const int rows = max(0, min(BS, nv - j * BS));
                if (rows == 0) continue;
                if (bid[j] < 0 || bid[j] >= a.num_blocks) { bad = true; continue; }
                bytes += 2u * rows * D * 2;
            }
            if (bad) raise_status(PKV_DEV_RANGE);
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
            for (int j = 0; j < C::BPT; ++j) {
                const int rows = max(0, min(BS, nv - j * BS));
                if (rows == 0 || bid[j] < 0 || bid[j] >= a.num_blocks) continue;
                const uint32_t nb = (uint32_t)rows * D * 2;
                const size_t off = (size_t)bid[j] * block_stride;
                bulk_g2s(dK + j * BS * D * 2, kbase + off, nb, bar, pol);
                bulk_g2s(dV + j * BS * D * 2, vbase + off, nb, bar, pol);
            }
        }
    };

    const int npro = min(STAGES, my_n);
    for (int i = 0; i < npro; ++i) issue(i);

    // q of the G heads of this kv head, 8 dims per lane, pre-scaled
    float2 qf[G][4];
    {
        const uint16_t* qp = a.q + ((size_t)seq * Hkv * G + (size_t)kvh * G) * D + sub * 8;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const uint4 w = __ldg(reinterpret_cast<const uint4*>(qp + (size_t)g * D));
            const float2 s2 = make_float2(a.qscale, a.qscale);
            qf[g][0] = __fmul2_rn(bf16x2_to_float2(w.x), s2);
            qf[g][1] = __fmul2_rn(bf16x2_to_float2(w.y), s2);
            qf[g][2] = __fmul2_rn(bf16x2_to_float2(w.z), s2);
            qf[g][3] = __fmul2_rn(bf16x2_to_float2(w.w), s2);
        }
    }

    WarpState<G> ws;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        ws.m[g] = -INFINITY;
#pragma unroll
        for (int k = 0; k < 4; ++k) ws.acc[g][k] = make_float2(0.f, 0.f);
    }
    ws.z = 0.f;

    int failed_at = -1;
    for (int i = 0; i < my_n; ++i) {
        const int st = i % STAGES;
        const uint32_t parity = (uint32_t)(i / STAGES) & 1u;
        const bool ok = mbar_wait_bounded(smem_addr(&bars[st]), parity, WAIT_LIMIT_NS);
        if (__any_sync(FULL, !ok)) { failed_at = i; break; }
        const int tok0 = t0 + (warp + i * NW) * C::TILE;
        const int nv = min(C::TILE, t1 - tok0);
        const unsigned char* sK = ring + (size_t)st * C::STAGE_BYTES;
        const unsigned char* sV = sK + C::TILE_BYTES;
        if (nv == C::TILE)
            consume_tile<D, G, BS, NW, false>(ws, qf, sK, sV, nv, grp, sub, hsel);
        else
            consume_tile<D, G, BS, NW, true>(ws, qf, sK, sV, nv, grp, sub, hsel);
        __syncwarp();
        if (i + STAGES < my_n) issue(i + STAGES);
    }
    if (failed_at >= 0) {
        if (lane == 0) raise_status(PKV_DEV_TIMEOUT);
        // let this warp's copies still in flight land before the CTA exits
        const int last = min(failed_at + STAGES, my_n);
        for (int i = failed_at; i < last; ++i)
            mbar_wait_bounded(smem_addr(&bars[i % STAGES]), (uint32_t)(i / STAGES) & 1u,
                              DRAIN_LIMIT_NS);
    }

    // ---- warp result: sum over token groups, then to shared memory -------------
#pragma unroll
    for (int off = C::LG; off < 32; off <<= 1) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                ws.acc[g][k].x += __shfl_xor_sync(FULL, ws.acc[g][k].x, off);
                ws.acc[g][k].y += __shfl_xor_sync(FULL, ws.acc[g][k].y, off);
            }
        ws.z += __shfl_xor_sync(FULL, ws.z, off);
    }
    float* wsm = mscratch + warp * G * C::MERGE_STRIDE;
    if (grp == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float* o = wsm + g * C::MERGE_STRIDE + 2 + sub * 8;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                o[2 * k] = ws.acc[g][k].x;
                o[2 * k + 1] = ws.acc[g][k].y;
            }
        }
        if (sub % C::DUP == 0) {
            wsm[hsel * C::MERGE_STRIDE + 0] = pick<G>(ws.m, hsel);
            wsm[hsel * C::MERGE_STRIDE + 1] = ws.z;
        }
    }
    __syncthreads();

    // ---- CTA merge over warps (max-rescaled) ------------------------------------
    const size_t pbase = unit * a.num_partitions;
    for (int e = threadIdx.x; e < G * D; e += NW * 32) {
        const int g = e / D;
        const int dim = e - g * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, mscratch[(w * G + g) * C::MERGE_STRIDE]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float* r = mscratch + (w * G + g) * C::MERGE_STRIDE;
            if (r[0] == -INFINITY) continue;   // warp had no tile
            const float c = fast_exp2(r[0] - M);
            num = fmaf(c, r[2 + dim], num);
            den = fmaf(c, r[1], den);
        }
        if (nparts == 1) {
            out[(size_t)g * D + dim] = f32_to_bf16_bits(num / den);
        } else {
            a.part_o[((pbase + part) * G + g) * D + dim] = num;
            if (dim == 0) a.part_mz[(pbase + part) * G + g] = make_float2(M, den);
        }
    }
    if (nparts == 1) return;

    // ---- split-K: the last partition of this (sequence, kv head) merges --------
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(a.counters + unit, 1u);
        s_last = (prev == (unsigned)(nparts - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x == 0) a.counters[unit] = 0u;   // ready for the next launch
    for (int e = threadIdx.x; e < G * D; e += NW * 32) {
        const int g = e / D;
        const int dim = e - g * D;
        float M = -INFINITY;
        for (int r = 0; r < nparts; ++r) M = fmaxf(M, __ldcg(&a.part_mz[(pbase + r) * G + g].x));
        float num = 0.f, den = 0.f;
        for (int r = 0; r < nparts; ++r) {
            const float2 mz = __ldcg(&a.part_mz[(pbase + r) * G + g]);
            const float c = fast_exp2(mz.x - M);
            num = fmaf(c, __ldcg(&a.part_o[((pbase + r) * G + g) * D + dim]), num);
            den = fmaf(c, mz.y, den);
        }
        out[(size_t)g * D + dim] = f32_to_bf16_bits(num / den);
    }
}

}  // namespace pkv
