// Warp-level pieces of the paged decode attention kernel: tensor-core
// fragments (mma.sync m16n8k16, bf16 in, fp32 accumulate), shared-memory
// tile addressing for TMA-swizzled K/V tiles, and the online-softmax update
// of one 16-token sub-tile.
//
// What one sub-tile update computes ("Infra: PagedAttention", section 按
// Block 分配): scores s_i = scale * q_h . k_i for 16 tokens and the G query
// heads h of one kv head, then the running (max m, Z = sum e^{s-m},
// unnormalised sum e^{s-m} v) is rescaled to the new max and extended.
// Scores are kept in base 2 (multiplied by scale*log2 e), so every
// exponential is exp2 of a base-2 score: the same softmax.
//
// Fragment layout.  S = Q K^T with the G query heads as the M rows of the
// 16-row MMA tile (rows G..15 are zero), the 16 tokens as N (two n8 tiles)
// and head_dim as K.  The S accumulators, exponentiated and packed to bf16,
// are exactly the A fragment of O += P V (the 16 tokens become the K of the
// second MMA), so P never leaves registers.
#pragma once

#include "pkv_device.cuh"

namespace pkv {

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // default bounded wait on a stage
constexpr uint64_t DRAIN_LIMIT_NS = 500000000ull;   // bounded drain after a timeout (fixed)
// Per-device limit of the wait on a stage (pkv_set_wait_limit_ns).
__device__ unsigned long long g_wait_limit_ns = WAIT_LIMIT_NS;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

template <int G>
__device__ __forceinline__ float pick(const float (&v)[G], int idx) {
    float r = v[0];
#pragma unroll
    for (int g = 1; g < G; ++g) r = (idx == g) ? v[g] : r;
    return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
}

// Shared-memory geometry of one staged tile of TILE tokens (32 at head_dim
// 64, 16 at head_dim 128 or with 4-token blocks; never less than one block)
// for head dimension D and block size BS.  TMA writes each physical block's rows
// with the 128-byte swizzle, 64 dims (128 bytes) per row per half; a block
// starts on a 1024-byte boundary (blocks of fewer than 8 rows are padded to
// 8), so the 16-byte chunk c of smem row r sits at chunk c ^ (r & 7).
template <int D, int BS>
struct TileSmem {
    static constexpr int TILE = BS >= 32 ? BS : ((D == 64 && BS >= 8) ? 32 : 16);   // tokens per stage
    static constexpr int BPT = TILE / BS;                // physical blocks per stage
    static constexpr int RPB = BS < 8 ? 8 : BS;          // smem rows per block
    static constexpr int TROWS = BPT * RPB;              // smem rows per tile
    static constexpr int HALVES = D / 64;                // 128-byte row halves
    static constexpr int HALF_BYTES = TROWS * 128;
    static constexpr int KT_BYTES = HALVES * HALF_BYTES; // one K (or V) tile
    static_assert(HALF_BYTES % 1024 == 0, "tiles must stay 1024-byte aligned");

    // byte offset of (token, 16-byte chunk c of the row) inside a tile
    __device__ __forceinline__ static uint32_t offset(int token, int c) {
        const int srow = (token / BS) * RPB + token % BS;
        const int half = c >> 3;
        return (uint32_t)(half * HALF_BYTES + srow * 128 + (((c & 7) ^ (srow & 7)) << 4));
    }
    // byte offset of the start of a token's row in half `half`
    __device__ __forceinline__ static uint32_t row_offset(int token, int half) {
        const int srow = (token / BS) * RPB + token % BS;
        return (uint32_t)(half * HALF_BYTES + srow * 128);
    }
};

// Per-warp softmax state for one (sequence, kv head): lane t holds row
// g = t/4 of the 16-row tile (query head g when g < G), its running max m
// (base 2), its partial Z over the columns it owns, and the O accumulator
// fragments (D/8 n8 tiles x 4 floats; entries 2,3 are the zero rows g+8).
template <int D>
struct MmaState {
    float o[D / 8][4];
    float m;
    float l;

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        m = -INFINITY;
        l = 0.f;
    }
};

// A fragments of Q (rows = query heads, K = head_dim) from the unit's q
// staged in shared memory as bf16 [G][D]; rows >= G are zero.
template <int D, int G>
__device__ __forceinline__ void load_q_frags(uint32_t (&qa)[D / 16][4], const uint16_t* sq, int lane) {
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
        uint32_t lo = 0, hi = 0;
        if (g < G) {
            lo = *reinterpret_cast<const uint32_t*>(sq + g * D + 16 * k + 2 * c);
            hi = *reinterpret_cast<const uint32_t*>(sq + g * D + 16 * k + 8 + 2 * c);
        }
        qa[k][0] = lo;
        qa[k][1] = 0u;
        qa[k][2] = hi;
        qa[k][3] = 0u;
    }
}

// One staged tile of TILE tokens (TILE/16 sub-tiles of 16 handled jointly:
// one max and one rescale per tile); tokens at or past nv are masked (their V
// rows have been zeroed by the caller).
template <int D, int BS, bool MASKED>
__device__ __forceinline__ void mma_tile(MmaState<D>& st, const uint32_t (&qa)[D / 16][4],
                                         uint32_t sK, uint32_t sV, int nv, float qscale, int lane) {
    using TS = TileSmem<D, BS>;
    constexpr int NSUB = TS::TILE / 16;
    // ---- S = Q K^T: per sub-tile two n8 tiles of tokens, D/16 k-steps ----
    float s[NSUB][2][4];
#pragma unroll
    for (int u = 0; u < NSUB; ++u)
#pragma unroll
        for (int n = 0; n < 2; ++n) s[u][n][0] = s[u][n][1] = s[u][n][2] = s[u][n][3] = 0.f;
    {
        const int tok = (lane & 7) + ((lane >> 4) << 3);
        const int csel = (lane >> 3) & 1;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
#pragma unroll
            for (int u = 0; u < NSUB; ++u) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(sK + TS::offset(16 * u + tok, 2 * k + csel), b0, b1, b2, b3);
                mma_bf16_16816(s[u][0], qa[k], b0, b1);
                mma_bf16_16816(s[u][1], qa[k], b2, b3);
            }
        }
    }
    // ---- online softmax on row g = lane/4 (columns 2c, 2c+1 of each n8 tile) ----
    const int c = lane & 3;
    float x[NSUB][4];
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < NSUB; ++u) {
        x[u][0] = s[u][0][0] * qscale;
        x[u][1] = s[u][0][1] * qscale;
        x[u][2] = s[u][1][0] * qscale;
        x[u][3] = s[u][1][1] * qscale;
        if (MASKED) {
            const int b = 16 * u + 2 * c;
            if (b >= nv) x[u][0] = -INFINITY;
            if (b + 1 >= nv) x[u][1] = -INFINITY;
            if (b + 8 >= nv) x[u][2] = -INFINITY;
            if (b + 9 >= nv) x[u][3] = -INFINITY;
        }
        mx = fmaxf(mx, fmaxf(fmaxf(x[u][0], x[u][1]), fmaxf(x[u][2], x[u][3])));
    }
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
    const float mnew = fmaxf(st.m, mx);            // finite: every tile has a valid token
    const float alpha = fast_exp2(st.m - mnew);    // 0 on a unit's first tile (m = -inf)
    st.m = mnew;
    uint32_t pa[NSUB][4];
    float psum = 0.f;
#pragma unroll
    for (int u = 0; u < NSUB; ++u) {
        const float p0 = fast_exp2(x[u][0] - mnew), p1 = fast_exp2(x[u][1] - mnew);
        const float p2 = fast_exp2(x[u][2] - mnew), p3 = fast_exp2(x[u][3] - mnew);
        psum += (p0 + p1) + (p2 + p3);
        pa[u][0] = pack_bf16x2(p0, p1);
        pa[u][1] = 0u;
        pa[u][2] = pack_bf16x2(p2, p3);
        pa[u][3] = 0u;
    }
    st.l = st.l * alpha + psum;
    if (__any_sync(FULL, alpha != 1.0f)) {
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            st.o[n][0] *= alpha;
            st.o[n][1] *= alpha;
        }
    }
    // ---- O += P V: P (row g, 16 tokens per sub-tile) is the A fragment; V^T via ldmatrix.trans ----
    {
        const int tok = (lane & 7) + (((lane >> 3) & 1) << 3);
        const int cadd = lane >> 4;
#pragma unroll
        for (int u = 0; u < NSUB; ++u) {
            if (MASKED && 16 * u >= nv) break;     // whole sub-tile past the end: P = 0
#pragma unroll
            for (int j = 0; j < D / 8; j += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(sV + TS::offset(16 * u + tok, j + cadd), b0, b1, b2, b3);
                mma_bf16_16816(st.o[j], pa[u], b0, b1);
                mma_bf16_16816(st.o[j + 1], pa[u], b2, b3);
            }
        }
    }
}

}  // namespace pkv
