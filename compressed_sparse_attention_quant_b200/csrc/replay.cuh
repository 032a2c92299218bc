// replay.cuh -- K9: window attention of L consecutive query tokens (SWA
// bounded replay and the window part of a Full-mode prefill).
// Page "DeepSeek V4 1-Flash 架构拆解…" (blog.zulogic.cn), section 5 "Bounded
// Replay" and page "DeepSeek V4.1 Flash 模型架構與推論優化技術規格剖析"
// (infernews.com), section 2: instead of storing the sliding-window state,
// the last 128 tokens are replayed; page neodrop.ai, architecture part 3.
// Query j of sequence b (position T - L + j) attends to the window rows
// j .. j + 127 of swa[b] (row r holds position T - (128 + L - 1) + r; rows at
// negative positions are skipped): causal attention in a band of 128.
//
// One CTA (8 warps) per tile of 8 consecutive queries of one sequence; warp w
// is query j0 + w with its 16 heads as the MMA rows. The band of the tile,
// window rows j0 .. j0 + 143 (135 used), is staged once in shared memory and
// serves every query of the tile, so a window row crosses L2 once per tile
// instead of once per query.
//   QK   bf16 mma.sync m16n8k16 straight on the staged bf16 rows and the
//        query (exact inputs, fp32 accumulate), over nine 64-channel chunks;
//        the window channels and the query of chunk c + 2 are copied
//        (cp.async) while chunk c is multiplied. The 16 x 144 scores of a
//        query stay in the warp's registers.
//   softmax  the whole band of a query is in registers: one maximum, exp2,
//        probabilities rounded to f16 (the same values feed the sum).
//   PV   the staged tile is converted in place to f16 under one power-of-two
//        exponent (so any bf16 magnitude keeps f16 precision), then f16
//        mma.sync with the probabilities as the A operand (the score
//        accumulators' layout) and ldmatrix.trans of the tile as B, one
//        64-channel output chunk at a time.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kRpQueries = 8;                          // queries per CTA (one warp each)
constexpr int kRpThreads = kRpQueries * 32;
constexpr int kRpKeys = 144;                           // band rows staged per tile (>= 128 + 8 - 1)
constexpr int kRpRowBytes = kDim * 2;                  // 1152: one bf16 / f16 row
constexpr int kRpChunks = kDim / 64;                   // 9 chunks of 64 channels
constexpr int kRpQRows = kRpQueries * kHeads;          // 128 query rows (query, head)

struct RpSmem {
    alignas(128) uint8_t win[kRpKeys * kRpRowBytes];             // 165,888: the band, 16-byte chunks swizzled
    alignas(128) uint8_t q[2][kRpQRows * 128];                   // 32,768: one 64-channel chunk of the queries
    float red[kRpQueries];
    int s_exp;
};
constexpr size_t kRpSmemBytes = sizeof(RpSmem);

struct RpParams {
    const __nv_bfloat16 *q;        // [B][L][16][576]
    const __nv_bfloat16 *swa;      // [B][128 + L - 1][576]
    const int32_t *seq_lens;       // [B]
    int L;
    float scale_log2;
    float *out;                    // [B][L][16][576]
    float *lse;                    // [B][L][16]
};

// Byte offset of 16-byte chunk c of staged row r (chunks XOR-swizzled by the
// row's low 3 bits, so the 8 rows an ldmatrix reads hit 8 bank groups).
__device__ __forceinline__ uint32_t rp_off(int r, int c, int row_bytes) {
    return static_cast<uint32_t>(r * row_bytes + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kRpThreads, 1)
swa_replay_kernel(const RpParams P) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    RpSmem &sm = *reinterpret_cast<RpSmem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tig = lane & 3;
    const int b = blockIdx.y;
    const int j0 = blockIdx.x * kRpQueries;
    const int L = P.L;
    const int n_rows = kWindow + L - 1;                    // window rows of the sequence
    int T = P.seq_lens[b];
    const bool bad_len = T < L;
    if (bad_len) {
        if (tid == 0 && blockIdx.x == 0) flag_status(kStatusBounds);
        T = -1;
    }
    const int first_pos = T - n_rows;                      // position of window row 0
    const __nv_bfloat16 *wrow0 = P.swa + (static_cast<int64_t>(b) * n_rows) * kDim;
    const __nv_bfloat16 *qrow0 = P.q + (static_cast<int64_t>(b) * L) * kHeads * kDim;

    // Copies of chunk c (64 channels): the band rows' channels into their
    // place in the tile, the queries' channels into q[c & 1].
    auto issue = [&](int c) {
        if (c < kRpChunks) {
            for (int i = tid; i < kRpKeys * 8; i += kRpThreads) {
                const int r = i >> 3, part = i & 7;
                const int row = j0 + r;
                const bool ok = row < n_rows && T >= 0 && first_pos + row >= 0;
                const void *src = ok ? static_cast<const void *>(wrow0 + static_cast<int64_t>(row) * kDim + c * 64 + part * 8)
                                     : static_cast<const void *>(P.swa);
                cp_async16(sm.win + rp_off(r, c * 8 + part, kRpRowBytes), src, ok ? 16u : 0u);
            }
            for (int i = tid; i < kRpQRows * 8; i += kRpThreads) {
                const int r = i >> 3, part = i & 7;
                const int qj = j0 + (r >> 4);
                const bool ok = qj < L;
                const void *src = ok ? static_cast<const void *>(qrow0 + (static_cast<int64_t>(qj) * kHeads + (r & 15)) * kDim +
                                                                c * 64 + part * 8)
                                     : static_cast<const void *>(P.q);
                cp_async16(sm.q[c & 1] + rp_off(r, part, 128), src, ok ? 16u : 0u);
            }
        }
        cp_async_commit();
    };

    pdl_wait();
    pdl_trigger();
    issue(0);
    issue(1);

    // ---------------- S = Q K^T over the band (bf16, exact inputs)
    float s[18][4];
#pragma unroll
    for (int nt = 0; nt < 18; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
    for (int c = 0; c < kRpChunks; ++c) {
        cp_async_wait<1>();
        __syncthreads();                                   // chunk c of the band and the queries is in
        const uint8_t *qb = sm.q[c & 1];
#pragma unroll
        for (int t = 0; t < 4; ++t) {                      // k-steps of 16 channels
            uint32_t a0, a1, a2, a3;
            ldsm_x4(a0, a1, a2, a3, qb + rp_off(warp * 16 + (lane & 15), 2 * t + (lane >> 4), 128));
#pragma unroll
            for (int nt = 0; nt < 18; nt += 2) {
                // keys of n-tiles nt, nt + 1; channels 16t .. 16t + 15 of the chunk
                uint32_t b0, b1, b2, b3;
                const int key = nt * 8 + (lane & 7) + 8 * (lane >> 4);
                ldsm_x4(b0, b1, b2, b3, sm.win + rp_off(key, c * 8 + 2 * t + ((lane >> 3) & 1), kRpRowBytes));
                mma_bf16_16816(s[nt], a0, a1, a2, a3, b0, b1);
                mma_bf16_16816(s[nt + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        __syncthreads();                                   // q[c & 1] is free again
        issue(c + 2);
    }
    cp_async_wait<0>();

    // ---------------- softmax over the band of query j = j0 + warp
    const int j = j0 + warp;
    float m[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 18; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int n = nt * 8 + 2 * tig + e;               // band row j0 + n
            const bool ok = j < L && T >= 0 && n >= warp && n <= warp + kWindow - 1 && j0 + n < n_rows &&
                            first_pos + j0 + n >= 0;
            s[nt][e] = ok ? s[nt][e] * P.scale_log2 : -INFINITY;
            s[nt][2 + e] = ok ? s[nt][2 + e] * P.scale_log2 : -INFINITY;
            m[0] = fmaxf(m[0], s[nt][e]);
            m[1] = fmaxf(m[1], s[nt][2 + e]);
        }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        m[hh] = fmaxf(m[hh], __shfl_xor_sync(0xffffffffu, m[hh], 1));
        m[hh] = fmaxf(m[hh], __shfl_xor_sync(0xffffffffu, m[hh], 2));
    }
    float l[2] = {0.0f, 0.0f};
    uint32_t pa[9][4];                                     // f16 probability fragments, k-step = 16 keys
#pragma unroll
    for (int nt = 0; nt < 18; ++nt) {
        float p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float mm = m[e >> 1];
            p[e] = (mm == -INFINITY || s[nt][e] == -INFINITY) ? 0.0f : exp2f(s[nt][e] - mm);
        }
        const __half2 h01 = __floats2half2_rn(p[0], p[1]), h23 = __floats2half2_rn(p[2], p[3]);
        const float2 r01 = __half22float2(h01), r23 = __half22float2(h23);
        l[0] += r01.x + r01.y;
        l[1] += r23.x + r23.y;
        // k-step nt / 2: n-tile 2s gives a0 (head g) / a1 (head g + 8), n-tile 2s + 1 gives a2 / a3
        pa[nt >> 1][(nt & 1) * 2 + 0] = *reinterpret_cast<const uint32_t *>(&h01);
        pa[nt >> 1][(nt & 1) * 2 + 1] = *reinterpret_cast<const uint32_t *>(&h23);
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], 1);
        l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], 2);
    }

    // ---------------- the tile in f16 under one power-of-two exponent
    __syncthreads();                                       // every warp is done reading the bf16 tile
    float mx = 0.0f;
    for (int i = tid; i < kRpKeys * kRpRowBytes / 16; i += kRpThreads) {
        const uint4 v = *reinterpret_cast<const uint4 *>(sm.win + i * 16);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
            mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(w4[q] << 16)), fabsf(__uint_as_float(w4[q] & 0xffff0000u))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) sm.red[warp] = mx;
    __syncthreads();
    if (tid == 0) {
        float t = sm.red[0];
        for (int w = 1; w < kRpQueries; ++w) t = fmaxf(t, sm.red[w]);
        int e = 0;
        if (t > 0.0f && !(t >= 0.0625f && t < 32768.0f))
            e = max(-100, min(100, static_cast<int>((__float_as_uint(t) >> 23) & 0xffu) - 127 - 10));
        sm.s_exp = e;
    }
    __syncthreads();
    const int vexp = sm.s_exp;
    const float vdown = exp2f(static_cast<float>(-vexp));
    for (int i = tid; i < kRpKeys * kRpRowBytes / 16; i += kRpThreads) {
        uint4 v = *reinterpret_cast<const uint4 *>(sm.win + i * 16);
        uint32_t *w4 = &v.x;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float lo = __uint_as_float(w4[q] << 16) * vdown, hi = __uint_as_float(w4[q] & 0xffff0000u) * vdown;
            __half2 h = __floats2half2_rn(lo, hi);
            w4[q] = *reinterpret_cast<uint32_t *>(&h);
        }
        *reinterpret_cast<uint4 *>(sm.win + i * 16) = v;
    }
    __syncthreads();

    // ---------------- O = P V, one 64-channel chunk at a time
    const float omul = exp2f(static_cast<float>(vexp));
    const float inv0 = l[0] > 0.0f ? omul / l[0] : 0.0f, inv1 = l[1] > 0.0f ? omul / l[1] : 0.0f;
    float *orow = P.out + (static_cast<int64_t>(b) * L + j) * kHeads * kDim;
    for (int c2 = 0; c2 < kRpChunks; ++c2) {
        float o[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;
#pragma unroll
        for (int ks = 0; ks < 9; ++ks) {
            const int key = ks * 16 + 8 * ((lane >> 3) & 1) + (lane & 7);
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(b0, b1, b2, b3, sm.win + rp_off(key, c2 * 8 + 2 * p + (lane >> 4), kRpRowBytes));
                mma_f16_16816(o[2 * p], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b0, b1);
                mma_f16_16816(o[2 * p + 1], pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3], b2, b3);
            }
        }
        if (j < L) {
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const int ch = c2 * 64 + n * 8 + 2 * tig;
                *reinterpret_cast<float2 *>(orow + g * kDim + ch) = make_float2(o[n][0] * inv0, o[n][1] * inv0);
                *reinterpret_cast<float2 *>(orow + (g + 8) * kDim + ch) = make_float2(o[n][2] * inv1, o[n][3] * inv1);
            }
        }
    }
    if (j < L && tig == 0) {
        float *lrow = P.lse + (static_cast<int64_t>(b) * L + j) * kHeads;
        lrow[g] = l[0] > 0.0f ? (m[0] + log2f(l[0])) * 0.69314718055994530942f : -INFINITY;
        lrow[g + 8] = l[1] > 0.0f ? (m[1] + log2f(l[1])) * 0.69314718055994530942f : -INFINITY;
    }
}

}  // namespace csa2
