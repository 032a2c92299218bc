// attn.cuh -- K4/K5: sparse attention over the selected FP4 entries plus the
// sliding window, merged by online softmax.
// Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2 (attention reads only the top-K addressed entries of the shared main
// KV) and part 3 (E2M1 + E4M3 per 16 channels); page "DeepSeek V4 1-Flash
// 架构拆解…" (blog.zulogic.cn), section 4 (a 128-token window kept per layer
// beside the global compressed state).
//
// One CTA (8 warps) per (query token, split of its key list). The key list
// is the k selected positions followed by the 128 window rows. Per tile of 64
// keys:
//   gather   4 threads per key: 16-byte loads of the 288 packed bytes and
//            2-byte loads of the group scales (or of the bf16 window row),
//            hardware E2M1x2 -> f16x2 and E4M3x2 -> f16x2 conversion, one
//            exact f16 multiply, 16-byte stores into a [64][584] f16 tile;
//   QK       warp (key group kg, channel quarter cq): 4 n-tiles x 9 k-steps of
//            m16n8k16 f16 MMA, query fragments resident in registers; the four
//            channel quarters are summed through shared memory;
//   softmax  two heads per warp, warp-shuffle max / sum in the exp2 domain,
//            probabilities rounded to f16 (the same values feed the sum);
//   PV       warp w owns 72 output channels (9 n-tiles), ldmatrix.trans of the
//            same f16 tile serves as the value operand.
// Splits write unnormalised partials (m, l, O) that K5 merges.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kAttThreads = 256;
constexpr int kAttTile = 64;
constexpr int kKhPitch = kDim + 8;          // halfs per tile row (1168 B: conflict-free ldmatrix)
constexpr int kPPitch = kAttTile + 8;       // halfs per probability row
constexpr int kRedPitch = 36;               // floats per partial-score row

struct AttSmem {
    alignas(128) __half kh[kAttTile][kKhPitch];
    alignas(16) float red[8][16][kRedPitch];
    alignas(16) __half p[16][kPPitch];
    float m_run[16];
    float l_run[16];
    float alpha[16];
    int valid[kAttTile];
};

struct AttParams {
    const __nv_bfloat16 *q;        // [R][16][576]
    const uint8_t *kv_fp4;         // [pages][64][288]
    const uint8_t *kv_scale;       // [pages][64][36]
    int64_t num_pages;
    const int32_t *page_table;     // [B][max_pages]
    int max_pages;
    const int32_t *seq_lens;       // [B]
    const int32_t *topk_idx;       // [R][k]
    int k;
    const __nv_bfloat16 *swa;      // [B][W + Sq - 1][576]
    int Sq;
    float scale_log2;              // softmax scale * log2(e)
    float *out;                    // [R][16][576]
    float *lse;                    // [R][16]
    float *part_o;                 // [R][S][16][576]
    float2 *part_ml;               // [R][S][16]
    int n_splits;
    int tiles_per_split;
};

__global__ void __launch_bounds__(kAttThreads, 2)
sparse_attn_kernel(const AttParams P) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    AttSmem &sm = *reinterpret_cast<AttSmem *>(smem_raw);
    const int row = blockIdx.y;
    const int split = blockIdx.x;
    const int b = row / P.Sq, j = row % P.Sq;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tig = lane & 3;
    const int n_rows_swa = kWindow + P.Sq - 1;

    int T = P.seq_lens[b];
    if (T < P.Sq || T > P.max_pages * kPage) {
        if (tid == 0 && split == 0) flag_status(kStatusBounds);
        T = -1;                                   // no valid key at all
    }
    const int n_slots = P.k + kWindow;
    const int n_tiles = (n_slots + kAttTile - 1) / kAttTile;
    const int tile0 = split * P.tiles_per_split;
    const int tile1 = min(tile0 + P.tiles_per_split, n_tiles);

    if (tid < 16) {
        sm.m_run[tid] = -INFINITY;
        sm.l_run[tid] = 0.0f;
    }

    // Query fragments for QK: warp (kg, cq) covers channels cq*144 .. +143.
    const int kg = warp >> 2, cq = warp & 3;
    uint32_t qa[9][4];
    {
        const __nv_bfloat16 *qrow = P.q + static_cast<int64_t>(row) * kHeads * kDim;
#pragma unroll
        for (int ks = 0; ks < 9; ++ks) {
            const int cb = cq * 144 + ks * 16 + tig * 2;
            qa[ks][0] = bf16x2_to_f16x2(*reinterpret_cast<const uint32_t *>(qrow + g * kDim + cb));
            qa[ks][1] = bf16x2_to_f16x2(*reinterpret_cast<const uint32_t *>(qrow + (g + 8) * kDim + cb));
            qa[ks][2] = bf16x2_to_f16x2(*reinterpret_cast<const uint32_t *>(qrow + g * kDim + cb + 8));
            qa[ks][3] = bf16x2_to_f16x2(*reinterpret_cast<const uint32_t *>(qrow + (g + 8) * kDim + cb + 8));
        }
    }

    float o[9][4];
#pragma unroll
    for (int nt = 0; nt < 9; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;

    for (int tile = tile0; tile < tile1; ++tile) {
        // ---------------- gather + dequantize one tile of 64 keys
        {
            const int key = tid >> 2, part = tid & 3;
            const int slot = tile * kAttTile + key;
            __half *dst = sm.kh[key];
            bool valid = false;
            if (slot < P.k && T > 0) {
                const int ti = P.topk_idx[static_cast<int64_t>(row) * P.k + slot];
                int64_t phys_slot = -1;
                if (ti >= 0) {
                    if (ti < T) {
                        const int64_t ph = P.page_table[static_cast<int64_t>(b) * P.max_pages + (ti >> 6)];
                        if (ph >= 0 && ph < P.num_pages) phys_slot = ph * kPage + (ti & 63);
                        else flag_status(kStatusBounds);
                    } else {
                        flag_status(kStatusBounds);
                    }
                }
                if (phys_slot >= 0) {
                    valid = true;
                    const uint8_t *src = P.kv_fp4 + phys_slot * kFp4Bytes;
                    const uint8_t *ssrc = P.kv_scale + phys_slot * kScaleBytes;
                    uint4 raw[5];
                    uint32_t sc[5];
#pragma unroll
                    for (int i = 0; i < 5; ++i) {
                        const int c = part + 4 * i;      // 16-byte chunk = 32 channels
                        if (c < 18) {
                            raw[i] = __ldg(reinterpret_cast<const uint4 *>(src + c * 16));
                            sc[i] = __ldg(reinterpret_cast<const unsigned short *>(ssrc + c * 2));
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 5; ++i) {
                        const int c = part + 4 * i;
                        if (c < 18) {
                            const uint32_t sf = e4m3x2_to_f16x2(sc[i]);          // (scale 2c, scale 2c+1)
                            const uint32_t s_lo = __byte_perm(sf, 0, 0x1010);     // broadcast low half
                            const uint32_t s_hi = __byte_perm(sf, 0, 0x3232);     // broadcast high half
                            const uint32_t wv[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
                            for (int q4 = 0; q4 < 4; ++q4) {
                                const uint32_t s2 = q4 < 2 ? s_lo : s_hi;
                                uint4 h;
                                h.x = hmul2_u32(e2m1x2_to_f16x2(wv[q4] & 0xffu), s2);
                                h.y = hmul2_u32(e2m1x2_to_f16x2((wv[q4] >> 8) & 0xffu), s2);
                                h.z = hmul2_u32(e2m1x2_to_f16x2((wv[q4] >> 16) & 0xffu), s2);
                                h.w = hmul2_u32(e2m1x2_to_f16x2(wv[q4] >> 24), s2);
                                *reinterpret_cast<uint4 *>(dst + c * 32 + q4 * 8) = h;
                            }
                        }
                    }
                }
            } else if (slot >= P.k && slot < n_slots && T > 0) {
                const int r = j + (slot - P.k);              // window row of this query
                if (T - n_rows_swa + r >= 0) {
                    valid = true;
                    const uint4 *src = reinterpret_cast<const uint4 *>(
                        P.swa + (static_cast<int64_t>(b) * n_rows_swa + r) * kDim);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint4 raw[9];
#pragma unroll
                        for (int i = 0; i < 9; ++i) raw[i] = __ldg(src + part + 4 * (half * 9 + i));
#pragma unroll
                        for (int i = 0; i < 9; ++i) {
                            uint4 h;
                            h.x = bf16x2_to_f16x2(raw[i].x);
                            h.y = bf16x2_to_f16x2(raw[i].y);
                            h.z = bf16x2_to_f16x2(raw[i].z);
                            h.w = bf16x2_to_f16x2(raw[i].w);
                            *reinterpret_cast<uint4 *>(dst + (part + 4 * (half * 9 + i)) * 8) = h;
                        }
                    }
                }
            }
            if (!valid) {
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                for (int c = part; c < kDim / 8; c += 4) *reinterpret_cast<uint4 *>(dst + c * 8) = z;
            }
            if (part == 0) sm.valid[key] = valid ? 1 : 0;
        }
        __syncthreads();

        // ---------------- S = Q K^T over this warp's channel quarter
        {
            float acc[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
            const int m = lane >> 3, r = lane & 7;
#pragma unroll
            for (int ks = 0; ks < 9; ++ks) {
                const int cb = cq * 144 + ks * 16;
#pragma unroll
                for (int pr = 0; pr < 2; ++pr) {
                    const int key = kg * 32 + (2 * pr + (m >> 1)) * 8 + r;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(b0, b1, b2, b3, &sm.kh[key][cb + (m & 1) * 8]);
                    mma_f16_16816(acc[2 * pr], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
                    mma_f16_16816(acc[2 * pr + 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                sm.red[warp][g][nt * 8 + tig * 2] = acc[nt][0];
                sm.red[warp][g][nt * 8 + tig * 2 + 1] = acc[nt][1];
                sm.red[warp][g + 8][nt * 8 + tig * 2] = acc[nt][2];
                sm.red[warp][g + 8][nt * 8 + tig * 2 + 1] = acc[nt][3];
            }
        }
        __syncthreads();

        // ---------------- online softmax, two heads per warp
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int h = warp * 2 + hh;
            float s[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int key = lane + 32 * u;          // key group u
                const float v = sm.red[u * 4 + 0][h][lane] + sm.red[u * 4 + 1][h][lane] +
                                sm.red[u * 4 + 2][h][lane] + sm.red[u * 4 + 3][h][lane];
                s[u] = sm.valid[key] ? v * P.scale_log2 : -INFINITY;
            }
            float mx = fmaxf(s[0], s[1]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_old = sm.m_run[h];
            const float m_new = fmaxf(m_old, mx);
            float alpha, p0, p1;
            if (m_new == -INFINITY) {
                alpha = 1.0f;
                p0 = p1 = 0.0f;
            } else {
                alpha = exp2f(m_old - m_new);
                p0 = exp2f(s[0] - m_new);
                p1 = exp2f(s[1] - m_new);
            }
            const __half h0 = __float2half_rn(p0), h1 = __float2half_rn(p1);
            sm.p[h][lane] = h0;
            sm.p[h][lane + 32] = h1;
            float sum = __half2float(h0) + __half2float(h1);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            __syncwarp();
            if (lane == 0) {
                sm.l_run[h] = sm.l_run[h] * alpha + sum;
                sm.m_run[h] = m_new;
                sm.alpha[h] = alpha;
            }
        }
        __syncthreads();

        // ---------------- O = alpha * O + P V over this warp's 72 channels
        {
            const float a_lo = sm.alpha[g], a_hi = sm.alpha[g + 8];
#pragma unroll
            for (int nt = 0; nt < 9; ++nt) {
                o[nt][0] *= a_lo;
                o[nt][1] *= a_lo;
                o[nt][2] *= a_hi;
                o[nt][3] *= a_hi;
            }
            const int m = lane >> 3, r = lane & 7;
            const int c0 = warp * 72;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(a0, a1, a2, a3, &sm.p[r + 8 * (m & 1)][kk * 16 + 8 * (m >> 1)]);
                const int key = kk * 16 + 8 * (m & 1) + r;
#pragma unroll
                for (int pr = 0; pr < 4; ++pr) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(b0, b1, b2, b3, &sm.kh[key][c0 + pr * 16 + 8 * (m >> 1)]);
                    mma_f16_16816(o[2 * pr], a0, a1, a2, a3, b0, b1);
                    mma_f16_16816(o[2 * pr + 1], a0, a1, a2, a3, b2, b3);
                }
                uint32_t b0, b1;
                ldsm_x2_t(b0, b1, &sm.kh[key][c0 + 64]);
                mma_f16_16816(o[8], a0, a1, a2, a3, b0, b1);
            }
        }
        __syncthreads();
    }

    // ---------------- epilogue: final output or split partial
    const int c0 = warp * 72;
    if (P.n_splits == 1) {
        const float l_lo = sm.l_run[g], l_hi = sm.l_run[g + 8];
        const float inv_lo = l_lo > 0.0f ? 1.0f / l_lo : 0.0f;
        const float inv_hi = l_hi > 0.0f ? 1.0f / l_hi : 0.0f;
        float *orow = P.out + static_cast<int64_t>(row) * kHeads * kDim;
#pragma unroll
        for (int nt = 0; nt < 9; ++nt) {
            const int c = c0 + nt * 8 + tig * 2;
            *reinterpret_cast<float2 *>(orow + g * kDim + c) = make_float2(o[nt][0] * inv_lo, o[nt][1] * inv_lo);
            *reinterpret_cast<float2 *>(orow + (g + 8) * kDim + c) = make_float2(o[nt][2] * inv_hi, o[nt][3] * inv_hi);
        }
        if (tid < 16) {
            const float l = sm.l_run[tid];
            P.lse[static_cast<int64_t>(row) * kHeads + tid] =
                l > 0.0f ? (sm.m_run[tid] + log2f(l)) * 0.69314718055994530942f : -INFINITY;
        }
    } else {
        const int64_t pidx = static_cast<int64_t>(row) * P.n_splits + split;
        float *po = P.part_o + pidx * kHeads * kDim;
#pragma unroll
        for (int nt = 0; nt < 9; ++nt) {
            const int c = c0 + nt * 8 + tig * 2;
            *reinterpret_cast<float2 *>(po + g * kDim + c) = make_float2(o[nt][0], o[nt][1]);
            *reinterpret_cast<float2 *>(po + (g + 8) * kDim + c) = make_float2(o[nt][2], o[nt][3]);
        }
        if (tid < 16) P.part_ml[pidx * kHeads + tid] = make_float2(sm.m_run[tid], sm.l_run[tid]);
    }
}

// K5: merge split partials: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads)
attn_merge_kernel(const float *__restrict__ part_o, const float2 *__restrict__ part_ml, int n_splits,
                  float *__restrict__ out, float *__restrict__ lse) {
    extern __shared__ float wgt[];     // [n_splits][16]
    const int row = blockIdx.x;
    const float2 *ml = part_ml + static_cast<int64_t>(row) * n_splits * kHeads;
    if (threadIdx.x < kHeads) {
        const int h = threadIdx.x;
        float M = -INFINITY;
        for (int s = 0; s < n_splits; ++s) M = fmaxf(M, ml[s * kHeads + h].x);
        float L = 0.0f;
        for (int s = 0; s < n_splits; ++s) {
            const float2 v = ml[s * kHeads + h];
            const float e = (M == -INFINITY || v.y == 0.0f) ? 0.0f : exp2f(v.x - M);
            wgt[s * kHeads + h] = e;
            L += e * v.y;
        }
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        for (int s = 0; s < n_splits; ++s) wgt[s * kHeads + h] *= inv;
        lse[static_cast<int64_t>(row) * kHeads + h] = L > 0.0f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
    }
    __syncthreads();
    const float4 *po = reinterpret_cast<const float4 *>(part_o + static_cast<int64_t>(row) * n_splits * kHeads * kDim);
    float4 *orow = reinterpret_cast<float4 *>(out + static_cast<int64_t>(row) * kHeads * kDim);
    constexpr int kVec = kHeads * kDim / 4;   // 2304 float4 per row
    for (int i = threadIdx.x; i < kVec; i += kMergeThreads) {
        const int h = (i * 4) / kDim;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < n_splits; ++s) {
            const float wv = wgt[s * kHeads + h];
            if (wv != 0.0f) {
                const float4 v = __ldcg(po + static_cast<int64_t>(s) * kVec + i);
                acc.x += wv * v.x;
                acc.y += wv * v.y;
                acc.z += wv * v.z;
                acc.w += wv * v.w;
            }
        }
        orow[i] = acc;
    }
}

}  // namespace csa2
