// indexer.cuh -- K2: lightweight-indexer scores over every cached token.
// Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2 (indexer keys shared across layers, top-K addressing), and page
// "DeepSeek V4 1-Flash 架构拆解…" (blog.zulogic.cn), section 3 (the Full owner
// holds "indexer K / scale"). The pages print no score formula; the kernel
// computes the DSA-style reading
//     s_t = sum_h w_h * max(0, sigma_t * <q_h, k_t>)
// for every token t of the sequence (tokens past a query's position are
// scored too and ignored by the selection).
//
// Data path: HBM-bound streaming of 68 B per cached token. Each CTA walks a
// contiguous run of logical pages of one sequence. One thread issues bulk
// copies (cp.async.bulk, no multicast) of whole 4 KB key pages and their
// 256 B scale rows into a 4-stage shared-memory ring completed by mbarriers;
// all eight warps consume: ldmatrix of 16-token x 32-channel E4M3 tiles (the
// page is stored in 8x16-byte core matrices, so the loads are conflict
// free), FP8 tensor-core MMA (m16n8k32 e4m3, fp32 accumulate) against the
// query operand held in registers (columns = query token x head), then the
// ReLU / sigma / head-weight epilogue and a 4-byte score store.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kIdxThreads = 256;        // 8 warps
constexpr int kIdxPagesPerStage = 2;    // warps 0-3 -> page 0, warps 4-7 -> page 1
constexpr int kIdxStages = 4;
constexpr int kIdxPagesPerCta = 32;     // 2048 tokens per CTA

struct IdxSmem {
    alignas(128) uint8_t k[kIdxStages][kIdxPagesPerStage][kKidxPageBytes];
    alignas(16) float sig[kIdxStages][kIdxPagesPerStage][kPage];
    alignas(8) uint64_t full[kIdxStages];
};

// Per-row selection state shared by the top-k passes (topk.cuh).
struct TopkRow {
    uint32_t prefix;     // resolved high bits of the k-th largest key
    int32_t bits;        // how many high bits are resolved (0..32)
    int32_t remaining;   // how many elements with key prefix == prefix are taken
    int32_t n_valid;     // scored positions 0 .. n_valid-1
    int32_t eq_count;    // elements whose key prefix == prefix
    int32_t done;        // 1 once no further radix level is needed
    int32_t pad[2];
};

constexpr int kTopkBins = 2048;

__device__ __forceinline__ int idx_row_len(const int32_t *seq_lens, int b, int Sq, int max_pages) {
    const int T = seq_lens[b];
    if (T < Sq || T > max_pages * kPage) return -1;
    return T;
}

__global__ void __launch_bounds__(kIdxThreads)
indexer_score_kernel(const uint8_t *__restrict__ q_idx, const float *__restrict__ w,
                     const uint8_t *__restrict__ kidx, const float *__restrict__ kidx_scale,
                     int64_t num_pages, const int32_t *__restrict__ page_table, int max_pages,
                     const int32_t *__restrict__ seq_lens, int Sq, int k, float *__restrict__ scores,
                     int64_t t_cap, TopkRow *__restrict__ rows, uint32_t *__restrict__ hist,
                     uint32_t *__restrict__ counters) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    IdxSmem &sm = *reinterpret_cast<IdxSmem *>(smem_raw);
    const int b = blockIdx.y;
    const int tid = threadIdx.x;
    const int T = idx_row_len(seq_lens, b, Sq, max_pages);

    // Selection state of this sequence's query rows (read by the next kernel).
    if (blockIdx.x == 0) {
        for (int j = 0; j < Sq; ++j) {
            const int row = b * Sq + j;
            for (int i = tid; i < kTopkBins; i += kIdxThreads) hist[static_cast<int64_t>(row) * kTopkBins + i] = 0u;
            if (tid == 0) {
                const int n_valid = T < 0 ? 0 : T - Sq + j + 1;
                TopkRow r;
                r.prefix = 0u;
                r.bits = 0;
                r.n_valid = n_valid;
                r.remaining = n_valid < k ? n_valid : k;
                r.eq_count = n_valid;
                r.done = n_valid <= k ? 1 : 0;
                r.pad[0] = r.pad[1] = 0;
                rows[row] = r;
                counters[row] = 0u;
                if (T < 0) flag_status(kStatusBounds);
            }
        }
    }
    if (T < 0) return;
    const int n_pages_b = (T + kPage - 1) / kPage;
    const int p0 = blockIdx.x * kIdxPagesPerCta;
    const int p1 = min(p0 + kIdxPagesPerCta, n_pages_b);
    if (p0 >= p1) return;
    const int iters = (p1 - p0 + kIdxPagesPerStage - 1) / kIdxPagesPerStage;

    if (tid == 0) {
        for (int s = 0; s < kIdxStages; ++s) mbar_init(&sm.full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto issue = [&](int it) {
        const int stage = it % kIdxStages;
        int64_t phys[kIdxPagesPerStage];
        uint32_t bytes = 0;
#pragma unroll
        for (int pp = 0; pp < kIdxPagesPerStage; ++pp) {
            const int p = p0 + it * kIdxPagesPerStage + pp;
            phys[pp] = -1;
            if (p < p1) {
                const int64_t ph = page_table[static_cast<int64_t>(b) * max_pages + p];
                if (ph >= 0 && ph < num_pages) {
                    phys[pp] = ph;
                    bytes += kKidxPageBytes + kPage * 4;
                } else {
                    flag_status(kStatusBounds);
                }
            }
        }
        mbar_arrive_expect_tx(&sm.full[stage], bytes);
#pragma unroll
        for (int pp = 0; pp < kIdxPagesPerStage; ++pp) {
            if (phys[pp] >= 0) {
                bulk_g2s(sm.k[stage][pp], kidx + phys[pp] * kKidxPageBytes, kKidxPageBytes, &sm.full[stage]);
                bulk_g2s(sm.sig[stage][pp], kidx_scale + phys[pp] * kPage, kPage * 4, &sm.full[stage]);
            }
        }
    };
    if (tid == 0) {
        for (int it = 0; it < kIdxStages && it < iters; ++it) issue(it);
    }

    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tig = lane & 3;
    const int pp = warp >> 2;        // page within the stage
    const int mt = warp & 3;         // 16-token m-tile within the page
    const int n_tiles = (4 * Sq + 7) / 8;   // query-token x head columns, 8 per MMA

    // Query operand: B[k = channel][n = query * 4 + head], two k-steps of 32.
    uint32_t bq[2][2][2];   // [n-tile][k-step][reg]
    float wq[2][2];         // head weights of this thread's two accumulator columns
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int n = nt * 8 + g;
        const int qq = n >> 2, h = n & 3;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            uint32_t r0 = 0u, r1 = 0u;
            if (nt < n_tiles && qq < Sq) {
                const uint8_t *qp = q_idx + ((static_cast<int64_t>(b) * Sq + qq) * kIdxHeads + h) * kIdxDim;
                r0 = *reinterpret_cast<const uint32_t *>(qp + 32 * s + tig * 4);
                r1 = *reinterpret_cast<const uint32_t *>(qp + 32 * s + 16 + tig * 4);
            }
            bq[nt][s][0] = r0;
            bq[nt][s][1] = r1;
        }
        const int nc = nt * 8 + tig * 2;
        const int qc = nc >> 2;
        wq[nt][0] = wq[nt][1] = 0.0f;
        if (nt < n_tiles && qc < Sq) {
            const float *wp = w + (static_cast<int64_t>(b) * Sq + qc) * kIdxHeads + (nc & 3);
            wq[nt][0] = wp[0];
            wq[nt][1] = wp[1];
        }
    }

    for (int it = 0; it < iters; ++it) {
        const int stage = it % kIdxStages;
        mbar_wait_bounded(&sm.full[stage], (it / kIdxStages) & 1);
        const int p = p0 + it * kIdxPagesPerStage + pp;
        if (p < p1) {
            const uint8_t *base = sm.k[stage][pp];
            uint32_t a[2][4];
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const int m = lane >> 3, r = lane & 7;
                const int tg = 2 * mt + (m & 1);          // 8-token core-matrix group
                const int chunk = 2 * s + (m >> 1);       // 16-channel chunk
                ldsm_x4(a[s][0], a[s][1], a[s][2], a[s][3], base + tg * 512 + chunk * 128 + r * 16);
            }
            const float sig0 = sm.sig[stage][pp][mt * 16 + g];
            const float sig1 = sm.sig[stage][pp][mt * 16 + g + 8];
            const int64_t t0 = static_cast<int64_t>(p) * kPage + mt * 16 + g;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                if (nt < n_tiles) {
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_e4m3_16832(acc, a[0][0], a[0][1], a[0][2], a[0][3], bq[nt][0][0], bq[nt][0][1]);
                    mma_e4m3_16832(acc, a[1][0], a[1][1], a[1][2], a[1][3], bq[nt][1][0], bq[nt][1][1]);
                    // columns tig*2, tig*2+1 = two heads of one query token
                    const float part0 = wq[nt][0] * fmaxf(0.0f, sig0 * acc[0]) + wq[nt][1] * fmaxf(0.0f, sig0 * acc[1]);
                    const float part1 = wq[nt][0] * fmaxf(0.0f, sig1 * acc[2]) + wq[nt][1] * fmaxf(0.0f, sig1 * acc[3]);
                    const float oth0 = __shfl_xor_sync(0xffffffffu, part0, 1);
                    const float oth1 = __shfl_xor_sync(0xffffffffu, part1, 1);
                    const int qq = nt * 2 + (tig >> 1);
                    if (qq < Sq) {
                        float *srow = scores + (static_cast<int64_t>(b) * Sq + qq) * t_cap;
                        // heads 0,1 (even tig) + heads 2,3 (odd tig)
                        if ((tig & 1) == 0) srow[t0] = part0 + oth0;
                        else srow[t0 + 8] = oth1 + part1;
                    }
                }
            }
        }
        __syncthreads();   // every warp is done with this stage
        if (tid == 0 && it + kIdxStages < iters) issue(it + kIdxStages);
    }
}

}  // namespace csa2
