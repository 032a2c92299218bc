// indexer.cuh -- K2: lightweight-indexer scores over every cached token,
// with the first top-k histogram fused into the epilogue.
// Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2 (indexer keys shared across layers, top-K addressing), and page
// "DeepSeek V4 1-Flash 架构拆解…" (blog.zulogic.cn), section 3 (the Full owner
// holds "indexer K / scale"). The pages print no score formula; the kernel
// computes the DSA-style reading
//     s_t = sum_h w_h * max(0, sigma_t * <q_h, k_t>)
// for every token t of the sequence's pages.
//
// Data path: HBM-bound streaming of 68 B per cached token. One CTA per SM;
// each warp owns a contiguous run of the flattened (sequence, page) space and
// runs its own three-slot ring: lane 0 issues bulk copies (cp.async.bulk, no
// multicast) of a whole 4 KB key page and its 256 B scale row into a slot,
// completing on that slot's mbarrier, two pages ahead of the page being
// computed (keys marked evict-first in L2, scores evict-last), so about
// 140 KB per SM are in flight without holding them in
// registers and without any cross-warp synchronisation. Page-table entries
// are resolved 32 pages at a time by one coalesced warp load, one batch
// ahead. Compute reads the page from shared memory: lane (g, tig) loads
// channels tig*16 .. tig*16+15 of token rows g and g+8 of each 16-token tile
// (the page stores 8x16-byte core matrices, so a warp's load covers 512
// contiguous bytes, free of bank conflicts). The MMA's k index
// tig*4 + j (+16) is mapped to channel tig*16 + 8*step + j (+4) for the keys
// and the query alike, which leaves the dot product unchanged. FP8 tensor-core
// MMA (m16n8k32 e4m3, fp32 accumulate); columns = query token x head. The
// epilogue applies sigma, ReLU and the head weights, stores the score and adds
// each valid score's top 11 key bits to a shared-memory histogram per query
// row (rows past the shared slots go straight to the global histogram).
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kIdxMaxRing = 4;
constexpr int kTopkBins = 2048;                 // top 11 bits of the key
constexpr int kTopkDigitShift = 21;
constexpr int kIdxSlotBytes = kKidxPageBytes + kPage * 4;

// Launch shapes: one query token per sequence -> 16 warps and 2 histogram
// rows; more query tokens -> 12 warps and 8 histogram rows; 3-slot rings.
struct IdxShape {
    int warps;
    int ring;
    int hist_rows;
};
inline IdxShape idx_shape(int Sq) { return Sq == 1 ? IdxShape{16, 3, 2} : IdxShape{12, 3, 8}; }
inline size_t idx_smem_bytes(const IdxShape &s) {
    return static_cast<size_t>(s.warps) * s.ring * (kIdxSlotBytes + 16) +
           static_cast<size_t>(s.hist_rows) * kTopkBins * 4;
}

struct IdxArgs {
    const uint8_t *q_idx;        // [B][Sq][4][64]
    const float *w;              // [B][Sq][4]
    const uint8_t *kidx;         // [pages][4096]
    const float *kidx_scale;     // [pages][64]
    int64_t num_pages;
    const int32_t *page_table;   // [B][max_pages]
    int max_pages;
    const int32_t *seq_lens;     // [B]
    int B;
    int Sq;
    float *scores;               // [B*Sq][t_cap]
    int64_t t_cap;
    uint32_t *hist;              // [B*Sq][kTopkBins], zero on entry
    int hist_rows;               // shared-memory histogram rows per CTA
    int ring;                    // ring slots per warp (<= kIdxMaxRing)
};

__device__ __forceinline__ int idx_seq_len(const int32_t *seq_lens, int b, int Sq, int max_pages) {
    const int T = seq_lens[b];
    if (T < Sq || T > max_pages * kPage) return -1;
    return T;
}

__global__ void __launch_bounds__(512, 1)
indexer_score_kernel(const IdxArgs A) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int n_warps = blockDim.x >> 5;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tig = lane & 3;
    const int Sq = A.Sq;
    const int ring = A.ring;
    // shared layout: [warps][ring] slots (keys then scales), barriers, meta, histogram
    uint8_t *slots = smem_raw;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + static_cast<size_t>(n_warps) * ring * kIdxSlotBytes);
    int2 *metas = reinterpret_cast<int2 *>(bars + n_warps * ring);
    uint32_t *hist = reinterpret_cast<uint32_t *>(metas + n_warps * ring);
    uint8_t *my_slots = slots + static_cast<size_t>(warp) * ring * kIdxSlotBytes;
    uint64_t *my_bars = bars + warp * ring;
    int2 *my_meta = metas + warp * ring;

    const int64_t n_flat = static_cast<int64_t>(A.B) * A.max_pages;
    const int64_t cta0 = n_flat * blockIdx.x / gridDim.x;
    const int64_t cta1 = n_flat * (blockIdx.x + 1) / gridDim.x;
    const int64_t f_begin = cta0 + (cta1 - cta0) * warp / n_warps;
    const int64_t f_end = cta0 + (cta1 - cta0) * (warp + 1) / n_warps;
    const int b_first = static_cast<int>(cta0 / A.max_pages);

    if (lane == 0) {
        for (int s = 0; s < ring; ++s) mbar_init(&my_bars[s], 1);
        fence_mbar_init();
    }
    for (int i = tid; i < A.hist_rows * kTopkBins; i += blockDim.x) hist[i] = 0u;
    pdl_wait();                                         // cache pages and zeroed histograms are ready
    pdl_trigger();
    __syncthreads();

    const int n_tiles = (4 * Sq + 7) / 8;
    uint4 bq[2];                 // query operand per n-tile: row n = nt*8 + g, channels tig*16 .. +15
    float wq[2][2];              // head weights of this lane's two accumulator columns
    int cur_b = -1, cur_T = 0;
    auto load_query = [&](int b) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int n = nt * 8 + g;
            const int qq = n >> 2, h = n & 3;
            bq[nt] = make_uint4(0u, 0u, 0u, 0u);
            if (nt < n_tiles && qq < Sq)
                bq[nt] = *reinterpret_cast<const uint4 *>(
                    A.q_idx + ((static_cast<int64_t>(b) * Sq + qq) * kIdxHeads + h) * kIdxDim + tig * 16);
            const int nc = nt * 8 + tig * 2;
            const int qc = nc >> 2;
            wq[nt][0] = wq[nt][1] = 0.0f;
            if (nt < n_tiles && qc < Sq) {
                const float *wp = A.w + (static_cast<int64_t>(b) * Sq + qc) * kIdxHeads + (nc & 3);
                wq[nt][0] = wp[0];
                wq[nt][1] = wp[1];
            }
        }
    };

    // Per-lane resolution of the 32 pages of batch bi: physical page (-2: no
    // page to score, -1: bad page-table entry), sequence and logical page.
    const int64_t n_batches = (f_end - f_begin + 31) / 32;
    auto resolve = [&](int64_t bi, int64_t &phys, int &pb, int &pp) {
        phys = -2;
        pb = 0;
        pp = 0;
        const int64_t f = f_begin + bi * 32 + lane;
        if (bi < n_batches && f < f_end) {
            pb = static_cast<int>(f / A.max_pages);
            pp = static_cast<int>(f - static_cast<int64_t>(pb) * A.max_pages);
            const int T = idx_seq_len(A.seq_lens, pb, Sq, A.max_pages);
            if (T < 0) {
                if (pp == 0) flag_status(kStatusBounds);
            } else if (pp * kPage < T) {
                const int64_t ph = A.page_table[static_cast<int64_t>(pb) * A.max_pages + pp];
                if (ph >= 0 && ph < A.num_pages) {
                    phys = ph;
                } else {
                    phys = -1;
                    flag_status(kStatusBounds);
                }
            }
        }
    };
    int64_t ph_c, ph_n;
    int pb_c, pp_c, pb_n, pp_n;
    resolve(0, ph_c, pb_c, pp_c);
    resolve(1, ph_n, pb_n, pp_n);
    int64_t bi_issue = 0;
    uint32_t todo = __ballot_sync(0xffffffffu, ph_c != -2);
    int issued = 0, consumed = 0;
    // Keys stream through L2 once; scores are re-read by the selection.
    const uint64_t pol_stream = l2_policy_evict_first();
    const uint64_t pol_keep = l2_policy_evict_last();

    auto try_issue = [&]() {
        while (todo == 0u && bi_issue + 1 < n_batches) {
            ++bi_issue;
            ph_c = ph_n;
            pb_c = pb_n;
            pp_c = pp_n;
            resolve(bi_issue + 1, ph_n, pb_n, pp_n);
            todo = __ballot_sync(0xffffffffu, ph_c != -2);
        }
        if (todo == 0u || issued - consumed >= ring) return;
        const int li = __ffs(todo) - 1;
        todo &= todo - 1u;
        const int64_t ph = __shfl_sync(0xffffffffu, ph_c, li);
        const int b = __shfl_sync(0xffffffffu, pb_c, li);
        const int p = __shfl_sync(0xffffffffu, pp_c, li);
        const int slot = issued % ring;
        if (lane == 0) {
            my_meta[slot] = make_int2(b, p);
            uint8_t *dst = my_slots + slot * kIdxSlotBytes;
            mbar_arrive_expect_tx(&my_bars[slot], ph >= 0 ? static_cast<uint32_t>(kIdxSlotBytes) : 0u);
            if (ph >= 0) {
                bulk_g2s(dst, A.kidx + ph * kKidxPageBytes, kKidxPageBytes, &my_bars[slot], pol_stream);
                bulk_g2s(dst + kKidxPageBytes, A.kidx_scale + ph * kPage, kPage * 4, &my_bars[slot], pol_stream);
            }
        }
        ++issued;
    };

    for (int s = 0; s < ring; ++s) try_issue();
    while (consumed < issued) {
        const int slot = consumed % ring;
        mbar_wait_bounded(&my_bars[slot], (consumed / ring) & 1);
        __syncwarp();
        const int2 meta = my_meta[slot];
        if (meta.x != cur_b) {
            cur_b = meta.x;
            cur_T = A.seq_lens[cur_b];
            load_query(cur_b);
        }
        const uint8_t *kp = my_slots + slot * kIdxSlotBytes;
        const float *sp = reinterpret_cast<const float *>(kp + kKidxPageBytes);
        const int hrow0 = (cur_b - b_first) * Sq;          // shared histogram row of query 0
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
            const uint4 r0 = *reinterpret_cast<const uint4 *>(kp + (2 * mt) * 512 + tig * 128 + g * 16);
            const uint4 r1 = *reinterpret_cast<const uint4 *>(kp + (2 * mt + 1) * 512 + tig * 128 + g * 16);
            const float s0 = sp[mt * 16 + g], s1 = sp[mt * 16 + g + 8];
            const int t_lo = meta.y * kPage + mt * 16 + g;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                if (nt < n_tiles) {
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_e4m3_16832(acc, r0.x, r1.x, r0.y, r1.y, bq[nt].x, bq[nt].y);
                    mma_e4m3_16832(acc, r0.z, r1.z, r0.w, r1.w, bq[nt].z, bq[nt].w);
                    const float part0 = wq[nt][0] * fmaxf(0.0f, s0 * acc[0]) + wq[nt][1] * fmaxf(0.0f, s0 * acc[1]);
                    const float part1 = wq[nt][0] * fmaxf(0.0f, s1 * acc[2]) + wq[nt][1] * fmaxf(0.0f, s1 * acc[3]);
                    const float oth0 = __shfl_xor_sync(0xffffffffu, part0, 1);
                    const float oth1 = __shfl_xor_sync(0xffffffffu, part1, 1);
                    const int qq = nt * 2 + (tig >> 1);
                    // even tig: token t_lo (heads 0,1 + heads 2,3); odd tig: token t_lo + 8
                    const int t = t_lo + ((tig & 1) ? 8 : 0);
                    const float score = (tig & 1) ? oth1 + part1 : part0 + oth0;
                    if (qq < Sq) {
                        st_policy(&A.scores[(static_cast<int64_t>(cur_b) * Sq + qq) * A.t_cap + t], score, pol_keep);
                        if (t <= cur_T - Sq + qq) {
                            const uint32_t bin = float_key(score) >> kTopkDigitShift;
                            const int hr = hrow0 + qq;
                            if (hr < A.hist_rows) atomicAdd(&hist[hr * kTopkBins + bin], 1u);
                            else atomicAdd(&A.hist[(static_cast<int64_t>(cur_b) * Sq + qq) * kTopkBins + bin], 1u);
                        }
                    }
                }
            }
        }
        __syncwarp();                                   // every lane is done with the slot
        ++consumed;
        try_issue();
    }

    __syncthreads();
    // Flush the shared histograms of the rows this CTA touched.
    const int b_last = static_cast<int>((cta1 > cta0 ? cta1 - 1 : cta0) / A.max_pages);
    const int n_rows = min(A.hist_rows, (b_last - b_first + 1) * Sq);
    for (int i = tid; i < n_rows * kTopkBins; i += blockDim.x) {
        const uint32_t c = hist[i];
        if (c) atomicAdd(&A.hist[static_cast<int64_t>(b_first) * Sq * kTopkBins + i], c);
    }
}

}  // namespace csa2
