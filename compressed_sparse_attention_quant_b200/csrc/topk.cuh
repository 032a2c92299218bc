// topk.cuh -- K3: exact, deterministic top-k over the indexer scores.
// Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2: the "Top-K sparse addressing index"; page "DeepSeek V4 1-Flash
// 架构拆解…" (blog.zulogic.cn), section 3: Full and Reindex run the selection.
//
// Rule: the k largest scores of positions 0 .. n_valid-1, ties to the lower
// position, emitted in ascending position order, -1 padded.
//
// Method: a radix select over order-preserving 32-bit keys, levels of
// 11 + 11 + 10 bits, run by one thread-block cluster of C CTAs per query row
// (C = 1..16). CTA r of the cluster owns the position windows
// [(i*C + r)*W, +W) for rounds i = 0, 1, ... (a single round unless the row
// exceeds C * 2^17 positions).
//   level 1  the indexer already built the row's histogram of the top 11 key
//            bits: every CTA finds the bin b1 holding the k-th largest key.
//   pass A   one read of the CTA's scores (L2-resident; a single-round
//            window streams through two 64 KB shared-memory slots filled by
//            bulk copies issued ahead, the first two before level 1): keys in
//            bins above b1 are certainly selected and set bits of a
//            shared-memory bitmap over the window; keys in bin b1 are
//            candidates, counted into a histogram of their next 11 bits and
//            kept (key, position) in shared memory while they fit.
//   level 2/3 the CTAs sum their histograms through distributed shared
//            memory (every CTA reads every peer's), so each CTA picks the same
//            digit; level 3 is skipped when the level-2 bin is taken whole.
//   emit     candidates above the threshold key join the bitmap, candidates
//            equal to it go to a tie bitmap; one exchange of (selected, ties)
//            counts across the cluster gives each CTA its first tie rank and
//            output offset, ties are taken lowest position first, and each
//            thread writes the positions of its contiguous bitmap words (and,
//            when asked, their scores: the context-parallel candidates).
// If some CTA's candidates overflow its shared list, or the row needs more
// than one round, the levels and the emission re-read the scores instead of
// the list (same result, more L2 reads). Cluster barriers are the only
// waits, and every CTA of a cluster takes the same branches.
#pragma once

#include "common.cuh"
#include "indexer.cuh"

#include <cooperative_groups.h>

namespace csa2 {

constexpr int kTkThreads = 1024;
constexpr int kTkWin = 1 << 17;                  // positions per CTA window
constexpr int kTkWinWords = kTkWin / 32;
constexpr int kTkCandCap = 4096;                 // candidates kept in shared memory per CTA
constexpr int kTkMaxCluster = 16;
constexpr int kTkUnroll = 4;                     // float4 loads in flight per thread
constexpr int kTkGrp = 4 * kTkThreads * kTkUnroll; // positions of one pass-A group (64 KB of scores)

// Zeroes the per-row level-1 histograms before the indexer accumulates them.
__global__ void __launch_bounds__(256) topk_zero_kernel(uint4 *__restrict__ p, int64_t n16) {
    pdl_wait();                                         // the previous selection has read them
    pdl_trigger();
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        p[i] = make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ int topk_n_valid(const int32_t *seq_lens, int row, int Sq, int max_pages) {
    const int b = row / Sq, j = row % Sq;
    const int T = seq_lens[b];
    if (T < Sq || T > max_pages * kPage) return 0;
    return T - Sq + j + 1;
}

// Warp-level inclusive scan helper.
__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

// Exclusive block scan of one value per thread. wbuf holds >= nwarps + 1
// words. Returns the exclusive prefix; *total receives the block sum.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *wbuf, uint32_t *total) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t incl = warp_incl_scan(v);
    if (lane == 31) wbuf[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t wv = lane < NW ? wbuf[lane] : 0u;
        const uint32_t wi = warp_incl_scan(wv);
        if (lane < NW) wbuf[lane] = wi - wv;
        if (lane == NW - 1) wbuf[NW] = wi;
    }
    __syncthreads();
    const uint32_t res = wbuf[warp] + incl - v;
    *total = wbuf[NW];
    __syncthreads();
    return res;
}

// Exclusive block scan of a pair of counts packed in 64 bits (one scan for
// two quantities). wbuf holds >= nwarps + 1 entries.
template <int NT>
__device__ __forceinline__ uint64_t block_excl_scan64(uint64_t v, uint64_t *wbuf, uint64_t *total) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wbuf[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint64_t wv = lane < NW ? wbuf[lane] : 0ull;
        uint64_t wi = wv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint64_t y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < NW) wbuf[lane] = wi - wv;
        if (lane == NW - 1) wbuf[NW] = wi;
    }
    __syncthreads();
    const uint64_t res = wbuf[warp] + incl - v;
    *total = wbuf[NW];
    __syncthreads();
    return res;
}

// From the row's 2048-bin histogram (global), the bin holding the need-th
// largest key, and how many keys lie in higher bins. Every thread of the
// block gets the answer.
template <int NT>
__device__ __forceinline__ void find_threshold_bin(const uint32_t *__restrict__ gh, uint32_t need,
                                                   uint32_t *wbuf, int *s_bin, uint32_t *s_above,
                                                   int *bin_out, uint32_t *above_out) {
    constexpr int PER = kTopkBins / NT;
    const int top = kTopkBins - 1 - threadIdx.x * PER;   // this thread's bins: top, top-1, ...
    uint32_t c[PER];
    uint32_t local = 0u;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        c[i] = __ldcg(&gh[top - i]);
        local += c[i];
    }
    if (threadIdx.x == 0) {                 // stays if the counts fall short of need (corrupt input)
        *s_bin = 0;
        *s_above = 0u;
    }
    uint32_t tot;
    uint32_t run = block_excl_scan<NT>(local, wbuf, &tot);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        if (run < need && run + c[i] >= need) {
            *s_bin = top - i;
            *s_above = run;
        }
        run += c[i];
    }
    __syncthreads();
    *bin_out = *s_bin;
    *above_out = *s_above;
}

// Warp-level pick over a histogram of nbins (<= 2048, a multiple of 64) bins
// in shared or global memory: the bin holding the need-th largest element
// (bins scanned from the top) and the count in higher bins. Lane l owns the 64
// bins 2047 - 64 l - 63 .. 2047 - 64 l: their sum, a warp scan, then the one
// lane holding the crossing rescans its bins. Every lane of the warp gets the
// answer; when the counts fall short of need (corrupt input) it is (0, 0).
// Histograms read by a warp-level pick are stored with one padding word per
// 64 bins (bin b at b + b / 64), so that the 32 lanes of the pick, 64 bins
// apart, fall in 32 different banks.
__device__ __forceinline__ int hpad(int b) { return b + (b >> 6); }
constexpr int kTopkBinsPadded = kTopkBins + kTopkBins / 64;

// Warp-level pick over a histogram of nbins (<= 2048, a multiple of 64) bins:
// the bin holding the need-th largest element (bins scanned from the top) and
// the count in higher bins. Lane l owns the 64 bins 2047 - 64 l - 63 ..
// 2047 - 64 l: their sum, a warp scan, then the one lane holding the crossing
// rescans its bins. kGlobal: a plain [2048] histogram in global memory; else a
// padded one (hpad) in shared memory. Every lane of the warp gets the answer;
// when the counts fall short of need (corrupt input) it is (0, 0).
template <bool kGlobal>
__device__ __forceinline__ uint32_t pick_ld(const uint32_t *h, int b) {
    return kGlobal ? __ldcg(h + b) : h[hpad(b)];
}

template <bool kGlobal>
__device__ __forceinline__ void warp_pick(const uint32_t *h, int nbins, uint32_t need, uint32_t &bin,
                                          uint32_t &above) {
    const int lane = threadIdx.x & 31;
    const int lo = kTopkBins - 64 * (lane + 1);                // this lane's bins: lo .. lo + 63
    uint32_t local = 0u;
    if (lo < nbins) {
        if (kGlobal) {
#pragma unroll 4
            for (int i = 0; i < 16; ++i) {
                const uint4 v = __ldcg(reinterpret_cast<const uint4 *>(h + lo) + i);
                local += v.x + v.y + v.z + v.w;
            }
        } else {
#pragma unroll 8
            for (int i = 0; i < 64; ++i) local += h[hpad(lo) + i];   // one padded run of 64
        }
    }
    const uint32_t incl = warp_incl_scan(local);
    const uint32_t run0 = incl - local;                         // elements in bins above this lane's
    const bool mine = run0 < need && incl >= need;
    const uint32_t who = __ballot_sync(0xffffffffu, mine);
    uint32_t b_out = 0u, a_out = 0u;
    if (mine) {
        uint32_t run = run0;
        for (int i = 63; i >= 0; --i) {                         // from the top bin down
            const uint32_t c = pick_ld<kGlobal>(h, lo + i);
            if (run < need && run + c >= need) {
                b_out = static_cast<uint32_t>(lo + i);
                a_out = run;
            }
            run += c;
        }
    }
    const int src = who ? __ffs(who) - 1 : 0;
    bin = who ? __shfl_sync(0xffffffffu, b_out, src) : 0u;
    above = who ? __shfl_sync(0xffffffffu, a_out, src) : 0u;
}

struct TkSmem {
    alignas(128) float ring[2][kTkGrp]; // 128 KB: scores of pass-A groups, filled by bulk copies ahead
    uint64_t ring_full[2];
    uint32_t sel[kTkWinWords];          // 16 KB: selected positions of the window
    uint32_t tie[kTkWinWords];          // 16 KB: positions whose key equals the threshold
    uint32_t ckey[kTkCandCap];          // 16 KB: candidate keys (bin b1)
    int32_t cpos[kTkCandCap];           // 16 KB: candidate positions
    uint32_t hloc[2][kTopkBins];        // this CTA's level-2 / level-3 histograms (read by peers)
    uint32_t hsum[kTopkBins];           // cluster-wide sum of the current level
    uint32_t wbuf[kTkThreads / 32 + 1];
    uint64_t wbuf64[kTkThreads / 32 + 1];
    uint32_t xchg[2][2];                // per round parity: (selected before ties, ties), read by peers
    uint32_t n_cand;
    int s_bin;
    uint32_t s_above;
    uint32_t s_digit;
    uint32_t s_cum;
    uint32_t s_flag;
    uint32_t s_base[4];
};

// Digit of the need-th largest element of a histogram of nbins (<= 2048)
// bins, and the count of elements in higher bins.
__device__ __forceinline__ void tk_pick(TkSmem &sm, const uint32_t *h, int nbins, uint32_t need, uint32_t &digit,
                                        uint32_t &above) {
    const int top = kTopkBins - 1 - static_cast<int>(threadIdx.x) * 2;
    if (threadIdx.x == 0) {                 // stays if the counts fall short of need (corrupt input)
        sm.s_digit = 0u;
        sm.s_cum = 0u;
    }
    const uint32_t c0 = top < nbins ? h[top] : 0u;
    const uint32_t c1 = top - 1 < nbins ? h[top - 1] : 0u;
    uint32_t tot;
    const uint32_t run = block_excl_scan<kTkThreads>(c0 + c1, sm.wbuf, &tot);
    if (run < need && run + c0 >= need) {
        sm.s_digit = static_cast<uint32_t>(top);
        sm.s_cum = run;
    } else if (run + c0 < need && run + c0 + c1 >= need) {
        sm.s_digit = static_cast<uint32_t>(top - 1);
        sm.s_cum = run + c0;
    }
    __syncthreads();
    digit = sm.s_digit;
    above = sm.s_cum;
    __syncthreads();
}

// Guarded float4 of scores at positions p .. p+3 (< w1 only).
__device__ __forceinline__ float4 tk_load(const float *srow, int64_t p, int64_t w1, bool live) {
    if (live && p + 4 <= w1) return __ldcg(reinterpret_cast<const float4 *>(srow + p));
    float t[4] = {0.f, 0.f, 0.f, 0.f};
    if (live)
#pragma unroll
        for (int u = 0; u < 4; ++u)
            if (p + u < w1) t[u] = __ldcg(srow + p + u);
    return make_float4(t[0], t[1], t[2], t[3]);
}

// OR of a 4-bit group over the 8 lanes sharing one 32-position bitmap word.
__device__ __forceinline__ uint32_t tk_word(uint32_t nib) {
    uint32_t w = nib << ((threadIdx.x & 7) * 4);
    w |= __shfl_xor_sync(0xffffffffu, w, 1);
    w |= __shfl_xor_sync(0xffffffffu, w, 2);
    w |= __shfl_xor_sync(0xffffffffu, w, 4);
    return w;
}

__global__ void __launch_bounds__(kTkThreads, 1)
topk_cluster_kernel(const float *__restrict__ scores, int64_t t_cap, const uint32_t *__restrict__ hist,
                    const int32_t *__restrict__ seq_lens, int Sq, int max_pages, int k, int32_t *__restrict__ out,
                    float *__restrict__ out_scores) {
    namespace cg = cooperative_groups;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    TkSmem &sm = *reinterpret_cast<TkSmem *>(smem_raw);
    cg::cluster_group cluster = cg::this_cluster();
    const int C = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int row = blockIdx.x / C;
    const int tid = threadIdx.x;
    if (tid == 0) {
        mbar_init(&sm.ring_full[0], 1);
        mbar_init(&sm.ring_full[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    // The sequence lengths are an input no earlier kernel of the step writes:
    // read before the wait.
    const int n_valid = topk_n_valid(seq_lens, row, Sq, max_pages);
    pdl_wait();                                         // scores and histograms are complete
    pdl_trigger();
    int32_t *orow = out + static_cast<int64_t>(row) * k;
    float *srow_out = out_scores ? out_scores + static_cast<int64_t>(row) * k : nullptr;
    const float *srow = scores + static_cast<int64_t>(row) * t_cap;
    if (n_valid <= k) {                                 // every valid position is selected
        for (int i = rank * kTkThreads + tid; i < k; i += C * kTkThreads) {
            orow[i] = i < n_valid ? i : -1;
            if (srow_out) srow_out[i] = i < n_valid ? __ldcg(srow + i) : -INFINITY;
        }
        return;                                         // no distributed shared memory was touched
    }
    const int64_t per = (static_cast<int64_t>(n_valid) + C - 1) / C;
    const int64_t Wn = min(static_cast<int64_t>(kTkWin), (per + 31) / 32 * 32);
    const int rounds = static_cast<int>((n_valid + C * Wn - 1) / (C * Wn));
    const bool fast = rounds == 1;
    auto win = [&](int r, int64_t &w0, int64_t &w1, int &n_it) {
        w0 = (static_cast<int64_t>(r) * C + rank) * Wn;
        w1 = min(w0 + Wn, static_cast<int64_t>(n_valid));
        n_it = w1 > w0 ? static_cast<int>((w1 - w0 + 4 * kTkThreads - 1) / (4 * kTkThreads)) : 0;
    };

    // Single-round rows stream their window's scores through two 64 KB slots
    // of shared memory (one pass-A group each), filled by bulk copies (no
    // multicast) issued ahead of the reads: the first two before level 1.
    int64_t fw0 = 0, fw1 = 0;
    int fn_it = 0;
    if (fast) win(0, fw0, fw1, fn_it);
    const int n_grp = (fn_it + kTkUnroll - 1) / kTkUnroll;
    auto issue_grp = [&](int gi) {
        const int64_t p0 = fw0 + static_cast<int64_t>(gi) * kTkGrp;
        const int64_t cnt = min(static_cast<int64_t>(kTkGrp), fw1 - p0);
        const uint32_t bytes = static_cast<uint32_t>((cnt * 4 + 15) & ~static_cast<int64_t>(15));
        mbar_arrive_expect_tx(&sm.ring_full[gi & 1], bytes);
        bulk_g2s(sm.ring[gi & 1], srow + p0, bytes, &sm.ring_full[gi & 1], l2_policy_evict_first());
    };
    if (tid == 0)
        for (int gi = 0; gi < min(2, n_grp); ++gi) issue_grp(gi);

    for (int i = tid; i < 2 * kTopkBins; i += kTkThreads) (&sm.hloc[0][0])[i] = 0u;
    if (tid == 0) sm.n_cand = 0u;
    // ---- level 1: from the indexer's histogram
    int b1;
    uint32_t above1;
    find_threshold_bin<kTkThreads>(hist + static_cast<int64_t>(row) * kTopkBins, static_cast<uint32_t>(k), sm.wbuf,
                                   &sm.s_bin, &sm.s_above, &b1, &above1);
    uint32_t need = static_cast<uint32_t>(k) - above1;

    // ---- pass A: sure bits, level-2 histogram, candidate list
    // With a positive threshold bin (1024 < b1 < 2047) a score is above b1,
    // or in b1, exactly when its IEEE bits as a signed integer are at least
    // hi_bits, or in [lo_bits, hi_bits): negative scores and -0 fall below
    // both. That skips the key transform for all but the candidates.
    const bool pos = b1 > 1024 && b1 < kTopkBins - 1;
    const int32_t lo_bits = (b1 - 1024) << kTopkDigitShift;
    const int32_t hi_bits = (b1 - 1023) << kTopkDigitShift;
    for (int r = 0; r < rounds; ++r) {
        int64_t w0, w1;
        int n_it;
        win(r, w0, w1, n_it);
        for (int i0 = 0; i0 < n_it; i0 += kTkUnroll) {
            float4 f[kTkUnroll];
            const int gi = i0 / kTkUnroll;
            if (fast) {
                // positions past w1 in the slot are stale and masked below
                mbar_wait_bounded(&sm.ring_full[gi & 1], static_cast<uint32_t>((gi >> 1) & 1));
                const float4 *slot = reinterpret_cast<const float4 *>(sm.ring[gi & 1]);
#pragma unroll
                for (int u = 0; u < kTkUnroll; ++u)
                    f[u] = i0 + u < n_it ? slot[u * kTkThreads + tid] : make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
#pragma unroll
                for (int u = 0; u < kTkUnroll; ++u)
                    f[u] = tk_load(srow, w0 + static_cast<int64_t>(i0 + u) * (4 * kTkThreads) + tid * 4, w1,
                                   i0 + u < n_it);
            }
            uint32_t cmask = 0u;                         // 4 bits per unrolled load
#pragma unroll
            for (int u = 0; u < kTkUnroll; ++u) {
                const int64_t p = w0 + static_cast<int64_t>(i0 + u) * (4 * kTkThreads) + tid * 4;
                const float fv[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
                uint32_t s4 = 0u;
                // one bounds check per float4; per element only on the ragged tail
                const bool full4 = i0 + u < n_it && p + 4 <= w1;
                if (pos && full4) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int32_t bits = __float_as_int(fv[e]);
                        if (bits >= lo_bits) {
                            if (bits >= hi_bits) {
                                s4 |= 1u << e;
                            } else {
                                cmask |= 1u << (4 * u + e);
                                atomicAdd(&sm.hloc[0][(static_cast<uint32_t>(bits) >> 10) & (kTopkBins - 1)], 1u);
                            }
                        }
                    }
                } else if (pos) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int32_t bits = __float_as_int(fv[e]);
                        if (i0 + u < n_it && p + e < w1 && bits >= lo_bits) {
                            if (bits >= hi_bits) {
                                s4 |= 1u << e;
                            } else {
                                cmask |= 1u << (4 * u + e);
                                atomicAdd(&sm.hloc[0][(static_cast<uint32_t>(bits) >> 10) & (kTopkBins - 1)], 1u);
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t key = float_key(fv[e]);
                        const int bin = static_cast<int>(key >> kTopkDigitShift);
                        if (i0 + u < n_it && p + e < w1) {
                            if (bin > b1) s4 |= 1u << e;
                            if (bin == b1) {
                                cmask |= 1u << (4 * u + e);
                                atomicAdd(&sm.hloc[0][(key >> 10) & (kTopkBins - 1)], 1u);
                            }
                        }
                    }
                }
                if (fast) {
                    const uint32_t w = tk_word(s4);
                    if ((tid & 7) == 0 && i0 + u < n_it) sm.sel[(i0 + u) * (kTkThreads / 8) + (tid >> 3)] = w;
                }
            }
            if (fast && __any_sync(0xffffffffu, cmask != 0u)) {
                const uint32_t cnt = __popc(cmask);
                const uint32_t incl = warp_incl_scan(cnt);
                uint32_t base = 0u;
                if ((tid & 31) == 31) base = atomicAdd(&sm.n_cand, incl);
                base = __shfl_sync(0xffffffffu, base, 31) + incl - cnt;
                while (cmask) {
                    const int bit = __ffs(cmask) - 1;
                    cmask &= cmask - 1u;
                    const int u = bit >> 2, e = bit & 3;
                    float4 fu = f[0];
#pragma unroll
                    for (int uu = 1; uu < kTkUnroll; ++uu)
                        if (u == uu) fu = f[uu];                 // register select, no local array
                    const float v = e == 0 ? fu.x : e == 1 ? fu.y : e == 2 ? fu.z : fu.w;
                    if (base < static_cast<uint32_t>(kTkCandCap)) {
                        sm.ckey[base] = float_key(v);
                        sm.cpos[base] = static_cast<int32_t>(w0 + static_cast<int64_t>(i0 + u) * (4 * kTkThreads) +
                                                             tid * 4 + e);
                    }
                    ++base;
                }
            }
            if (fast) {
                __syncthreads();                         // every thread has read slot gi & 1
                if (tid == 0 && gi + 2 < n_grp) issue_grp(gi + 2);
            }
        }
    }
    cluster.sync();                                     // every CTA's level-2 histogram and list are complete

    // ---- level 2: cluster-wide histogram of the candidates' next 11 bits
    for (int i = tid; i < kTopkBins; i += kTkThreads) {
        uint32_t v = 0u;
        for (int q = 0; q < C; ++q) v += cluster.map_shared_rank(&sm.hloc[0][0], q)[i];
        sm.hsum[i] = v;
    }
    if (tid == 0) {
        uint32_t of = 0u;
        for (int q = 0; q < C; ++q) of |= *cluster.map_shared_rank(&sm.n_cand, q) > static_cast<uint32_t>(kTkCandCap);
        sm.s_flag = of;
    }
    __syncthreads();
    const bool use_list = fast && sm.s_flag == 0u;
    uint32_t d2, above2;
    tk_pick(sm, sm.hsum, kTopkBins, need, d2, above2);
    const uint32_t cnt2 = sm.hsum[d2];
    need -= above2;
    uint32_t prefix = (static_cast<uint32_t>(b1) << 11) | d2;
    int bits = 22;
    if (cnt2 != need) {
        // ---- level 3: the low 10 bits of the keys with this 22-bit prefix
        if (use_list) {
            const uint32_t nc = sm.n_cand;
            for (uint32_t i = tid; i < nc; i += kTkThreads) {
                const uint32_t key = sm.ckey[i];
                if ((key >> 10) == prefix) atomicAdd(&sm.hloc[1][key & 1023u], 1u);
            }
        } else {
            for (int r = 0; r < rounds; ++r) {
                int64_t w0, w1;
                int n_it;
                win(r, w0, w1, n_it);
                for (int i = 0; i < n_it; ++i) {
                    const int64_t p = w0 + static_cast<int64_t>(i) * (4 * kTkThreads) + tid * 4;
                    const float4 f = tk_load(srow, p, w1, true);
                    const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t key = float_key(fv[e]);
                        if (p + e < w1 && (key >> 10) == prefix) atomicAdd(&sm.hloc[1][key & 1023u], 1u);
                    }
                }
            }
        }
        cluster.sync();
        for (int i = tid; i < 1024; i += kTkThreads) {
            uint32_t v = 0u;
            for (int q = 0; q < C; ++q) v += cluster.map_shared_rank(&sm.hloc[1][0], q)[i];
            sm.hsum[i] = v;
        }
        __syncthreads();
        uint32_t d3, above3;
        tk_pick(sm, sm.hsum, 1024, need, d3, above3);
        need -= above3;
        prefix = (prefix << 10) | d3;
        bits = 32;
    }
    // Threshold: keys whose top `bits` bits exceed `prefix` are selected;
    // among keys equal to it, the `need` lowest positions.

    // ---- emission, one round at a time (positions ascend with the round)
    uint32_t out_base = 0u, tie_base = 0u;
    for (int r = 0; r < rounds; ++r) {
        int64_t w0, w1;
        int n_it;
        win(r, w0, w1, n_it);
        const int nw = w1 > w0 ? static_cast<int>((w1 - w0 + 31) / 32) : 0;
        __syncthreads();                                // the previous round's bitmaps are consumed
        if (use_list) {
            for (int i = tid; i < nw; i += kTkThreads) sm.tie[i] = 0u;
            __syncthreads();
            const uint32_t nc = sm.n_cand;
            for (uint32_t i = tid; i < nc; i += kTkThreads) {
                const uint32_t key = sm.ckey[i];
                const uint32_t top = bits == 32 ? key : key >> 10;
                const int64_t rel = sm.cpos[i] - w0;
                if (top > prefix) atomicOr(&sm.sel[rel >> 5], 1u << (rel & 31));
                else if (top == prefix) atomicOr(&sm.tie[rel >> 5], 1u << (rel & 31));
            }
        } else {
            for (int i = 0; i < n_it; ++i) {
                const int64_t p = w0 + static_cast<int64_t>(i) * (4 * kTkThreads) + tid * 4;
                const float4 f = tk_load(srow, p, w1, true);
                const float fv[4] = {f.x, f.y, f.z, f.w};
                uint32_t s4 = 0u, t4 = 0u;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t key = float_key(fv[e]);
                    const uint32_t top = bits == 32 ? key : key >> 10;
                    if (p + e < w1) {
                        if (top > prefix) s4 |= 1u << e;
                        else if (top == prefix) t4 |= 1u << e;
                    }
                }
                const uint32_t ws = tk_word(s4), wt = tk_word(t4);
                if ((tid & 7) == 0) {
                    sm.sel[i * (kTkThreads / 8) + (tid >> 3)] = ws;
                    sm.tie[i * (kTkThreads / 8) + (tid >> 3)] = wt;
                }
            }
        }
        __syncthreads();
        // thread t owns the contiguous words [wb, we)
        const int wper = (nw + kTkThreads - 1) / kTkThreads;
        const int wb = min(tid * wper, nw), we = min(wb + wper, nw);
        uint32_t n_tie = 0u, n_sel = 0u;
        for (int i = wb; i < we; ++i) {
            n_tie += __popc(sm.tie[i]);
            n_sel += __popc(sm.sel[i]);
        }
        uint64_t tot2;                                   // (ties, selected) in one scan
        const uint64_t off2 =
            block_excl_scan64<kTkThreads>((static_cast<uint64_t>(n_tie) << 32) | n_sel, sm.wbuf64, &tot2);
        const uint32_t tie_off = static_cast<uint32_t>(off2 >> 32), sel_off = static_cast<uint32_t>(off2);
        const uint32_t cta_ties = static_cast<uint32_t>(tot2 >> 32), cta_sel = static_cast<uint32_t>(tot2);
        if (tid == 0) {
            sm.xchg[r & 1][0] = cta_sel;
            sm.xchg[r & 1][1] = cta_ties;
        }
        cluster.sync();
        if (tid == 0) {
            // Walk the cluster in position order: ranks, each with its ties
            // taken while the global tie rank is below `need`.
            uint32_t op = out_base, tp = tie_base;
            for (int q = 0; q < C; ++q) {
                const uint32_t *x = cluster.map_shared_rank(&sm.xchg[r & 1][0], q);
                const uint32_t s = x[0], t = x[1];
                if (q == rank) {
                    sm.s_base[0] = op;
                    sm.s_base[1] = tp;
                }
                const uint32_t taken = need > tp ? min(t, need - tp) : 0u;
                op += s + taken;
                tp += t;
            }
            sm.s_base[2] = op;
            sm.s_base[3] = tp;
        }
        __syncthreads();
        uint32_t tie_rank = sm.s_base[1] + tie_off;
        // Output offset: the CTA's base, the selected positions before this
        // thread's words, and the ties before them that are taken (global tie
        // ranks below need).
        const uint32_t ties_open = need > sm.s_base[1] ? need - sm.s_base[1] : 0u;
        uint32_t pos = sm.s_base[0] + sel_off + min(tie_off, ties_open);
        for (int i = wb; i < we; ++i) {
            uint32_t m = sm.sel[i];
            uint32_t tm = sm.tie[i];
            if (tm) {
                const uint32_t c = __popc(tm);
                if (tie_rank + c <= need) {
                    m |= tm;
                } else {
                    uint32_t tr = tie_rank;
                    while (tm) {
                        const uint32_t bit = tm & (0u - tm);
                        tm ^= bit;
                        if (tr < need) m |= bit;
                        ++tr;
                    }
                }
                tie_rank += c;
                sm.sel[i] = m;
            }
        }
        for (int i = wb; i < we; ++i) {
            uint32_t m = sm.sel[i];
            while (m) {
                const int bit = __ffs(m) - 1;
                m &= m - 1u;
                if (pos < static_cast<uint32_t>(k)) {
                    const int64_t t = w0 + i * 32 + bit;
                    orow[pos] = static_cast<int32_t>(t);
                    if (srow_out) srow_out[pos] = __ldcg(srow + t);
                }
                ++pos;
            }
        }
        out_base = sm.s_base[2];
        tie_base = sm.s_base[3];
    }
    cluster.sync();                                     // no CTA leaves while a peer may read its counts
}

}  // namespace csa2
