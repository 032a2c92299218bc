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
// exceeds C * 2^17 positions); inside a window each thread owns a contiguous
// run of positions and the bitmap words over them.
//   level 1  the indexer already built the row's histogram of the top 11 key
//            bits: every CTA finds the bin b1 holding the k-th largest key.
//   pass A   one read of the CTA's scores (L2-resident): keys in bins above
//            b1 are certainly selected and set bits of a shared-memory
//            bitmap over the window; keys in bin b1 are candidates, counted
//            into a histogram of their next 11 bits and marked in a second
//            bitmap (both bitmaps assembled from 4-bit pieces by shuffles).
//   level 2/3 the CTAs sum their histograms through distributed shared
//            memory (every CTA reads every peer's), so each CTA picks the same
//            digit; level 3 is skipped when the level-2 bin is taken whole.
//   emit     candidates above the threshold key join the bitmap, candidates
//            equal to it go to a tie bitmap (level 3 and the emission re-read
//            only the candidates' scores, each thread over its own bitmap
//            words); one exchange of (selected, ties)
//            counts across the cluster gives each CTA its first tie rank and
//            output offset, ties are taken lowest position first, and each
//            thread writes the positions of its contiguous bitmap words.
// If the row needs more than one round of windows, the levels and the
// emission re-read all the scores instead of the candidate bitmap (same
// result, more L2 reads). Cluster barriers are the only waits, and every
// CTA of a cluster takes the same branches.
#pragma once

#include "common.cuh"
#include "indexer.cuh"

#include <cooperative_groups.h>

namespace csa2 {

constexpr int kTkThreads = 1024;
constexpr int kTkWin = 1 << 17;                  // positions per CTA window
constexpr int kTkWinWords = kTkWin / 32;
constexpr int kTkMaxCluster = 16;

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
    uint32_t sel[kTkWinWords];          // 16 KB: selected positions of the window
    uint32_t tie[kTkWinWords];          // 16 KB: positions whose key equals the threshold
    uint32_t cand[kTkWinWords];         // 16 KB: positions whose key is in the level-1 bin b1
    uint32_t hloc[2][kTopkBins];        // this CTA's level-2 / level-3 histograms (read by peers)
    uint32_t hsum[kTopkBinsPadded];     // cluster-wide sum of the current level (padded, hpad)
    uint32_t wsel[kTkThreads / 32];     // per-warp counts of the emission
    uint32_t wtie[kTkThreads / 32];
    uint32_t xchg[2][2];                // per round parity: (selected before ties, ties), read by peers
    uint32_t s_pick[2];                 // (bin / digit, count above) of the current level
};

// Guarded float4 of scores at positions p .. p+3 (< w1 only).
__device__ __forceinline__ float4 tk_load(const float *srow, int64_t p, int64_t w1) {
    if (p + 4 <= w1) return __ldcg(reinterpret_cast<const float4 *>(srow + p));
    float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < 4; ++u)
        if (p + u < w1) t[u] = __ldcg(srow + p + u);
    return make_float4(t[0], t[1], t[2], t[3]);
}

// Work layout: in each round the CTA's window of Wn positions is split into
// contiguous runs of P = Wn / 1024 positions (a multiple of 32), one per
// thread, so a thread's bitmap words hold only its own positions and need no
// exchange between lanes. Warp-level scans replace block-wide ones: every
// level and the emission take one CTA barrier plus, for the cluster-wide
// counts, one cluster barrier.
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
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();                                         // scores and histograms are complete
    pdl_trigger();
    const int n_valid = topk_n_valid(seq_lens, row, Sq, max_pages);
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
    const int NW = static_cast<int>((Wn / 32 + kTkThreads - 1) / kTkThreads);   // bitmap words per thread: 1 .. 4
    const int P = 32 * NW;                              // positions per thread (threads past Wn have none)
    const int rounds = static_cast<int>((n_valid + C * Wn - 1) / (C * Wn));
    const bool fast = rounds == 1;
    auto win = [&](int r, int64_t &w0, int64_t &w1) {
        w0 = (static_cast<int64_t>(r) * C + rank) * Wn;
        w1 = min(w0 + Wn, static_cast<int64_t>(n_valid));
    };

    for (int i = tid; i < 2 * kTopkBins; i += kTkThreads) (&sm.hloc[0][0])[i] = 0u;
    // ---- level 1: one warp scans the indexer's histogram of the row
    if (warp == 0) {
        uint32_t b1w, a1w;
        warp_pick<true>(hist + static_cast<int64_t>(row) * kTopkBins, kTopkBins, static_cast<uint32_t>(k), b1w, a1w);
        if (lane == 0) {
            sm.s_pick[0] = b1w;
            sm.s_pick[1] = a1w;
        }
    }
    __syncthreads();
    const int b1 = static_cast<int>(sm.s_pick[0]);
    uint32_t need = static_cast<uint32_t>(k) - sm.s_pick[1];

    // ---- pass A: sure bits, level-2 histogram, candidate list
    // With a positive threshold bin (1024 < b1 < 2047) a score is above b1,
    // or in b1, exactly when its IEEE bits as a signed integer are at least
    // hi_bits, or in [lo_bits, hi_bits): negative scores and -0 fall below
    // both. Otherwise the order-preserving key decides.
    const bool pos = b1 > 1024 && b1 < kTopkBins - 1;
    const int32_t lo_bits = (b1 - 1024) << kTopkDigitShift;
    const int32_t hi_bits = (b1 - 1023) << kTopkDigitShift;
    auto classify = [&](float f, int64_t p, int64_t w1, bool &sure, bool &cand, uint32_t &key) {
        key = float_key(f);
        if (p >= w1) {
            sure = cand = false;
        } else if (pos) {
            const int32_t bits = __float_as_int(f);
            sure = bits >= hi_bits;
            cand = !sure && bits >= lo_bits;
        } else {
            const int bin = static_cast<int>(key >> kTopkDigitShift);
            sure = bin > b1;
            cand = bin == b1;
        }
    };
    // Loads are coalesced: lane L of warp w reads positions wb + 128 j + 4 L
    // .. + 3 (wb = the warp's first position); the eight lanes 8q .. 8q + 7
    // of iteration j cover one 32-position bitmap word, which three
    // shuffles assemble from their 4-bit pieces. The words are the same ones
    // the owning threads read later.
    for (int r = 0; r < rounds; ++r) {
        int64_t w0, w1;
        win(r, w0, w1);
        const int64_t wb = w0 + static_cast<int64_t>(warp) * 32 * P;
        const int n_it = P / 4;                          // 8 * NW iterations of 128 positions
        for (int j0 = 0; j0 < n_it; j0 += 4) {
            float4 f[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) f[u] = tk_load(srow, wb + 128 * (j0 + u) + 4 * lane, w1);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t p = wb + 128 * (j0 + u) + 4 * lane;
                const float fv[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
                uint32_t sn = 0u, cn = 0u;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    bool su, ca;
                    uint32_t key;
                    classify(fv[e], p + e, w1, su, ca, key);
                    sn |= (su ? 1u : 0u) << e;
                    if (ca) {
                        cn |= 1u << e;
                        atomicAdd(&sm.hloc[0][(key >> 10) & (kTopkBins - 1)], 1u);
                    }
                }
                if (fast) {
                    uint32_t sw = sn << (4 * (lane & 7));
                    sw |= __shfl_xor_sync(0xffffffffu, sw, 1);
                    sw |= __shfl_xor_sync(0xffffffffu, sw, 2);
                    sw |= __shfl_xor_sync(0xffffffffu, sw, 4);
                    if ((lane & 7) == 0) sm.sel[(p - w0) >> 5] = sw;
                }
                if (fast) {                                  // candidate word (bin b1), same assembly
                    uint32_t cw = cn << (4 * (lane & 7));
                    cw |= __shfl_xor_sync(0xffffffffu, cw, 1);
                    cw |= __shfl_xor_sync(0xffffffffu, cw, 2);
                    cw |= __shfl_xor_sync(0xffffffffu, cw, 4);
                    if ((lane & 7) == 0) sm.cand[(p - w0) >> 5] = cw;
                }
            }
        }
    }
    cluster.sync();                                     // every CTA's level-2 histogram and list are complete

    // ---- level 2: cluster-wide histogram of the candidates' next 11 bits
    for (int i = tid; i < kTopkBins; i += kTkThreads) {
        uint32_t v = 0u;
        for (int q = 0; q < C; ++q) v += cluster.map_shared_rank(&sm.hloc[0][0], q)[i];
        sm.hsum[hpad(i)] = v;
    }
    __syncthreads();
    const bool use_list = fast;                         // the candidate words of a single-round window
    if (warp == 0) {
        uint32_t d, a;
        warp_pick<false>(sm.hsum, kTopkBins, need, d, a);
        if (lane == 0) {
            sm.s_pick[0] = d;
            sm.s_pick[1] = a;
        }
    }
    __syncthreads();
    const uint32_t d2 = sm.s_pick[0], above2 = sm.s_pick[1];
    const uint32_t cnt2 = sm.hsum[hpad(static_cast<int>(d2))];
    need -= above2;
    uint32_t prefix = (static_cast<uint32_t>(b1) << 11) | d2;
    int bits = 22;
    if (cnt2 != need) {
        // ---- level 3: the low 10 bits of the keys with this 22-bit prefix
        if (use_list) {
            int64_t w0, w1;
            win(0, w0, w1);
            const int64_t t0 = w0 + static_cast<int64_t>(tid) * P;
            for (int wi = 0; wi < NW; ++wi) {
                uint32_t m = sm.cand[tid * NW + wi];
                while (m) {                                  // four candidates' loads in flight at a time
                    int bit[4];
                    float f[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        bit[u] = m ? __ffs(m) - 1 : -1;
                        m &= m - 1u;
                        f[u] = bit[u] >= 0 ? __ldcg(srow + t0 + 32 * wi + bit[u]) : 0.0f;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t key = float_key(f[u]);
                        if (bit[u] >= 0 && (key >> 10) == prefix) atomicAdd(&sm.hloc[1][key & 1023u], 1u);
                    }
                }
            }
        } else {
            for (int r = 0; r < rounds; ++r) {
                int64_t w0, w1;
                win(r, w0, w1);
                const int64_t t0 = w0 + static_cast<int64_t>(tid) * P;
                for (int i = 0; i < P; i += 4) {
                    const float4 f = tk_load(srow, t0 + i, w1);
                    const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t key = float_key(fv[e]);
                        if (t0 + i + e < w1 && (key >> 10) == prefix) atomicAdd(&sm.hloc[1][key & 1023u], 1u);
                    }
                }
            }
        }
        cluster.sync();
        for (int i = tid; i < 1024; i += kTkThreads) {
            uint32_t v = 0u;
            for (int q = 0; q < C; ++q) v += cluster.map_shared_rank(&sm.hloc[1][0], q)[i];
            sm.hsum[hpad(i)] = v;
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t d, a;
            warp_pick<false>(sm.hsum, 1024, need, d, a);
            if (lane == 0) {
                sm.s_pick[0] = d;
                sm.s_pick[1] = a;
            }
        }
        __syncthreads();
        const uint32_t d3 = sm.s_pick[0], above3 = sm.s_pick[1];
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
        win(r, w0, w1);
        const int64_t t0 = w0 + static_cast<int64_t>(tid) * P;
        if (use_list) {
            // this thread's candidate words: above the threshold -> selected, equal -> tie
            for (int wi = 0; wi < NW; ++wi) {
                uint32_t m = sm.cand[tid * NW + wi], s4 = 0u, t4 = 0u;
                while (m) {                                  // four candidates' loads in flight at a time
                    int bit[4];
                    float f[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        bit[u] = m ? __ffs(m) - 1 : -1;
                        m &= m - 1u;
                        f[u] = bit[u] >= 0 ? __ldcg(srow + t0 + 32 * wi + bit[u]) : 0.0f;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        if (bit[u] < 0) continue;
                        const uint32_t key = float_key(f[u]);
                        const uint32_t top = bits == 32 ? key : key >> 10;
                        if (top > prefix) s4 |= 1u << bit[u];
                        else if (top == prefix) t4 |= 1u << bit[u];
                    }
                }
                sm.sel[tid * NW + wi] |= s4;
                sm.tie[tid * NW + wi] = t4;
            }
        } else {
            for (int wi = 0; wi < NW; ++wi) {
                uint32_t s4 = 0u, t4 = 0u;
                for (int i = 0; i < 32; i += 4) {
                    const int64_t p = t0 + 32 * wi + i;
                    const float4 f = tk_load(srow, p, w1);
                    const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint32_t key = float_key(fv[e]);
                        const uint32_t top = bits == 32 ? key : key >> 10;
                        if (p + e < w1) {
                            if (top > prefix) s4 |= 1u << (i + e);
                            else if (top == prefix) t4 |= 1u << (i + e);
                        }
                    }
                }
                sm.sel[tid * NW + wi] = s4;
                sm.tie[tid * NW + wi] = t4;
            }
        }
        __syncthreads();
        // counts of this thread's words, then of its warp (warp-level scans)
        uint32_t n_sel = 0u, n_tie = 0u;
        for (int wi = 0; wi < NW; ++wi) {
            n_sel += __popc(sm.sel[tid * NW + wi]);
            n_tie += __popc(sm.tie[tid * NW + wi]);
        }
        const uint32_t is_ = warp_incl_scan(n_sel), it_ = warp_incl_scan(n_tie);
        if (lane == 31) {
            sm.wsel[warp] = is_;
            sm.wtie[warp] = it_;
        }
        __syncthreads();
        uint32_t cta_sel = 0u, cta_tie = 0u, wsel_before = 0u, wtie_before = 0u;
        for (int w = 0; w < kTkThreads / 32; ++w) {
            const uint32_t a = sm.wsel[w], t = sm.wtie[w];
            if (w < warp) {
                wsel_before += a;
                wtie_before += t;
            }
            cta_sel += a;
            cta_tie += t;
        }
        if (tid == 0) {
            sm.xchg[r & 1][0] = cta_sel;
            sm.xchg[r & 1][1] = cta_tie;
        }
        cluster.sync();
        // Walk the cluster in position order: ranks, each with its ties
        // taken while the global tie rank is below `need` (every thread
        // computes the same bases).
        uint32_t op = out_base, tp = tie_base, my_op = 0u, my_tp = 0u;
        for (int q = 0; q < C; ++q) {
            const uint32_t *x = cluster.map_shared_rank(&sm.xchg[r & 1][0], q);
            const uint32_t sq = x[0], tq = x[1];
            if (q == rank) {
                my_op = op;
                my_tp = tp;
            }
            const uint32_t taken = need > tp ? min(tq, need - tp) : 0u;
            op += sq + taken;
            tp += tq;
        }
        uint32_t tie_rank = my_tp + wtie_before + it_ - n_tie;
        // this thread's outputs: its selected positions plus its kept ties
        uint32_t kept = 0u;
        {
            uint32_t tr = tie_rank;
            for (int wi = 0; wi < NW; ++wi) {
                uint32_t tm = sm.tie[tid * NW + wi];
                const uint32_t c = __popc(tm);
                if (tr + c <= need) {
                    kept += c;
                } else {
                    while (tm) {
                        const uint32_t bit = tm & (0u - tm);
                        tm ^= bit;
                        if (tr < need) ++kept;
                        ++tr;
                    }
                    tr -= c;
                }
                tr += c;
            }
        }
        // output offset: selected and kept ties before this thread, in position order
        const uint32_t mine = n_sel + kept;
        const uint32_t incl = warp_incl_scan(mine);
        __syncthreads();                                // the warp totals of the counts above are read
        if (lane == 31) sm.wsel[warp] = incl;
        __syncthreads();
        uint32_t wout_before = 0u;
        for (int w = 0; w < warp; ++w) wout_before += sm.wsel[w];
        uint32_t pos_out = my_op + wout_before + incl - mine;
        for (int wi = 0; wi < NW; ++wi) {
            uint32_t m = sm.sel[tid * NW + wi];
            uint32_t tm = sm.tie[tid * NW + wi];
            while (tm) {                                // keep ties while the global tie rank allows
                const uint32_t bit = tm & (0u - tm);
                tm ^= bit;
                if (tie_rank < need) m |= bit;
                ++tie_rank;
            }
            while (m) {
                const int bit = __ffs(m) - 1;
                m &= m - 1u;
                if (pos_out < static_cast<uint32_t>(k)) {
                    const int64_t t = t0 + 32 * wi + bit;
                    orow[pos_out] = static_cast<int32_t>(t);
                    if (srow_out) srow_out[pos_out] = __ldcg(srow + t);
                }
                ++pos_out;
            }
        }
        out_base = op;
        tie_base = tp;
        __syncthreads();                                // the next round rewrites the bitmaps
    }
    cluster.sync();                                     // no CTA leaves while a peer may read its counts
}

}  // namespace csa2
