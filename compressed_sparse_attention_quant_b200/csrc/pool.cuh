// pool.cuh -- K6: top-k inside a candidate pool (hierarchical sparse indexer).
// Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2: later indexing layers filter only within the candidate pool built
// by the first Full layer, so their cost no longer grows with the context.
// The pool is the Full layer's top-C (ascending token indices, -1 padded, as
// K3 emits it); the layer scores only those tokens with its own query.
//
// One thread-block cluster of S CTAs (S = 1 or 2, 512 threads each) per
// query row; CTA q owns the q-th contiguous slice of the pool, so the slices
// are in pool order.
//   slots   each thread resolves 8 of its slice's entries at a time (pool
//           index, then page-table entry, loads of all 8 in flight) to
//           physical cache slots, kept in shared memory.
//   score   warps take 4 groups of 16 entries at a time: their indexer keys
//           (64 bytes each) and scales are loaded together, the keys are the
//           A operand (16 entries x 32 channels per k-step) of FP8 mma.sync
//           m16n8k32 against the row's query (4 heads as B columns), fp32
//           accumulation. ReLU, sigma and the head weights follow; the
//           score's order-preserving 32-bit key replaces the slot (0 marks an
//           empty or invalid entry: no finite score maps there).
//   select  radix select on the keys, 11 + 11 + 10 bits: each level a shared
//           histogram per CTA, summed over the cluster through distributed
//           shared memory, and a warp-level pick; it gives the k-th largest
//           key T and the number of ties to keep.
//   emit    entries above T and the first ties in pool order (pool order is
//           ascending token order, so these are the lowest token indices),
//           compacted in order: per-thread runs, warp scans, one exchange of
//           counts across the cluster.
// A pool entry after the row's query position (causal bound), past the
// sequence or with a bad page sets the status word and is skipped. Scores
// equal the mathematical value whenever every partial sum is exact in fp32
// (small-integer E4M3 inputs, sigma = 1 or a power of two, power-of-two
// weights), like K2.
//
// Merge mode (context-parallel decode): the entries are the shards' top-k
// lists with their scores given, in shard order (each list ascending, the
// shards owning increasing position ranges, so the concatenation ascends);
// the same selection gives the top-k of the union, which is the top-k of the
// whole context, and each shard may take the entries it owns as local
// positions.
#pragma once

#include "common.cuh"
#include "topk.cuh"

#include <cooperative_groups.h>

namespace csa2 {

constexpr int kPoolThreads = 512;
constexpr int kPoolWarps = kPoolThreads / 32;
constexpr int kPoolBins = 2048;
static_assert(kPoolBins == kTopkBins, "the pool shares warp_pick and its padded histogram with K3");
constexpr int kPoolMax = 32768;                  // largest pool per row
constexpr int kPoolMaxCluster = 2;
constexpr int kPoolBatch = 8;                    // entries per thread resolved together (pass 1)
constexpr int kPoolGroups = 4;                   // 16-entry groups per warp scored together (pass 2)

struct PoolSmemFixed {
    uint32_t qb[kIdxHeads * kIdxDim / 4];        // the row's query, E4M3 bytes (4 per word)
    float w[kIdxHeads];
    uint32_t hloc[kPoolBins];                    // this CTA's histogram of the current level (read by peers)
    uint32_t hsum[kTopkBinsPadded];              // cluster-wide sum, padded (hpad) as warp_pick reads it
    uint32_t wcnt[2][kPoolWarps];
    uint32_t xchg[3];                            // (valid entries, selected, ties) of this CTA, read by peers
    uint32_t s_pick[2];                          // (bin, count above) of the current level
};

constexpr size_t pool_smem_bytes(int slice) {
    return sizeof(PoolSmemFixed) + static_cast<size_t>(slice) * sizeof(uint32_t);
}

struct PoolArgs {
    const uint8_t *q_idx;        // [R][4][64] E4M3 (scoring mode)
    const float *w;              // [R][4]
    const uint8_t *kidx;         // [pages][4096]
    const float *kidx_scale;     // [pages][64]
    int64_t num_pages;
    const int32_t *page_table;   // [B][max_pages]
    int max_pages;
    const int32_t *seq_lens;     // [B]
    int Sq;
    // Entry i of row r is at pool[(i / seg) * seg_stride + r * row_stride + i % seg]
    // (one segment [R][C] for a candidate pool; [shards][R][k_shard] for a merge).
    const int32_t *pool;
    int C;
    int seg;
    int64_t seg_stride;
    int64_t row_stride;
    const float *given;          // merge mode: the entries' scores (same addressing), no scoring
    int k;
    int32_t *out;                // [R][k] (may be null in merge mode)
    int32_t *out_local;          // merge mode: [R][k] entries in [lo, hi) minus lo, else -1 (or null)
    int32_t lo, hi;
    int slice;                   // entries per CTA of the cluster (a multiple of 16)
};

__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kPoolThreads)
pool_topk_kernel(const PoolArgs A) {
    namespace cg = cooperative_groups;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    PoolSmemFixed &fs = *reinterpret_cast<PoolSmemFixed *>(smem_raw);
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw + sizeof(PoolSmemFixed));
    cg::cluster_group cluster = cg::this_cluster();
    const int S = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int row = blockIdx.x / S, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tig = lane & 3;
    const int b = row / A.Sq;
    const int e0 = rank * A.slice;                              // this CTA's entries [e0, e1)
    const int e1 = min(e0 + A.slice, A.C);

    // Inputs no earlier kernel of the step writes: the query and weights.
    if (!A.given) {
        if (tid < kIdxHeads * kIdxDim / 4)
            fs.qb[tid] = __ldg(reinterpret_cast<const uint32_t *>(A.q_idx + static_cast<int64_t>(row) * kIdxHeads * kIdxDim) + tid);
        if (tid < kIdxHeads) fs.w[tid] = A.w[static_cast<int64_t>(row) * kIdxHeads + tid];
    }
    int T = A.given ? A.Sq : A.seq_lens[b];
    pdl_wait();                                                 // the pool is written by the previous kernel
    pdl_trigger();
    if (T < A.Sq || T > A.max_pages * kPage) {
        if (tid == 0 && rank == 0) flag_status(kStatusBounds);
        T = A.Sq - 1 - row % A.Sq;                              // no valid token for any query of the row
    }
    // Query j of the sequence sits at position T - Sq + j and is causal: a
    // pool entry after it is out of range.
    const int lim = T - A.Sq + row % A.Sq + 1;
    for (int i = tid; i < kPoolBins; i += kPoolThreads) fs.hloc[i] = 0u;
    __syncthreads();                                            // query, weights in; histogram zero
    auto entry = [&](int i) -> int64_t {
        return static_cast<int64_t>(i / A.seg) * A.seg_stride + static_cast<int64_t>(row) * A.row_stride + i % A.seg;
    };

    // ---------------- keys of this CTA's entries
    const int n_mine = max(e1 - e0, 0);
    uint32_t n_valid = 0u;
    if (A.given) {
        for (int i = e0 + tid; i < e1; i += kPoolThreads) {
            const int t = A.pool[entry(i)];
            uint32_t key = 0u;
            if (t >= 0) {
                if (i > 0 && A.pool[entry(i - 1)] >= t) flag_status(kStatusBounds);   // must ascend
                key = float_key(__ldg(A.given + entry(i)));
                ++n_valid;
            }
            keys[i - e0] = key;
        }
    } else {
        // ---- pass 1: the slice's physical slots (pool index -> page -> slot,
        // -1 for an empty or invalid entry), written in place into keys[];
        // kPoolBatch entries per thread have their loads in flight together
        for (int base = 0; base < n_mine; base += kPoolThreads * kPoolBatch) {
            int tk[kPoolBatch], tprev[kPoolBatch];
            int64_t pg[kPoolBatch];
#pragma unroll
            for (int u = 0; u < kPoolBatch; ++u) {
                const int il = base + u * kPoolThreads + tid, i = e0 + il;
                tk[u] = il < n_mine ? A.pool[entry(i)] : -1;
                tprev[u] = il < n_mine && i > 0 ? A.pool[entry(i - 1)] : -1;
            }
#pragma unroll
            for (int u = 0; u < kPoolBatch; ++u)
                pg[u] = tk[u] >= 0 && tk[u] < lim ? A.page_table[static_cast<int64_t>(b) * A.max_pages + (tk[u] >> 6)] : -1;
#pragma unroll
            for (int u = 0; u < kPoolBatch; ++u) {
                const int il = base + u * kPoolThreads + tid;
                if (il >= n_mine) continue;
                int slot = -1;
                const int t = tk[u];
                if (t >= 0) {
                    if (tprev[u] >= t) flag_status(kStatusBounds);                // the pool must ascend
                    if (t >= lim || pg[u] < 0 || pg[u] >= A.num_pages) {
                        flag_status(kStatusBounds);
                    } else {
                        slot = static_cast<int>(pg[u] * kPage + (t & 63));
                        ++n_valid;
                    }
                }
                keys[il] = static_cast<uint32_t>(slot);
            }
        }
        __syncthreads();
        // ---- pass 2: scores. A warp takes kPoolGroups groups of 16 entries at
        // a time (all their key and sigma loads in flight), one MMA per group.
        // query B fragments: head g (< 4) channels 4 tig .. +3 and 16 + 4 tig .. +3 of each k-step
        uint32_t qf[2][2];
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            qf[ks][0] = g < kIdxHeads ? fs.qb[(g * kIdxDim + ks * 32 + 4 * tig) / 4] : 0u;
            qf[ks][1] = g < kIdxHeads ? fs.qb[(g * kIdxDim + ks * 32 + 16 + 4 * tig) / 4] : 0u;
        }
        const float wlo = fs.w[2 * (tig & 1)], whi = fs.w[2 * (tig & 1) + 1];
        const int n_groups = (n_mine + 15) / 16;
        for (int g0 = warp * kPoolGroups; g0 < n_groups; g0 += kPoolWarps * kPoolGroups) {
            int sl[kPoolGroups][2];
            uint32_t a[kPoolGroups][2][4];
            float sg[kPoolGroups][2];
#pragma unroll
            for (int q = 0; q < kPoolGroups; ++q)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int il = (g0 + q) * 16 + g + 8 * h;
                    sl[q][h] = g0 + q < n_groups && il < n_mine ? static_cast<int>(keys[il]) : -1;
                }
#pragma unroll
            for (int q = 0; q < kPoolGroups; ++q)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int sv = sl[q][h];
                    const uint8_t *kb = A.kidx + (sv >= 0 ? static_cast<int64_t>(sv >> 6) * kKidxPageBytes +
                                                                ((sv & 63) >> 3) * 512 + (sv & 7) * 16 + 4 * tig
                                                          : 0);
#pragma unroll
                    for (int c = 0; c < 4; ++c)                 // 16-byte chunk c = channels 16c .. 16c + 15
                        a[q][c >> 1][(c & 1) * 2 + h] = sv >= 0 ? __ldg(reinterpret_cast<const uint32_t *>(kb + c * 128)) : 0u;
                    sg[q][h] = sv >= 0 ? __ldg(A.kidx_scale + sv) : 0.0f;
                }
#pragma unroll
            for (int q = 0; q < kPoolGroups; ++q) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                    mma_e4m3_16832(acc, a[q][ks][0], a[q][ks][1], a[q][ks][2], a[q][ks][3], qf[ks][0], qf[ks][1]);
                // lanes with tig 0 / 1 hold heads 0, 1 / 2, 3 of entries g and g + 8
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float part = wlo * fmaxf(0.0f, sg[q][h] * acc[2 * h]) + whi * fmaxf(0.0f, sg[q][h] * acc[2 * h + 1]);
                    part += __shfl_xor_sync(0xffffffffu, part, 1);   // heads 0..3
                    const int il = (g0 + q) * 16 + g + 8 * h;
                    if (tig == 0 && g0 + q < n_groups && il < n_mine) keys[il] = sl[q][h] >= 0 ? float_key(part) : 0u;
                }
            }
        }
    }
    // valid entries of the whole row (cluster)
    {
        const uint32_t wv = warp_incl_scan(n_valid);
        if (lane == 31) fs.wcnt[0][warp] = wv;
        __syncthreads();
        if (tid == 0) {
            uint32_t t = 0u;
            for (int w = 0; w < kPoolWarps; ++w) t += fs.wcnt[0][w];
            fs.xchg[0] = t;
        }
        cluster.sync();
    }
    uint32_t row_valid = 0u;
    for (int q = 0; q < S; ++q) row_valid += *cluster.map_shared_rank(&fs.xchg[0], q);
    const uint32_t need = min(static_cast<uint32_t>(A.k), row_valid);

    // ---------------- threshold key T: the need-th largest key over the cluster
    uint32_t thr = 0u, n_gt = 0u;                // select keys > thr, then (need - n_gt) ties == thr
    const bool all = need == row_valid;          // every valid entry is kept (also when there is none)
    if (!all) {
        uint32_t prefix = 0u, above = 0u;
#pragma unroll 1
        for (int lvl = 0; lvl < 3; ++lvl) {
            const int wdt = lvl < 2 ? 11 : 10;               // key bits 31..21, 20..10, 9..0
            const int shift = lvl == 0 ? 21 : (lvl == 1 ? 10 : 0);
            if (lvl > 0) {
                cluster.sync();                              // every peer has read this CTA's previous level
                for (int i = tid; i < kPoolBins; i += kPoolThreads) fs.hloc[i] = 0u;
                __syncthreads();
            }
            for (int i = tid; i < n_mine; i += kPoolThreads) {
                const uint32_t kk = keys[i];
                if (kk == 0u) continue;
                if (lvl > 0 && (kk >> (shift + wdt)) != prefix) continue;
                atomicAdd(&fs.hloc[(kk >> shift) & ((1u << wdt) - 1u)], 1u);
            }
            cluster.sync();
            for (int i = tid; i < kPoolBins; i += kPoolThreads) {
                uint32_t v = 0u;
                for (int q = 0; q < S; ++q) v += cluster.map_shared_rank(&fs.hloc[0], q)[i];
                fs.hsum[hpad(i)] = v;
            }
            __syncthreads();
            if (warp == 0) {
                uint32_t bin, ab;
                warp_pick<false>(fs.hsum, 1 << wdt, need - above, bin, ab);
                if (lane == 0) {
                    fs.s_pick[0] = bin;
                    fs.s_pick[1] = ab;
                }
            }
            __syncthreads();
            above += fs.s_pick[1];
            prefix = (prefix << wdt) | fs.s_pick[0];
        }
        thr = prefix;
        n_gt = above;
    }

    // ---------------- emit, in pool order: keys > thr, then the first ties
    const int seg = (n_mine + kPoolThreads - 1) / kPoolThreads;
    const int i0 = min(tid * seg, n_mine), i1 = min(i0 + seg, n_mine);
    uint32_t n_sel = 0u, n_tie = 0u;
    for (int i = i0; i < i1; ++i) {
        const uint32_t kk = keys[i];
        if (kk == 0u) continue;
        if (all || kk > thr) ++n_sel;
        else if (kk == thr) ++n_tie;
    }
    const uint32_t is_ = warp_incl_scan(n_sel), it_ = warp_incl_scan(n_tie);
    __syncthreads();                                            // wcnt[0] of the count above is read
    if (lane == 31) {
        fs.wcnt[0][warp] = is_;
        fs.wcnt[1][warp] = it_;
    }
    __syncthreads();
    uint32_t cta_sel = 0u, cta_tie = 0u, sel_before = is_ - n_sel, tie_before = it_ - n_tie;
    for (int w = 0; w < kPoolWarps; ++w) {
        if (w < warp) {
            sel_before += fs.wcnt[0][w];
            tie_before += fs.wcnt[1][w];
        }
        cta_sel += fs.wcnt[0][w];
        cta_tie += fs.wcnt[1][w];
    }
    if (tid == 0) {
        fs.xchg[1] = cta_sel;
        fs.xchg[2] = cta_tie;
    }
    cluster.sync();
    const uint32_t ties_keep = need - n_gt;
    uint32_t sel_base = 0u, tie_base = 0u;
    for (int q = 0; q < rank; ++q) {
        sel_base += cluster.map_shared_rank(&fs.xchg[0], q)[1];
        tie_base += cluster.map_shared_rank(&fs.xchg[0], q)[2];
    }
    // Position of an entry = selected strictly-greater entries before it plus
    // kept ties before it (both over the whole cluster, in pool order).
    uint32_t gt_before = sel_base + sel_before;
    uint32_t tb = tie_base + tie_before;
    int32_t *orow = A.out ? A.out + static_cast<int64_t>(row) * A.k : nullptr;
    int32_t *lrow = A.out_local ? A.out_local + static_cast<int64_t>(row) * A.k : nullptr;
    auto put = [&](uint32_t pos, int32_t t) {
        if (orow) orow[pos] = t;
        if (lrow) lrow[pos] = (t >= A.lo && t < A.hi) ? t - A.lo : -1;
    };
    for (int i = i0; i < i1; ++i) {
        const uint32_t kk = keys[i];
        if (kk == 0u) continue;
        if (all || kk > thr) {
            const uint32_t pos = gt_before + min(tb, ties_keep);
            if (pos < need) put(pos, A.pool[entry(e0 + i)]);
            ++gt_before;
        } else if (kk == thr) {
            if (tb < ties_keep && gt_before + tb < need) put(gt_before + tb, A.pool[entry(e0 + i)]);
            ++tb;
        }
    }
    for (int i = static_cast<int>(need) + rank * kPoolThreads + tid; i < A.k; i += S * kPoolThreads)
        put(static_cast<uint32_t>(i), -1);
    cluster.sync();                                             // no CTA leaves while a peer may read its counts
}

// Cluster size: 2 when every CTA still holds at least 1024 entries and all
// clusters fit in one wave of two CTAs per SM, else 1.
inline cudaError_t launch_pool_topk(PoolArgs A, int rows, int sm_count, cudaStream_t stream) {
    int S = 1;
    while (S * 2 <= kPoolMaxCluster && static_cast<int64_t>(rows) * S * 2 <= 2 * sm_count && A.C / (S * 2) >= 1024)
        S *= 2;
    A.slice = (A.C + S - 1) / S;
    A.slice = (A.slice + 15) / 16 * 16;
    return launch_pdl_cluster(pool_topk_kernel, dim3(static_cast<unsigned>(rows * S)), dim3(kPoolThreads),
                              pool_smem_bytes(A.slice), stream, S, A);
}

}  // namespace csa2
