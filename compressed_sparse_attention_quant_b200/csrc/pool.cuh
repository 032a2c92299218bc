// pool.cuh -- K6: top-k inside a candidate pool (hierarchical sparse indexer).
// Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2: later indexing layers filter only within the candidate pool built
// by the first Full layer, so their cost no longer grows with the context.
// The pool is the Full layer's top-C (ascending token indices, -1 padded, as
// K3 emits it); the layer scores only those tokens with its own query.
//
// One CTA (512 threads) per query row. A pool entry after the row's query
// position (causal bound), past the sequence or with a bad page sets the status
// word and is skipped.
//   score   thread i takes pool entries i, i + 512, ...: the token's 64-byte
//           indexer key (four 16-byte chunks of its page's core-matrix
//           layout) and sigma; four fp32 dot products with the row's query
//           (converted from E4M3 once into shared memory), ReLU, head
//           weights; the score's order-preserving 32-bit key goes to shared
//           memory (0 marks an empty or invalid entry: no finite score maps
//           there).
//   select  radix select on the keys, 11 + 11 + 10 bits, each level a shared
//           histogram and a block scan from the top, gives the k-th largest
//           key T and the number of ties to keep. The entries above T and the
//           first ties in pool order (pool order is ascending token order, so
//           these are the lowest token indices) are compacted in order.
// Scores equal the mathematical value whenever every partial sum is exact in
// fp32 (small-integer E4M3 inputs, sigma = 1, power-of-two weights), like K2.
//
// Merge mode (context-parallel decode): the entries are the shards' top-k
// lists with their scores given, in shard order (each list ascending, the
// shards owning increasing position ranges, so the concatenation ascends);
// the same selection gives the top-k of the union, which is the top-k of the
// whole context, and each shard may take the entries it owns as local
// positions.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kPoolThreads = 512;
constexpr int kPoolBins = 2048;
constexpr int kPoolMax = 32768;                  // largest pool per row (128 KB of keys)

struct PoolSmemFixed {
    float q[kIdxHeads][kIdxDim];                 // the row's query, fp32
    float w[kIdxHeads];
    uint32_t hist[kPoolBins];
    uint64_t wbuf64[kPoolThreads / 32 + 1];
    uint32_t wbuf[kPoolThreads / 32 + 1];
    uint32_t s_bin, s_above;
};

constexpr size_t pool_smem_bytes(int pool_size) {
    return sizeof(PoolSmemFixed) + static_cast<size_t>(pool_size) * sizeof(uint32_t);
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
};

// From a shared 2048-bin histogram, the bin holding the need-th largest key
// and the count of keys in higher bins (each thread owns 4 bins from the top).
__device__ __forceinline__ void pool_pick(PoolSmemFixed &fs, uint32_t need, uint32_t &bin, uint32_t &above) {
    constexpr int PER = kPoolBins / kPoolThreads;
    const int top = kPoolBins - 1 - static_cast<int>(threadIdx.x) * PER;
    uint32_t c[PER];
    uint32_t local = 0u;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        c[i] = fs.hist[top - i];
        local += c[i];
    }
    if (threadIdx.x == 0) {                      // stays if the counts fall short of need
        fs.s_bin = 0u;
        fs.s_above = 0u;
    }
    uint32_t tot;
    uint32_t run = block_excl_scan<kPoolThreads>(local, fs.wbuf, &tot);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        if (run < need && run + c[i] >= need) {
            fs.s_bin = static_cast<uint32_t>(top - i);
            fs.s_above = run;
        }
        run += c[i];
    }
    __syncthreads();
    bin = fs.s_bin;
    above = fs.s_above;
    __syncthreads();
}

__global__ void __launch_bounds__(kPoolThreads)
pool_topk_kernel(const PoolArgs A) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    PoolSmemFixed &fs = *reinterpret_cast<PoolSmemFixed *>(smem_raw);
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw + sizeof(PoolSmemFixed));
    const int row = blockIdx.x, tid = threadIdx.x;
    const int b = row / A.Sq;

    // Inputs no earlier kernel of the step writes: the query and weights.
    if (!A.given && tid < kIdxHeads * kIdxDim / 2) {
        const uint8_t *qb = A.q_idx + static_cast<int64_t>(row) * kIdxHeads * kIdxDim + 2 * tid;
        const uint32_t h2 = e4m3x2_to_f16x2(qb[0] | (static_cast<uint32_t>(qb[1]) << 8));
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h2));
        (&fs.q[0][0])[2 * tid] = f.x;
        (&fs.q[0][0])[2 * tid + 1] = f.y;
    }
    if (!A.given && tid < kIdxHeads) fs.w[tid] = A.w[static_cast<int64_t>(row) * kIdxHeads + tid];
    int T = A.given ? A.Sq : A.seq_lens[b];
    pdl_wait();                                  // the pool is written by the previous kernel
    pdl_trigger();
    if (T < A.Sq || T > A.max_pages * kPage) {
        if (tid == 0) flag_status(kStatusBounds);
        T = A.Sq - 1 - row % A.Sq;               // no valid token for any query of the row
    }
    // Query j of the sequence sits at position T - Sq + j and is causal: a
    // pool entry after it is out of range.
    const int lim = T - A.Sq + row % A.Sq + 1;
    __syncthreads();

    // ---------------- score every pool entry
    auto entry = [&](int i) -> int64_t {
        return static_cast<int64_t>(i / A.seg) * A.seg_stride + static_cast<int64_t>(row) * A.row_stride + i % A.seg;
    };
    uint32_t n_valid = 0u;
    for (int i = tid; i < A.C; i += kPoolThreads) {
        const int t = A.pool[entry(i)];
        uint32_t key = 0u;
        if (t >= 0 && A.given) {
            if (i > 0 && A.pool[entry(i - 1)] >= t) flag_status(kStatusBounds);      // must ascend
            key = float_key(__ldg(A.given + entry(i)));
            ++n_valid;
        } else if (t >= 0) {
            const int64_t page = t < lim ? A.page_table[static_cast<int64_t>(b) * A.max_pages + (t >> 6)] : -1;
            if (i > 0 && A.pool[entry(i - 1)] >= t) flag_status(kStatusBounds);      // pool must ascend
            if (page >= 0 && page < A.num_pages) {
                const int r = t & 63;
                const uint8_t *kb = A.kidx + page * kKidxPageBytes + (r >> 3) * 512 + (r & 7) * 16;
                const float sg = A.kidx_scale[page * kPage + r];
                float dot[kIdxHeads] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c16 = 0; c16 < 4; ++c16) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(kb + c16 * 128);
                    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t lo = e4m3x2_to_f16x2(wd[j] & 0xffffu);
                        const uint32_t hi = e4m3x2_to_f16x2(wd[j] >> 16);
                        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&lo));
                        const float2 c = __half22float2(*reinterpret_cast<const __half2 *>(&hi));
                        const int ch = c16 * 16 + j * 4;
#pragma unroll
                        for (int h = 0; h < kIdxHeads; ++h) {
                            const float4 qv = *reinterpret_cast<const float4 *>(&fs.q[h][ch]);
                            dot[h] = fmaf(qv.x, a.x, dot[h]);
                            dot[h] = fmaf(qv.y, a.y, dot[h]);
                            dot[h] = fmaf(qv.z, c.x, dot[h]);
                            dot[h] = fmaf(qv.w, c.y, dot[h]);
                        }
                    }
                }
                float score = 0.0f;
#pragma unroll
                for (int h = 0; h < kIdxHeads; ++h) score += fs.w[h] * fmaxf(sg * dot[h], 0.0f);
                key = float_key(score);
                ++n_valid;
            } else {
                flag_status(kStatusBounds);
            }
        }
        keys[i] = key;
    }
    {
        uint32_t tot;
        block_excl_scan<kPoolThreads>(n_valid, fs.wbuf, &tot);
        n_valid = tot;                           // every thread: valid entries of the row
    }
    const uint32_t need = min(static_cast<uint32_t>(A.k), n_valid);

    // ---------------- threshold key T: the need-th largest key
    uint32_t thr = 0u, n_gt = 0u;                // select keys > thr, then (need - n_gt) ties == thr
    if (need > 0u && need < n_valid) {
        uint32_t prefix = 0u, above = 0u;
#pragma unroll 1
        for (int lvl = 0; lvl < 3; ++lvl) {
            const int wdt = lvl < 2 ? 11 : 10;               // key bits 31..21, 20..10, 9..0
            const int shift = lvl == 0 ? 21 : (lvl == 1 ? 10 : 0);
            for (int i = tid; i < kPoolBins; i += kPoolThreads) fs.hist[i] = 0u;
            __syncthreads();
            for (int i = tid; i < A.C; i += kPoolThreads) {
                const uint32_t kk = keys[i];
                if (kk == 0u) continue;
                if (lvl > 0 && (kk >> (shift + wdt)) != prefix) continue;
                atomicAdd(&fs.hist[(kk >> shift) & ((1u << wdt) - 1u)], 1u);
            }
            __syncthreads();
            uint32_t bin, ab;
            pool_pick(fs, need - above, bin, ab);
            above += ab;
            prefix = (prefix << wdt) | bin;
        }
        thr = prefix;
        n_gt = above;
    }

    // ---------------- emit, in pool order: keys > thr, then the first ties
    const bool all = need == n_valid;           // every valid entry is kept (also when there is none)
    const int seg = (A.C + kPoolThreads - 1) / kPoolThreads;
    const int i0 = min(tid * seg, A.C), i1 = min(i0 + seg, A.C);
    uint32_t n_sel = 0u, n_tie = 0u;
    for (int i = i0; i < i1; ++i) {
        const uint32_t kk = keys[i];
        if (kk == 0u) continue;
        if (all || kk > thr) ++n_sel;
        else if (kk == thr) ++n_tie;
    }
    uint64_t tot64;
    const uint64_t pre = block_excl_scan64<kPoolThreads>((static_cast<uint64_t>(n_tie) << 32) | n_sel, fs.wbuf64,
                                                        &tot64);
    uint32_t tie_before = static_cast<uint32_t>(pre >> 32);
    const uint32_t ties_keep = need - n_gt;
    // Position of an entry = selected strictly-greater entries before it plus
    // kept ties before it.
    uint32_t gt_before = static_cast<uint32_t>(pre & 0xffffffffu);
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
            const uint32_t pos = gt_before + min(tie_before, ties_keep);
            if (pos < need) put(pos, A.pool[entry(i)]);
            ++gt_before;
        } else if (kk == thr) {
            if (tie_before < ties_keep && gt_before + tie_before < need) put(gt_before + tie_before, A.pool[entry(i)]);
            ++tie_before;
        }
    }
    for (int i = static_cast<int>(need) + tid; i < A.k; i += kPoolThreads) put(static_cast<uint32_t>(i), -1);
}

inline cudaError_t launch_pool_topk(const PoolArgs &A, int rows, cudaStream_t stream) {
    return launch_pdl(pool_topk_kernel, dim3(static_cast<unsigned>(rows)), dim3(kPoolThreads), pool_smem_bytes(A.C),
                      stream, A);
}

}  // namespace csa2
