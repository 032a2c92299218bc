// topk.cuh -- K3: exact, deterministic top-k over the indexer scores.
// Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2: the "Top-K sparse addressing index"; page "DeepSeek V4 1-Flash
// 架构拆解…" (blog.zulogic.cn), section 3: Full and Reindex run the selection.
//
// Selection rule: the k largest scores of positions 0 .. n_valid-1, ties to
// the lower position, emitted in ascending position order, -1 padded.
//
// Method (multi-CTA per query row, no inter-CTA waiting):
//   1. radix levels on the order-preserving 32-bit key of each score, 11 + 11
//      + 10 bits from the top: every CTA histograms the next digit of the
//      keys that match the prefix resolved so far (shared-memory atomics,
//      then one global add per non-empty bin); the last CTA of the row to
//      arrive (atomic counter, no spin) picks the digit holding the k-th key
//      and stops early once every element of that digit is taken.
//   2. count: per 4096-element chunk, elements above the threshold prefix
//      and equal to it; the last CTA scans the chunk counts into output
//      offsets.
//   3. write: each chunk emits its selected positions in order (block scan
//      of per-thread counts); among keys equal to the threshold only the
//      lowest positions, up to the number still needed, are taken.
// Scores stay L2-resident between the passes (4 B per cached token).
#pragma once

#include "common.cuh"
#include "indexer.cuh"

namespace csa2 {

constexpr int kTopkThreads = 256;
constexpr int kTopkPerThread = 16;
constexpr int kTopkChunk = kTopkThreads * kTopkPerThread;   // 4096

__device__ __forceinline__ int topk_digit_width(int level) { return level < 2 ? 11 : 10; }

// Exclusive block scan of one value per thread (256 threads). Returns the
// exclusive prefix; *total receives the block sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *warp_buf, uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_buf[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        uint32_t wv = lane < (kTopkThreads / 32) ? warp_buf[lane] : 0u;
        uint32_t wi = wv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < (kTopkThreads / 32)) warp_buf[lane] = wi - wv;   // exclusive warp offsets
        if (lane == kTopkThreads / 32 - 1) warp_buf[kTopkThreads / 32] = wi;
    }
    __syncthreads();
    const uint32_t res = warp_buf[warp] + incl - v;
    *total = warp_buf[kTopkThreads / 32];
    __syncthreads();
    return res;
}

// Loads this thread's 16 consecutive keys of the chunk; positions >= n get
// valid = false.
__device__ __forceinline__ void load_keys(const float *__restrict__ srow, int64_t c0, int n,
                                          uint32_t (&key)[kTopkPerThread], uint32_t &valid_mask) {
    const int64_t e0 = c0 + static_cast<int64_t>(threadIdx.x) * kTopkPerThread;
    valid_mask = 0u;
    if (e0 + kTopkPerThread <= n) {
        const float4 *p = reinterpret_cast<const float4 *>(srow + e0);
#pragma unroll
        for (int v = 0; v < kTopkPerThread / 4; ++v) {
            const float4 f = __ldcg(p + v);
            key[4 * v + 0] = float_key(f.x);
            key[4 * v + 1] = float_key(f.y);
            key[4 * v + 2] = float_key(f.z);
            key[4 * v + 3] = float_key(f.w);
        }
        valid_mask = 0xffffu;
    } else {
#pragma unroll
        for (int i = 0; i < kTopkPerThread; ++i) {
            if (e0 + i < n) {
                key[i] = float_key(__ldcg(srow + e0 + i));
                valid_mask |= 1u << i;
            } else {
                key[i] = 0u;
            }
        }
    }
}

__device__ __forceinline__ uint32_t key_prefix(uint32_t key, int bits) {
    return bits == 0 ? 0u : (key >> (32 - bits));
}

// One radix level: histogram of the next digit, then the last CTA picks it.
__global__ void __launch_bounds__(kTopkThreads)
topk_radix_kernel(const float *__restrict__ scores, int64_t t_cap, TopkRow *__restrict__ rows,
                  uint32_t *__restrict__ hist, uint32_t *__restrict__ counters, int level) {
    __shared__ uint32_t sh[kTopkBins];
    __shared__ uint32_t wbuf[kTopkThreads / 32 + 1];
    __shared__ int is_last;
    const int row = blockIdx.y;
    const TopkRow st = rows[row];
    if (st.done) return;                        // uniform over the row's CTAs
    const int width = topk_digit_width(level);
    const int nb = 1 << width;
    const int bits_after = st.bits + width;
    for (int i = threadIdx.x; i < nb; i += kTopkThreads) sh[i] = 0u;
    __syncthreads();

    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTopkChunk;
    if (c0 < st.n_valid) {
        uint32_t key[kTopkPerThread];
        uint32_t vm;
        load_keys(scores + static_cast<int64_t>(row) * t_cap, c0, st.n_valid, key, vm);
#pragma unroll
        for (int i = 0; i < kTopkPerThread; ++i) {
            if (((vm >> i) & 1u) && key_prefix(key[i], st.bits) == st.prefix) {
                atomicAdd(&sh[(key[i] >> (32 - bits_after)) & (nb - 1)], 1u);
            }
        }
    }
    __syncthreads();
    uint32_t *gh = hist + static_cast<int64_t>(row) * kTopkBins;
    for (int i = threadIdx.x; i < nb; i += kTopkThreads)
        if (sh[i]) atomicAdd(&gh[i], sh[i]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = (atomicAdd(&counters[row], 1u) == gridDim.x - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();

    // Last CTA of the row: find the digit holding the remaining-th largest key.
    const int per = nb / kTopkThreads;          // 8 or 4 bins per thread
    // thread t owns bins [hi_t - per + 1, hi_t] counted from the top
    const int top = nb - 1 - threadIdx.x * per;
    uint32_t local = 0u;
    for (int i = 0; i < per; ++i) {
        const uint32_t c = __ldcg(&gh[top - i]);
        sh[top - i] = c;
        local += c;
    }
    uint32_t tot;
    const uint32_t above = block_excl_scan(local, wbuf, &tot);   // keys in higher bins
    const uint32_t need = static_cast<uint32_t>(st.remaining);
    uint32_t run = above;
    for (int i = 0; i < per; ++i) {
        const int bin = top - i;
        const uint32_t c = sh[bin];
        if (run < need && run + c >= need) {
            TopkRow r = st;
            r.prefix = (st.bits == 0 ? 0u : (st.prefix << width)) | static_cast<uint32_t>(bin);
            r.bits = bits_after;
            r.remaining = static_cast<int32_t>(need - run);
            r.eq_count = static_cast<int32_t>(c);
            r.done = (c == need - run || bits_after == 32) ? 1 : 0;
            rows[row] = r;
        }
        run += c;
    }
    // leave the histogram and counter zeroed for the next level
    for (int i = threadIdx.x; i < kTopkBins; i += kTopkThreads) gh[i] = 0u;
    if (threadIdx.x == 0) counters[row] = 0u;
}

// Chunk counts of keys above / equal to the threshold prefix, then offsets.
__global__ void __launch_bounds__(kTopkThreads)
topk_count_kernel(const float *__restrict__ scores, int64_t t_cap, const TopkRow *__restrict__ rows,
                  uint32_t *__restrict__ counters, uint2 *__restrict__ chunk_cnt,
                  uint2 *__restrict__ chunk_off, int n_chunks) {
    __shared__ uint32_t wbuf[kTopkThreads / 32 + 1];
    __shared__ int is_last;
    const int row = blockIdx.y;
    const TopkRow st = rows[row];
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTopkChunk;
    uint32_t gt = 0u, eq = 0u;
    if (c0 < st.n_valid) {
        uint32_t key[kTopkPerThread];
        uint32_t vm;
        load_keys(scores + static_cast<int64_t>(row) * t_cap, c0, st.n_valid, key, vm);
#pragma unroll
        for (int i = 0; i < kTopkPerThread; ++i) {
            if ((vm >> i) & 1u) {
                const uint32_t pf = key_prefix(key[i], st.bits);
                gt += pf > st.prefix;
                eq += pf == st.prefix;
            }
        }
    }
    uint32_t tgt, teq;
    block_excl_scan(gt, wbuf, &tgt);
    block_excl_scan(eq, wbuf, &teq);
    uint2 *cc = chunk_cnt + static_cast<int64_t>(row) * n_chunks;
    if (threadIdx.x == 0) cc[blockIdx.x] = make_uint2(tgt, teq);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = (atomicAdd(&counters[row], 1u) == gridDim.x - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    // Offsets: output position of each chunk's first selection, and the number
    // of threshold-equal keys in earlier chunks.
    uint2 *co = chunk_off + static_cast<int64_t>(row) * n_chunks;
    uint32_t gt_before = 0u, eq_before = 0u;
    for (int base = 0; base < n_chunks; base += kTopkThreads) {
        const int c = base + threadIdx.x;
        uint2 v = make_uint2(0u, 0u);
        if (c < n_chunks) v = __ldcg(&cc[c]);
        uint32_t sg, se;
        const uint32_t pg = block_excl_scan(v.x, wbuf, &sg);
        const uint32_t pe = block_excl_scan(v.y, wbuf, &se);
        if (c < n_chunks) {
            const uint32_t eb = eq_before + pe;
            const uint32_t take = min(eb, static_cast<uint32_t>(st.remaining));
            co[c] = make_uint2(gt_before + pg + take, eb);
        }
        gt_before += sg;
        eq_before += se;
    }
    if (threadIdx.x == 0) counters[row] = 0u;
}

// Emit the selected positions of each chunk in ascending order.
__global__ void __launch_bounds__(kTopkThreads)
topk_write_kernel(const float *__restrict__ scores, int64_t t_cap, const TopkRow *__restrict__ rows,
                  const uint2 *__restrict__ chunk_off, int n_chunks, int k, int32_t *__restrict__ out) {
    __shared__ uint32_t wbuf[kTopkThreads / 32 + 1];
    const int row = blockIdx.y;
    const TopkRow st = rows[row];
    int32_t *orow = out + static_cast<int64_t>(row) * k;
    if (blockIdx.x == 0) {
        const int n_sel = min(k, st.n_valid);
        for (int i = n_sel + threadIdx.x; i < k; i += kTopkThreads) orow[i] = -1;
    }
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTopkChunk;
    if (c0 >= st.n_valid) return;               // uniform over the CTA
    const uint2 off = chunk_off[static_cast<int64_t>(row) * n_chunks + blockIdx.x];
    uint32_t key[kTopkPerThread];
    uint32_t vm;
    load_keys(scores + static_cast<int64_t>(row) * t_cap, c0, st.n_valid, key, vm);
    uint32_t gtm = 0u, eqm = 0u;
#pragma unroll
    for (int i = 0; i < kTopkPerThread; ++i) {
        if ((vm >> i) & 1u) {
            const uint32_t pf = key_prefix(key[i], st.bits);
            if (pf > st.prefix) gtm |= 1u << i;
            if (pf == st.prefix) eqm |= 1u << i;
        }
    }
    uint32_t tot;
    const uint32_t eq_rank0 = off.y + block_excl_scan(__popc(eqm), wbuf, &tot);
    // threshold-equal keys are taken while their global rank < remaining
    uint32_t selm = gtm;
    uint32_t r = eq_rank0;
#pragma unroll
    for (int i = 0; i < kTopkPerThread; ++i) {
        if ((eqm >> i) & 1u) {
            if (r < static_cast<uint32_t>(st.remaining)) selm |= 1u << i;
            ++r;
        }
    }
    uint32_t pos = off.x + block_excl_scan(__popc(selm), wbuf, &tot);
    const int64_t e0 = c0 + static_cast<int64_t>(threadIdx.x) * kTopkPerThread;
#pragma unroll
    for (int i = 0; i < kTopkPerThread; ++i) {
        if ((selm >> i) & 1u) {
            if (pos < static_cast<uint32_t>(k)) orow[pos] = static_cast<int32_t>(e0 + i);
            ++pos;
        }
    }
}

}  // namespace csa2
