// attn.cuh -- K4/K5: sparse attention over the selected FP4 entries plus the
// sliding window, merged by online softmax.
// Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2 (attention reads only the top-K addressed entries of the shared main
// KV) and part 3 (E2M1 + E4M3 per 16 channels); page "DeepSeek V4 1-Flash
// 架构拆解…" (blog.zulogic.cn), section 4 (a 128-token window kept per layer
// beside the global compressed state).
//
// Work: the key list of a query row is its 128 window rows (none when the
// caller passes no window) followed by its k selected entries (padded to a
// multiple of 16), cut into steps of 16 keys.
// The steps of all rows form one flat sequence that is split into equal
// contiguous ranges, one per CTA (persistent: about two CTAs per SM). A CTA
// writes a row's result directly when its range covers the whole row, else an
// unnormalised partial (m, l, O) of its first or last row; K5 merges those.
//
// K4, one CTA = 4 warps; warp w owns channels [144 w, 144 w + 144) of every
// key, query head and output:
//   staging  cp.async copies of the packed FP4 records and scales (or the bf16
//            window rows) of step i + 3 into a 4-stage ring, zero-filled for
//            empty keys. Physical slots (top-k index -> page table) are
//            resolved a chunk of 8 steps ahead, each load issued two steps
//            before its value is used.
//   QK       lane (g, tig) converts keys g and g + 8 of the step straight into
//            m16n8k16 B fragments: channels are taken in an order in which a
//            lane's four channels of a k-step are contiguous (16 per 64-channel
//            unit, one scale group), the query fragments (held in registers
//            for the row) use the same order, so each product q_c k_c is
//            summed once. FP4 -> f16 is the hardware E2M1x2 conversion times
//            the E4M3 scale (exact in f16); the window's bf16 -> f16 goes
//            through a per-warp power-of-two exponent that keeps it in range.
//   reduce   the four warps' partial scores meet in shared memory; every warp
//            sums them in the same order and runs the same online softmax
//            (exp2 domain, probabilities rounded to f16), so no further
//            exchange is needed.
//   PV       movmatrix transposes the key fragments of QK into the value
//            fragments (keys = values), and the score accumulators are the
//            probability operand, so the value tile never goes to shared
//            memory. The O accumulator (16 heads x 144 channels) stays in
//            registers with a per-warp power-of-two exponent.
// Warp-level mma.sync is used deliberately: with 16 heads the MMA N extent is
// 16, and at that width the warp MMAs issue faster than tcgen05 single-thread
// MMAs. Two barriers per step: the staged data is complete, and the partial
// scores are complete.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kAttThreads = 128;
constexpr int kAttWarps = kAttThreads / 32;
constexpr int kAttStepKeys = 16;
constexpr int kAttWinSteps = kWindow / kAttStepKeys;          // 8
constexpr int kAttStageBytes = kAttStepKeys * kDim * 2;       // 18,432: 16 window rows of bf16
constexpr int kAttRecBytes = kAttStepKeys * kFp4Bytes;        // 4,608: 16 packed FP4 records
constexpr int kAttScaleWin = 48;                              // 16-byte aligned window holding 36 scale bytes
constexpr int kAttStages = 4;
constexpr int kAttAhead = kAttStages - 1;                     // steps staged ahead of the one computed
constexpr int kAttChunkSteps = 8;                             // steps per slot-resolution chunk
constexpr int kAttChunkKeys = kAttChunkSteps * kAttStepKeys;  // 128 = one key per thread
constexpr int kAttQuarter = kDim / kAttWarps;                 // 144 channels per warp
static_assert(kAttChunkKeys == kAttThreads, "one key of a chunk per thread");

struct AttSmem {
    alignas(128) uint8_t stage[kAttStages][kAttStageBytes];   // 73,728
    float4 spart[2][kAttWarps][2][32];                        // 8,192: partial scores per warp
    int slot[2][kAttChunkKeys];                               // physical slots of two chunks
    uint8_t soff[kAttStages][kAttStepKeys];                   // scale offset inside the 48-byte window
    uint32_t vmask[kAttStages];                               // valid keys of a staged step
};
constexpr size_t kAttSmemBytes = sizeof(AttSmem);

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
    float *part_o;                 // [2 * grid][16][576]
    float2 *part_ml;               // [2 * grid][16]: (m in the log2 domain, l)
    int n_win;                     // window steps per row: 8 (128 rows), or 0 without a window
    int n_st;                      // steps per row: n_win + ceil(k / 16)
    int64_t total_steps;           // R * n_st
};

// First step of CTA c's range (the same formula on host and device).
__host__ __device__ __forceinline__ int64_t att_range_start(int64_t total, int c, int grid) {
    return total * c / grid;
}

// CTA whose range holds step s.
__host__ __device__ __forceinline__ int att_cta_of(int64_t total, int64_t s, int grid) {
    int c = static_cast<int>(s * grid / total);
    while (c + 1 < grid && att_range_start(total, c + 1, grid) <= s) ++c;
    while (c > 0 && att_range_start(total, c, grid) > s) --c;
    return c;
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// bf16x2 -> f32 pair (exact).
__device__ __forceinline__ float2 bf16x2_f32(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

__device__ __forceinline__ uint32_t f32x2_f16x2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Power-of-two exponent e such that values up to m, scaled by 2^-e, are
// represented in f16 without overflow and with full relative precision for
// the largest ones: 0 for m in [2^-4, 2^15) (the common case, no scaling),
// else the exponent that puts m near 2^10. Clamped to [-100, 100].
__device__ __forceinline__ int f16_exponent(float m) {
    if (!(m > 0.0f) || (m >= 0.0625f && m < 32768.0f)) return 0;
    const int e = static_cast<int>((__float_as_uint(m) >> 23) & 0xffu) - 127 - 10;
    return max(-100, min(100, e));
}

// Row state of a query row resolved once per segment.
struct AttRow {
    int row, b, j, T, pos;   // T < 0: no valid key at all
};

__device__ __forceinline__ AttRow att_row(const AttParams &P, int row) {
    AttRow r;
    r.row = row;
    r.b = row / P.Sq;
    r.j = row - r.b * P.Sq;
    r.T = P.seq_lens[r.b];
    if (r.T < P.Sq || r.T > P.max_pages * kPage) r.T = -1;
    r.pos = r.T - P.Sq + r.j;
    return r;
}

__global__ void __launch_bounds__(kAttThreads, 2)
sparse_attn_kernel(const AttParams P) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    AttSmem &sm = *reinterpret_cast<AttSmem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tig = lane & 3;
    const int grid = static_cast<int>(gridDim.x);
    const int64_t st0 = att_range_start(P.total_steps, blockIdx.x, grid);
    const int n_my = static_cast<int>(att_range_start(P.total_steps, blockIdx.x + 1, grid) - st0);
    const int n_st = P.n_st;
    const int n_rows_swa = kWindow + P.Sq - 1;
    const int cbase = warp * kAttQuarter;            // this warp's first channel

    // ------------------------------------------------ staging helpers (all threads)
    // Physical slot (or -1) of key `t` of chunk `ch` of this CTA, in two
    // halves so the dependent loads can be spread over iterations.
    auto chunk_key = [&](int ch, int t, int &row, int &s) -> bool {
        const int64_t gs = st0 + static_cast<int64_t>(ch) * kAttChunkSteps + t / kAttStepKeys;
        if (gs >= st0 + n_my) return false;
        row = static_cast<int>(gs / n_st);
        s = static_cast<int>(gs - static_cast<int64_t>(row) * n_st);
        return s >= P.n_win;
    };
    auto load_idx = [&](int ch, int t, int &row_out) -> int {
        int row, s;
        row_out = -1;
        if (!chunk_key(ch, t, row, s)) return -1;
        const int i = (s - P.n_win) * kAttStepKeys + (t % kAttStepKeys);
        if (i >= P.k) return -1;
        row_out = row;
        return P.topk_idx[static_cast<int64_t>(row) * P.k + i];
    };
    // idx -> (checked) page-table entry; returns the physical slot or -1.
    auto resolve = [&](int row, int idx) -> int {
        if (row < 0 || idx < 0) return -1;
        const AttRow r = att_row(P, row);
        if (r.T < 0 || idx > r.pos) {               // past the query (causal) or a bad length
            flag_status(kStatusBounds);
            return -1;
        }
        const int64_t ph = P.page_table[static_cast<int64_t>(r.b) * P.max_pages + (idx >> 6)];
        if (ph < 0 || ph >= P.num_pages) {
            flag_status(kStatusBounds);
            return -1;
        }
        return static_cast<int>(ph * kPage + (idx & 63));
    };
    // Issue the copies of CTA step i into its stage (one commit group).
    auto issue = [&](int i) {
        if (i < n_my) {
            const int st = i % kAttStages;
            const int64_t gs = st0 + i;
            const int row = static_cast<int>(gs / n_st);
            const int s = static_cast<int>(gs - static_cast<int64_t>(row) * n_st);
            uint8_t *dst = sm.stage[st];
            if (s < P.n_win) {
                // 16 window rows: 16 x 72 chunks of 16 bytes, chunk c of key e
                // at position c ^ (e & 7) (conflict-free reads).
                const AttRow r = att_row(P, row);
                const int first = r.pos - (kWindow - 1) + s * kAttStepKeys;   // position of key 0
                const __nv_bfloat16 *src0 =
                    P.swa + (static_cast<int64_t>(r.b) * n_rows_swa + r.j + s * kAttStepKeys) * kDim;
#pragma unroll
                for (int m = 0; m < kAttStepKeys * (kDim / 8) / kAttThreads; ++m) {
                    const int c = tid + m * kAttThreads;
                    const int e = c / (kDim / 8), ch = c - e * (kDim / 8);
                    const bool ok = r.T >= 0 && first + e >= 0;
                    const uint8_t *src = reinterpret_cast<const uint8_t *>(ok ? src0 + e * kDim + ch * 8 : P.swa);
                    cp_async16(dst + e * (kDim * 2) + ((ch ^ (e & 7)) << 4), src, ok ? 16u : 0u);
                }
                if (warp == 0) {
                    const bool v = lane < kAttStepKeys && r.T >= 0 && first + lane >= 0;
                    const uint32_t m = __ballot_sync(0xffffffffu, v);
                    if (lane == 0) sm.vmask[st] = m;
                }
            } else {
                // 16 FP4 records (18 chunks each) + 16 scale windows (3 chunks).
                const int *sl = sm.slot[(i / kAttChunkSteps) & 1] + (i % kAttChunkSteps) * kAttStepKeys;
                for (int c = tid; c < kAttStepKeys * 21; c += kAttThreads) {
                    const int e = c / 21, part = c - e * 21;
                    const int slot = sl[e];
                    if (part < 18) {
                        const uint8_t *src = slot >= 0 ? P.kv_fp4 + static_cast<int64_t>(slot) * kFp4Bytes + part * 16
                                                       : P.kv_fp4;
                        cp_async16(dst + e * kFp4Bytes + part * 16, src, slot >= 0 ? 16u : 0u);
                    } else {
                        const int64_t sb = static_cast<int64_t>(slot) * kScaleBytes;
                        const uint8_t *src = slot >= 0 ? P.kv_scale + (sb & ~static_cast<int64_t>(15)) + (part - 18) * 16
                                                       : P.kv_scale;
                        cp_async16(dst + kAttRecBytes + e * kAttScaleWin + (part - 18) * 16, src, slot >= 0 ? 16u : 0u);
                        if (part == 18) sm.soff[st][e] = static_cast<uint8_t>(slot >= 0 ? (sb & 15) : 0);
                    }
                }
                if (warp == 0) {
                    const uint32_t m = __ballot_sync(0xffffffffu, lane < kAttStepKeys && sl[lane & 15] >= 0);
                    if (lane == 0) sm.vmask[st] = m;
                }
            }
        }
        cp_async_commit();
    };

    // ------------------------------------------------ per-row (segment) state
    uint32_t qa[9][4];          // query fragments (heads g, g + 8) of this warp's channels
    float q_mul = 1.0f;         // 2^eq: query exponent of this warp
    float o[18][4];             // O accumulator, units of 2^o_exp
    int o_exp = 0;
    float m_run[2], l_run[2];   // heads g, g + 8 (log2 domain)

    auto load_query = [&](int row) {
        const __nv_bfloat16 *qr = P.q + static_cast<int64_t>(row) * kHeads * kDim;
        uint4 v[2][4];
        uint2 tl[2];
        float mx = 0.0f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint4 *hp = reinterpret_cast<const uint4 *>(qr + (g + 8 * hh) * kDim + cbase);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                v[hh][2 * u] = __ldg(hp + (64 * u + 16 * tig) / 8);
                v[hh][2 * u + 1] = __ldg(hp + (64 * u + 16 * tig) / 8 + 1);
            }
            tl[hh] = __ldg(reinterpret_cast<const uint2 *>(qr + (g + 8 * hh) * kDim + cbase + 128 + 4 * tig));
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t w[10] = {v[hh][0].x, v[hh][0].y, v[hh][0].z, v[hh][0].w, v[hh][1].x, v[hh][1].y,
                                    v[hh][1].z, v[hh][1].w, tl[hh].x, tl[hh].y};
#pragma unroll
            for (int i = 0; i < 10; ++i) {
                const float2 f = bf16x2_f32(w[i]);
                mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float2 f = bf16x2_f32((&v[hh][2].x)[i]);
                mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const int eq = f16_exponent(mx);
        const float sdown = exp2f(static_cast<float>(-eq));
        q_mul = exp2f(static_cast<float>(eq));
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            // 16 channels per unit: k-step s of unit u takes channels 4s .. 4s+3
            // (words 2s, 2s+1); the tail k-step takes the tail's two words.
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint32_t w[8] = {v[hh][2 * u].x, v[hh][2 * u].y, v[hh][2 * u].z, v[hh][2 * u].w,
                                       v[hh][2 * u + 1].x, v[hh][2 * u + 1].y, v[hh][2 * u + 1].z,
                                       v[hh][2 * u + 1].w};
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const float2 a = bf16x2_f32(w[2 * s]), c = bf16x2_f32(w[2 * s + 1]);
                    qa[4 * u + s][hh] = f32x2_f16x2(a.x * sdown, a.y * sdown);        // a0 / a1
                    qa[4 * u + s][2 + hh] = f32x2_f16x2(c.x * sdown, c.y * sdown);    // a2 / a3
                }
            }
            const float2 a = bf16x2_f32(tl[hh].x), c = bf16x2_f32(tl[hh].y);
            qa[8][hh] = f32x2_f16x2(a.x * sdown, a.y * sdown);
            qa[8][2 + hh] = f32x2_f16x2(c.x * sdown, c.y * sdown);
        }
    };
    auto reset_row = [&]() {
#pragma unroll
        for (int n = 0; n < 18; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;
        o_exp = 0;
        m_run[0] = m_run[1] = -INFINITY;
        l_run[0] = l_run[1] = 0.0f;
    };
    // Result of the segment [s_first, s_last] of row r.
    auto finish_row = [&](const AttRow &r, int s_first, int s_last, int part_slot) {
        float l[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float v = l_run[hh];
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            l[hh] = v;
        }
        const float omul = exp2f(static_cast<float>(o_exp));
        const bool whole = s_first == 0 && s_last == n_st - 1;
        float *dst;
        float mul[2];
        if (whole) {
            dst = P.out + static_cast<int64_t>(r.row) * kHeads * kDim;
            mul[0] = l[0] > 0.0f ? omul / l[0] : 0.0f;
            mul[1] = l[1] > 0.0f ? omul / l[1] : 0.0f;
        } else {
            dst = P.part_o + static_cast<int64_t>(part_slot) * kHeads * kDim;
            mul[0] = mul[1] = omul;
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float *hrow = dst + (g + 8 * hh) * kDim + cbase;
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    const int n = 2 * (4 * u + s);
                    *reinterpret_cast<float4 *>(hrow + 64 * u + 16 * tig + 4 * s) =
                        make_float4(o[n][2 * hh] * mul[hh], o[n][2 * hh + 1] * mul[hh], o[n + 1][2 * hh] * mul[hh],
                                    o[n + 1][2 * hh + 1] * mul[hh]);
                }
            *reinterpret_cast<float4 *>(hrow + 128 + 4 * tig) =
                make_float4(o[16][2 * hh] * mul[hh], o[16][2 * hh + 1] * mul[hh], o[17][2 * hh] * mul[hh],
                            o[17][2 * hh + 1] * mul[hh]);
        }
        if (warp == 0 && tig == 0) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int h = g + 8 * hh;
                if (whole)
                    P.lse[static_cast<int64_t>(r.row) * kHeads + h] =
                        l[hh] > 0.0f ? (m_run[hh] + log2f(l[hh])) * 0.69314718055994530942f : -INFINITY;
                else
                    P.part_ml[static_cast<int64_t>(part_slot) * kHeads + h] = make_float2(m_run[hh], l[hh]);
            }
        }
    };

    if (n_my <= 0) return;                              // no work (uniform)

    // ------------------------------------------------ prologue
    // The query, window rows, lengths and page table are inputs no earlier
    // kernel of the step writes: the first row's query fragments load before
    // the wait for the selection.
    int64_t gs = st0;
    int row = static_cast<int>(gs / n_st);
    int s = static_cast<int>(gs - static_cast<int64_t>(row) * n_st);
    load_query(row);
    reset_row();
    pdl_wait();                                         // the top-k indices are ready
    pdl_trigger();
    {
        int rr;
        const int idx = load_idx(0, tid, rr);
        sm.slot[0][tid] = resolve(rr, idx);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kAttAhead; ++i) issue(i);

    AttRow cur = att_row(P, row);
    if (cur.T < 0 && tid == 0) flag_status(kStatusBounds);
    int seg_first = s;                                   // first step of the current segment
    int seg_no = 0;                                      // segments finished so far
    int nrow = -1, nidx = -1;                            // slot resolution of the next chunk in flight
    int32_t npage = -1;

    for (int i = 0; i < n_my; ++i) {
        // ---- next chunk's slots: index load, page load, store (two steps apart)
        const int ch = i / kAttChunkSteps, ph = i % kAttChunkSteps;
        if (ph == 0) nidx = load_idx(ch + 1, tid, nrow);
        if (ph == 2) {
            npage = -1;
            if (nrow >= 0 && nidx >= 0) {
                const AttRow r = att_row(P, nrow);
                if (r.T >= 0 && nidx <= r.pos) npage = P.page_table[static_cast<int64_t>(r.b) * P.max_pages + (nidx >> 6)];
            }
        }
        if (ph == 4) {
            int slot = -1;
            if (nrow >= 0 && nidx >= 0) {
                const AttRow r = att_row(P, nrow);
                if (r.T < 0 || nidx > r.pos || npage < 0 || npage >= P.num_pages) flag_status(kStatusBounds);
                else slot = npage * kPage + (nidx & 63);
            }
            sm.slot[(ch + 1) & 1][tid] = slot;
        }
        issue(i + kAttAhead);
        cp_async_wait<kAttAhead>();                     // step i has landed (this thread's copies)
        __syncthreads();                                // ... everyone's; slot stores visible

        const int st = i % kAttStages;
        const uint8_t *stg = sm.stage[st];
        const uint32_t vm = sm.vmask[st];
        const bool win = s < P.n_win;

        // ---- key fragments of keys g and g + 8 (n-tiles 0, 1)
        uint32_t kb[2][9][2];
        int k_exp = 0;
        if (!win) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int e = nt * 8 + g;
                const uint8_t *rec = stg + e * kFp4Bytes + cbase / 2;
                const uint8_t *sc = stg + kAttRecBytes + e * kAttScaleWin + sm.soff[st][e] + warp * 9;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint2 rv = *reinterpret_cast<const uint2 *>(rec + 32 * u + 8 * tig);
                    const uint32_t s2 = e4m3x2_to_f16x2(static_cast<uint32_t>(sc[4 * u + tig]) * 0x0101u);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t wv = q < 2 ? rv.x : rv.y;
                        kb[nt][4 * u + q][0] = hmul2_u32(e2m1x2_to_f16x2((wv >> (16 * (q & 1))) & 0xffu), s2);
                        kb[nt][4 * u + q][1] = hmul2_u32(e2m1x2_to_f16x2((wv >> (16 * (q & 1) + 8)) & 0xffu), s2);
                    }
                }
                const uint32_t tv = *reinterpret_cast<const unsigned short *>(rec + 64 + 2 * tig);
                const uint32_t s2 = e4m3x2_to_f16x2(static_cast<uint32_t>(sc[8]) * 0x0101u);
                kb[nt][8][0] = hmul2_u32(e2m1x2_to_f16x2(tv & 0xffu), s2);
                kb[nt][8][1] = hmul2_u32(e2m1x2_to_f16x2(tv >> 8), s2);
            }
        } else {
            // bf16 window rows: read, take this warp's maximum, convert under
            // the exponent that keeps them in f16 range.
            uint4 w4[2][4];
            uint2 w2[2];
            float mx = 0.0f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int e = nt * 8 + g;
                const uint8_t *rowp = stg + e * (kDim * 2);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c0 = (cbase + 64 * u + 16 * tig) / 8;        // 16-byte chunk of channel base
                    w4[nt][2 * u] = *reinterpret_cast<const uint4 *>(rowp + ((c0 ^ (e & 7)) << 4));
                    w4[nt][2 * u + 1] = *reinterpret_cast<const uint4 *>(rowp + (((c0 + 1) ^ (e & 7)) << 4));
                }
                const int ct = cbase + 128 + 4 * tig;
                w2[nt] = *reinterpret_cast<const uint2 *>(rowp + (((ct / 8) ^ (e & 7)) << 4) + (ct % 8) * 2);
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
                    const uint32_t wv[4] = {w4[nt][i4].x, w4[nt][i4].y, w4[nt][i4].z, w4[nt][i4].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 f = bf16x2_f32(wv[q]);
                        mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
                    }
                }
                const float2 f0 = bf16x2_f32(w2[nt].x), f1 = bf16x2_f32(w2[nt].y);
                mx = fmaxf(mx, fmaxf(fmaxf(fabsf(f0.x), fabsf(f0.y)), fmaxf(fabsf(f1.x), fabsf(f1.y))));
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            k_exp = f16_exponent(mx);
            const float sdown = exp2f(static_cast<float>(-k_exp));
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint32_t wv[8] = {w4[nt][2 * u].x, w4[nt][2 * u].y, w4[nt][2 * u].z, w4[nt][2 * u].w,
                                            w4[nt][2 * u + 1].x, w4[nt][2 * u + 1].y, w4[nt][2 * u + 1].z,
                                            w4[nt][2 * u + 1].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 a = bf16x2_f32(wv[2 * q]), c = bf16x2_f32(wv[2 * q + 1]);
                        kb[nt][4 * u + q][0] = f32x2_f16x2(a.x * sdown, a.y * sdown);
                        kb[nt][4 * u + q][1] = f32x2_f16x2(c.x * sdown, c.y * sdown);
                    }
                }
                const float2 a = bf16x2_f32(w2[nt].x), c = bf16x2_f32(w2[nt].y);
                kb[nt][8][0] = f32x2_f16x2(a.x * sdown, a.y * sdown);
                kb[nt][8][1] = f32x2_f16x2(c.x * sdown, c.y * sdown);
            }
        }

        // ---- partial scores over this warp's channels
        float acc[2][2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int a = 0; a < 2; ++a) acc[nt][a][0] = acc[nt][a][1] = acc[nt][a][2] = acc[nt][a][3] = 0.0f;
#pragma unroll
        for (int ks = 0; ks < 9; ++ks)
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
                mma_f16_16816(acc[nt][ks & 1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], kb[nt][ks][0],
                              kb[nt][ks][1]);
        {
            const float smul = q_mul * exp2f(static_cast<float>(k_exp));   // undo the two exponents
            float4 p0 = make_float4((acc[0][0][0] + acc[0][1][0]) * smul, (acc[0][0][1] + acc[0][1][1]) * smul,
                                    (acc[0][0][2] + acc[0][1][2]) * smul, (acc[0][0][3] + acc[0][1][3]) * smul);
            float4 p1 = make_float4((acc[1][0][0] + acc[1][1][0]) * smul, (acc[1][0][1] + acc[1][1][1]) * smul,
                                    (acc[1][0][2] + acc[1][1][2]) * smul, (acc[1][0][3] + acc[1][1][3]) * smul);
            sm.spart[i & 1][warp][0][lane] = p0;
            sm.spart[i & 1][warp][1][lane] = p1;
        }
        // value fragments: the key fragments transposed (keys = values)
        uint32_t vb[9][2][2];
#pragma unroll
        for (int ks = 0; ks < 9; ++ks)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                vb[ks][h][0] = movmatrix_t(kb[0][ks][h]);
                vb[ks][h][1] = movmatrix_t(kb[1][ks][h]);
            }
        __syncthreads();                                // all partial scores are in shared memory

        // ---- full scores (same summation order in every warp), online softmax
        float sc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float4 t = sm.spart[i & 1][0][nt][lane];
#pragma unroll
            for (int w = 1; w < kAttWarps; ++w) {
                const float4 u4 = sm.spart[i & 1][w][nt][lane];
                t.x += u4.x;
                t.y += u4.y;
                t.z += u4.z;
                t.w += u4.w;
            }
            // keys of this lane: nt * 8 + 2 tig + {0, 1}; c0/c1 head g, c2/c3 head g + 8
            const bool v0 = (vm >> (nt * 8 + 2 * tig)) & 1u, v1 = (vm >> (nt * 8 + 2 * tig + 1)) & 1u;
            sc[nt][0] = v0 ? t.x * P.scale_log2 : -INFINITY;
            sc[nt][1] = v1 ? t.y * P.scale_log2 : -INFINITY;
            sc[nt][2] = v0 ? t.z * P.scale_log2 : -INFINITY;
            sc[nt][3] = v1 ? t.w * P.scale_log2 : -INFINITY;
        }
        float alpha[2];
        uint32_t pa[4];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float mx = fmaxf(fmaxf(sc[0][2 * hh], sc[0][2 * hh + 1]), fmaxf(sc[1][2 * hh], sc[1][2 * hh + 1]));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            // The running maximum moves only when the step's maximum passes it
            // by more than 8 (probabilities stay below 2^8, exact in f16 range).
            const float m_new = (mx > m_run[hh] + 8.0f || m_run[hh] == -INFINITY) ? mx : m_run[hh];
            alpha[hh] = (m_new == m_run[hh] || m_run[hh] == -INFINITY) ? 1.0f : exp2f(m_run[hh] - m_new);
            if (m_run[hh] == -INFINITY) alpha[hh] = 1.0f;      // O and l are still zero
            m_run[hh] = m_new;
            float p[2][2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float x = sc[nt][2 * hh + e];
                    p[nt][e] = (m_new == -INFINITY || x == -INFINITY) ? 0.0f : exp2f(x - m_new);
                }
            const __half2 h0 = __floats2half2_rn(p[0][0], p[0][1]);
            const __half2 h1 = __floats2half2_rn(p[1][0], p[1][1]);
            const float2 r0 = __half22float2(h0), r1 = __half22float2(h1);
            l_run[hh] = l_run[hh] * alpha[hh] + (r0.x + r0.y + r1.x + r1.y);
            pa[hh] = *reinterpret_cast<const uint32_t *>(&h0);          // a0 (head g) / a1 (head g + 8)
            pa[2 + hh] = *reinterpret_cast<const uint32_t *>(&h1);      // a2 / a3
        }
        // ---- O = alpha O + P V, keeping O in units of 2^k_exp for this step
        {
            const float ex = exp2f(static_cast<float>(o_exp - k_exp));
            const float a0 = alpha[0] * ex, a1 = alpha[1] * ex;
            if (__any_sync(0xffffffffu, a0 != 1.0f || a1 != 1.0f)) {
#pragma unroll
                for (int n = 0; n < 18; ++n) {
                    o[n][0] *= a0;
                    o[n][1] *= a0;
                    o[n][2] *= a1;
                    o[n][3] *= a1;
                }
            }
            o_exp = k_exp;
        }
#pragma unroll
        for (int ks = 0; ks < 9; ++ks)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                mma_f16_16816(o[2 * ks + h], pa[0], pa[1], pa[2], pa[3], vb[ks][h][0], vb[ks][h][1]);

        // ---- segment end: the row ends here or the range does
        const bool last_of_row = s == n_st - 1;
        if (last_of_row || i == n_my - 1) {
            // partial slot: the first segment of the range uses 2c, a later one 2c + 1
            finish_row(cur, seg_first, s, 2 * static_cast<int>(blockIdx.x) + (seg_no > 0 ? 1 : 0));
            ++seg_no;
            if (i + 1 < n_my) {
                ++row;
                s = 0;
                seg_first = 0;
                cur = att_row(P, row);
                if (cur.T < 0 && tid == 0) flag_status(kStatusBounds);
                load_query(row);
                reset_row();
            }
        } else {
            ++s;
        }
    }
    cp_async_wait<0>();
}

// K5: merge the partials of the rows whose steps were split over CTAs:
// O = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c. One CTA per (query row,
// group of 4 heads); a row held whole by one CTA was written by K4 and is
// skipped. CTA c holds its partial of the row in slot 2c, except the first
// CTA covering the row when its range began in an earlier row (then the row
// is its second segment: slot 2c + 1). Each thread owns 3 float4 of the
// group's 4 x 576 outputs and loads the partials 4 at a time.
constexpr int kMergeThreads = 192;
constexpr int kMergeHeads = 4;
constexpr int kMergeVec = kMergeHeads * kDim / 4;        // 576 float4 per CTA
constexpr int kMergePer = kMergeVec / kMergeThreads;    // 3

__global__ void __launch_bounds__(kMergeThreads)
attn_merge_kernel(const float *__restrict__ part_o, const float2 *__restrict__ part_ml, int64_t total_steps,
                  int n_st, int grid, float *__restrict__ out, float *__restrict__ lse) {
    __shared__ float s_red[kMergeThreads / 32][kMergeHeads];
    __shared__ float s_M[kMergeHeads], s_L[kMergeHeads];
    pdl_wait();
    pdl_trigger();
    const int row = blockIdx.x, hg = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t r0 = static_cast<int64_t>(row) * n_st, r1 = r0 + n_st - 1;
    const int c0 = att_cta_of(total_steps, r0, grid), c1 = att_cta_of(total_steps, r1, grid);
    if (c0 == c1) return;                                 // one CTA held the row: already final
    const int n_parts = c1 - c0 + 1;
    const int first_slot = 2 * c0 + (att_range_start(total_steps, c0, grid) < r0 ? 1 : 0);
    auto slot_of = [&](int p) { return p == 0 ? first_slot : 2 * (c0 + p); };
    const float2 *ml = part_ml + hg * kMergeHeads;

    // block-wide reduction of one value per head (op 0: max, 1: sum)
    auto reduce4 = [&](float (&v)[kMergeHeads], int op, float *dst) {
#pragma unroll
        for (int h = 0; h < kMergeHeads; ++h) {
            float x = v[h];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float y = __shfl_xor_sync(0xffffffffu, x, off);
                x = op == 0 ? fmaxf(x, y) : x + y;
            }
            if (lane == 0) s_red[warp][h] = x;
        }
        __syncthreads();
        if (tid < kMergeHeads) {
            float x = s_red[0][tid];
            for (int w = 1; w < kMergeThreads / 32; ++w) x = op == 0 ? fmaxf(x, s_red[w][tid]) : x + s_red[w][tid];
            dst[tid] = x;
        }
        __syncthreads();
    };
    float mv[kMergeHeads];
#pragma unroll
    for (int h = 0; h < kMergeHeads; ++h) mv[h] = -INFINITY;
    for (int p = tid; p < n_parts; p += kMergeThreads) {
        const int64_t sl = slot_of(p);
#pragma unroll
        for (int h = 0; h < kMergeHeads; ++h) {
            const float2 v = __ldcg(ml + sl * kHeads + h);
            if (v.y > 0.0f) mv[h] = fmaxf(mv[h], v.x);
        }
    }
    reduce4(mv, 0, s_M);
    float lv[kMergeHeads];
#pragma unroll
    for (int h = 0; h < kMergeHeads; ++h) lv[h] = 0.0f;
    for (int p = tid; p < n_parts; p += kMergeThreads) {
        const int64_t sl = slot_of(p);
#pragma unroll
        for (int h = 0; h < kMergeHeads; ++h) {
            const float2 v = __ldcg(ml + sl * kHeads + h);
            if (v.y > 0.0f) lv[h] += exp2f(v.x - s_M[h]) * v.y;
        }
    }
    reduce4(lv, 1, s_L);

    constexpr int kRowVec = kHeads * kDim / 4;              // 2304 float4 per partial
    const float4 *po = reinterpret_cast<const float4 *>(part_o) + hg * kMergeVec;
    float4 acc[kMergePer];
    int hc[kMergePer];
#pragma unroll
    for (int c = 0; c < kMergePer; ++c) {
        acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        hc[c] = (c * kMergeThreads + tid) / (kDim / 4);
    }
    for (int p0 = 0; p0 < n_parts; p0 += 4) {
        float4 v[4][kMergePer];
        float wt[4][kMergePer];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const bool live = p0 + u < n_parts;
            const int64_t sl = live ? slot_of(p0 + u) : 0;
#pragma unroll
            for (int c = 0; c < kMergePer; ++c) {
                v[u][c] = live ? __ldcg(po + sl * kRowVec + c * kMergeThreads + tid) : make_float4(0.f, 0.f, 0.f, 0.f);
                const float2 m = live ? __ldcg(ml + sl * kHeads + hc[c]) : make_float2(0.f, 0.f);
                wt[u][c] = m.y > 0.0f ? exp2f(m.x - s_M[hc[c]]) : 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int c = 0; c < kMergePer; ++c) {
                acc[c].x += wt[u][c] * v[u][c].x;
                acc[c].y += wt[u][c] * v[u][c].y;
                acc[c].z += wt[u][c] * v[u][c].z;
                acc[c].w += wt[u][c] * v[u][c].w;
            }
    }
    float4 *orow = reinterpret_cast<float4 *>(out + static_cast<int64_t>(row) * kHeads * kDim) + hg * kMergeVec;
#pragma unroll
    for (int c = 0; c < kMergePer; ++c) {
        const float L = s_L[hc[c]];
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        orow[c * kMergeThreads + tid] = make_float4(acc[c].x * inv, acc[c].y * inv, acc[c].z * inv, acc[c].w * inv);
    }
    if (tid < kMergeHeads) {
        const float L = s_L[tid];
        lse[static_cast<int64_t>(row) * kHeads + hg * kMergeHeads + tid] =
            L > 0.0f ? (s_M[tid] + log2f(L)) * 0.69314718055994530942f : -INFINITY;
    }
}

// K8: one softmax over disjoint key sets from per-part results (context-
// parallel shards): with L = log sum_p exp(lse_p), out = sum_p exp(lse_p - L)
// o_p and lse = L; a part with lse = -inf (no key) weighs 0. One CTA per
// (query row, group of 4 heads), parts in the natural-log domain.
__global__ void __launch_bounds__(kMergeThreads)
lse_merge_kernel(const float *__restrict__ o_parts, const float *__restrict__ lse_parts, int n_parts, int R,
                 float *__restrict__ out, float *__restrict__ lse) {
    __shared__ float s_M[kMergeHeads], s_S[kMergeHeads];
    pdl_wait();
    pdl_trigger();
    const int row = blockIdx.x, hg = blockIdx.y, tid = threadIdx.x;
    if (tid < kMergeHeads) {
        float M = -INFINITY;
        for (int p = 0; p < n_parts; ++p)
            M = fmaxf(M, __ldg(lse_parts + (static_cast<int64_t>(p) * R + row) * kHeads + hg * kMergeHeads + tid));
        float S = 0.0f;
        if (M != -INFINITY)
            for (int p = 0; p < n_parts; ++p) {
                const float l = __ldg(lse_parts + (static_cast<int64_t>(p) * R + row) * kHeads + hg * kMergeHeads + tid);
                if (l != -INFINITY) S += expf(l - M);
            }
        s_M[tid] = M;
        s_S[tid] = S;
        lse[static_cast<int64_t>(row) * kHeads + hg * kMergeHeads + tid] = S > 0.0f ? M + logf(S) : -INFINITY;
    }
    __syncthreads();
    constexpr int kRowVec = kHeads * kDim / 4;
    float4 acc[kMergePer];
#pragma unroll
    for (int c = 0; c < kMergePer; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p = 0; p < n_parts; ++p) {
        const float4 *po = reinterpret_cast<const float4 *>(o_parts) + (static_cast<int64_t>(p) * R + row) * kRowVec +
                           hg * kMergeVec;
#pragma unroll
        for (int c = 0; c < kMergePer; ++c) {
            const int h = (c * kMergeThreads + tid) / (kDim / 4);
            const float l = __ldg(lse_parts + (static_cast<int64_t>(p) * R + row) * kHeads + hg * kMergeHeads + h);
            if (l == -INFINITY || s_S[h] == 0.0f) continue;
            const float wt = expf(l - s_M[h]) / s_S[h];
            const float4 v = __ldg(po + c * kMergeThreads + tid);
            acc[c].x += wt * v.x;
            acc[c].y += wt * v.y;
            acc[c].z += wt * v.z;
            acc[c].w += wt * v.w;
        }
    }
    float4 *orow = reinterpret_cast<float4 *>(out + static_cast<int64_t>(row) * kHeads * kDim) + hg * kMergeVec;
#pragma unroll
    for (int c = 0; c < kMergePer; ++c) orow[c * kMergeThreads + tid] = acc[c];
}

}  // namespace csa2
