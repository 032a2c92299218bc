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
// K4, one CTA = 9 warps; warp w owns the 64-channel unit [64 w, 64 w + 64)
// (scale groups 4w .. 4w + 3) of every key, query head and output:
//   staging  cp.async copies of the packed FP4 records and scales (or the bf16
//            window rows) of step i + 4 into the stage step i has just
//            released (4-stage ring), zero-filled for empty keys. Physical slots (top-k index -> page table) are
//            resolved a chunk of 8 steps ahead, each load issued two steps
//            before its value is used.
//   QK       lane (g, tig) converts keys g and g + 8 of the step straight into
//            m16n8k16 B fragments: in k-step s it takes channels
//            16 tig + 4 s .. + 3 of the unit, so its four k-steps are one
//            8-byte load and one scale; the query fragments (held in
//            registers for the row) use the same order, so each product
//            q_c k_c is summed once. FP4 -> f16 is the hardware E2M1x2
//            conversion times the E4M3 scale (exact in f16); the window's
//            bf16 -> f16 goes through a per-warp power-of-two exponent that
//            keeps it in range.
//   softmax  the nine warps' partial scores meet in shared memory; warp w < 8
//            sums them for heads 2w, 2w + 1 (one key per lane) and runs the
//            online softmax of those heads (exp2 domain, exact running
//            maximum, probabilities rounded to f16, the same values feed the
//            sum), writing the f16 probabilities and the rescale factors.
//   PV       movmatrix transposes the key fragments of QK into the value
//            fragments (keys = values), so the value tile never goes to
//            shared memory; the probabilities are the A operand (ldmatrix).
//            The O accumulator (16 heads x 64 channels) stays in registers
//            with a per-warp power-of-two exponent.
// Warp-level mma.sync is used deliberately: with 16 heads the MMA N extent is
// 16, and at that width the warp MMAs issue faster than tcgen05 single-thread
// MMAs. Two barriers per step: the partial scores are complete (and the step's
// stage is free), and the probabilities together with the next step's stage.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kAttWarps = 9;                                   // one 64-channel unit each
constexpr int kAttThreads = kAttWarps * 32;                    // 288
constexpr int kAttStepKeys = 16;
constexpr int kAttWinSteps = kWindow / kAttStepKeys;          // 8
constexpr int kAttStageBytes = kAttStepKeys * kDim * 2;       // 18,432: 16 window rows of bf16
constexpr int kAttRecBytes = kAttStepKeys * kFp4Bytes;        // 4,608: 16 packed FP4 records
constexpr int kAttScaleWin = 48;                              // 16-byte aligned window holding 36 scale bytes
constexpr int kAttStages = 4;
constexpr int kAttChunkSteps = 8;                             // steps per slot-resolution chunk
constexpr int kAttChunkKeys = kAttChunkSteps * kAttStepKeys;  // 128 (threads 0..127 resolve one key each)
constexpr int kAttUnit = 64;                                  // channels per warp
static_assert(kAttWarps * kAttUnit == kDim, "nine 64-channel units");

struct AttSmem {
    alignas(128) uint8_t stage[kAttStages][kAttStageBytes];   // 73,728
    float4 spart[2][kAttWarps][2][32];                        // 18,432: partial scores per warp
    alignas(16) uint8_t p16[kHeads * kAttStepKeys * 2];       // 512: f16 probabilities [head][key], chunks swizzled
    float alpha[kHeads];                                      // rescale of O for this step, per head
    float l_fin[kHeads];                                      // running sum, m_fin: running max (segment end)
    float m_fin[kHeads];
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

__global__ void __maxnreg__(104)
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
    const int cbase = warp * kAttUnit;                 // this warp's first channel

    // ------------------------------------------------ staging helpers
    // (row, step-in-row) of CTA step i, by division (used once per chunk).
    auto step_of = [&](int i, int &row, int &s) {
        const int64_t gs = st0 + i;
        row = static_cast<int>(gs / n_st);
        s = static_cast<int>(gs - static_cast<int64_t>(row) * n_st);
    };
    // Top-k index of key t (< 128) of chunk ch, or -1 (window step, padding, past the range).
    auto load_idx = [&](int ch, int t, int &row_out) -> int {
        row_out = -1;
        const int i = ch * kAttChunkSteps + t / kAttStepKeys;
        if (t >= kAttChunkKeys || i >= n_my) return -1;
        int row, s;
        step_of(i, row, s);
        if (s < P.n_win) return -1;
        const int e = (s - P.n_win) * kAttStepKeys + (t % kAttStepKeys);
        if (e >= P.k) return -1;
        row_out = row;
        return P.topk_idx[static_cast<int64_t>(row) * P.k + e];
    };
    // Issue the copies of CTA step i (its row and step given) into its stage (one commit group).
    auto issue = [&](int i, int row, int s) {
        if (i < n_my) {
            const int st = i % kAttStages;
            uint8_t *dst = sm.stage[st];
            if (s < P.n_win) {
                // 16 window rows: 16 x 72 chunks of 16 bytes, chunk c of key e
                // at position c ^ (e & 7) (conflict-free reads).
                const AttRow r = att_row(P, row);
                const int first = r.pos - (kWindow - 1) + s * kAttStepKeys;   // position of key 0
                const __nv_bfloat16 *src0 =
                    P.swa + (static_cast<int64_t>(r.b) * n_rows_swa + r.j + s * kAttStepKeys) * kDim;
                for (int c = tid; c < kAttStepKeys * (kDim / 8); c += kAttThreads) {
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
    uint32_t qa[4][4];          // query fragments (heads g, g + 8) of this warp's unit
    float q_mul = 1.0f;         // 2^eq: query exponent of this warp
    float o[8][4];              // O accumulator (heads g, g + 8 x the unit), units of 2^o_exp
    int o_exp = 0;
    float m_run = -INFINITY, l_run = 0.0f;   // softmax lanes: head 2 warp + (lane >> 4)

    auto load_query = [&](int row) {
        const __nv_bfloat16 *qr = P.q + static_cast<int64_t>(row) * kHeads * kDim;
        uint4 v[2][2];
        float mx = 0.0f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint4 *hp = reinterpret_cast<const uint4 *>(qr + (g + 8 * hh) * kDim + cbase + 16 * tig);
            v[hh][0] = __ldg(hp);
            v[hh][1] = __ldg(hp + 1);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float2 f = bf16x2_f32((&v[hh][0].x)[i]);
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
            // k-step s takes channels 16 tig + 4 s .. + 3 (words 2s, 2s + 1 of the lane's 16 channels)
#pragma unroll
            for (int st = 0; st < 4; ++st) {
                const float2 a = bf16x2_f32((&v[hh][0].x)[2 * st]), c = bf16x2_f32((&v[hh][0].x)[2 * st + 1]);
                qa[st][hh] = f32x2_f16x2(a.x * sdown, a.y * sdown);        // a0 / a1
                qa[st][2 + hh] = f32x2_f16x2(c.x * sdown, c.y * sdown);    // a2 / a3
            }
        }
    };
    auto reset_row = [&]() {
#pragma unroll
        for (int n = 0; n < 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;
        o_exp = 0;
        m_run = -INFINITY;
        l_run = 0.0f;
    };
    // Result of the segment [s_first, s_last] of row r (all threads).
    auto finish_row = [&](const AttRow &r, int s_first, int s_last, int part_slot) {
        if (warp < kHeads / 2 && (lane & 15) == 0) {
            const int h = 2 * warp + (lane >> 4);
            sm.l_fin[h] = l_run;
            sm.m_fin[h] = m_run;
        }
        __syncthreads();
        const float l0 = sm.l_fin[g], l1 = sm.l_fin[g + 8];
        const float omul = exp2f(static_cast<float>(o_exp));
        const bool whole = s_first == 0 && s_last == n_st - 1;
        float *dst;
        float mul[2];
        if (whole) {
            dst = P.out + static_cast<int64_t>(r.row) * kHeads * kDim;
            mul[0] = l0 > 0.0f ? omul / l0 : 0.0f;
            mul[1] = l1 > 0.0f ? omul / l1 : 0.0f;
        } else {
            dst = P.part_o + static_cast<int64_t>(part_slot) * kHeads * kDim;
            mul[0] = mul[1] = omul;
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float *hrow = dst + (g + 8 * hh) * kDim + cbase + 16 * tig;
#pragma unroll
            for (int st = 0; st < 4; ++st) {
                const int n = 2 * st;
                *reinterpret_cast<float4 *>(hrow + 4 * st) =
                    make_float4(o[n][2 * hh] * mul[hh], o[n][2 * hh + 1] * mul[hh], o[n + 1][2 * hh] * mul[hh],
                                o[n + 1][2 * hh + 1] * mul[hh]);
            }
        }
        if (tid < kHeads) {
            const float l = sm.l_fin[tid], m = sm.m_fin[tid];
            if (whole)
                P.lse[static_cast<int64_t>(r.row) * kHeads + tid] =
                    l > 0.0f ? (m + log2f(l)) * 0.69314718055994530942f : -INFINITY;
            else
                P.part_ml[static_cast<int64_t>(part_slot) * kHeads + tid] = make_float2(m, l);
        }
    };

    if (n_my <= 0) return;                              // no work (uniform)

    // ------------------------------------------------ prologue
    // The query, window rows, lengths and page table are inputs no earlier
    // kernel of the step writes: the first row's query fragments load before
    // the wait for the selection.
    int row, s;
    step_of(0, row, s);
    load_query(row);
    reset_row();
    pdl_wait();                                         // the top-k indices are ready
    pdl_trigger();
    {
        int rr;
        const int idx = load_idx(0, tid, rr);
        int slot = -1;
        if (rr >= 0 && idx >= 0) {
            const AttRow r = att_row(P, rr);
            if (r.T < 0 || idx > r.pos) {               // past the query (causal) or a bad length
                flag_status(kStatusBounds);
            } else {
                const int64_t ph = P.page_table[static_cast<int64_t>(r.b) * P.max_pages + (idx >> 6)];
                if (ph < 0 || ph >= P.num_pages) flag_status(kStatusBounds);
                else slot = static_cast<int>(ph * kPage + (idx & 63));
            }
        }
        if (tid < kAttChunkKeys) sm.slot[0][tid] = slot;
    }
    __syncthreads();
    // the issue pointer (row, step) runs kAttStages steps ahead of the compute pointer
    int irow = row, is = s;
    for (int i = 0; i < kAttStages; ++i) {
        issue(i, irow, is);
        if (++is == n_st) { is = 0; ++irow; }
    }
    cp_async_wait<kAttStages - 1>();                    // step 0 has landed (this thread's copies)
    __syncthreads();                                    // ... everyone's

    AttRow cur = att_row(P, row);
    if (cur.T < 0 && tid == 0) flag_status(kStatusBounds);
    int seg_first = s;                                   // first step of the current segment
    int seg_no = 0;                                      // segments finished so far
    int nrow = -1, nidx = -1;                            // slot resolution of the next chunk in flight
    int64_t npage = -1;
    const int sh = warp < kHeads / 2 ? 2 * warp + (lane >> 4) : 0;     // softmax head of this lane
    const int sk = lane & 15;                                          // softmax key of this lane

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
        if (ph == 4 && tid < kAttChunkKeys) {
            int slot = -1;
            if (nrow >= 0 && nidx >= 0) {
                const AttRow r = att_row(P, nrow);
                if (r.T < 0 || nidx > r.pos || npage < 0 || npage >= P.num_pages) flag_status(kStatusBounds);
                else slot = static_cast<int>(npage * kPage + (nidx & 63));
            }
            sm.slot[(ch + 1) & 1][tid] = slot;
        }
        // step i's stage is complete and visible (barrier at the end of the previous step)
        const int st = i % kAttStages;
        const uint8_t *stg = sm.stage[st];
        const uint32_t vm = sm.vmask[st];
        const bool win = s < P.n_win;

        // ---- key fragments of keys g and g + 8 (n-tiles 0, 1)
        uint32_t kb[2][4][2];
        int k_exp = 0;
        if (!win) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int e = nt * 8 + g;
                const uint2 rv = *reinterpret_cast<const uint2 *>(stg + e * kFp4Bytes + cbase / 2 + 8 * tig);
                const uint8_t sc = stg[kAttRecBytes + e * kAttScaleWin + sm.soff[st][e] + 4 * warp + tig];
                const uint32_t s2 = e4m3x2_to_f16x2(static_cast<uint32_t>(sc) * 0x0101u);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t wv = q < 2 ? rv.x : rv.y;
                    kb[nt][q][0] = hmul2_u32(e2m1x2_to_f16x2((wv >> (16 * (q & 1))) & 0xffu), s2);
                    kb[nt][q][1] = hmul2_u32(e2m1x2_to_f16x2((wv >> (16 * (q & 1) + 8)) & 0xffu), s2);
                }
            }
        } else {
            // bf16 window rows: read, take this warp's maximum, convert under
            // the exponent that keeps them in f16 range.
            uint4 w4[2][2];
            float mx = 0.0f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int e = nt * 8 + g;
                const uint8_t *rowp = stg + e * (kDim * 2);
                const int c0 = (cbase + 16 * tig) / 8;                     // 16-byte chunk of the lane's channels
                w4[nt][0] = *reinterpret_cast<const uint4 *>(rowp + ((c0 ^ (e & 7)) << 4));
                w4[nt][1] = *reinterpret_cast<const uint4 *>(rowp + (((c0 + 1) ^ (e & 7)) << 4));
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float2 f = bf16x2_f32((&w4[nt][0].x)[q]);
                    mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            k_exp = f16_exponent(mx);
            const float sdown = exp2f(static_cast<float>(-k_exp));
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 a = bf16x2_f32((&w4[nt][0].x)[2 * q]), c = bf16x2_f32((&w4[nt][0].x)[2 * q + 1]);
                    kb[nt][q][0] = f32x2_f16x2(a.x * sdown, a.y * sdown);
                    kb[nt][q][1] = f32x2_f16x2(c.x * sdown, c.y * sdown);
                }
        }

        // ---- partial scores over this warp's unit
        {
            float acc[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
                    mma_f16_16816(acc[nt], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], kb[nt][ks][0], kb[nt][ks][1]);
            const float smul = q_mul * exp2f(static_cast<float>(k_exp)) * P.scale_log2;   // undo the exponents
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
                sm.spart[i & 1][warp][nt][lane] =
                    make_float4(acc[nt][0] * smul, acc[nt][1] * smul, acc[nt][2] * smul, acc[nt][3] * smul);
        }
        // value fragments: the key fragments transposed (keys = values)
        uint32_t vb[4][2][2];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                vb[ks][h][0] = movmatrix_t(kb[0][ks][h]);
                vb[ks][h][1] = movmatrix_t(kb[1][ks][h]);
            }
        __syncthreads();                                // all partial scores are in; step i's stage is free
        // stage the copies of step i + 4 into the stage step i no longer reads
        issue(i + kAttStages, irow, is);
        if (++is == n_st) { is = 0; ++irow; }

        // ---- softmax of heads 2 warp, 2 warp + 1 (warps 0..7), one key per lane
        if (warp < kHeads / 2) {
            // partial of (head sh, key sk) sits in lane (sh % 8) * 4 + (sk % 8) / 2 of n-tile sk / 8,
            // component (sh / 8) * 2 + sk % 2
            const int L = (sh & 7) * 4 + ((sk & 7) >> 1), nt = sk >> 3, comp = (sh >> 3) * 2 + (sk & 1);
            float x = 0.0f;
#pragma unroll
            for (int w = 0; w < kAttWarps; ++w) x += (&sm.spart[i & 1][w][nt][L].x)[comp];
            x = ((vm >> sk) & 1u) ? x : -INFINITY;
            float mx = x;
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_new = fmaxf(m_run, mx);
            const float alpha = (m_run == -INFINITY) ? 1.0f : exp2f(m_run - m_new);   // O and l still zero when -inf
            const float p = (m_new == -INFINITY || x == -INFINITY) ? 0.0f : exp2f(x - m_new);
            const __half ph16 = __float2half_rn(p);
            float ps = __half2float(ph16);
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
            l_run = l_run * alpha + ps;
            m_run = m_new;
            // P[head][key]: 32-byte rows, the two 16-byte chunks swizzled by the head
            *reinterpret_cast<__half *>(sm.p16 + sh * 32 + ((((sk >> 3) ^ ((sh >> 2) & 1))) << 4) + (sk & 7) * 2) = ph16;
            if (sk == 0) sm.alpha[sh] = alpha;
        }
        cp_async_wait<kAttStages - 1>();                // step i + 1 has landed (this thread's copies)
        __syncthreads();                                // probabilities, rescale factors, step i + 1's stage are in

        // ---- O = alpha O + P V, keeping O in units of 2^k_exp for this step
        {
            const float ex = exp2f(static_cast<float>(o_exp - k_exp));
            const float a0 = sm.alpha[g] * ex, a1 = sm.alpha[g + 8] * ex;
            if (__any_sync(0xffffffffu, a0 != 1.0f || a1 != 1.0f)) {
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    o[n][0] *= a0;
                    o[n][1] *= a0;
                    o[n][2] *= a1;
                    o[n][3] *= a1;
                }
            }
            o_exp = k_exp;
            uint32_t pa0, pa1, pa2, pa3;
            const int prow = lane & 15, pch = lane >> 4;
            ldsm_x4(pa0, pa1, pa2, pa3, sm.p16 + prow * 32 + ((pch ^ ((prow >> 2) & 1)) << 4));
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                for (int h = 0; h < 2; ++h) mma_f16_16816(o[2 * ks + h], pa0, pa1, pa2, pa3, vb[ks][h][0], vb[ks][h][1]);
        }

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
constexpr int kMergeMaxParts = 512;                      // >= 2 x CTAs of one wave
constexpr int kMergeBatch = 8;                           // partials loaded together

__global__ void __launch_bounds__(kMergeThreads)
attn_merge_kernel(const float *__restrict__ part_o, const float2 *__restrict__ part_ml, int64_t total_steps,
                  int n_st, int grid, float *__restrict__ out, float *__restrict__ lse) {
    __shared__ float2 s_ml[kMergeMaxParts][kMergeHeads];     // (m, l), then (weight, -)
    __shared__ int s_slot[kMergeMaxParts];
    __shared__ float s_L[kMergeHeads];
    pdl_wait();
    pdl_trigger();
    const int row = blockIdx.x, hg = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t r0 = static_cast<int64_t>(row) * n_st, r1 = r0 + n_st - 1;
    const int c0 = att_cta_of(total_steps, r0, grid), c1 = att_cta_of(total_steps, r1, grid);
    if (c0 == c1) return;                                 // one CTA held the row: already final
    const int n_parts = min(c1 - c0 + 1, kMergeMaxParts);
    const int first_slot = 2 * c0 + (att_range_start(total_steps, c0, grid) < r0 ? 1 : 0);
    for (int p = tid; p < n_parts; p += kMergeThreads) s_slot[p] = p == 0 ? first_slot : 2 * (c0 + p);
    __syncthreads();
    for (int i = tid; i < n_parts * kMergeHeads; i += kMergeThreads)
        s_ml[i / kMergeHeads][i % kMergeHeads] =
            __ldcg(part_ml + static_cast<int64_t>(s_slot[i / kMergeHeads]) * kHeads + hg * kMergeHeads + i % kMergeHeads);
    __syncthreads();
    // one warp per head: maximum, weights 2^(m - M), normaliser
    if (warp < kMergeHeads) {
        float M = -INFINITY;
        for (int p = lane; p < n_parts; p += 32)
            if (s_ml[p][warp].y > 0.0f) M = fmaxf(M, s_ml[p][warp].x);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float L = 0.0f;
        for (int p = lane; p < n_parts; p += 32) {
            const float2 v = s_ml[p][warp];
            const float e = v.y > 0.0f ? exp2f(v.x - M) : 0.0f;
            L += e * v.y;
            s_ml[p][warp].x = e;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
        if (lane == 0) {
            s_L[warp] = L;
            lse[static_cast<int64_t>(row) * kHeads + hg * kMergeHeads + warp] =
                L > 0.0f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
        }
    }
    __syncthreads();
    constexpr int kRowVec = kHeads * kDim / 4;              // 2304 float4 per partial
    const float4 *po = reinterpret_cast<const float4 *>(part_o) + hg * kMergeVec;
    float4 acc[kMergePer];
    int hc[kMergePer];
#pragma unroll
    for (int c = 0; c < kMergePer; ++c) {
        acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        hc[c] = (c * kMergeThreads + tid) / (kDim / 4);
    }
    for (int p0 = 0; p0 < n_parts; p0 += kMergeBatch) {
        float4 v[kMergeBatch][kMergePer];
#pragma unroll
        for (int u = 0; u < kMergeBatch; ++u)
#pragma unroll
            for (int c = 0; c < kMergePer; ++c)
                v[u][c] = p0 + u < n_parts
                              ? __ldcg(po + static_cast<int64_t>(s_slot[p0 + u]) * kRowVec + c * kMergeThreads + tid)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < kMergeBatch; ++u) {
            if (p0 + u >= n_parts) break;
#pragma unroll
            for (int c = 0; c < kMergePer; ++c) {
                const float wt = s_ml[p0 + u][hc[c]].x;
                acc[c].x += wt * v[u][c].x;
                acc[c].y += wt * v[u][c].y;
                acc[c].z += wt * v[u][c].z;
                acc[c].w += wt * v[u][c].w;
            }
        }
    }
    float4 *orow = reinterpret_cast<float4 *>(out + static_cast<int64_t>(row) * kHeads * kDim) + hg * kMergeVec;
#pragma unroll
    for (int c = 0; c < kMergePer; ++c) {
        const float L = s_L[hc[c]];
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        orow[c * kMergeThreads + tid] = make_float4(acc[c].x * inv, acc[c].y * inv, acc[c].z * inv, acc[c].w * inv);
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
