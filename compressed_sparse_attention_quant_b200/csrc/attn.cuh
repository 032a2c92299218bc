// attn.cuh -- K4/K5: sparse attention over the selected FP4 entries plus the
// sliding window, merged by online softmax.
// Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2 (attention reads only the top-K addressed entries of the shared main
// KV) and part 3 (E2M1 + E4M3 per 16 channels); page "DeepSeek V4 1-Flash
// 架构拆解…" (blog.zulogic.cn), section 4 (a 128-token window kept per layer
// beside the global compressed state).
//
// Work: the key list of a query row is its 128 window rows (none when the
// caller passes no window) followed by its k selected entries, cut into
// blocks of 128 keys. The blocks of all rows form one flat sequence that is
// split into equal contiguous ranges, one per CTA (persistent, one CTA per
// SM). A CTA writes a row's result directly when its range covers the whole
// row, else an unnormalised partial (m, l, O) of its first or last row; K5
// merges those.
//
// K4 runs both products on the tensor cores (tcgen05, accumulators in tensor
// memory), with the keys as the MMA's M side so that the 16 heads are its N:
//   S^T [128 keys x 16 heads] = K [keys x 576] . Q^T        (36 MMAs, K = 16)
//   O^T [576 x 16] += V^T [576 x keys] . P^T [keys x 16]    (5 x 8 MMAs)
// Keys are values, so one f16 tile of the block serves both: it is stored as
// 72 slabs of 128 keys x 8 channels (16 bytes per key), which is the K-major
// operand layout of the QK product and the MN-major one of the PV product.
// The fifth 128-channel tile of O reads 64 channels past the end of the slab
// tile; those rows of its accumulator are never read.
//   producers (warps 4..7, one key each): gather the block's packed FP4
//            records by bulk copy into a staging buffer one block ahead,
//            convert E2M1 x E4M3 scale to f16 (exact in f16) into the slab
//            tile, group by group of 128 channels as the previous block's PV
//            releases each group; window rows are bf16 and are copied into
//            the tile unchanged (cp.async, zero-filled before position 0).
//            At a row's first block they stage its query twice: bf16 as is
//            (for the window block) and f16 under a power-of-two exponent
//            that keeps it in range (for the FP4 blocks).
//   MMA      (warp 8, one thread): QK of the block as its groups arrive, one
//            commit; after the probabilities, PV tile by tile, one commit per
//            tile (each releases that channel group to the producers).
//   softmax  (warps 0..3, one key per thread, the block's S row from tensor
//            memory): exp2 domain, a reference maximum per head that rises
//            only when a block exceeds it by more than 8 (then O is rescaled
//            in tensor memory first; otherwise probabilities up to 2^8 stay
//            as they are, at the same relative precision),
//            probabilities rounded to f16 (FP4 blocks) or split into two bf16
//            terms hi + lo (the window block, bf16 operands), and the sum of
//            exactly the values the MMA uses. At the end of a row segment
//            they read O from tensor memory and write the result or partial.
// Every wait is an mbarrier wait with a time limit.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kAttBlk = 128;                                   // keys per block (MMA M)
constexpr int kAttSoftWarps = 4;                               // warps 0..3
constexpr int kAttProdWarps = 4;                               // warps 4..7
constexpr int kAttMmaWarp = 8;
constexpr int kAttThreads = 9 * 32;                            // 288
constexpr int kAttGroups = 5;                                  // channel groups of 128 (the last holds 64)
constexpr int kAttSlab = kAttBlk * 16;                         // 2,048: 128 keys x 8 channels of 16 bits
constexpr int kAttTileBytes = (kDim / 8) * kAttSlab;           // 147,456
constexpr int kAttQBytes = kHeads * kDim * 2;                  // 18,432
constexpr int kAttPBytes = kAttBlk * kHeads * 2;               // 4,096
constexpr int kAttRawStride = 304;                             // 288-byte record + 16 (conflict-free 16-byte reads)
constexpr int kAttRawBytes = kAttBlk * kAttRawStride;          // 38,912
constexpr int kAttTmemCols = 128;
constexpr int kAttSCol = 0;                                    // S^T: 16 columns
constexpr int kAttOCol = 16;                                   // O^T: 5 tiles x 16 columns
constexpr float kAttSlack = 8.0f;                              // log2 units a block may exceed the reference max
constexpr uint32_t kIdescBf16 = (1u << 7) | (1u << 10);        // A and B format BF16 (kind::f16)
// Operand strides (bytes between adjacent 8 x 16-byte core matrices).
// K-major: LBO = along K, SBO = along M/N.
constexpr uint32_t kTileLboK = kAttSlab, kTileSboK = 128;      // A of QK: channel groups / key groups
constexpr uint32_t kQLbo = 256, kQSbo = 128;                   // B of QK: channel groups / head groups
// MN-major: LBO = along K, SBO = along M/N.
constexpr uint32_t kTileLboMN = 128, kTileSboMN = kAttSlab;    // A of PV: key groups / channel groups
constexpr uint32_t kPLbo = 256, kPSbo = 128;                   // B of PV: key groups / head groups

struct AttSmem {
    alignas(128) uint8_t tile[kAttTileBytes];                 // f16 (FP4 block) or bf16 (window) keys
    alignas(16) uint8_t qf[kAttQBytes];                        // must follow the tile (read past its end)
    alignas(16) uint8_t qb[kAttQBytes];
    alignas(16) uint8_t p_hi[kAttPBytes];
    alignas(16) uint8_t p_lo[kAttPBytes];
    alignas(16) uint8_t raw[kAttRawBytes];                     // packed FP4 records of the next block
    uint64_t deq_done[kAttGroups];                             // producers -> MMA (group t of the tile is in)
    uint64_t pv_done[kAttGroups];                              // MMA -> producers, softmax (PV tile t done)
    uint64_t s_full;                                           // MMA -> softmax (S of the block)
    uint64_t p_ready;                                          // softmax -> MMA (P, rescaled O)
    uint64_t raw_full;                                         // bulk copies -> producers
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t mask[2][4];                                       // valid keys of a block, by block parity
    int eq[2];                                                 // query exponent of a block
    float qmax[2][kAttProdWarps];
    alignas(16) float red_m[kAttSoftWarps][kHeads];
    float red_l[kAttSoftWarps][kHeads];
};
constexpr size_t kAttSmemBytes = sizeof(AttSmem);
static_assert(offsetof(AttSmem, qf) == kAttTileBytes, "the PV tail tile reads on into qf");
static_assert(kAttSmemBytes <= 232448, "one CTA per SM");

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
    int n_win;                     // window blocks per row: 1, or 0 without a window
    int n_st;                      // blocks per row: n_win + ceil(k / 128)
    int64_t total_steps;           // R * n_st
};

// First block of CTA c's range (the same formula on host and device).
__host__ __device__ __forceinline__ int64_t att_range_start(int64_t total, int c, int grid) {
    return total * c / grid;
}

// CTA whose range holds block s.
__host__ __device__ __forceinline__ int att_cta_of(int64_t total, int64_t s, int grid) {
    int c = static_cast<int>(s * grid / total);
    while (c + 1 < grid && att_range_start(total, c + 1, grid) <= s) ++c;
    while (c > 0 && att_range_start(total, c, grid) > s) --c;
    return c;
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

// Row state of a query row.
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

// Block i of a CTA's range.
struct AttBlk {
    int row, j;        // query row, block of the row
    bool win;          // the window block
    int e0, n;         // first selected entry, keys in the block
    bool first, last;  // first / last block of a row segment of this CTA
};

__device__ __forceinline__ AttBlk att_blk(const AttParams &P, int64_t b0, int nblk, int i) {
    AttBlk k;
    const int64_t gb = b0 + i;
    k.row = static_cast<int>(gb / P.n_st);
    k.j = static_cast<int>(gb - static_cast<int64_t>(k.row) * P.n_st);
    k.win = k.j < P.n_win;
    k.e0 = k.win ? 0 : (k.j - P.n_win) * kAttBlk;
    k.n = k.win ? kAttBlk : min(kAttBlk, P.k - k.e0);
    k.first = i == 0 || k.j == 0;
    k.last = i == nblk - 1 || k.j == P.n_st - 1;
    return k;
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
          "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
          "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
          "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
          "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
          "r"(__float_as_uint(v[15]))
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// Barrier over n threads that also ORs a predicate across them.
__device__ __forceinline__ bool bar_red_or(int id, int n, bool v) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res) : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n) : "memory");
    return res != 0u;
}

__device__ __forceinline__ void named_bar(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Bulk global -> shared copy completing on an mbarrier (default L2 policy).
__device__ __forceinline__ void bulk_g2s_plain(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Reduction of 16 per-lane values over the warp's 32 lanes, one head per
// lane pair: lane L returns the result for head L >> 1 (16 shuffles).
template <bool kMax>
__device__ __forceinline__ float warp_reduce16(const float (&v)[16]) {
    const int lane = threadIdx.x & 31;
    auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
    float a[8], b[4], c[2];
    {
        const bool up = lane & 16;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float send = up ? v[i] : v[i + 8], keep = up ? v[i + 8] : v[i];
            a[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 16));
        }
    }
    {
        const bool up = lane & 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float send = up ? a[i] : a[i + 4], keep = up ? a[i + 4] : a[i];
            b[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 8));
        }
    }
    {
        const bool up = lane & 4;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float send = up ? b[i] : b[i + 2], keep = up ? b[i + 2] : b[i];
            c[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 4));
        }
    }
    const bool up = lane & 2;
    float d = op(up ? c[1] : c[0], __shfl_xor_sync(0xffffffffu, up ? c[0] : c[1], 2));
    return op(d, __shfl_xor_sync(0xffffffffu, d, 1));
}

__device__ __forceinline__ uint32_t slab_off(int key, int cgroup) {
    return static_cast<uint32_t>(cgroup * kAttSlab + (key >> 3) * 128 + (key & 7) * 16);
}

// ------------------------------------------------------------------ producers
// Physical slot of key r of fp4 block i (top-k index idx, its page entry
// pg), or -1; flags out-of-range data.
__device__ __forceinline__ int att_slot(const AttParams &P, const AttBlk &k, const AttRow &rw, int r, int idx,
                                        int64_t pg) {
    if (r >= k.n || idx < 0) return -1;                  // padding
    if (rw.T < 0 || idx > rw.pos || pg < 0 || pg >= P.num_pages) {
        flag_status(kStatusBounds);
        return -1;
    }
    return static_cast<int>(pg * kPage + (idx & 63));
}

__device__ __forceinline__ bool att_producers(const AttParams &P, AttSmem &sm, int64_t b0, int nblk) {
    const int r = threadIdx.x - kAttSoftWarps * 32;       // key of the block
    const int pw = r >> 5, lane = r & 31;
    const int n_rows_swa = kWindow + P.Sq - 1;
    const uint32_t mykey = static_cast<uint32_t>((r >> 3) * 128 + (r & 7) * 16);
    auto next_fp4 = [&](int i) {
        while (i < nblk && att_blk(P, b0, nblk, i).win) ++i;
        return i;
    };
    auto load_idx = [&](int i) -> int {
        if (i >= nblk) return -1;
        const AttBlk k = att_blk(P, b0, nblk, i);
        return r < k.n ? __ldg(P.topk_idx + static_cast<int64_t>(k.row) * P.k + k.e0 + r) : -1;
    };
    auto load_page = [&](int i, int idx) -> int64_t {
        if (i >= nblk || idx < 0) return -1;
        const AttBlk k = att_blk(P, b0, nblk, i);
        const AttRow rw = att_row(P, k.row);
        if (rw.T < 0 || idx > rw.pos) return -1;
        return __ldg(P.page_table + static_cast<int64_t>(rw.b) * P.max_pages + (idx >> 6));
    };
    auto resolve = [&](int i, int idx, int64_t pg) -> int {
        if (i >= nblk) return -1;
        const AttBlk k = att_blk(P, b0, nblk, i);
        return att_slot(P, k, att_row(P, k.row), r, idx, pg);
    };
    uint32_t sc_next[9];
    auto issue = [&](int slot) {                          // copy + scales of this key's next record
        if (slot >= 0) {
            mbar_arrive_expect_tx(&sm.raw_full, kFp4Bytes);
            bulk_g2s_plain(sm.raw + r * kAttRawStride, P.kv_fp4 + static_cast<int64_t>(slot) * kFp4Bytes, kFp4Bytes,
                           &sm.raw_full);
            const uint32_t *sp = reinterpret_cast<const uint32_t *>(P.kv_scale + static_cast<int64_t>(slot) * kScaleBytes);
#pragma unroll
            for (int u = 0; u < 9; ++u) sc_next[u] = __ldg(sp + u);
        } else {
            mbar_arrive(&sm.raw_full);
#pragma unroll
            for (int u = 0; u < 9; ++u) sc_next[u] = 0u;  // zero scale: the key's tile row is zero
        }
    };
    // The row's query: a bf16 copy and an f16 copy under exponent eq. Before
    // overwriting, the previous block's QK must be done (its PV tile 0 is).
    int eq = 0, qrow_par = 0;
    auto stage_q = [&](const AttBlk &k, const AttRow &rw, int i) -> bool {
        const uint32_t pp = static_cast<uint32_t>((i - 1) & 1);
        // ---- the row's query: bf16 copy and f16 copy under exponent eq
        if (rw.T < 0 && r == 0) flag_status(kStatusBounds);
        const __nv_bfloat16 *qr = P.q + static_cast<int64_t>(k.row) * kHeads * kDim;
        uint4 qv[9];
        float mx = 0.0f;
#pragma unroll
        for (int u = 0; u < 9; ++u) {
            const int c = u * 128 + r, h = c & 15, jg = c >> 4;
            qv[u] = __ldg(reinterpret_cast<const uint4 *>(qr + h * kDim + 8 * jg));
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = bf16x2_f32((&qv[u].x)[e]);
                mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) sm.qmax[qrow_par][pw] = mx;
        named_bar(2, kAttProdWarps * 32);
        mx = fmaxf(fmaxf(sm.qmax[qrow_par][0], sm.qmax[qrow_par][1]), fmaxf(sm.qmax[qrow_par][2], sm.qmax[qrow_par][3]));
        qrow_par ^= 1;
        eq = f16_exponent(mx);
        const float sdown = exp2f(static_cast<float>(-eq));
        // the previous block's QK has read the old query once its PV tile 0 is done
        if (i > 0 && !mbar_wait_bounded(&sm.pv_done[0], pp)) return false;
#pragma unroll
        for (int u = 0; u < 9; ++u) {
            const int c = u * 128 + r, h = c & 15, jg = c >> 4;
            const uint32_t off = static_cast<uint32_t>(jg * 256 + (h >> 3) * 128 + (h & 7) * 16);
            *reinterpret_cast<uint4 *>(sm.qb + off) = qv[u];
            uint32_t hv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = bf16x2_f32((&qv[u].x)[e]);
                hv[e] = f32x2_f16x2(f.x * sdown, f.y * sdown);
            }
            *reinterpret_cast<uint4 *>(sm.qf + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        }
        return true;
    };
    // Window rows j .. j + 127 of the band into the tile, one cp.async group
    // per channel group, each issued once the previous block's PV has
    // released it.
    auto win_issue = [&](const AttRow &rw, int i) -> bool {
        const uint32_t pp = static_cast<uint32_t>((i - 1) & 1);
        const bool valid = rw.T >= 0 && rw.pos - (kWindow - 1) + r >= 0;
        const __nv_bfloat16 *src = P.swa + (static_cast<int64_t>(rw.b) * n_rows_swa + rw.j + r) * kDim;
#pragma unroll 1
        for (int t = 0; t < kAttGroups; ++t) {
            if (i > 0 && !mbar_wait_bounded(&sm.pv_done[t], pp)) return false;
            const int g1 = t < 4 ? 16 * t + 16 : 72;
            for (int jg = 16 * t; jg < g1; ++jg)
                cp_async16(sm.tile + jg * kAttSlab + mykey, valid ? src + 8 * jg : P.swa, valid ? 16u : 0u);
            cp_async_commit();
        }
        return true;
    };
    // The first block's query (and window rows) are inputs that no kernel
    // of this path writes: they are staged before waiting for the selection
    // of the previous kernel, while it finishes.
    {
        const AttBlk k0 = att_blk(P, b0, nblk, 0);
        const AttRow rw0 = att_row(P, k0.row);
        stage_q(k0, rw0, 0);
        if (k0.win) win_issue(rw0, 0);
    }
    pdl_wait();                                           // the top-k indices are ready
    // pipeline: the next fp4 block's copy is in flight; the one after has its top-k index loaded
    int f1 = next_fp4(0);
    int slot1 = -1;
    if (f1 < nblk) {
        const int idx = load_idx(f1);
        slot1 = resolve(f1, idx, load_page(f1, idx));
        issue(slot1);
    }
    int f2 = next_fp4(f1 + 1);
    int idx2 = load_idx(f2);
    uint32_t raw_par = 0u;

    for (int i = 0; i < nblk; ++i) {
        const AttBlk k = att_blk(P, b0, nblk, i);
        const AttRow rw = att_row(P, k.row);
        const uint32_t pp = static_cast<uint32_t>((i - 1) & 1);
        if (k.first && i > 0 && !stage_q(k, rw, i)) return false;
        if (!k.win) {
            // ---- FP4 block: its records are (being) staged; resolve the one after next
            const int64_t pg2 = load_page(f2, idx2);
            const bool valid = slot1 >= 0;
            if (!mbar_wait_bounded(&sm.raw_full, raw_par)) return false;
            raw_par ^= 1u;
            const uint8_t *rr = sm.raw + r * kAttRawStride;
#pragma unroll
            for (int t = 0; t < kAttGroups; ++t) {
                if (i > 0 && !mbar_wait_bounded(&sm.pv_done[t], pp)) return false;
                // scale bytes 8t .. 8t + 7 (pieces 4t .. 4t + 3): two words, selected without indexing
                uint32_t sw0 = 0u, sw1 = 0u;
#pragma unroll
                for (int u = 0; u < 9; ++u) {
                    sw0 = u == 2 * t ? sc_next[u] : sw0;
                    sw1 = u == 2 * t + 1 ? sc_next[u] : sw1;
                }
                const int npc = t < kAttGroups - 1 ? 4 : 2;
#pragma unroll
                for (int mm = 0; mm < 4; ++mm) {                 // channels 32m .. 32m + 31, m = 4t + mm
                    if (mm < npc) {
                        const int m = 4 * t + mm;
                        const uint4 v = *reinterpret_cast<const uint4 *>(rr + 16 * m);
                        const uint32_t sw = mm < 2 ? sw0 : sw1;
                        const uint32_t s2 = e4m3x2_to_f16x2((sw >> (16 * (mm & 1))) & 0xffffu);
                        const uint32_t sa = (s2 & 0xffffu) | (s2 << 16), sb = (s2 >> 16) | (s2 & 0xffff0000u);
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const uint32_t w = (&v.x)[u], s = u < 2 ? sa : sb;
                            const uint4 o = make_uint4(hmul2_u32(e2m1x2_to_f16x2(w & 0xffu), s),
                                                       hmul2_u32(e2m1x2_to_f16x2((w >> 8) & 0xffu), s),
                                                       hmul2_u32(e2m1x2_to_f16x2((w >> 16) & 0xffu), s),
                                                       hmul2_u32(e2m1x2_to_f16x2(w >> 24), s));
                            *reinterpret_cast<uint4 *>(sm.tile + (4 * m + u) * kAttSlab + mykey) = o;
                        }
                    }
                }
                if (t == kAttGroups - 1) {
                    const uint32_t mk = __ballot_sync(0xffffffffu, valid);
                    if (lane == 0) sm.mask[i & 1][pw] = mk;
                    if (r == 0) sm.eq[i & 1] = eq;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.deq_done[t]);
            }
            // this thread's staging row is consumed: start the next fp4 block's copy
            f1 = f2;
            slot1 = resolve(f1, idx2, pg2);
            if (f1 < nblk) issue(slot1);
            f2 = next_fp4(f1 + 1);
            idx2 = load_idx(f2);
        } else {
            // ---- window block: its copies (issued here, or for block 0 before the
            // wait for the selection) are published in order as they land
            const bool valid = rw.T >= 0 && rw.pos - (kWindow - 1) + r >= 0;
            if (i > 0 && !win_issue(rw, i)) return false;
            const uint32_t mk = __ballot_sync(0xffffffffu, valid);
            if (lane == 0) sm.mask[i & 1][pw] = mk;
            if (r == 0) sm.eq[i & 1] = 0;
#define ATT_WIN_DONE(T)                                                                  \
            cp_async_wait<kAttGroups - 1 - (T)>();                                       \
            fence_proxy_async_smem();                                                    \
            __syncwarp();                                                                \
            if (lane == 0) mbar_arrive(&sm.deq_done[T]);
            ATT_WIN_DONE(0)
            ATT_WIN_DONE(1)
            ATT_WIN_DONE(2)
            ATT_WIN_DONE(3)
            ATT_WIN_DONE(4)
#undef ATT_WIN_DONE
        }
        // ---- the next block starts a row: pull its query and window band into L2
        if (i + 1 < nblk) {
            const AttBlk kn = att_blk(P, b0, nblk, i + 1);
            if (kn.j == 0) {
                const uint8_t *qn = reinterpret_cast<const uint8_t *>(P.q + static_cast<int64_t>(kn.row) * kHeads * kDim);
                for (int l = r; l < kAttQBytes / 128; l += kAttBlk) prefetch_l2(qn + l * 128);
                const AttRow rn = att_row(P, kn.row);
                if (kn.win && rn.T >= 0 && rn.pos - (kWindow - 1) + r >= 0) {
                    const uint8_t *wr = reinterpret_cast<const uint8_t *>(
                        P.swa + (static_cast<int64_t>(rn.b) * n_rows_swa + rn.j + r) * kDim);
#pragma unroll
                    for (int l = 0; l < kDim * 2 / 128; ++l) prefetch_l2(wr + l * 128);
                }
            }
        }
    }
    return true;
}

// ------------------------------------------------------------------ MMA issue
// Every MMA operand is a base descriptor plus a compile-time offset, and the
// instruction descriptor and accumulate flag are compile-time constants (one
// instantiation per block kind): with descriptors or flags computed at run
// time, the issue of each MMA was measured to take about twice as long.
template <bool kWin>
__device__ __forceinline__ bool att_qk(AttSmem &sm, uint32_t tmem, uint64_t d_kt, uint64_t d_q, uint32_t par) {
    constexpr uint32_t id = umma_idesc(kAttBlk, kHeads, false, false) | (kWin ? kIdescBf16 : 0u);
#pragma unroll
    for (int t = 0; t < kAttGroups; ++t) {
        if (!mbar_wait_bounded(&sm.deq_done[t], par)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 8 * t; ks < (t < kAttGroups - 1 ? 8 * t + 8 : kDim / 16); ++ks)
            umma_f16(tmem + kAttSCol, d_kt + static_cast<uint64_t>((ks * 2 * kAttSlab) >> 4),
                     d_q + static_cast<uint64_t>((ks * 512) >> 4), id, ks > 0 ? 1u : 0u);
    }
    umma_commit(&sm.s_full);
    return true;
}

template <bool kWin, bool kFirst>
__device__ __forceinline__ void att_pv(AttSmem &sm, uint32_t tmem, uint64_t d_vt, uint64_t d_ph, uint64_t d_pl) {
    constexpr uint32_t id = umma_idesc(kAttBlk, kHeads, true, true) | (kWin ? kIdescBf16 : 0u);
#pragma unroll
    for (int t = 0; t < kAttGroups; ++t) {
#pragma unroll
        for (int ks = 0; ks < kAttBlk / 16; ++ks) {
            const uint64_t a = d_vt + static_cast<uint64_t>((t * 16 * kAttSlab + ks * 256) >> 4);
            umma_f16(tmem + kAttOCol + 16 * t, a, d_ph + static_cast<uint64_t>((ks * 512) >> 4), id,
                     (kFirst && ks == 0) ? 0u : 1u);
            if (kWin) umma_f16(tmem + kAttOCol + 16 * t, a, d_pl + static_cast<uint64_t>((ks * 512) >> 4), id, 1u);
        }
        umma_commit(&sm.pv_done[t]);
    }
}

__device__ __forceinline__ bool att_mma(const AttParams &P, AttSmem &sm, uint32_t tmem, int64_t b0, int nblk) {
    const uint64_t d_kt = umma_desc(smem_u32(sm.tile), kTileLboK, kTileSboK, 0);
    const uint64_t d_vt = umma_desc(smem_u32(sm.tile), kTileLboMN, kTileSboMN, 0);
    const uint64_t d_qf = umma_desc(smem_u32(sm.qf), kQLbo, kQSbo, 0);
    const uint64_t d_qb = umma_desc(smem_u32(sm.qb), kQLbo, kQSbo, 0);
    const uint64_t d_ph = umma_desc(smem_u32(sm.p_hi), kPLbo, kPSbo, 0);
    const uint64_t d_pl = umma_desc(smem_u32(sm.p_lo), kPLbo, kPSbo, 0);
    for (int i = 0; i < nblk; ++i) {
        const AttBlk k = att_blk(P, b0, nblk, i);
        const uint32_t par = static_cast<uint32_t>(i & 1);
        const bool ok = k.win ? att_qk<true>(sm, tmem, d_kt, d_qb, par) : att_qk<false>(sm, tmem, d_kt, d_qf, par);
        if (!ok || !mbar_wait_bounded(&sm.p_ready, par)) return false;
        tc_fence_after();
        if (k.win) {
            if (k.first) att_pv<true, true>(sm, tmem, d_vt, d_ph, d_pl);
            else att_pv<true, false>(sm, tmem, d_vt, d_ph, d_pl);
        } else {
            if (k.first) att_pv<false, true>(sm, tmem, d_vt, d_ph, d_pl);
            else att_pv<false, false>(sm, tmem, d_vt, d_ph, d_pl);
        }
    }
    return true;
}

// ------------------------------------------------------------------ softmax, epilogue
__device__ __forceinline__ bool att_softmax(const AttParams &P, AttSmem &sm, uint32_t tmem, int64_t b0, int nblk) {
    const int q = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = threadIdx.x;                                  // key of the block (TMEM lane)
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16);
    float m_run[kHeads], l_acc[kHeads];
    int seg_j0 = 0, seg_no = 0;
    for (int i = 0; i < nblk; ++i) {
        const AttBlk k = att_blk(P, b0, nblk, i);
        const uint32_t par = static_cast<uint32_t>(i & 1);
        if (k.first) {
#pragma unroll
            for (int h = 0; h < kHeads; ++h) {
                m_run[h] = -INFINITY;
                l_acc[h] = 0.0f;
            }
            seg_j0 = k.j;
        }
        if (!mbar_wait_bounded(&sm.deq_done[kAttGroups - 1], par)) return false;   // mask, exponent
        if (!mbar_wait_bounded(&sm.s_full, par)) return false;
        tc_fence_after();
        float s[kHeads];
        tmem_ld16(trow + kAttSCol, s);
        const bool valid = (sm.mask[i & 1][q] >> lane) & 1u;
        const float sc = P.scale_log2 * (k.win ? 1.0f : exp2f(static_cast<float>(sm.eq[i & 1])));
#pragma unroll
        for (int h = 0; h < kHeads; ++h) s[h] = valid ? s[h] * sc : -INFINITY;
        // Reference maximum per head: the first finite block maximum, raised
        // only when a block exceeds it by more than kAttSlack (then O and l
        // are rescaled); otherwise probabilities up to 2^kAttSlack are kept,
        // which f16 and the bf16 pair represent with the same relative error.
        // In the common case no key exceeds it and the block's maximum is not
        // needed: one barrier-reduction over the 128 keys decides (a segment's
        // first block always exceeds the empty reference).
        bool exceed = false;
#pragma unroll
        for (int h = 0; h < kHeads; ++h) exceed |= s[h] > m_run[h] + kAttSlack;
        float alpha[kHeads];
#pragma unroll
        for (int h = 0; h < kHeads; ++h) alpha[h] = 1.0f;
        bool rescale = false;
        if (bar_red_or(1, kAttSoftWarps * 32, exceed)) {
            {
                const float mh = warp_reduce16<true>(s);
                if ((lane & 1) == 0) sm.red_m[q][lane >> 1] = mh;
            }
            named_bar(1, kAttSoftWarps * 32);
#pragma unroll
            for (int h4 = 0; h4 < kHeads / 4; ++h4) {
                const float4 a = reinterpret_cast<const float4 *>(sm.red_m[0])[h4];
                const float4 b = reinterpret_cast<const float4 *>(sm.red_m[1])[h4];
                const float4 c = reinterpret_cast<const float4 *>(sm.red_m[2])[h4];
                const float4 d = reinterpret_cast<const float4 *>(sm.red_m[3])[h4];
                const float mbv[4] = {fmaxf(fmaxf(a.x, b.x), fmaxf(c.x, d.x)), fmaxf(fmaxf(a.y, b.y), fmaxf(c.y, d.y)),
                                      fmaxf(fmaxf(a.z, b.z), fmaxf(c.z, d.z)), fmaxf(fmaxf(a.w, b.w), fmaxf(c.w, d.w))};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int h = 4 * h4 + e;
                    const float mb = mbv[e];
                    if (m_run[h] == -INFINITY) {
                        m_run[h] = mb;                   // O and l of this head are still zero
                    } else if (mb > m_run[h] + kAttSlack) {
                        alpha[h] = exp2f(m_run[h] - mb);
                        m_run[h] = mb;
                        rescale = true;
                    }
                }
            }
        }
        // probabilities of this key: f16 (FP4 block) or bf16 hi + lo (window block)
        {
            uint32_t hi[8], lo[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                float p0 = s[2 * u] == -INFINITY ? 0.0f : exp2f(s[2 * u] - m_run[2 * u]);
                float p1 = s[2 * u + 1] == -INFINITY ? 0.0f : exp2f(s[2 * u + 1] - m_run[2 * u + 1]);
                if (!k.win) {
                    const __half2 h2 = __floats2half2_rn(p0, p1);
                    hi[u] = *reinterpret_cast<const uint32_t *>(&h2);
                    const float2 used = __half22float2(h2);
                    p0 = used.x;
                    p1 = used.y;
                } else {
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                    const float2 bh = __bfloat1622float2(b2);
                    const __nv_bfloat162 c2 = __floats2bfloat162_rn(p0 - bh.x, p1 - bh.y);
                    const float2 bl = __bfloat1622float2(c2);
                    hi[u] = *reinterpret_cast<const uint32_t *>(&b2);
                    lo[u] = *reinterpret_cast<const uint32_t *>(&c2);
                    p0 = bh.x + bl.x;
                    p1 = bh.y + bl.y;
                }
                l_acc[2 * u] = l_acc[2 * u] * alpha[2 * u] + p0;
                l_acc[2 * u + 1] = l_acc[2 * u + 1] * alpha[2 * u + 1] + p1;
            }
            const uint32_t po = static_cast<uint32_t>((r >> 3) * 256 + (r & 7) * 16);
            *reinterpret_cast<uint4 *>(sm.p_hi + po) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(sm.p_hi + po + 128) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
            if (k.win) {
                *reinterpret_cast<uint4 *>(sm.p_lo + po) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                *reinterpret_cast<uint4 *>(sm.p_lo + po + 128) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
            }
        }
        if (!k.first && rescale) {
            // the reference maximum rose: O *= alpha once the previous block's PV is done
            if (!mbar_wait_bounded(&sm.pv_done[kAttGroups - 1], par ^ 1u)) return false;
            tc_fence_after();
#pragma unroll 1
            for (int t = 0; t < kAttGroups; ++t) {
                float o[kHeads];
                tmem_ld16(trow + kAttOCol + 16 * t, o);
#pragma unroll
                for (int h = 0; h < kHeads; ++h) o[h] *= alpha[h];
                tmem_st16(trow + kAttOCol + 16 * t, o);
            }
            tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_ready);
        if (!k.last) continue;

        // ---- end of a row segment: read O, write the result or the partial
        if (!mbar_wait_bounded(&sm.pv_done[kAttGroups - 1], par)) return false;
        tc_fence_after();
        {
            const float lh = warp_reduce16<false>(l_acc);
            if ((lane & 1) == 0) sm.red_l[q][lane >> 1] = lh;
        }
        named_bar(1, kAttSoftWarps * 32);
        float l[kHeads], mul[kHeads];
        const bool whole = seg_j0 == 0 && k.j == P.n_st - 1;
#pragma unroll
        for (int h = 0; h < kHeads; ++h) {
            l[h] = (sm.red_l[0][h] + sm.red_l[1][h]) + (sm.red_l[2][h] + sm.red_l[3][h]);
            mul[h] = whole ? (l[h] > 0.0f ? 1.0f / l[h] : 0.0f) : 1.0f;
        }
        const int slot = 2 * static_cast<int>(blockIdx.x) + (seg_no > 0 ? 1 : 0);
        float *dst = whole ? P.out + static_cast<int64_t>(k.row) * kHeads * kDim
                           : P.part_o + static_cast<int64_t>(slot) * kHeads * kDim;
#pragma unroll 1
        for (int t = 0; t < kAttGroups; ++t) {
            float o[kHeads];
            tmem_ld16(trow + kAttOCol + 16 * t, o);
            const int c = 128 * t + r;
            if (c < kDim) {
#pragma unroll
                for (int h = 0; h < kHeads; ++h) dst[h * kDim + c] = o[h] * mul[h];
            }
        }
        if (r < kHeads) {
            float lr = 0.0f, mr = 0.0f;
#pragma unroll
            for (int h = 0; h < kHeads; ++h)
                if (h == r) {
                    lr = l[h];
                    mr = m_run[h];
                }
            if (whole)
                P.lse[static_cast<int64_t>(k.row) * kHeads + r] = lr > 0.0f ? (mr + log2f(lr)) * 0.69314718055994530942f
                                                                            : -INFINITY;
            else
                P.part_ml[static_cast<int64_t>(slot) * kHeads + r] = make_float2(mr, lr);
        }
        tc_fence_before();
        ++seg_no;
    }
    return true;
}

__global__ void __launch_bounds__(kAttThreads, 1)
sparse_attn_kernel(const AttParams P) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    AttSmem &sm = *reinterpret_cast<AttSmem *>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int grid = static_cast<int>(gridDim.x);
    const int64_t b0 = att_range_start(P.total_steps, blockIdx.x, grid);
    const int nblk = static_cast<int>(att_range_start(P.total_steps, blockIdx.x + 1, grid) - b0);
    if (nblk <= 0) return;                                      // uniform
    if (tid == 0) {
        for (int t = 0; t < kAttGroups; ++t) {
            mbar_init(&sm.deq_done[t], kAttProdWarps);
            mbar_init(&sm.pv_done[t], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.p_ready, kAttSoftWarps);
        mbar_init(&sm.raw_full, kAttProdWarps * 32);
        mbar_init(&sm.drain, 1);
        fence_mbar_init();
    }
    if (warp == kAttMmaWarp) {
        tmem_alloc(&sm.tmem_base, kAttTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    pdl_trigger();                                              // producers wait for the selection themselves
    if (warp < kAttSoftWarps) {
        att_softmax(P, sm, tmem, b0, nblk);
    } else if (warp < kAttSoftWarps + kAttProdWarps) {
        att_producers(P, sm, b0, nblk);
    } else if ((tid & 31) == 0) {
        const bool ok = att_mma(P, sm, tmem, b0, nblk);
        if (!ok) {                                              // let every MMA issued finish before the release
            umma_commit(&sm.drain);
            mbar_wait_bounded(&sm.drain, 0);
        }
    }
    cp_async_wait<0>();
    tc_fence_before();
    __syncthreads();
    if (warp == kAttMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kAttTmemCols);
    }
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
