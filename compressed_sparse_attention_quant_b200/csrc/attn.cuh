// attn.cuh -- K4/K5: sparse attention over the selected FP4 entries plus the
// sliding window, merged by online softmax.
// Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2 (attention reads only the top-K addressed entries of the shared main
// KV) and part 3 (E2M1 + E4M3 per 16 channels); page "DeepSeek V4 1-Flash
// 架构拆解…" (blog.zulogic.cn), section 4 (a 128-token window kept per layer
// beside the global compressed state).
//
// Work: the key list of a query row is its k selected entries in ceil(k/64)
// tiles of 64 keys (the last one padded) followed by its 128 window rows in two
// tiles of their own (none when the caller passes no window). Each row's tiles
// are split into S runs, one CTA each (8 warps, two CTAs per SM), S chosen by
// the host so that all CTAs fit one wave. A run writes the row's result when
// S = 1; else an unnormalised partial (m, l, O) that K5 merges.
//   set-up   before waiting for the selection of the previous kernel (the
//            query is an input): the query row is rounded to f16 while its
//            largest magnitude is taken, and written again under 2^-eq in the
//            rare case that it asks for a power-of-two exponent eq != 0; it is
//            stored in the QK operand order (qk_pos) and each warp takes its
//            fragments with ldmatrix. The run's selected positions are then
//            resolved to physical cache slots 12 tiles at a time (top-k index
//            -> page table, all loads of a chunk in flight);
//   prefetch cp.async (16-byte and 4-byte LDGSTS, zero-filled for padding)
//            fetches the next tile's packed FP4 records and scales as soon as
//            the current tile's QK has consumed them, overlapping the softmax
//            and PV;
//   QK       warp (32-key group, 144-channel quarter): each lane converts the
//            FP4 bytes of its key (hardware E2M1x2 -> f16x2, E4M3 -> f16 and
//            one exact f16 multiply) directly into m16n8k16 B fragments, and
//            stores the same f16 values into a [64][576] tile whose 16-byte
//            chunks are XOR-swizzled by key; the quarters are summed through
//            shared memory. Window tiles are first written to the f16 tile by
//            all threads (bf16 -> f16 while the tile's largest magnitude is
//            taken, again under 2^-ew in the rare other case), and QK reads
//            its fragments from there;
//   softmax  two heads per warp, warp-shuffle max / sum in the exp2 domain
//            (logits carry 2^(eq + ew)), probabilities rounded to f16 (the
//            same values feed the sum) and written over partial rows that no
//            other warp reads, so three CTA barriers per tile remain (data in,
//            QK done, P ready);
//   PV       warp w owns 72 output channels; ldmatrix.trans of the f16 tile
//            is the value operand; a window tile's exponent scales O around
//            its products.
// Warp-level mma.sync is used deliberately: with 16 heads the MMA N extent is
// 16; measured on the B200, one tcgen05 kind::f16 M128 N16 K16 MMA costs ~45
// cycles (728 useful MAC/clk/SM) while mma.sync m16n8k16 sustains 1024
// MAC/clk/SM with its operands in registers.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kAttThreads = 256;
constexpr int kAttTile = 64;
constexpr int kKhRow = kDim * 2;            // 1152 bytes per f16 key row (no padding: swizzled chunks)
constexpr int kMaxTilesPerSplit = 12;

struct AttSmem {
    alignas(128) uint8_t kh[kAttTile * kKhRow];            // 73,728: f16 keys / values
    alignas(16) float red[8][16][32];                      // 16,384: QK partials; P reuses the start
    alignas(16) uint8_t raw[kAttTile][kFp4Bytes];          // 18,432: staged packed FP4 of the next tile
    alignas(16) uint8_t rsc[kAttTile][kScaleBytes];        // 2,304: staged scales of the next tile
    int slot[kMaxTilesPerSplit * kAttTile];                // 3,072: physical slot of each selected key
    float m_run[16];
    float l_run[16];
    float alpha[16];
    float wmax[kAttThreads / 32];
    int valid[kAttTile];
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
    float *part_o;                 // [R][S][16][576]
    float2 *part_ml;               // [R][S][16]
    int n_splits;
    int tiles_per_split;
    int n_win;                     // window tiles per row: 2, or 0 without a window
};

// bf16x2 -> f32 pair (exact).
__device__ __forceinline__ float2 bf16x2_f32(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

__device__ __forceinline__ uint32_t f32x2_f16x2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float bf16x4_absmax(const uint4 &v, float mx) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = bf16x2_f32((&v.x)[e]);
        mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    return mx;
}

// 8 bf16 values scaled by 2^-e (exact) and rounded to f16.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4 &v, float sdown) {
    uint32_t h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = bf16x2_f32((&v.x)[e]);
        h[e] = f32x2_f16x2(f.x * sdown, f.y * sdown);
    }
    return make_uint4(h[0], h[1], h[2], h[3]);
}

// Power-of-two exponent e such that values up to m, scaled by 2^-e, are
// represented in f16 without overflow and with full relative precision for
// the largest ones: 0 for m in [2^-4, 2^15) (the common case, no scaling),
// else the exponent that puts m near 2^10. Clamped to [-60, 60] (O is scaled
// by 2^+-e in f32 around a window tile's products).
__device__ __forceinline__ int f16_exponent(float m) {
    if (!(m > 0.0f) || (m >= 0.0625f && m < 32768.0f)) return 0;
    const int e = static_cast<int>((__float_as_uint(m) >> 23) & 0xffu) - 127 - 10;
    return max(-60, min(60, e));
}

// Largest magnitude over the CTA (one CTA barrier; every thread gets it).
template <typename Smem>
__device__ __forceinline__ float att_cta_max(Smem &sm, float mx) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if ((threadIdx.x & 31) == 0) sm.wmax[threadIdx.x >> 5] = mx;
    __syncthreads();
    float m = sm.wmax[0];
#pragma unroll
    for (int w = 1; w < kAttThreads / 32; ++w) m = fmaxf(m, sm.wmax[w]);
    return m;
}

// Pull the 128-byte line holding p into L2 (no register result).
__device__ __forceinline__ void prefetch_l2_line(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Byte offset of 8-channel chunk `chunk` (0..71) of key row `key`: chunks are
// XOR-swizzled by the key's low 3 bits so that the 8 rows an ldmatrix reads
// fall in 8 different bank groups.
__device__ __forceinline__ uint32_t kh_off(int key, int chunk) {
    return static_cast<uint32_t>(key * kKhRow + ((chunk ^ (key & 7)) << 4));
}

// Float index of (head, key-in-group) in a warp's QK partial block: columns
// XOR-swizzled by the head (in 8-float blocks) so that the four heads a
// half-warp's float2 fragment stores touch land in four different bank groups.
__device__ __forceinline__ int red_col(int head, int col) { return col ^ ((head & 3) << 3); }

// f16 probabilities of head h for the tile's 64 keys: the 128 bytes of
// red[0][h] (a row only the softmax warp of head h reads), with 16-byte chunks
// XOR-swizzled by the head so the 8 rows an ldmatrix reads hit 8 bank groups.
__device__ __forceinline__ uint8_t *p_row(AttSmem &sm, int h) {
    return reinterpret_cast<uint8_t *>(&sm.red[0][h][0]);
}
__device__ __forceinline__ int p_off(int h, int key) { return (((key >> 3) ^ (h & 7)) << 4) + (key & 7) * 2; }

// Position, in the operand order of the QK phase, of the physical channel
// pair (c, c + 1), c even. Warp quarter cq of the QK phase owns channels
// [144 cq, 144 cq + 144): two 64-channel units in which lane quad tig holds
// channels 16 tig .. 16 tig + 15 of its key (one scale group, four k-steps),
// then a 16-channel tail in which lane quad tig holds channels 4 tig .. 4 tig + 3.
// k-step s of a unit puts channels 16 tig + 4 s + {0, 1} on MMA rows
// k = 2 tig + {0, 1} and 16 tig + 4 s + {2, 3} on rows 2 tig + 8 + {0, 1}.
// The query is stored in the same order, so every product q_c k_c is still
// summed exactly once.
__device__ __forceinline__ int qk_pos(int c) {
    const int cq = c / 144, r = c - cq * 144;
    const int ks = r < 128 ? (r >> 6) * 4 + ((r >> 2) & 3) : 8;
    const int tig = r < 128 ? (r >> 4) & 3 : (r - 128) >> 2;
    const int y = r & 3;
    return cq * 144 + ks * 16 + 2 * tig + (y & 1) + ((y >> 1) << 3);
}

// QK over one warp's 32 keys x 144-channel quarter, in the operand order of
// qk_pos. kFused: every key of the tile is a selected cache entry; the lane
// converts its FP4 bytes straight into B fragments and also writes them to
// the f16 tile for PV. Otherwise every key row is already in the f16 tile.
template <bool kFused>
__device__ __forceinline__ void qk_quarter(AttSmem &sm, const uint32_t (&qa)[9][4], float (&acc)[4][4], int kg,
                                           int cq, int g, int tig) {
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const int key = kg * 32 + nt * 8 + g;
        const uint8_t *rrow = sm.raw[key];
        const uint8_t *srow = sm.rsc[key];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int cb = cq * 144 + u * 64 + tig * 16;            // physical channel of h[0]
            uint4 *d0 = reinterpret_cast<uint4 *>(sm.kh + kh_off(key, cb >> 3));
            uint4 *d1 = reinterpret_cast<uint4 *>(sm.kh + kh_off(key, (cb >> 3) + 1));
            uint32_t h[8];
            if (kFused) {
                const uint2 rv = *reinterpret_cast<const uint2 *>(rrow + (cb >> 1));
                const uint32_t s2 = e4m3x2_to_f16x2(static_cast<uint32_t>(srow[cb >> 4]) * 0x0101u);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    h[i] = hmul2_u32(e2m1x2_to_f16x2(((i < 4 ? rv.x : rv.y) >> (8 * (i & 3))) & 0xffu), s2);
                *d0 = make_uint4(h[0], h[1], h[2], h[3]);
                *d1 = make_uint4(h[4], h[5], h[6], h[7]);
            } else {
                const uint4 a = *d0, b = *d1;
                h[0] = a.x; h[1] = a.y; h[2] = a.z; h[3] = a.w;
                h[4] = b.x; h[5] = b.y; h[6] = b.z; h[7] = b.w;
            }
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_f16_16816(acc[nt], qa[4 * u + s][0], qa[4 * u + s][1], qa[4 * u + s][2], qa[4 * u + s][3],
                              h[2 * s], h[2 * s + 1]);
        }
        {
            const int cb = cq * 144 + 128 + tig * 4;
            uint2 *d = reinterpret_cast<uint2 *>(sm.kh + kh_off(key, cb >> 3) + (cb & 7) * 2);
            uint32_t h0, h1;
            if (kFused) {
                const uint32_t rv = *reinterpret_cast<const unsigned short *>(rrow + (cb >> 1));
                const uint32_t s2 = e4m3x2_to_f16x2(static_cast<uint32_t>(srow[cb >> 4]) * 0x0101u);
                h0 = hmul2_u32(e2m1x2_to_f16x2(rv & 0xffu), s2);
                h1 = hmul2_u32(e2m1x2_to_f16x2(rv >> 8), s2);
                *d = make_uint2(h0, h1);
            } else {
                const uint2 v = *d;
                h0 = v.x;
                h1 = v.y;
            }
            mma_f16_16816(acc[nt], qa[8][0], qa[8][1], qa[8][2], qa[8][3], h0, h1);
        }
    }
}

__global__ void __launch_bounds__(kAttThreads, 2)
sparse_attn_kernel(const AttParams P) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    AttSmem &sm = *reinterpret_cast<AttSmem *>(smem_raw);
    const int row = blockIdx.y;
    const int split = blockIdx.x;
    const int b = row / P.Sq, j = row % P.Sq;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tig = lane & 3;
    const int n_rows_swa = kWindow + P.Sq - 1;

    // Inputs that no earlier kernel of the step writes are read before the
    // wait for the selection: the query, the sequence length and (into L2)
    // the sequence's page-table row. The query goes through the (still free)
    // f16 tile: 16-byte loads, f16 rounding, a scatter into the QK operand
    // order, then one ldmatrix per k-step. Warp (kg, cq) covers channels
    // cq*144 .. +143.
    const int kg = warp >> 2, cq = warp & 3;
    uint32_t qa[9][4];
    int eq = 0;
    {
        // f16 under 2^-eq: written with eq = 0 while the row's largest
        // magnitude is taken, and written again in the (rare) case that it
        // asks for another exponent
        const uint4 *qg = reinterpret_cast<const uint4 *>(P.q + static_cast<int64_t>(row) * kHeads * kDim);
        auto stage = [&](float sdown) -> float {
            float mx = 0.0f;
            for (int i = tid; i < kHeads * kDim / 8; i += kAttThreads) {
                const int h = i / (kDim / 8), c = (i - h * (kDim / 8)) * 8;
                const uint4 v = __ldg(qg + i);
                mx = bf16x4_absmax(v, mx);
                const uint4 f = bf16x8_to_f16x8(v, sdown);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int L = qk_pos(c + 2 * p);
                    *reinterpret_cast<uint32_t *>(sm.kh + kh_off(h, L >> 3) + (L & 7) * 2) = (&f.x)[p];
                }
            }
            return mx;
        };
        eq = f16_exponent(att_cta_max(sm, stage(1.0f)));
        if (eq != 0) {
            stage(exp2f(static_cast<float>(-eq)));
            __syncthreads();
        }
#pragma unroll
        for (int ks = 0; ks < 9; ++ks)
            ldsm_x4(qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], sm.kh + kh_off(lane & 15, 18 * cq + 2 * ks + (lane >> 4)));
    }
    int T = P.seq_lens[b];
    for (int i = tid * 32; i < P.max_pages; i += kAttThreads * 32)           // 128-byte lines of the row
        prefetch_l2_line(P.page_table + static_cast<int64_t>(b) * P.max_pages + i);
    pdl_wait();                                         // the selection's indices are ready
    pdl_trigger();

    if (T < P.Sq || T > P.max_pages * kPage) {
        if (tid == 0 && split == 0) flag_status(kStatusBounds);
        T = -1;                                          // no valid key at all
    }
    // tiles: ceil(k / 64) of selected entries (the last one padded), then the
    // window's n_win tiles of 64 rows
    const int n_fp4_tiles = (P.k + kAttTile - 1) / kAttTile;
    const int n_tiles = n_fp4_tiles + P.n_win;
    const int tile0 = split * P.tiles_per_split;
    const int tile1 = min(tile0 + P.tiles_per_split, n_tiles);
    const int n_it = max(tile1 - tile0, 0);

    if (tid < 16) {
        sm.m_run[tid] = -INFINITY;
        sm.l_run[tid] = 0.0f;
    }
    // Physical slots of the selected keys of tiles c0 .. c0 + 11 (a chunk of
    // the run): all index loads first, then all page-table loads, so only two
    // load latencies are exposed per chunk. Positions after the query's own
    // (pos = T - Sq + j) are flagged and skipped.
    const int pos = T - P.Sq + j;
    auto resolve_chunk = [&](int c0) {
        constexpr int kPer = (kMaxTilesPerSplit * kAttTile + kAttThreads - 1) / kAttThreads;   // 3
        const int n_keys = min(kMaxTilesPerSplit, tile1 - c0) * kAttTile;
        int ti[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int i = tid + u * kAttThreads;
            const int slot = c0 * kAttTile + i;
            ti[u] = (i < n_keys && slot < P.k && T > 0) ? P.topk_idx[static_cast<int64_t>(row) * P.k + slot] : -1;
        }
        int64_t ph[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            ph[u] = -1;
            if (ti[u] >= 0) {
                if (ti[u] <= pos) ph[u] = P.page_table[static_cast<int64_t>(b) * P.max_pages + (ti[u] >> 6)];
                else flag_status(kStatusBounds);
            }
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int i = tid + u * kAttThreads;
            if (i < n_keys) {
                int phys_slot = -1;
                if (ti[u] >= 0 && ti[u] <= pos) {
                    if (ph[u] >= 0 && ph[u] < P.num_pages) phys_slot = static_cast<int>(ph[u] * kPage + (ti[u] & 63));
                    else flag_status(kStatusBounds);
                }
                sm.slot[i] = phys_slot;
            }
        }
    };
    resolve_chunk(tile0);

    float o[9][4];
#pragma unroll
    for (int nt = 0; nt < 9; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
    __syncthreads();                                     // slot table ready

    const int gkey = tid >> 2, gpart = tid & 3;          // gather role: 4 threads per key
    auto prefetch = [&](int tile) {
        if (tile >= n_fp4_tiles) return;                 // window rows are not staged here
        const int ps = sm.slot[((tile - tile0) % kMaxTilesPerSplit) * kAttTile + gkey];   // -1: padding, zero-filled
        const uint32_t nb16 = ps >= 0 ? 16u : 0u, nb4 = ps >= 0 ? 4u : 0u;
        const uint8_t *src = P.kv_fp4 + (ps >= 0 ? static_cast<int64_t>(ps) * kFp4Bytes : 0);
        const uint8_t *ssrc = P.kv_scale + (ps >= 0 ? static_cast<int64_t>(ps) * kScaleBytes : 0);
        for (int c = gpart; c < kFp4Bytes / 16; c += 4) cp_async16(&sm.raw[gkey][c * 16], src + c * 16, nb16);
        for (int wd = gpart; wd < kScaleBytes / 4; wd += 4) cp_async4(&sm.rsc[gkey][wd * 4], ssrc + wd * 4, nb4);
    };
    if (n_it > 0) prefetch(tile0);
    cp_async_commit();

    for (int tile = tile0; tile < tile1; ++tile) {
        const int it = tile - tile0;
        cp_async_wait<0>();                              // this tile's raw records have landed
        __syncthreads();
        // Every key of the tile is a selected cache entry: QK converts the FP4
        // records itself. Otherwise all threads first write the tile's key
        // rows (FP4 -> f16, window bf16 -> f16, or zeros) to the f16 tile.
        const bool fused = tile < n_fp4_tiles;
        int ew = 0;                                      // exponent of a window tile
        if (fused && gpart == 0) sm.valid[gkey] = sm.slot[(it % kMaxTilesPerSplit) * kAttTile + gkey] >= 0 ? 1 : 0;
        if (!fused) {
            // a window tile: rows j + 64 wt .. of the band, bf16 -> f16 under
            // the tile's exponent ew (written with ew = 0 while the largest
            // magnitude is taken; written again in the rare other case)
            const int r = j + (tile - n_fp4_tiles) * kAttTile + gkey;
            const bool valid = T > 0 && T - n_rows_swa + r >= 0;
            const uint4 *src = reinterpret_cast<const uint4 *>(P.swa + (static_cast<int64_t>(b) * n_rows_swa + r) * kDim);
            uint8_t *kh = sm.kh;
            auto rows = [&](float sdown) -> float {
                float mx = 0.0f;
                if (valid) {
                    // Thread p of a key takes chunks 8m + 2p + {0,1}: the
                    // chunks of a store phase share their parity per key.
#pragma unroll
                    for (int third = 0; third < 3; ++third) {
                        uint4 rv[6];
#pragma unroll
                        for (int i = 0; i < 6; ++i) {
                            const int e = third * 6 + i;
                            rv[i] = __ldg(src + 8 * (e >> 1) + 2 * gpart + (e & 1));
                        }
#pragma unroll
                        for (int i = 0; i < 6; ++i) {
                            const int e = third * 6 + i;
                            mx = bf16x4_absmax(rv[i], mx);
                            *reinterpret_cast<uint4 *>(kh + kh_off(gkey, 8 * (e >> 1) + 2 * gpart + (e & 1))) =
                                bf16x8_to_f16x8(rv[i], sdown);
                        }
                    }
                } else {
                    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                    for (int c = gpart; c < kDim / 8; c += 4) *reinterpret_cast<uint4 *>(kh + kh_off(gkey, c)) = z;
                }
                return mx;
            };
            ew = f16_exponent(att_cta_max(sm, rows(1.0f)));
            if (ew != 0) rows(exp2f(static_cast<float>(-ew)));
            if (gpart == 0) sm.valid[gkey] = valid ? 1 : 0;
        }
        if (!fused) __syncthreads();

        // ---------------- S = Q K^T over this warp's 32 keys x channel quarter
        {
            float acc[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
            if (fused) qk_quarter<true>(sm, qa, acc, kg, cq, g, tig);
            else qk_quarter<false>(sm, qa, acc, kg, cq, g, tig);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int col = nt * 8 + tig * 2;
                *reinterpret_cast<float2 *>(&sm.red[warp][g][red_col(g, col)]) = make_float2(acc[nt][0], acc[nt][1]);
                *reinterpret_cast<float2 *>(&sm.red[warp][g + 8][red_col(g + 8, col)]) =
                    make_float2(acc[nt][2], acc[nt][3]);
            }
        }
        __syncthreads();                                 // partials and the f16 tile are complete; raw is free
        if (tile + 1 < tile1 && (tile + 1 - tile0) % kMaxTilesPerSplit == 0) {
            resolve_chunk(tile + 1);                     // the next chunk of the run
            __syncthreads();
        }
        if (tile + 1 < tile1) prefetch(tile + 1);        // overlaps this tile's softmax and PV
        cp_async_commit();

        // ---------------- online softmax, two heads per warp
        {
            const float sc = P.scale_log2 * exp2f(static_cast<float>(eq + ew));
            float pv[2][2], alpha[2], m_new[2], psum[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int h = warp * 2 + hh;
                float s[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int key = lane + 32 * u;          // key group u
                    const int cc = red_col(h, lane);
                    const float v = sm.red[u * 4 + 0][h][cc] + sm.red[u * 4 + 1][h][cc] +
                                    sm.red[u * 4 + 2][h][cc] + sm.red[u * 4 + 3][h][cc];
                    s[u] = sm.valid[key] ? v * sc : -INFINITY;
                }
                float mx = fmaxf(s[0], s[1]);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                const float m_old = sm.m_run[h];
                m_new[hh] = fmaxf(m_old, mx);
                if (m_new[hh] == -INFINITY) {
                    alpha[hh] = 1.0f;
                    pv[hh][0] = pv[hh][1] = 0.0f;
                } else {
                    alpha[hh] = exp2f(m_old - m_new[hh]);
                    pv[hh][0] = exp2f(s[0] - m_new[hh]);
                    pv[hh][1] = exp2f(s[1] - m_new[hh]);
                }
                pv[hh][0] = __half2float(__float2half_rn(pv[hh][0]));
                pv[hh][1] = __half2float(__float2half_rn(pv[hh][1]));
                float sum = pv[hh][0] + pv[hh][1];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                psum[hh] = sum;
            }
            // Row h of every partial block is read by this warp alone, so the
            // probabilities of head h go into the 128 bytes of red[0][h]
            // without a CTA barrier (the warp's own reads are complete: the
            // shuffles above consumed them).
            __syncwarp();
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int h = warp * 2 + hh;
                *reinterpret_cast<__half *>(p_row(sm, h) + p_off(h, lane)) = __float2half_rn(pv[hh][0]);
                *reinterpret_cast<__half *>(p_row(sm, h) + p_off(h, lane + 32)) = __float2half_rn(pv[hh][1]);
                if (lane == 0) {
                    sm.l_run[h] = sm.l_run[h] * alpha[hh] + psum[hh];
                    sm.m_run[h] = m_new[hh];
                    sm.alpha[h] = alpha[hh];
                }
            }
        }
        __syncthreads();

        // ---------------- O = alpha * O + P V over this warp's 72 channels
        {
            // a window tile's values are f16 under 2^-ew: O enters its frame and leaves it
            const float down = exp2f(static_cast<float>(-ew));
            const float a_lo = sm.alpha[g] * down, a_hi = sm.alpha[g + 8] * down;
#pragma unroll
            for (int nt = 0; nt < 9; ++nt) {
                o[nt][0] *= a_lo;
                o[nt][1] *= a_lo;
                o[nt][2] *= a_hi;
                o[nt][3] *= a_hi;
            }
            const int m = lane >> 3, r = lane & 7;
            const int c0 = warp * 72;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(a0, a1, a2, a3, p_row(sm, r + 8 * (m & 1)) + p_off(r + 8 * (m & 1), kk * 16 + 8 * (m >> 1)));
                const int key = kk * 16 + 8 * (m & 1) + r;
#pragma unroll
                for (int pr = 0; pr < 4; ++pr) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(b0, b1, b2, b3, sm.kh + kh_off(key, ((c0 + pr * 16) >> 3) + (m >> 1)));
                    mma_f16_16816(o[2 * pr], a0, a1, a2, a3, b0, b1);
                    mma_f16_16816(o[2 * pr + 1], a0, a1, a2, a3, b2, b3);
                }
                uint32_t b0, b1;
                ldsm_x2_t(b0, b1, sm.kh + kh_off(key, (c0 + 64) >> 3));
                mma_f16_16816(o[8], a0, a1, a2, a3, b0, b1);
            }
            if (ew != 0) {
                const float up = exp2f(static_cast<float>(ew));
#pragma unroll
                for (int nt = 0; nt < 9; ++nt) {
                    o[nt][0] *= up;
                    o[nt][1] *= up;
                    o[nt][2] *= up;
                    o[nt][3] *= up;
                }
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---------------- epilogue: final output or split partial
    const int c0 = warp * 72;
    if (P.n_splits == 1) {
        const float l_lo = sm.l_run[g], l_hi = sm.l_run[g + 8];
        const float inv_lo = l_lo > 0.0f ? 1.0f / l_lo : 0.0f;
        const float inv_hi = l_hi > 0.0f ? 1.0f / l_hi : 0.0f;
        float *orow = P.out + static_cast<int64_t>(row) * kHeads * kDim;
#pragma unroll
        for (int nt = 0; nt < 9; ++nt) {
            const int c = c0 + nt * 8 + tig * 2;
            *reinterpret_cast<float2 *>(orow + g * kDim + c) = make_float2(o[nt][0] * inv_lo, o[nt][1] * inv_lo);
            *reinterpret_cast<float2 *>(orow + (g + 8) * kDim + c) = make_float2(o[nt][2] * inv_hi, o[nt][3] * inv_hi);
        }
        if (tid < 16) {
            const float l = sm.l_run[tid];
            P.lse[static_cast<int64_t>(row) * kHeads + tid] =
                l > 0.0f ? (sm.m_run[tid] + log2f(l)) * 0.69314718055994530942f : -INFINITY;
        }
    } else {
        const int64_t pidx = static_cast<int64_t>(row) * P.n_splits + split;
        float *po = P.part_o + pidx * kHeads * kDim;
#pragma unroll
        for (int nt = 0; nt < 9; ++nt) {
            const int c = c0 + nt * 8 + tig * 2;
            *reinterpret_cast<float2 *>(po + g * kDim + c) = make_float2(o[nt][0], o[nt][1]);
            *reinterpret_cast<float2 *>(po + (g + 8) * kDim + c) = make_float2(o[nt][2], o[nt][3]);
        }
        if (tid < 16) P.part_ml[pidx * kHeads + tid] = make_float2(sm.m_run[tid], sm.l_run[tid]);
    }
}

// K5: merge the S partials of each query row:
// O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s. One CTA per (query row,
// group of 4 heads); run s of row r holds slot r * S + s. Each thread owns 3
// float4 of the group's 4 x 576 outputs and loads the partials 8 at a time.
constexpr int kMergeThreads = 192;
constexpr int kMergeHeads = 4;
constexpr int kMergeVec = kMergeHeads * kDim / 4;        // 576 float4 per CTA
constexpr int kMergePer = kMergeVec / kMergeThreads;    // 3
constexpr int kMergeMaxParts = 512;                      // largest S
constexpr int kMergeBatch = 8;                           // partials loaded together

__global__ void __launch_bounds__(kMergeThreads)
attn_merge_kernel(const float *__restrict__ part_o, const float2 *__restrict__ part_ml, int n_splits,
                  float *__restrict__ out, float *__restrict__ lse) {
    __shared__ float2 s_ml[kMergeMaxParts][kMergeHeads];     // (m, l), then (weight, -)
    __shared__ int s_slot[kMergeMaxParts];
    __shared__ float s_L[kMergeHeads];
    pdl_wait();
    pdl_trigger();
    const int row = blockIdx.x, hg = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n_parts = min(n_splits, kMergeMaxParts);
    for (int p = tid; p < n_parts; p += kMergeThreads) s_slot[p] = row * n_splits + p;
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
