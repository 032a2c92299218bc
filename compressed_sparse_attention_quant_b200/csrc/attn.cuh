// attn.cuh -- K4/K5: sparse attention over the selected FP4 entries plus the
// sliding window, merged by online softmax.
// Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2 (attention reads only the top-K addressed entries of the shared main
// KV) and part 3 (E2M1 + E4M3 per 16 channels); page "DeepSeek V4 1-Flash
// 架构拆解…" (blog.zulogic.cn), section 4 (a 128-token window kept per layer
// beside the global compressed state).
//
// One CTA (8 warps, two CTAs per SM) per (query token, split of its key
// list). The key list is the k selected positions followed by the 128 window
// rows; a split owns a run of at most 12 tiles of 64 keys.
//   set-up   the query row is read with 16-byte loads, rounded to f16 and
//            stored in shared memory in the QK operand order (qk_pos), from
//            where each warp takes its fragments with ldmatrix; the split's
//            selected positions are resolved once to physical cache slots
//            (top-k index -> page table) in a shared table;
//   prefetch cp.async (16-byte and 4-byte LDGSTS, zero-filled for empty
//            slots) fetches the next tile's packed FP4 records and scales as
//            soon as the current tile's QK has consumed them, overlapping the
//            softmax and PV;
//   QK       warp (32-key group, 144-channel quarter): each lane converts the
//            FP4 bytes of its key (hardware E2M1x2 -> f16x2, E4M3 -> f16 and
//            one exact f16 multiply) directly into m16n8k16 B fragments, and
//            stores the same f16 values into a [64][576] tile whose 16-byte
//            chunks are XOR-swizzled by key; the query fragments stay in
//            registers; the quarters are summed through shared memory. Tiles
//            holding window rows (bf16 loads rounded to f16), padding, or the
//            end of the selected list are first written to the f16 tile by
//            all threads, and QK reads its fragments from there;
//   softmax  two heads per warp, warp-shuffle max / sum in the exp2 domain,
//            probabilities rounded to f16 (the same values feed the sum) and
//            written over partial rows that no other warp reads, so three
//            CTA barriers per tile remain (data in, QK done, P ready);
//   PV       warp w owns 72 output channels; ldmatrix.trans of the f16 tile
//            is the value operand.
// Warp-level mma.sync is used deliberately: with 16 heads the MMA N extent is
// 16, and at that width the warp MMAs issue faster than tcgen05 single-thread
// MMAs. Splits write unnormalised partials (m, l, O) that K5 merges.
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
};

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
    {
        const uint4 *qg = reinterpret_cast<const uint4 *>(P.q + static_cast<int64_t>(row) * kHeads * kDim);
        for (int i = tid; i < kHeads * kDim / 8; i += kAttThreads) {
            const int h = i / (kDim / 8), c = (i - h * (kDim / 8)) * 8;
            const uint4 v = __ldg(qg + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const int L = qk_pos(c + 2 * p);
                *reinterpret_cast<uint32_t *>(sm.kh + kh_off(h, L >> 3) + (L & 7) * 2) = bf16x2_to_f16x2(w[p]);
            }
        }
        __syncthreads();
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
    const int n_slots = P.k + kWindow;
    const int n_tiles = (n_slots + kAttTile - 1) / kAttTile;
    const int tile0 = split * P.tiles_per_split;
    const int tile1 = min(min(tile0 + P.tiles_per_split, n_tiles), tile0 + kMaxTilesPerSplit);
    const int n_it = max(tile1 - tile0, 0);

    if (tid < 16) {
        sm.m_run[tid] = -INFINITY;
        sm.l_run[tid] = 0.0f;
    }
    // Physical slots of this split's selected keys: all index loads first,
    // then all page-table loads, so only two load latencies are exposed.
    {
        constexpr int kPer = (kMaxTilesPerSplit * kAttTile + kAttThreads - 1) / kAttThreads;   // 3
        int ti[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int i = tid + u * kAttThreads;
            const int slot = tile0 * kAttTile + i;
            ti[u] = (i < n_it * kAttTile && slot < P.k && T > 0)
                        ? P.topk_idx[static_cast<int64_t>(row) * P.k + slot] : -1;
        }
        int64_t ph[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            ph[u] = -1;
            if (ti[u] >= 0) {
                if (ti[u] < T) ph[u] = P.page_table[static_cast<int64_t>(b) * P.max_pages + (ti[u] >> 6)];
                else flag_status(kStatusBounds);
            }
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int i = tid + u * kAttThreads;
            if (i < n_it * kAttTile) {
                int phys_slot = -1;
                if (ti[u] >= 0 && ti[u] < T) {
                    if (ph[u] >= 0 && ph[u] < P.num_pages) phys_slot = static_cast<int>(ph[u] * kPage + (ti[u] & 63));
                    else flag_status(kStatusBounds);
                }
                sm.slot[i] = phys_slot;
            }
        }
    }

    float o[9][4];
#pragma unroll
    for (int nt = 0; nt < 9; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
    __syncthreads();                                     // slot table ready

    const int gkey = tid >> 2, gpart = tid & 3;          // gather role: 4 threads per key
    auto prefetch = [&](int tile) {
        const int slot = tile * kAttTile + gkey;
        if (slot >= P.k) return;                         // window / padding keys are not staged
        const int ps = sm.slot[(tile - tile0) * kAttTile + gkey];
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
        const bool fused = (tile + 1) * kAttTile <= P.k;
        if (fused && gpart == 0) sm.valid[gkey] = sm.slot[it * kAttTile + gkey] >= 0 ? 1 : 0;
        if (!fused) {
            const int slot = tile * kAttTile + gkey;
            uint8_t *kh = sm.kh;
            bool valid = false;
            if (slot < P.k) {
                valid = sm.slot[it * kAttTile + gkey] >= 0;
                if (valid) {
                    // Threads 2 and 3 of a key walk the four 8-channel
                    // chunks of a record chunk in the order 2,3,0,1, so the
                    // 8 lanes of each 128-bit store phase hit 8 bank groups.
                    const bool rot = (gpart & 2) != 0;
                    // Record chunks c = gpart + 4i, software-pipelined: the
                    // next chunk's shared loads are issued before this one is
                    // converted.
                    constexpr int kCh = (kFp4Bytes / 16 + 3) / 4;           // 5
                    uint4 raw_n = *reinterpret_cast<const uint4 *>(&sm.raw[gkey][gpart * 16]);
                    uint32_t sc_n = *reinterpret_cast<const unsigned short *>(&sm.rsc[gkey][gpart * 2]);
#pragma unroll
                    for (int i = 0; i < kCh; ++i) {
                        const int c = gpart + 4 * i;
                        if (c >= kFp4Bytes / 16) break;
                        const uint4 raw = raw_n;
                        const uint32_t scv = sc_n;
                        if (c + 4 < kFp4Bytes / 16) {
                            raw_n = *reinterpret_cast<const uint4 *>(&sm.raw[gkey][(c + 4) * 16]);
                            sc_n = *reinterpret_cast<const unsigned short *>(&sm.rsc[gkey][(c + 4) * 2]);
                        }
                        const uint32_t sf = e4m3x2_to_f16x2(scv);                // (scale 2c, scale 2c+1)
                        const uint32_t s_lo = __byte_perm(sf, 0, 0x1010);
                        const uint32_t s_hi = __byte_perm(sf, 0, 0x3232);
                        const uint32_t w[4] = {rot ? raw.z : raw.x, rot ? raw.w : raw.y,
                                               rot ? raw.x : raw.z, rot ? raw.y : raw.w};
                        const uint32_t sa = rot ? s_hi : s_lo, sb = rot ? s_lo : s_hi;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint32_t wv = w[q];
                            const uint32_t s2 = q < 2 ? sa : sb;
                            uint4 h;
                            h.x = hmul2_u32(e2m1x2_to_f16x2(wv & 0xffu), s2);
                            h.y = hmul2_u32(e2m1x2_to_f16x2((wv >> 8) & 0xffu), s2);
                            h.z = hmul2_u32(e2m1x2_to_f16x2((wv >> 16) & 0xffu), s2);
                            h.w = hmul2_u32(e2m1x2_to_f16x2(wv >> 24), s2);
                            *reinterpret_cast<uint4 *>(kh + kh_off(gkey, 4 * c + (q ^ (rot ? 2 : 0)))) = h;
                        }
                    }
                }
            } else if (slot < n_slots && T > 0) {
                const int r = j + (slot - P.k);              // window row of this query
                if (T - n_rows_swa + r >= 0) {
                    valid = true;
                    const uint4 *src = reinterpret_cast<const uint4 *>(
                        P.swa + (static_cast<int64_t>(b) * n_rows_swa + r) * kDim);
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
                            uint4 h;
                            h.x = bf16x2_to_f16x2(rv[i].x);
                            h.y = bf16x2_to_f16x2(rv[i].y);
                            h.z = bf16x2_to_f16x2(rv[i].z);
                            h.w = bf16x2_to_f16x2(rv[i].w);
                            *reinterpret_cast<uint4 *>(kh + kh_off(gkey, 8 * (e >> 1) + 2 * gpart + (e & 1))) = h;
                        }
                    }
                }
            }
            if (!valid) {
                const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                for (int c = gpart; c < kDim / 8; c += 4) *reinterpret_cast<uint4 *>(kh + kh_off(gkey, c)) = z;
            }
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
        if (tile + 1 < tile1) prefetch(tile + 1);        // overlaps this tile's softmax and PV
        cp_async_commit();

        // ---------------- online softmax, two heads per warp
        {
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
                    s[u] = sm.valid[key] ? v * P.scale_log2 : -INFINITY;
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
            const float a_lo = sm.alpha[g], a_hi = sm.alpha[g + 8];
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

// K5: merge split partials: O = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s.
// One CTA per (query row, group of 4 heads): the (m, l) pairs are staged in
// shared memory by all threads at once, then each thread owns 3 float4 of the
// group's 4 x 576 outputs and issues the split loads 4 at a time, so the
// L2 round trips overlap instead of following one another.
constexpr int kMergeThreads = 192;
constexpr int kMergeHeads = 4;
constexpr int kMergeVec = kMergeHeads * kDim / 4;        // 576 float4 per CTA
constexpr int kMergePer = kMergeVec / kMergeThreads;    // 3

__global__ void __launch_bounds__(kMergeThreads)
attn_merge_kernel(const float *__restrict__ part_o, const float2 *__restrict__ part_ml, int n_splits,
                  float *__restrict__ out, float *__restrict__ lse) {
    extern __shared__ float2 mlw[];    // [n_splits][4]: (m, l), then (weight, -)
    pdl_wait();
    pdl_trigger();
    const int row = blockIdx.x, hg = blockIdx.y, tid = threadIdx.x;
    const float2 *ml = part_ml + static_cast<int64_t>(row) * n_splits * kHeads + hg * kMergeHeads;
    for (int i = tid; i < n_splits * kMergeHeads; i += kMergeThreads)
        mlw[i] = __ldcg(ml + (i / kMergeHeads) * kHeads + (i % kMergeHeads));
    __syncthreads();
    if (tid < kMergeHeads) {
        float M = -INFINITY;
        for (int s = 0; s < n_splits; ++s) M = fmaxf(M, mlw[s * kMergeHeads + tid].x);
        float L = 0.0f;
        for (int s = 0; s < n_splits; ++s) {
            const float2 v = mlw[s * kMergeHeads + tid];
            const float e = (M == -INFINITY || v.y == 0.0f) ? 0.0f : exp2f(v.x - M);
            mlw[s * kMergeHeads + tid].x = e;
            L += e * v.y;
        }
        const float inv = L > 0.0f ? 1.0f / L : 0.0f;
        for (int s = 0; s < n_splits; ++s) mlw[s * kMergeHeads + tid].x *= inv;
        lse[static_cast<int64_t>(row) * kHeads + hg * kMergeHeads + tid] =
            L > 0.0f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
    }
    __syncthreads();
    constexpr int kRowVec = kHeads * kDim / 4;              // 2304 float4 per split partial
    const float4 *po = reinterpret_cast<const float4 *>(part_o) +
                       static_cast<int64_t>(row) * n_splits * kRowVec + hg * kMergeVec;
    float4 acc[kMergePer];
#pragma unroll
    for (int c = 0; c < kMergePer; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < n_splits; s0 += 4) {
        float4 v[4][kMergePer];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int c = 0; c < kMergePer; ++c)
                v[u][c] = s0 + u < n_splits ? __ldcg(po + static_cast<int64_t>(s0 + u) * kRowVec + c * kMergeThreads + tid)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (s0 + u >= n_splits) break;
#pragma unroll
            for (int c = 0; c < kMergePer; ++c) {
                const float wv = mlw[(s0 + u) * kMergeHeads + (c * kMergeThreads + tid) / (kDim / 4)].x;
                acc[c].x += wv * v[u][c].x;
                acc[c].y += wv * v[u][c].y;
                acc[c].z += wv * v[u][c].z;
                acc[c].w += wv * v[u][c].w;
            }
        }
    }
    float4 *orow = reinterpret_cast<float4 *>(out + static_cast<int64_t>(row) * kHeads * kDim) + hg * kMergeVec;
#pragma unroll
    for (int c = 0; c < kMergePer; ++c) orow[c * kMergeThreads + tid] = acc[c];
}

}  // namespace csa2
