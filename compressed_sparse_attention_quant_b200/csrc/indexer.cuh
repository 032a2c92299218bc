// indexer.cuh -- K2: lightweight-indexer scores over every cached token,
// with the first top-k histogram fused into the epilogue.
// Page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2 (indexer keys shared across layers, top-K addressing), and page
// "DeepSeek V4 1-Flash 架构拆解…" (blog.zulogic.cn), section 3 (the Full owner
// holds "indexer K / scale"). The pages print no score formula; the kernel
// computes the DSA-style reading
//     s_t = sum_h w_h * max(0, sigma_t * <q_h, k_t>)
// for every token t of the sequence's pages.
//
// Data path: HBM-bound streaming of 68 B per cached token. One CTA per SM
// owns a contiguous run of "units" (up to eight consecutive pages of one
// sequence, 512 tokens) and runs a warp-specialised pipeline:
//   producer (1 warp)   resolves 32 units at a time, one batch ahead (one
//        coalesced page-table load per lane; the first batch before the
//        wait on the previous kernel, since the page table is an input),
//        and each lane with a unit copies its pages (4 KB key pages + 256 B
//        scale rows, cp.async.bulk without multicast, L2 evict-first) into
//        the next of S ring slots once that slot is free; the slot's "full"
//        mbarrier completes with the bytes. The launch's first S units are
//        issued one after another (the SM's bulk-copy engine serves copies
//        in issue order, so the first unit lands early); later units are
//        issued together by the lanes whose slots are free.
//   MMA (2 warps)       units alternate between two issuing threads (the
//        per-unit waits and the commit, not the tensor core, bound one
//        thread); each issues, per unit, eight tcgen05.mma kind::f8f6f4
//        (E4M3 x E4M3 -> fp32; four 128-token blocks x two 32-channel steps,
//        N = 16 query columns) from the slot straight into one of 4 TMEM
//        accumulators, and one commit (a commit costs several MMAs' worth
//        of issue time, so units are sized to amortise it). The key pages
//        are stored as 8 x 16-byte core matrices (byte (t, c) at
//        (t/8)*512 + (c/16)*128 + (t%8)*16 + c%16), the tensor core's
//        no-swizzle K-major operand layout, so they are used as copied. The
//        query (column n = query token * 4 + head) is written once per
//        sequence into the same layout (the CTA's first sequence while the
//        first copies are in flight).
//   epilogue (16 warps) 4 groups of 4 warps take the units in turn; warp q
//        of a group reads TMEM lanes 32q .. 32q+31 of every block (one token
//        per thread and block, all heads), applies sigma, ReLU and the head
//        weights, stores the scores (128-byte coalesced, L2 evict-last: the
//        selection re-reads them) and adds each valid score's top 11 key
//        bits to a shared-memory histogram per query row (rows past the
//        shared slots go straight to the global histogram).
// Every wait is a bounded mbarrier wait that sleeps between probes; a
// timeout sets the status word, stops the pipeline and the producer waits
// (bounded) for its copies before the CTA exits.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kTopkBins = 2048;                 // top 11 bits of the key
constexpr int kTopkDigitShift = 21;
constexpr int kIdxUnitPages = 8;                           // pages per unit
constexpr int kIdxBlocks = kIdxUnitPages / 2;               // M = 128-token MMA blocks per unit
constexpr int kIdxSlotKeys = kIdxUnitPages * kKidxPageBytes;   // 32 KB of keys
constexpr int kIdxSlotBytes = kIdxSlotKeys + kIdxUnitPages * kPage * 4;   // + scale rows
constexpr int kIdxEpiWarps = 16;
constexpr int kIdxGroups = kIdxEpiWarps / 4;
constexpr int kIdxAccBufs = kIdxGroups;                   // TMEM accumulators, one per group
constexpr int kIdxAccCols = 16;                           // N = 16 fp32 columns per block
constexpr int kIdxBufCols = kIdxBlocks * kIdxAccCols;      // one accumulator = all blocks of a unit
constexpr int kIdxTmemCols = kIdxAccBufs * kIdxBufCols;    // 256
constexpr int kIdxMmaWarps = 2;
constexpr int kIdxMmaWarp = kIdxEpiWarps;                 // first MMA warp
constexpr int kIdxProdWarp = kIdxEpiWarps + kIdxMmaWarps;
constexpr int kIdxThreads = (kIdxEpiWarps + kIdxMmaWarps + 1) * 32;
constexpr int kIdxQBytes = 16 * kIdxDim;                  // N = 16 rows x 64 B query operand

// Ring slots and shared histogram rows per launch shape (one query token per
// sequence, or more).
template <int Sq1>
struct IdxShape;
template <>
struct IdxShape<1> {
    static constexpr int kSlots = 6;
    static constexpr int kHistRows = 2;
};
template <>
struct IdxShape<0> {
    static constexpr int kSlots = 4;
    static constexpr int kHistRows = 8;
};

struct IdxUnitMeta {
    int b;          // sequence, or -1: stop mark
    int p0;         // first logical page
    int np;         // pages present (1 .. 8)
    int slot;       // ring slot
};

template <int Sq1>
struct IdxSmem {
    static constexpr int S = IdxShape<Sq1>::kSlots;
    alignas(128) uint8_t slot[S][kIdxSlotBytes];
    alignas(128) uint8_t qop[kIdxMmaWarps][kIdxQBytes];   // query operand per MMA warp
    uint32_t hist[IdxShape<Sq1>::kHistRows * kTopkBins];
    IdxUnitMeta meta[S];
    IdxUnitMeta acc_meta[kIdxAccBufs];
    uint64_t full[S];
    uint64_t empty[S];
    uint64_t acc_full[kIdxAccBufs];
    uint64_t acc_empty[kIdxAccBufs];
    uint64_t q_free[kIdxMmaWarps];
    uint32_t tmem_base;
};
template <int Sq1>
constexpr size_t idx_smem_bytes() { return sizeof(IdxSmem<Sq1>) + 128; }

struct IdxArgs {
    const uint8_t *q_idx;        // [B][Sq][4][64]
    const float *w;              // [B][Sq][4]
    const uint8_t *kidx;         // [pages][4096]
    const float *kidx_scale;     // [pages][64]
    int64_t num_pages;
    const int32_t *page_table;   // [B][max_pages]
    int max_pages;
    const int32_t *seq_lens;     // [B]
    int B;
    int Sq;
    float *scores;               // [B*Sq][t_cap]
    int64_t t_cap;
    uint32_t *hist;              // [B*Sq][kTopkBins], zero on entry
};

__device__ __forceinline__ int idx_seq_len(const int32_t *seq_lens, int b, int Sq, int max_pages) {
    const int T = seq_lens[b];
    if (T < Sq || T > max_pages * kPage) return -1;
    return T;
}

// D[tmem] (+)= A[smem] * B[smem] with E4M3 operands, one thread issues.
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate) : "memory");
}

// 32 lanes x 4 columns of 32-bit TMEM data: thread i gets lane (base + i).
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&v)[4]) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}

// Bounded wait by lane 0 for the whole warp (the result and the memory
// ordering reach every lane through the broadcast and __syncwarp).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait_bounded(bar, parity);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok;
}


template <int Sq1>
__global__ void __launch_bounds__(kIdxThreads, 1)
indexer_score_kernel(const IdxArgs A) {
    using Sm = IdxSmem<Sq1>;
    constexpr int S = Sm::S;
    constexpr int kRows = IdxShape<Sq1>::kHistRows;
    constexpr int kCols = Sq1 ? 4 : 16;                  // accumulator columns read per token
    extern __shared__ uint8_t smem_raw[];
    Sm &sm = *reinterpret_cast<Sm *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int Sq = A.Sq;

    const int ups = (A.max_pages + kIdxUnitPages - 1) / kIdxUnitPages;   // units per sequence
    const int64_t n_units = static_cast<int64_t>(A.B) * ups;
    const int64_t cta0 = n_units * blockIdx.x / gridDim.x;
    const int64_t cta1 = n_units * (blockIdx.x + 1) / gridDim.x;
    const int b_first = static_cast<int>(cta0 / ups);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 4);
        }
        for (int i = 0; i < kIdxAccBufs; ++i) {
            mbar_init(&sm.acc_full[i], 2);
            mbar_init(&sm.acc_empty[i], 4);
        }
        for (int i = 0; i < kIdxMmaWarps; ++i) mbar_init(&sm.q_free[i], 1);
        fence_mbar_init();
    }
    for (int i = tid; i < kRows * kTopkBins; i += blockDim.x) sm.hist[i] = 0u;
    for (int i = tid; i < kIdxMmaWarps * kIdxQBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(&sm.qop[0][0])[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();                           // the zero rows are read by the tensor core
    if (warp == kIdxMmaWarp) {
        tmem_alloc(&sm.tmem_base, kIdxTmemCols);
        tmem_relinquish();
    }
    // Lane-parallel resolution of unit u: sequence, first page, pages
    // present (the prefix below T with good page-table entries) and their
    // physical pages.
    struct Unit {
        int b, p0, np;
        int32_t ph[kIdxUnitPages];
    };
    auto resolve = [&](int64_t u, Unit &r) {
        r.b = 0;
        r.p0 = 0;
        r.np = 0;
        if (u >= cta1) return;
        r.b = static_cast<int>(u / ups);
        r.p0 = static_cast<int>(u - static_cast<int64_t>(r.b) * ups) * kIdxUnitPages;
        const int T = idx_seq_len(A.seq_lens, r.b, Sq, A.max_pages);
        if (T < 0) {
            if (r.p0 == 0) flag_status(kStatusBounds);
            return;
        }
        int32_t e[kIdxUnitPages];
#pragma unroll
        for (int pg = 0; pg < kIdxUnitPages; ++pg) {       // loads first, checks after
            const int p = r.p0 + pg;
            e[pg] = (p < A.max_pages && p * kPage < T) ? A.page_table[static_cast<int64_t>(r.b) * A.max_pages + p]
                                                       : -2;
        }
#pragma unroll
        for (int pg = 0; pg < kIdxUnitPages; ++pg) {
            r.ph[pg] = e[pg];
            if (r.np == pg && e[pg] != -2) {
                if (e[pg] >= 0 && e[pg] < A.num_pages) ++r.np;
                else flag_status(kStatusBounds);
            }
        }
    };
    // The page table and sequence lengths are inputs no earlier kernel of the
    // step writes: the producer resolves its first batch before the wait.
    Unit cur;
    if (warp == kIdxProdWarp) resolve(cta0 + lane, cur);
    pdl_wait();                                         // cache pages and zeroed histograms are ready
    pdl_trigger();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == kIdxProdWarp) {
        // ------------------------------------------------ producer
        const uint64_t pol_stream = l2_policy_evict_first();
        int64_t n_issued = 0;                           // units placed in the ring so far
        bool ok = true;
        auto slot_wait = [&](int64_t i) -> bool {       // the slot of ring index i is free
            if (i < S) return true;
            return mbar_wait_bounded(&sm.empty[i % S], static_cast<uint32_t>((i / S - 1) & 1));
        };
        Unit nxt;
        for (int64_t u0 = cta0; u0 < cta1 && ok; u0 += 32) {
            resolve(u0 + 32 + lane, nxt);               // the next batch's loads overlap this batch's copies
            const bool live = cur.np > 0;
            const uint32_t todo = __ballot_sync(0xffffffffu, live);
            const int rank = __popc(todo & ((1u << lane) - 1u));
            // Issue in chunks of S ring positions: a lane only waits on a slot
            // filled by an earlier chunk. The launch's first chunk goes one
            // unit at a time (all of rank r's copies before rank r + 1's): the
            // SM's bulk-copy engine takes copies in issue order, so the first
            // unit lands after its own copies instead of after the whole first
            // wave's. Later chunks issue together (lanes whose slots are free
            // do not wait for one another).
            const int n_live = __popc(todo);
            for (int r0 = 0; r0 < n_live;) {
                const int r1 = (n_issued == 0 && r0 < S) ? r0 + 1 : min(r0 - r0 % S + S, n_live);
                if (live && rank >= r0 && rank < r1) {
                    const int64_t i = n_issued + rank;
                    const int s = static_cast<int>(i % S);
                    if (slot_wait(i)) {
                        sm.meta[s] = IdxUnitMeta{cur.b, cur.p0, cur.np, s};
                        uint8_t *dst = sm.slot[s];
                        mbar_arrive_expect_tx(&sm.full[s], static_cast<uint32_t>((kKidxPageBytes + kPage * 4) * cur.np));
#pragma unroll
                        for (int pg = 0; pg < kIdxUnitPages; ++pg) {
                            if (pg < cur.np) {
                                const int64_t ph = cur.ph[pg];
                                bulk_g2s(dst + pg * kKidxPageBytes, A.kidx + ph * kKidxPageBytes, kKidxPageBytes,
                                         &sm.full[s], pol_stream);
                                bulk_g2s(dst + kIdxSlotKeys + pg * kPage * 4, A.kidx_scale + ph * kPage, kPage * 4,
                                         &sm.full[s], pol_stream);
                            }
                        }
                    } else {
                        ok = false;
                    }
                }
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                r0 = r1;
            }
            n_issued += __popc(todo);
            cur = nxt;
        }
        // One stop mark per epilogue group; the MMA warp forwards them.
        if (ok && lane < kIdxGroups) {
            const int64_t i = n_issued + lane;
            const int s = static_cast<int>(i % S);
            if (slot_wait(i)) {
                sm.meta[s] = IdxUnitMeta{-1, 0, 0, s};
                mbar_arrive(&sm.full[s]);
            } else {
                ok = false;
            }
        }
        // No copy may be in flight when the CTA exits: wait (bounded) for the
        // last filled phase of every slot.
        const int64_t n_total = n_issued + kIdxGroups;
        bool drain = true;                              // after a timeout give up at the first failure
        for (int s = lane; s < S && s < n_total && drain; s += 32) {
            const int64_t last = s + (n_total - 1 - s) / S * S;         // last ring index using slot s
            drain = mbar_wait_bounded(&sm.full[s], static_cast<uint32_t>((last / S) & 1));
        }
    } else if (warp >= kIdxMmaWarp) {
        // ------------------------------------------------ MMA issue: units i = mw, mw + 2, ...
        const int mw = warp - kIdxMmaWarp;
        constexpr uint32_t idesc = umma_idesc(128, kIdxAccCols, false, false);   // E4M3 x E4M3, fp32
        uint8_t *qop = sm.qop[mw];
        const uint32_t q_addr = smem_u32(qop);
        // column n = query token * 4 + head; 16 B chunk c of its 64 channels
        auto stage_q = [&](int b) {
            for (int k = lane; k < 4 * Sq * (kIdxDim / 16); k += 32) {
                const int n = k >> 2, c = k & 3;
                const uint4 v = *reinterpret_cast<const uint4 *>(
                    A.q_idx + (static_cast<int64_t>(b) * Sq * kIdxHeads + n) * kIdxDim + c * 16);
                *reinterpret_cast<uint4 *>(qop + (n >> 3) * 512 + c * 128 + (n & 7) * 16) = v;
            }
            fence_proxy_async_smem();                   // generic writes -> tensor-core reads
            __syncwarp();
        };
        // The CTA's first sequence is staged while the first copies are in flight.
        int cur_b = b_first, stops = 0;
        stage_q(cur_b);
        uint32_t q_phase = 0u;
        for (int64_t i = mw; stops < kIdxGroups / kIdxMmaWarps; i += kIdxMmaWarps) {
            const int s = static_cast<int>(i % S);
            const int buf = static_cast<int>(i % kIdxAccBufs);
            if (!warp_wait(&sm.full[s], static_cast<uint32_t>((i / S) & 1))) break;
            const IdxUnitMeta m = sm.meta[s];
            if (i >= kIdxAccBufs && !warp_wait(&sm.acc_empty[buf], static_cast<uint32_t>((i / kIdxAccBufs - 1) & 1)))
                break;
            tc_fence_after();
            if (m.b >= 0 && m.b != cur_b) {
                // New sequence: every MMA reading the old query must be done
                // before the operand is rewritten.
                if (lane == 0) umma_commit(&sm.q_free[mw]);
                if (!warp_wait(&sm.q_free[mw], q_phase)) break;
                q_phase ^= 1u;
                cur_b = m.b;
                stage_q(cur_b);
            }
            if (lane == 0) {
                sm.acc_meta[buf] = m;
                if (m.b >= 0) {
                    const uint32_t a_addr = smem_u32(sm.slot[s]);
#pragma unroll
                    for (int hf = 0; hf < kIdxBlocks; ++hf) {
                        if (2 * hf < m.np) {
                            const uint32_t d = tmem + buf * kIdxBufCols + hf * kIdxAccCols;
#pragma unroll
                            for (int ks = 0; ks < kIdxDim / 32; ++ks) {
                                const uint64_t ad = umma_desc(a_addr + hf * 2 * kKidxPageBytes + ks * 256, 128, 512, 0);
                                const uint64_t bd = umma_desc(q_addr + ks * 256, 128, 512, 0);
                                umma_e4m3(d, ad, bd, idesc, ks > 0 ? 1u : 0u);
                            }
                        }
                    }
                    umma_commit(&sm.acc_full[buf]);
                } else {
                    ++stops;
                    mbar_arrive(&sm.acc_full[buf]);     // stands in for the commit
                }
                mbar_arrive(&sm.acc_full[buf]);          // orders acc_meta for the epilogue
            }
            stops = __shfl_sync(0xffffffffu, stops, 0);
        }
    } else {
        // ------------------------------------------------ epilogue
        const int grp = warp >> 2, q = warp & 3;         // TMEM lanes 32q .. 32q+31
        const uint64_t pol_keep = l2_policy_evict_last();
        int cur_b = -1, cur_T = 0, hrow0 = 0;
        float wq[4][4];
        auto load_seq = [&](int b) {
            cur_b = b;
            cur_T = A.seq_lens[b];
            hrow0 = (b - b_first) * Sq;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
#pragma unroll
                for (int h = 0; h < 4; ++h)
                    wq[qq][h] = qq < Sq ? A.w[(static_cast<int64_t>(b) * Sq + qq) * kIdxHeads + h] : 0.0f;
        };
        load_seq(b_first);                              // while the first copies are in flight
        for (int64_t i = grp;; i += kIdxGroups) {
            const int buf = static_cast<int>(i % kIdxAccBufs);
            if (!warp_wait(&sm.acc_full[buf], static_cast<uint32_t>((i / kIdxAccBufs) & 1))) break;
            tc_fence_after();
            const IdxUnitMeta m = sm.acc_meta[buf];
            if (m.b < 0) {
                if (lane == 0) mbar_arrive(&sm.empty[m.slot]);
                break;
            }
            // this thread: token j of page 2*hf + (q >> 1) of the unit, for every block hf
            const int j = (q & 1) * 32 + lane;
            const float *sgp = reinterpret_cast<const float *>(sm.slot[m.slot] + kIdxSlotKeys);
            float sig[kIdxBlocks];
#pragma unroll
            for (int hf = 0; hf < kIdxBlocks; ++hf) sig[hf] = sgp[(2 * hf + (q >> 1)) * kPage + j];
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[m.slot]);
            if (m.b != cur_b) load_seq(m.b);
            // Scores of this thread's token in block hf from its accumulator row.
            auto emit = [&](int hf, const float *acc) {
                const int pg = 2 * hf + (q >> 1);
                if (pg >= m.np) return;
                const int t = (m.p0 + pg) * kPage + j;
                float *srow = A.scores + static_cast<int64_t>(cur_b) * Sq * A.t_cap + t;
#pragma unroll
                for (int qq = 0; qq < kCols / 4; ++qq) {
                    if (qq < Sq) {
                        float score = 0.0f;
#pragma unroll
                        for (int h = 0; h < 4; ++h) score += wq[qq][h] * fmaxf(0.0f, sig[hf] * acc[qq * 4 + h]);
                        st_policy(srow + qq * A.t_cap, score, pol_keep);
                        if (t <= cur_T - Sq + qq) {
                            const uint32_t bin = float_key(score) >> kTopkDigitShift;
                            const int hr = hrow0 + qq;
                            if (hr < kRows) atomicAdd(&sm.hist[hr * kTopkBins + bin], 1u);
                            else atomicAdd(&A.hist[(static_cast<int64_t>(cur_b) * Sq + qq) * kTopkBins + bin], 1u);
                        }
                    }
                }
            };
            const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16) + buf * kIdxBufCols;
            if constexpr (kCols == 4) {
                // all blocks to registers, release the accumulator, then score
                float acc[kIdxBlocks][4];
#pragma unroll
                for (int hf = 0; hf < kIdxBlocks; ++hf) tmem_ld4(trow + hf * kIdxAccCols, acc[hf]);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
#pragma unroll
                for (int hf = 0; hf < kIdxBlocks; ++hf) emit(hf, acc[hf]);
            } else {
                // 16 columns per block: one block at a time keeps registers low
#pragma unroll
                for (int hf = 0; hf < kIdxBlocks; ++hf) {
                    float acc[16];
                    tmem_ld16(trow + hf * kIdxAccCols, acc);
                    emit(hf, acc);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kIdxMmaWarp) {                         // the allocating warp frees TMEM
        tc_fence_after();
        tmem_dealloc(tmem, kIdxTmemCols);
    }
    // Flush the shared histograms of the rows this CTA touched.
    const int b_last = static_cast<int>((cta1 > cta0 ? cta1 - 1 : cta0) / ups);
    const int n_rows = min(kRows, (b_last - b_first + 1) * Sq);
    for (int i = tid; i < n_rows * kTopkBins; i += blockDim.x) {
        const uint32_t c = sm.hist[i];
        if (c) atomicAdd(&A.hist[static_cast<int64_t>(b_first) * Sq * kTopkBins + i], c);
    }
}

}  // namespace csa2
