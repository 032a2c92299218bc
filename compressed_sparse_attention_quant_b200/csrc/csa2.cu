// csa2.cu -- C-ABI entry points of the CSA2 FP4 sparse-decode library:
// argument validation, workspace layout and kernel launches. The kernels are
// in quant.cuh (K1), indexer.cuh (K2), topk.cuh (K3) and attn.cuh (K4/K5).
#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>

#include "attn.cuh"
#include "common.cuh"
#include "indexer.cuh"
#include "quant.cuh"
#include "topk.cuh"
#include "pool.cuh"
#include "replay.cuh"

namespace csa2 {

std::atomic<uint64_t> g_launches{0};

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    std::atomic<bool> ready{false};
    int sm_count = 0;
    int att_ctas_per_sm = 0;
    int q8_blocks = 0;            // resident blocks of the FP8 quantiser (whole device)
    int tk_max_cluster = 1;       // largest power-of-two top-k cluster the device can co-schedule
};
DeviceInfo g_dev[kMaxDevices];
// Serialises the one-time per-device set-up (attributes, occupancy, scratch
// address) when several host threads make their first call at once.
std::mutex g_init_mutex;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

cudaError_t device_info(DeviceInfo **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    DeviceInfo &d = g_dev[dev];
    if (d.ready.load(std::memory_order_acquire)) {
        *out = &d;
        return cudaSuccess;
    }
    std::lock_guard<std::mutex> lock(g_init_mutex);
    if (!d.ready.load(std::memory_order_relaxed)) {
        e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(indexer_score_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(idx_smem_bytes<1>()));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(indexer_score_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(idx_smem_bytes<0>()));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kAttSmemBytes));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(sizeof(TkSmem)));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(pool_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(pool_smem_bytes(kPoolMax)));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(swa_replay_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kRpSmemBytes));
        if (e != cudaSuccess) return e;
        // One shared-memory carveout for every kernel of the path, so that
        // consecutive launches do not reconfigure the SMs' L1 / shared split.
        const void *kernels[] = {reinterpret_cast<const void *>(quant_kv_fp4_kernel),
                                 reinterpret_cast<const void *>(indexer_score_kernel<1>),
                                 reinterpret_cast<const void *>(indexer_score_kernel<0>),
                                 reinterpret_cast<const void *>(topk_zero_kernel),
                                 reinterpret_cast<const void *>(topk_cluster_kernel),
                                 reinterpret_cast<const void *>(sparse_attn_kernel),
                                 reinterpret_cast<const void *>(attn_merge_kernel),
                                 reinterpret_cast<const void *>(quant_index_fp8_kernel),
                                 reinterpret_cast<const void *>(pool_topk_kernel),
                                 reinterpret_cast<const void *>(lse_merge_kernel),
                                 reinterpret_cast<const void *>(swa_replay_kernel)};
        for (const void *kf : kernels) {
            e = cudaFuncSetAttribute(kf, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
            if (e != cudaSuccess) return e;
        }

        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.att_ctas_per_sm, sparse_attn_kernel, kAttThreads,
                                                          kAttSmemBytes);
        if (e != cudaSuccess) return e;
        if (d.att_ctas_per_sm < 1) d.att_ctas_per_sm = 1;
        int q8 = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&q8, quant_index_fp8_kernel, kIdxQuantThreads, 0);
        if (e != cudaSuccess) return e;
        d.q8_blocks = std::max(1, q8) * d.sm_count;
        // Largest top-k cluster (<= 16 CTAs) that fits on the device at once.
        d.tk_max_cluster = 1;
        for (int cs = kTkMaxCluster; cs > 1; cs /= 2) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(cs);
            cfg.blockDim = dim3(kTkThreads);
            cfg.dynamicSmemBytes = sizeof(TkSmem);
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = cs;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n_clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&n_clusters, topk_cluster_kernel, &cfg) == cudaSuccess &&
                n_clusters >= 1) {
                d.tk_max_cluster = cs;
                break;
            }
            (void)cudaGetLastError();                      // clear a refusal of this size
        }
        d.ready.store(true, std::memory_order_release);
    }
    *out = &d;
    return cudaSuccess;
}

// ---------------------------------------------------------------- indexer / top-k workspace
struct IdxLayout {
    int64_t t_cap;
    size_t scores, hist, zero_end, total;
};

IdxLayout idx_layout(int B, int Sq, int max_pages, int k) {
    IdxLayout L{};
    const int64_t R = static_cast<int64_t>(B) * Sq;
    L.t_cap = static_cast<int64_t>(max_pages) * kPage;
    size_t off = 0;
    L.scores = off;    off = round_up(off + static_cast<size_t>(R * L.t_cap) * 4, 256);
    L.hist = off;      off = round_up(off + static_cast<size_t>(R) * kTopkBins * 4, 256);
    L.zero_end = off;
    L.total = off;
    return L;
}

// ---------------------------------------------------------------- attention work plan
struct AttPlan {
    int n_win;           // window tiles per query row (2, or 0 without a window)
    int n_st;            // tiles of 64 keys per query row
    int n_splits;        // S: runs per row, one CTA each
    int tps;             // tiles per run
    int R;
};

// Split each row's tiles into S runs so that the R * S CTAs fill the machine:
// minimise waves x tiles per CTA, with a small charge per run for writing and
// merging its partial.
AttPlan att_plan(int R, int k, int slots, bool window = true) {
    AttPlan pl;
    pl.R = R;
    pl.n_win = window ? kWindow / kAttTile : 0;
    pl.n_st = pl.n_win + (k + kAttTile - 1) / kAttTile;
    pl.n_splits = 1;
    pl.tps = pl.n_st;
    double best = 1e30;
    for (int s = 1; s <= pl.n_st && s <= kMergeMaxParts; ++s) {
        const int tps = (pl.n_st + s - 1) / s;
        const int s_eff = (pl.n_st + tps - 1) / tps;
        if (s_eff > 1 && static_cast<int64_t>(R) * s_eff > slots) break;   // split only within one wave
        const int64_t waves = (static_cast<int64_t>(R) * s_eff + slots - 1) / slots;
        const double cost = static_cast<double>(waves) * tps + (s_eff > 1 ? 0.25 * s_eff : 0.0);
        if (cost < best - 1e-9) {
            best = cost;
            pl.n_splits = s_eff;
            pl.tps = tps;
        }
    }
    return pl;
}

// Partials: one per (row, run) when a row is split.
size_t att_ws_bytes(const AttPlan &pl) {
    if (pl.n_splits <= 1) return 0;
    const size_t n = static_cast<size_t>(pl.R) * pl.n_splits;
    return round_up(n * kHeads * kDim * 4, 256) + round_up(n * kHeads * 8, 256);
}

csa2_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA; }

bool cache_ok(const csa2_paged_cache *c) {
    return c != nullptr && c->num_pages > 0 && c->num_pages <= (INT64_C(1) << 31) / kPage;
}

}  // namespace
}  // namespace csa2

using namespace csa2;

extern "C" {

csa2_status csa2_quant_kv_fp4(const void *x_bf16, int64_t n_tok, int dim, const int32_t *slot_mapping,
                              const void *kidx_in, const float *kidx_scale_in,
                              const csa2_paged_cache *cache, void *stream) {
    if (n_tok < 0 || !cache_ok(cache)) return CSA2_ERR_INVALID_ARG;
    if (dim != kDim) return CSA2_ERR_UNSUPPORTED;
    if (n_tok == 0) return CSA2_OK;
    if (!x_bf16 || !slot_mapping || !cache->kv_fp4 || !cache->kv_scale) return CSA2_ERR_INVALID_ARG;
    if (kidx_in && (!kidx_scale_in || !cache->kidx || !cache->kidx_scale)) return CSA2_ERR_INVALID_ARG;
    if (!aligned(x_bf16, 16) || !aligned(cache->kv_fp4, 16) || !aligned(slot_mapping, 4) ||
        (kidx_in && (!aligned(kidx_in, 16) || !aligned(cache->kidx, 16) || !aligned(cache->kidx_scale, 16) ||
                     !aligned(kidx_scale_in, 4))))
        return CSA2_ERR_ALIGNMENT;
    if (n_tok > (INT64_C(1) << 31) * kQuantThreads / (kDim / kGroup)) return CSA2_ERR_INVALID_ARG;
    return cuda_status(launch_quant_kv_fp4(x_bf16, n_tok, slot_mapping, kidx_in, kidx_scale_in, *cache,
                                           static_cast<cudaStream_t>(stream)));
}

csa2_status csa2_quant_indexer_fp8(const void *x_bf16, int64_t n_rows, int dim, void *codes_e4m3, float *sigma,
                                   void *stream) {
    if (n_rows < 0) return CSA2_ERR_INVALID_ARG;
    if (dim != kIdxDim) return CSA2_ERR_UNSUPPORTED;
    if (n_rows == 0) return CSA2_OK;
    if (!x_bf16 || !codes_e4m3 || !sigma) return CSA2_ERR_INVALID_ARG;
    if (!aligned(x_bf16, 16) || !aligned(codes_e4m3, 16) || !aligned(sigma, 4)) return CSA2_ERR_ALIGNMENT;
    if (n_rows > (INT64_C(1) << 40)) return CSA2_ERR_INVALID_ARG;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return CSA2_ERR_CUDA;
    return cuda_status(launch_quant_index_fp8(x_bf16, n_rows, codes_e4m3, sigma, dev->q8_blocks,
                                              static_cast<cudaStream_t>(stream)));
}

size_t csa2_indexer_topk_workspace_bytes(int B, int Sq, int max_pages, int k) {
    if (B <= 0 || Sq <= 0 || max_pages <= 0 || k <= 0) return 0;
    return idx_layout(B, Sq, max_pages, k).total;
}

}  // extern "C"

namespace csa2 {
namespace {

// csa2_indexer_topk, with the selected entries' scores written to out_scores
// when it is not null.
csa2_status indexer_topk_impl(const void *q_idx, const float *w, int B, int Sq, int idx_heads, int idx_dim,
                              const csa2_paged_cache *cache, const int32_t *page_table, int max_pages,
                              const int32_t *seq_lens, int k, int32_t *out_idx, float *out_scores, void *ws,
                              size_t ws_bytes, void *stream) {
    if (idx_heads != kIdxHeads || idx_dim != kIdxDim) return CSA2_ERR_UNSUPPORTED;
    if (B <= 0 || B > 65535 || Sq <= 0 || max_pages <= 0 || k <= 0 || k > 65536 || !cache_ok(cache))
        return CSA2_ERR_INVALID_ARG;
    if (Sq > 4) return CSA2_ERR_UNSUPPORTED;   // 4 query tokens x 4 heads = 16 MMA columns
    if (static_cast<int64_t>(B) * Sq > 65535) return CSA2_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(max_pages) * kPage > (INT64_C(1) << 30)) return CSA2_ERR_UNSUPPORTED;
    if (cache->num_pages > INT32_MAX) return CSA2_ERR_UNSUPPORTED;   // page-table entries are int32
    if (!q_idx || !w || !page_table || !seq_lens || !out_idx || !cache->kidx || !cache->kidx_scale)
        return CSA2_ERR_INVALID_ARG;
    if (!aligned(q_idx, 16) || !aligned(w, 16) || !aligned(cache->kidx, 16) || !aligned(cache->kidx_scale, 16) ||
        !aligned(page_table, 4) || !aligned(seq_lens, 4) || !aligned(out_idx, 4) ||
        (out_scores && !aligned(out_scores, 4)))
        return CSA2_ERR_ALIGNMENT;
    const IdxLayout L = idx_layout(B, Sq, max_pages, k);
    if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return CSA2_ERR_WORKSPACE;
    DeviceInfo *dev = nullptr;
    cudaError_t e = device_info(&dev);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *base = static_cast<uint8_t *>(ws);
    float *scores = reinterpret_cast<float *>(base + L.scores);
    uint32_t *hist = reinterpret_cast<uint32_t *>(base + L.hist);
    const int R = B * Sq;

    // The level-1 histograms start at zero.
    const int64_t n16 = static_cast<int64_t>((L.zero_end - L.hist) / 16);
    e = launch_pdl(topk_zero_kernel, dim3(static_cast<unsigned>(std::min<int64_t>((n16 + 255) / 256, 2 * dev->sm_count))),
                   dim3(256), 0, st, reinterpret_cast<uint4 *>(base + L.hist), n16);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;

    IdxArgs A;
    A.q_idx = static_cast<const uint8_t *>(q_idx);
    A.w = w;
    A.kidx = static_cast<const uint8_t *>(cache->kidx);
    A.kidx_scale = cache->kidx_scale;
    A.num_pages = cache->num_pages;
    A.page_table = page_table;
    A.max_pages = max_pages;
    A.seq_lens = seq_lens;
    A.B = B;
    A.Sq = Sq;
    A.scores = scores;
    A.t_cap = L.t_cap;
    A.hist = hist;
    const int64_t n_units = static_cast<int64_t>(B) * ((max_pages + kIdxUnitPages - 1) / kIdxUnitPages);
    const int grid1 = static_cast<int>(std::min<int64_t>(n_units, dev->sm_count));
    if (Sq == 1)
        e = launch_pdl(indexer_score_kernel<1>, dim3(grid1), dim3(kIdxThreads), idx_smem_bytes<1>(), st, A);
    else
        e = launch_pdl(indexer_score_kernel<0>, dim3(grid1), dim3(kIdxThreads), idx_smem_bytes<0>(), st, A);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
    // Top-k: one cluster of C CTAs per query row, C a power of two chosen so
    // that the R * C CTAs stay within one wave and every CTA keeps at least
    // 32768 positions (32 per thread: one bitmap word each).
    int C = 1;
    while (C * 2 <= dev->tk_max_cluster && static_cast<int64_t>(R) * C * 2 <= dev->sm_count &&
           L.t_cap / (C * 2) >= 32768)
        C *= 2;
    e = launch_pdl_cluster(topk_cluster_kernel, dim3(static_cast<unsigned>(R * C)), dim3(kTkThreads), sizeof(TkSmem),
                           st, C, static_cast<const float *>(scores), L.t_cap, static_cast<const uint32_t *>(hist),
                           seq_lens, Sq, max_pages, k, out_idx, out_scores);
    return cuda_status(e);
}

}  // namespace
}  // namespace csa2

extern "C" {

csa2_status csa2_indexer_topk(const void *q_idx, const float *w, int B, int Sq, int idx_heads, int idx_dim,
                              const csa2_paged_cache *cache, const int32_t *page_table, int max_pages,
                              const int32_t *seq_lens, int k, int32_t *out_idx, void *ws, size_t ws_bytes,
                              void *stream) {
    return indexer_topk_impl(q_idx, w, B, Sq, idx_heads, idx_dim, cache, page_table, max_pages, seq_lens, k, out_idx,
                             nullptr, ws, ws_bytes, stream);
}

csa2_status csa2_indexer_topk_scores(const void *q_idx, const float *w, int B, int Sq, int idx_heads, int idx_dim,
                                     const csa2_paged_cache *cache, const int32_t *page_table, int max_pages,
                                     const int32_t *seq_lens, int k, int32_t *out_idx, float *out_scores, void *ws,
                                     size_t ws_bytes, void *stream) {
    if (!out_scores) return CSA2_ERR_INVALID_ARG;
    return indexer_topk_impl(q_idx, w, B, Sq, idx_heads, idx_dim, cache, page_table, max_pages, seq_lens, k, out_idx,
                             out_scores, ws, ws_bytes, stream);
}

csa2_status csa2_indexer_pool_topk(const void *q_idx, const float *w, int B, int Sq, int idx_heads, int idx_dim,
                                   const csa2_paged_cache *cache, const int32_t *page_table, int max_pages,
                                   const int32_t *seq_lens, const int32_t *pool, int pool_size, int k,
                                   int32_t *out_idx, void *stream) {
    if (idx_heads != kIdxHeads || idx_dim != kIdxDim) return CSA2_ERR_UNSUPPORTED;
    if (B <= 0 || Sq <= 0 || max_pages <= 0 || k <= 0 || pool_size <= 0 || !cache_ok(cache))
        return CSA2_ERR_INVALID_ARG;
    if (pool_size > kPoolMax || static_cast<int64_t>(B) * Sq > 65535) return CSA2_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(max_pages) * kPage > (INT64_C(1) << 30)) return CSA2_ERR_UNSUPPORTED;
    if (cache->num_pages > INT32_MAX) return CSA2_ERR_UNSUPPORTED;
    if (!q_idx || !w || !page_table || !seq_lens || !pool || !out_idx || !cache->kidx || !cache->kidx_scale)
        return CSA2_ERR_INVALID_ARG;
    if (!aligned(cache->kidx, 16) || !aligned(cache->kidx_scale, 4) || !aligned(w, 4) || !aligned(page_table, 4) ||
        !aligned(seq_lens, 4) || !aligned(pool, 4) || !aligned(out_idx, 4))
        return CSA2_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return CSA2_ERR_CUDA;
    PoolArgs A;
    A.q_idx = static_cast<const uint8_t *>(q_idx);
    A.w = w;
    A.kidx = static_cast<const uint8_t *>(cache->kidx);
    A.kidx_scale = cache->kidx_scale;
    A.num_pages = cache->num_pages;
    A.page_table = page_table;
    A.max_pages = max_pages;
    A.seq_lens = seq_lens;
    A.Sq = Sq;
    A.pool = pool;
    A.C = pool_size;
    A.seg = pool_size;
    A.seg_stride = 0;
    A.row_stride = pool_size;
    A.given = nullptr;
    A.k = k;
    A.out = out_idx;
    A.out_local = nullptr;
    A.lo = 0;
    A.hi = 0;
    return cuda_status(launch_pool_topk(A, B * Sq, dev->sm_count, static_cast<cudaStream_t>(stream)));
}

csa2_status csa2_topk_merge(const float *cand_scores, const int32_t *cand_idx, int n_shards, int R, int k_shard,
                            int k, int32_t shard_lo, int32_t shard_hi, int32_t *out_idx, int32_t *out_local,
                            void *stream) {
    if (!cand_scores || !cand_idx || (!out_idx && !out_local) || n_shards <= 0 || R <= 0 || k_shard <= 0 || k <= 0)
        return CSA2_ERR_INVALID_ARG;
    if (R > 65535 || static_cast<int64_t>(n_shards) * k_shard > kPoolMax) return CSA2_ERR_UNSUPPORTED;
    if (!aligned(cand_scores, 4) || !aligned(cand_idx, 4) || (out_idx && !aligned(out_idx, 4)) ||
        (out_local && !aligned(out_local, 4)))
        return CSA2_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return CSA2_ERR_CUDA;
    PoolArgs A = {};
    A.Sq = 1;                                   // no sequence lengths in merge mode
    A.max_pages = 1;
    A.pool = cand_idx;
    A.C = n_shards * k_shard;
    A.seg = k_shard;
    A.seg_stride = static_cast<int64_t>(R) * k_shard;
    A.row_stride = k_shard;
    A.given = cand_scores;
    A.k = k;
    A.out = out_idx;
    A.out_local = out_local;
    A.lo = shard_lo;
    A.hi = shard_hi;
    return cuda_status(launch_pool_topk(A, R, dev->sm_count, static_cast<cudaStream_t>(stream)));
}

csa2_status csa2_swa_replay_attn(const void *q_bf16, int B, int L, int H, int D, const void *swa_bf16, int W,
                                 const int32_t *seq_lens, float softmax_scale, float *out, float *lse, void *stream) {
    if (H != kHeads || D != kDim || W != kWindow) return CSA2_ERR_UNSUPPORTED;
    if (B <= 0 || L <= 0 || !std::isfinite(softmax_scale)) return CSA2_ERR_INVALID_ARG;
    if (B > 65535 || L > (1 << 24)) return CSA2_ERR_UNSUPPORTED;
    if (!q_bf16 || !swa_bf16 || !seq_lens || !out || !lse) return CSA2_ERR_INVALID_ARG;
    if (!aligned(q_bf16, 16) || !aligned(swa_bf16, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
        !aligned(seq_lens, 4))
        return CSA2_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return CSA2_ERR_CUDA;
    RpParams P;
    P.q = static_cast<const __nv_bfloat16 *>(q_bf16);
    P.swa = static_cast<const __nv_bfloat16 *>(swa_bf16);
    P.seq_lens = seq_lens;
    P.L = L;
    P.scale_log2 = softmax_scale * 1.4426950408889634f;
    P.out = out;
    P.lse = lse;
    const dim3 grid(static_cast<unsigned>((L + kRpQueries - 1) / kRpQueries), static_cast<unsigned>(B));
    return cuda_status(launch_pdl(swa_replay_kernel, grid, dim3(kRpThreads), kRpSmemBytes,
                                  static_cast<cudaStream_t>(stream), P));
}

csa2_status csa2_lse_merge(const float *o_parts, const float *lse_parts, int n_parts, int R, float *out, float *lse,
                           void *stream) {
    if (!o_parts || !lse_parts || !out || !lse || n_parts <= 0 || R <= 0) return CSA2_ERR_INVALID_ARG;
    if (R > 65535) return CSA2_ERR_UNSUPPORTED;
    if (!aligned(o_parts, 16) || !aligned(out, 16) || !aligned(lse_parts, 4) || !aligned(lse, 4))
        return CSA2_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return CSA2_ERR_CUDA;
    return cuda_status(launch_pdl(lse_merge_kernel, dim3(R, kHeads / kMergeHeads), dim3(kMergeThreads), 0,
                                  static_cast<cudaStream_t>(stream), o_parts, lse_parts, n_parts, R, out, lse));
}

size_t csa2_sparse_attn_workspace_bytes(int B, int Sq, int k) {
    if (B <= 0 || Sq <= 0 || k < 0 || k > 65536 || static_cast<int64_t>(B) * Sq > 65535) return 0;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return 0;
    const int slots = dev->sm_count * dev->att_ctas_per_sm;
    return std::max(att_ws_bytes(att_plan(B * Sq, k, slots, true)), att_ws_bytes(att_plan(B * Sq, k, slots, false)));
}

csa2_status csa2_sparse_attn_decode(const void *q_bf16, int B, int Sq, int H, int D,
                                    const csa2_paged_cache *cache, const int32_t *page_table, int max_pages,
                                    const int32_t *seq_lens, const int32_t *topk_idx, int k,
                                    const void *swa_bf16, int W, float softmax_scale, float *out, float *lse,
                                    void *ws, size_t ws_bytes, void *stream) {
    if (H != kHeads || D != kDim || (W != kWindow && W != 0)) return CSA2_ERR_UNSUPPORTED;
    if (B <= 0 || Sq <= 0 || k < 0 || k > 65536 || max_pages <= 0 || !cache_ok(cache) ||
        !std::isfinite(softmax_scale) || (W == 0 && k == 0))
        return CSA2_ERR_INVALID_ARG;
    if (static_cast<int64_t>(B) * Sq > 65535) return CSA2_ERR_UNSUPPORTED;
    if (!q_bf16 || !page_table || !seq_lens || (k > 0 && !topk_idx) || (W > 0 && !swa_bf16) || !out || !lse ||
        !cache->kv_fp4 || !cache->kv_scale)
        return CSA2_ERR_INVALID_ARG;
    if (!aligned(q_bf16, 16) || (W > 0 && !aligned(swa_bf16, 16)) || !aligned(cache->kv_fp4, 16) ||
        !aligned(cache->kv_scale, 16) || !aligned(out, 16) || !aligned(lse, 4) || !aligned(page_table, 4) ||
        !aligned(seq_lens, 4) || (topk_idx && !aligned(topk_idx, 4)))
        return CSA2_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return CSA2_ERR_CUDA;
    const int R = B * Sq;
    const AttPlan pl = att_plan(R, k, dev->sm_count * dev->att_ctas_per_sm, W > 0);
    const size_t need = att_ws_bytes(pl);
    if (need > 0 && (!ws || !aligned(ws, 256) || ws_bytes < need)) return CSA2_ERR_WORKSPACE;

    AttParams P;
    P.q = static_cast<const __nv_bfloat16 *>(q_bf16);
    P.kv_fp4 = static_cast<const uint8_t *>(cache->kv_fp4);
    P.kv_scale = static_cast<const uint8_t *>(cache->kv_scale);
    P.num_pages = cache->num_pages;
    P.page_table = page_table;
    P.max_pages = max_pages;
    P.seq_lens = seq_lens;
    P.topk_idx = topk_idx;
    P.k = k;
    P.swa = static_cast<const __nv_bfloat16 *>(swa_bf16);
    P.Sq = Sq;
    P.scale_log2 = softmax_scale * 1.4426950408889634f;
    P.out = out;
    P.lse = lse;
    P.part_o = nullptr;
    P.part_ml = nullptr;
    P.n_win = pl.n_win;
    P.n_splits = pl.n_splits;
    P.tiles_per_split = pl.tps;
    if (need > 0) {
        uint8_t *base = static_cast<uint8_t *>(ws);
        P.part_o = reinterpret_cast<float *>(base);
        P.part_ml = reinterpret_cast<float2 *>(
            base + round_up(static_cast<size_t>(R) * pl.n_splits * kHeads * kDim * 4, 256));
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_pdl(sparse_attn_kernel, dim3(pl.n_splits, R), dim3(kAttThreads), kAttSmemBytes, st, P);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
    if (pl.n_splits > 1) {
        e = launch_pdl(attn_merge_kernel, dim3(R, kHeads / kMergeHeads), dim3(kMergeThreads), 0, st,
                       static_cast<const float *>(P.part_o), static_cast<const float2 *>(P.part_ml), pl.n_splits,
                       out, lse);
    }
    return cuda_status(e);
}

}  // extern "C"

namespace csa2 {
namespace {

// Library-owned scratch of csa2_sparse_attn_decode_noalloc: one copy per GPU
// that loads the library, alive until process exit.
__device__ __align__(256) uint8_t g_noalloc_scratch[CSA2_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device, looked up on the first call
// with that device current (the host-side symbol is not a device address).
void *g_noalloc_ptr[kMaxDevices] = {};

}  // namespace
}  // namespace csa2

extern "C" {

csa2_status csa2_sparse_attn_decode_noalloc(const void *q_bf16, int B, int Sq, int H, int D,
                                            const csa2_paged_cache *cache, const int32_t *page_table,
                                            int max_pages, const int32_t *seq_lens, const int32_t *topk_idx,
                                            int k, const void *swa_bf16, int W, float softmax_scale, float *out,
                                            float *lse, void *stream) {
    // The shape and range checks of csa2_sparse_attn_decode come first, so a
    // bad argument reports its own status rather than a workspace error.
    if (H != kHeads || D != kDim || (W != kWindow && W != 0)) return CSA2_ERR_UNSUPPORTED;
    if (B <= 0 || Sq <= 0 || k < 0 || k > 65536) return CSA2_ERR_INVALID_ARG;
    if (static_cast<int64_t>(B) * Sq > 65535) return CSA2_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CSA2_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_init_mutex);      // first call per device: one thread looks up
        if (g_noalloc_ptr[dev] == nullptr) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return CSA2_ERR_CUDA;
            g_noalloc_ptr[dev] = p;
        }
    }
    const size_t need = csa2_sparse_attn_workspace_bytes(B, Sq, k);
    if (need > CSA2_NOALLOC_SCRATCH_BYTES) return CSA2_ERR_WORKSPACE;
    return csa2_sparse_attn_decode(q_bf16, B, Sq, H, D, cache, page_table, max_pages, seq_lens, topk_idx, k,
                                   swa_bf16, W, softmax_scale, out, lse, g_noalloc_ptr[dev],
                                   CSA2_NOALLOC_SCRATCH_BYTES, stream);
}

csa2_status csa2_plan(const int *modes, int n_layers, int *kv_owner, int *index_src) {
    if (!modes || !kv_owner || !index_src || n_layers <= 0) return CSA2_ERR_INVALID_ARG;
    int owner = -1;
    for (int i = 0; i < n_layers; ++i) {
        switch (modes[i]) {
            case CSA2_FULL:
                owner = i;
                kv_owner[i] = i;
                index_src[i] = i;
                break;
            case CSA2_REINDEX:
                if (owner < 0) return CSA2_ERR_BAD_PLAN;
                kv_owner[i] = owner;
                index_src[i] = i;
                break;
            case CSA2_REUSE:
                if (owner < 0) return CSA2_ERR_BAD_PLAN;
                kv_owner[i] = owner;
                index_src[i] = owner;
                break;
            default:
                return CSA2_ERR_BAD_PLAN;
        }
    }
    return CSA2_OK;
}

csa2_status csa2_last_device_error(void *stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned int v = 0u;
    if (cudaMemcpyFromSymbolAsync(&v, g_status, sizeof v, 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return CSA2_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return CSA2_ERR_CUDA;
    if (v != 0u) {
        const unsigned int zero = 0u;
        if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
            return CSA2_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return CSA2_ERR_CUDA;
    }
    if (v & kStatusTimeout) return CSA2_ERR_TIMEOUT;
    if (v & kStatusBounds) return CSA2_ERR_DEVICE_BOUNDS;
    return CSA2_OK;
}

const char *csa2_status_string(csa2_status s) {
    switch (s) {
        case CSA2_OK: return "CSA2_OK";
        case CSA2_ERR_INVALID_ARG: return "CSA2_ERR_INVALID_ARG";
        case CSA2_ERR_UNSUPPORTED: return "CSA2_ERR_UNSUPPORTED";
        case CSA2_ERR_CUDA: return "CSA2_ERR_CUDA";
        case CSA2_ERR_BAD_PLAN: return "CSA2_ERR_BAD_PLAN";
        case CSA2_ERR_TIMEOUT: return "CSA2_ERR_TIMEOUT";
        case CSA2_ERR_DEVICE_BOUNDS: return "CSA2_ERR_DEVICE_BOUNDS";
        case CSA2_ERR_WORKSPACE: return "CSA2_ERR_WORKSPACE";
        case CSA2_ERR_ALIGNMENT: return "CSA2_ERR_ALIGNMENT";
    }
    return "CSA2_ERR_UNKNOWN";
}

uint64_t csa2_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
