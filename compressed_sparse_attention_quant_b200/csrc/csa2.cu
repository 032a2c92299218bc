// csa2.cu -- C-ABI entry points of the CSA2 FP4 sparse-decode library:
// argument validation, workspace layout and kernel launches. The kernels are
// in quant.cuh (K1), indexer.cuh (K2), topk.cuh (K3) and attn.cuh (K4/K5).
#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>

#include "attn.cuh"
#include "common.cuh"
#include "indexer.cuh"
#include "quant.cuh"
#include "topk.cuh"
#include "pool.cuh"

namespace csa2 {

std::atomic<uint64_t> g_launches{0};

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    int sm_count = 0;
    int att_ctas_per_sm = 0;
    int tk_max_cluster = 1;       // largest power-of-two top-k cluster the device can co-schedule
};
DeviceInfo g_dev[kMaxDevices];

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

cudaError_t device_info(DeviceInfo **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
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
                                 reinterpret_cast<const void *>(pool_topk_kernel)};
        for (const void *kf : kernels) {
            e = cudaFuncSetAttribute(kf, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
            if (e != cudaSuccess) return e;
        }

        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.att_ctas_per_sm, sparse_attn_kernel, kAttThreads,
                                                          kAttSmemBytes);
        if (e != cudaSuccess) return e;
        if (d.att_ctas_per_sm < 1) d.att_ctas_per_sm = 1;
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
        d.ready = true;
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

// ---------------------------------------------------------------- attention splits
struct AttSplit {
    int n_splits;
    int tiles_per_split;
};

// Split the (k + 128)-key list of each query row into S contiguous tile runs
// so that R * S CTAs fill the machine: minimise waves x tiles per CTA, with a
// small charge per split for writing and merging its partial.
AttSplit att_split(int R, int k, int slots) {
    const int n_tiles = (k + kWindow + kAttTile - 1) / kAttTile;
    const int s_min = (n_tiles + kMaxTilesPerSplit - 1) / kMaxTilesPerSplit;
    AttSplit best{s_min, (n_tiles + s_min - 1) / s_min};
    double best_cost = 1e30;
    for (int s = s_min; s <= n_tiles && s <= s_min + 64; ++s) {
        const int tps = (n_tiles + s - 1) / s;
        const int s_eff = (n_tiles + tps - 1) / tps;
        const int64_t ctas = static_cast<int64_t>(R) * s_eff;
        const int64_t waves = (ctas + slots - 1) / slots;
        const double cost = static_cast<double>(waves) * tps + (s_eff > 1 ? 0.25 * s_eff : 0.0);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = AttSplit{s_eff, tps};
        }
    }
    return best;
}

size_t att_ws_bytes(int R, const AttSplit &sp) {
    if (sp.n_splits <= 1) return 0;
    const size_t po = round_up(static_cast<size_t>(R) * sp.n_splits * kHeads * kDim * 4, 256);
    const size_t pm = round_up(static_cast<size_t>(R) * sp.n_splits * kHeads * 8, 256);
    return po + pm;
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
    return cuda_status(launch_quant_index_fp8(x_bf16, n_rows, codes_e4m3, sigma, dev->sm_count,
                                              static_cast<cudaStream_t>(stream)));
}

size_t csa2_indexer_topk_workspace_bytes(int B, int Sq, int max_pages, int k) {
    if (B <= 0 || Sq <= 0 || max_pages <= 0 || k <= 0) return 0;
    return idx_layout(B, Sq, max_pages, k).total;
}

csa2_status csa2_indexer_topk(const void *q_idx, const float *w, int B, int Sq, int idx_heads, int idx_dim,
                              const csa2_paged_cache *cache, const int32_t *page_table, int max_pages,
                              const int32_t *seq_lens, int k, int32_t *out_idx, void *ws, size_t ws_bytes,
                              void *stream) {
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
        !aligned(page_table, 4) || !aligned(seq_lens, 4) || !aligned(out_idx, 4))
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
    // 8192 positions.
    int C = 1;
    while (C * 2 <= dev->tk_max_cluster && static_cast<int64_t>(R) * C * 2 <= dev->sm_count &&
           L.t_cap / (C * 2) >= 8192)
        C *= 2;
    e = launch_pdl_cluster(topk_cluster_kernel, dim3(static_cast<unsigned>(R * C)), dim3(kTkThreads), sizeof(TkSmem),
                           st, C, static_cast<const float *>(scores), L.t_cap, static_cast<const uint32_t *>(hist),
                           seq_lens, Sq, max_pages, k, out_idx);
    return cuda_status(e);
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
    A.k = k;
    A.out = out_idx;
    return cuda_status(launch_pool_topk(A, B * Sq, static_cast<cudaStream_t>(stream)));
}

size_t csa2_sparse_attn_workspace_bytes(int B, int Sq, int k) {
    if (B <= 0 || Sq <= 0 || k < 0) return 0;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return 0;
    const int R = B * Sq;
    return att_ws_bytes(R, att_split(R, k, dev->sm_count * dev->att_ctas_per_sm));
}

csa2_status csa2_sparse_attn_decode(const void *q_bf16, int B, int Sq, int H, int D,
                                    const csa2_paged_cache *cache, const int32_t *page_table, int max_pages,
                                    const int32_t *seq_lens, const int32_t *topk_idx, int k,
                                    const void *swa_bf16, int W, float softmax_scale, float *out, float *lse,
                                    void *ws, size_t ws_bytes, void *stream) {
    if (H != kHeads || D != kDim || W != kWindow) return CSA2_ERR_UNSUPPORTED;
    if (B <= 0 || Sq <= 0 || k < 0 || k > 65536 || max_pages <= 0 || !cache_ok(cache) ||
        !std::isfinite(softmax_scale))
        return CSA2_ERR_INVALID_ARG;
    if (static_cast<int64_t>(B) * Sq > 65535) return CSA2_ERR_UNSUPPORTED;
    if (!q_bf16 || !page_table || !seq_lens || (k > 0 && !topk_idx) || !swa_bf16 || !out || !lse ||
        !cache->kv_fp4 || !cache->kv_scale)
        return CSA2_ERR_INVALID_ARG;
    if (!aligned(q_bf16, 16) || !aligned(swa_bf16, 16) || !aligned(cache->kv_fp4, 16) ||
        !aligned(cache->kv_scale, 4) || !aligned(out, 16) || !aligned(lse, 4) || !aligned(page_table, 4) ||
        !aligned(seq_lens, 4) || (topk_idx && !aligned(topk_idx, 4)))
        return CSA2_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return CSA2_ERR_CUDA;
    const int R = B * Sq;
    const AttSplit sp = att_split(R, k, dev->sm_count * dev->att_ctas_per_sm);
    const size_t need = att_ws_bytes(R, sp);
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
    P.n_splits = sp.n_splits;
    P.tiles_per_split = sp.tiles_per_split;
    P.part_o = nullptr;
    P.part_ml = nullptr;
    if (sp.n_splits > 1) {
        uint8_t *base = static_cast<uint8_t *>(ws);
        P.part_o = reinterpret_cast<float *>(base);
        P.part_ml = reinterpret_cast<float2 *>(
            base + round_up(static_cast<size_t>(R) * sp.n_splits * kHeads * kDim * 4, 256));
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    dim3 grid(sp.n_splits, R);
    cudaError_t e = launch_pdl(sparse_attn_kernel, grid, dim3(kAttThreads), kAttSmemBytes, st, P);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
    if (sp.n_splits > 1) {
        e = launch_pdl(attn_merge_kernel, dim3(R, kHeads / kMergeHeads), dim3(kMergeThreads),
                       sp.n_splits * kMergeHeads * sizeof(float2), st,
                       static_cast<const float *>(P.part_o), static_cast<const float2 *>(P.part_ml), sp.n_splits,
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
    if (B <= 0 || Sq <= 0 || k < 0) return CSA2_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CSA2_ERR_CUDA;
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return CSA2_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
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
