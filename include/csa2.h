/*
 * csa2.h -- C ABI of the B200 (sm_100a) library for the decode step of
 * Compressed Sparse Attention 2 (CSA2) over an FP4 main KV cache.
 *
 * Sources of the operations (page title and section):
 *   [NEO] "DeepSeek 首次公开 V4.1-Flash 技术报告：552B 骨干参数与 CED 架构亮相，
 *         KV 缓存压至 890 字节" (neodrop.ai), architecture part 2 (CSA2: three
 *         static modes, shared main KV and indexer keys, top-K indices reused
 *         across layers) and part 3 (FP4 main KV: E2M1 with one E4M3 scale per
 *         16 channels).
 *   [ZUL] "DeepSeek V4 1-Flash 架构拆解：CED、CSA2、Engram、mHC 与 DSp"
 *         (blog.zulogic.cn), section 3 (mode table; KV owner -> compressed
 *         global KV, indexer K / scale, top-K metadata -> consumer layers) and
 *         section 4 (a 128-token sliding window kept per layer beside the
 *         global KV).
 *   [INF] "DeepSeek V4.1 Flash 模型架構與推論優化技術規格剖析" (infernews.com),
 *         section 2 (the window is the last 128 tokens) and the section-4 table
 *         (row "CSA 2": modes Full / Index / Reuse).
 *
 * Conventions shared by every entry point:
 *   - Pointers marked "device" point to device memory owned by the caller. The
 *     library allocates nothing and never synchronises on the compute calls.
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream. Compute calls only enqueue work on it.
 *   - Argument errors (null pointers, unsupported shapes, misaligned buffers,
 *     too small workspace) are detected on the host before anything is
 *     enqueued and returned as a status; nothing runs in that case.
 *   - Out-of-range values found in device data (page-table entries, slot ids,
 *     top-k indices, sequence lengths) never fault: the kernel skips the
 *     access, treats the entry as empty and sets a sticky device status word
 *     that csa2_last_device_error() reads and clears.
 *   - The shapes are fixed by the model: 16 query heads, 576 latent channels
 *     (keys = values), 4 indexer heads of 64 channels, a 128-token window and
 *     64-token KV pages. Other values return CSA2_ERR_UNSUPPORTED.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Static per-layer mode ([NEO part 2], [ZUL section 3]). */
typedef enum csa2_mode {
    CSA2_FULL = 0,     /* builds KV + indexer state, selects top-k, attends   */
    CSA2_REINDEX = 1,  /* reuses the owner's KV; recomputes its own top-k      */
    CSA2_REUSE = 2     /* reuses the owner's KV and an earlier layer's top-k   */
} csa2_mode;

typedef enum csa2_status {
    CSA2_OK = 0,
    CSA2_ERR_INVALID_ARG = 1,   /* null / negative / inconsistent argument      */
    CSA2_ERR_UNSUPPORTED = 2,   /* shape other than the fixed model shape       */
    CSA2_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed         */
    CSA2_ERR_BAD_PLAN = 4,      /* a layer has no Full layer before it          */
    CSA2_ERR_TIMEOUT = 5,       /* a bounded device wait gave up                */
    CSA2_ERR_DEVICE_BOUNDS = 6, /* device data held an out-of-range entry       */
    CSA2_ERR_WORKSPACE = 7,     /* workspace missing, misaligned or too small   */
    CSA2_ERR_ALIGNMENT = 8      /* a device buffer is not 16-byte aligned       */
} csa2_status;

enum {
    CSA2_HEADS = 16,            /* attention heads per query token              */
    CSA2_DIM = 576,             /* latent channels (keys = values)              */
    CSA2_IDX_HEADS = 4,         /* indexer heads                                */
    CSA2_IDX_DIM = 64,          /* indexer channels                             */
    CSA2_WINDOW = 128,          /* sliding window ([ZUL section 4], [INF 2])    */
    CSA2_PAGE_TOKENS = 64,      /* tokens per KV page                           */
    CSA2_GROUP = 16,            /* channels per E4M3 scale ([NEO part 3])       */
    CSA2_FP4_BYTES = 288,       /* packed E2M1 bytes per token (576 / 2)        */
    CSA2_SCALE_BYTES = 36,      /* E4M3 scale bytes per token (576 / 16)        */
    CSA2_KIDX_PAGE_BYTES = 4096 /* indexer-key bytes per page (64 x 64)         */
};

/*
 * The paged global cache of one KV owner (a Full layer), shared by the layers
 * that alias it ([ZUL section 3]: KV owner -> compressed global KV, indexer
 * K / scale). A host-side struct of caller-owned device arrays, all indexed
 * by physical page p in [0, num_pages), each 16-byte aligned:
 *
 *   kv_fp4     uint8 [num_pages][64][288]  token-major; byte j of a token
 *              holds channel 2j in its low nibble and channel 2j+1 in its high
 *              nibble, each an E2M1 code (bit 3 sign, bits 2..0 magnitude code
 *              of {0, .5, 1, 1.5, 2, 3, 4, 6}).
 *   kv_scale   uint8 [num_pages][64][36]   E4M3FN scale of channels 16g..16g+15.
 *   kidx       uint8 [num_pages][4096]     indexer keys, E4M3FN, 64 tokens x 64
 *              channels; byte of (token t, channel c) at
 *              (t/8)*512 + (c/16)*128 + (t%8)*16 + c%16
 *              (8x16-byte core matrices, the no-swizzle K-major operand layout
 *              of the tensor cores).
 *   kidx_scale float [num_pages][64]       per-token indexer scale sigma.
 *
 * Token t of sequence b lives in physical page page_table[b][t / 64], row
 * t % 64. A slot id is page * 64 + row.
 */
typedef struct csa2_paged_cache {
    void *kv_fp4;
    void *kv_scale;
    void *kidx;
    float *kidx_scale;
    int64_t num_pages;
} csa2_paged_cache;

/*
 * csa2_quant_kv_fp4 -- Full mode: quantize and append KV ([NEO part 3]).
 *
 * For each of n_tok tokens, quantizes the bf16 latent x[t][0..dim) to FP4:
 * per 16-channel group, s = the E4M3FN value nearest to max|x|/6 (ties to
 * even, saturated at 448; 0 when max|x|/6 is at most 2^-10), and each channel
 * gets the E2M1 code nearest to |x|/s (ties to even code, saturated at 6,
 * canonical +0 for a zero magnitude; all codes 0 when s = 0). Inputs must be
 * finite. The packed bytes and scales go to slot slot_mapping[t] of `cache`.
 * When kidx_in is not NULL the token's indexer key kidx_in[t][0..64) (E4M3FN)
 * and its scale kidx_scale_in[t] are written to the same slot too.
 *
 *   x_bf16        device bf16 [n_tok][dim], dim must be 576
 *   slot_mapping  device int32 [n_tok]; a negative slot skips the token; a
 *                 slot >= 64 * num_pages sets CSA2_ERR_DEVICE_BOUNDS
 *   kidx_in       device uint8 [n_tok][64] or NULL
 *   kidx_scale_in device float [n_tok] (required iff kidx_in != NULL)
 *   cache         host pointer to the destination cache descriptor
 * Bulk cache builds (n_tok = B*T) and per-step appends (n_tok = B*Sq) use the
 * same call.
 */
csa2_status csa2_quant_kv_fp4(const void *x_bf16, int64_t n_tok, int dim,
                              const int32_t *slot_mapping,
                              const void *kidx_in, const float *kidx_scale_in,
                              const csa2_paged_cache *cache, void *stream);

/*
 * csa2_quant_indexer_fp8 -- indexer key / query quantiser ([ZUL section 3]:
 * the KV owner hands "indexer K / scale" to its consumer layers; [NEO part 2]:
 * the indexer scores with FP8 operands).
 *
 * For each of n_rows rows of 64 bf16 channels:
 *     sigma[r]    = the binary32 value nearest to amax_r / 448
 *     codes[r][c] = the E4M3FN value nearest to the exact quotient
 *                   x[r][c] / sigma[r] (one rounding, ties to even mantissa,
 *                   saturating at +-448, canonical +0)
 * An all-zero row gives sigma = 0 and zero codes. Inputs must be finite. The
 * pages print no scale rule; this is the plainest one (the row maximum lands
 * on the top E4M3 value). Keys: codes and sigma are the kidx_in and
 * kidx_scale_in of csa2_quant_kv_fp4. Queries: one row per (token, indexer
 * head); since sigma > 0 can be taken out of the ReLU, the head weight passed
 * to csa2_indexer_topk becomes w * sigma.
 *
 *   x_bf16      device bf16 [n_rows][dim], 16-byte aligned; dim must be 64
 *   codes_e4m3  device uint8 [n_rows][64], 16-byte aligned
 *   sigma       device float [n_rows], 4-byte aligned
 * HBM-bound: 128 B read and 68 B written per row.
 */
csa2_status csa2_quant_indexer_fp8(const void *x_bf16, int64_t n_rows, int dim,
                                   void *codes_e4m3, float *sigma, void *stream);

/*
 * csa2_indexer_topk -- Full / Reindex: score every cached token with the
 * lightweight indexer and select the top-k ([NEO part 2] "Top-K sparse
 * addressing index"; [ZUL section 3]: Full and Reindex compute the index).
 *
 * Query token j of sequence b sits at position pos = seq_lens[b] - Sq + j and
 * scores every cached token t <= pos:
 *     s_t = sum_h w[b][j][h] * max(0, sigma_t * <q[b][j][h], k_t>)
 * (the pages print no formula; this is the DSA-style reading). The dot
 * product of E4M3 operands runs on the FP8 tensor cores with fp32
 * accumulation. out_idx[b][j] receives the k tokens with the largest s_t, ties
 * to the lower token index, in ascending token order; when pos + 1 < k the
 * remaining entries are -1. The selection is exact and deterministic for the
 * scores as computed; scores equal the mathematical value whenever every
 * partial sum is exact in fp32 (e.g. small-integer E4M3 inputs, sigma = 1 and
 * power-of-two weights).
 *
 *   q_idx       device uint8 [B][Sq][4][64] (E4M3FN)
 *   w           device float [B][Sq][4]
 *   cache       host pointer; reads kidx and kidx_scale of the owner's cache
 *   page_table  device int32 [B][max_pages]
 *   seq_lens    device int32 [B]; Sq <= seq_lens[b] <= 64 * max_pages
 *   k           1 <= k <= 65536
 *   out_idx     device int32 [B][Sq][k]
 *   ws          device workspace of at least csa2_indexer_topk_workspace_bytes()
 *               bytes, 256-byte aligned; contents need no initialisation and
 *               are clobbered. When the call's work has completed on the
 *               stream, its first B * Sq * 64 * max_pages floats hold the
 *               scores as float [B * Sq][64 * max_pages]: entry (b * Sq + j, t)
 *               is s_t as computed (fp32) for every t <= pos; other entries
 *               are unspecified.
 *
 * Limits (else CSA2_ERR_UNSUPPORTED): 4 indexer heads x 64 channels,
 * Sq <= 4, B * Sq <= 65535, 64 * max_pages <= 2^30, cache->num_pages <=
 * INT32_MAX (physical page indices are int32).
 */
size_t csa2_indexer_topk_workspace_bytes(int B, int Sq, int max_pages, int k);
csa2_status csa2_indexer_topk(const void *q_idx, const float *w, int B, int Sq,
                              int idx_heads, int idx_dim,
                              const csa2_paged_cache *cache,
                              const int32_t *page_table, int max_pages,
                              const int32_t *seq_lens, int k, int32_t *out_idx,
                              void *ws, size_t ws_bytes, void *stream);

/*
 * csa2_indexer_topk_scores -- csa2_indexer_topk that also returns the scores
 * of the selected entries: out_scores[b][j][i] = s_t (fp32, as computed) of
 * t = out_idx[b][j][i], -inf where out_idx is -1. The context-parallel split
 * of one long sequence (scope table, multi-GPU part) exchanges these
 * (score, index) candidates between the shards that own its positions.
 *
 *   out_scores  device float [B][Sq][k]; every other argument, limit and
 *               status as csa2_indexer_topk
 */
csa2_status csa2_indexer_topk_scores(const void *q_idx, const float *w, int B, int Sq,
                                     int idx_heads, int idx_dim,
                                     const csa2_paged_cache *cache,
                                     const int32_t *page_table, int max_pages,
                                     const int32_t *seq_lens, int k, int32_t *out_idx,
                                     float *out_scores, void *ws, size_t ws_bytes,
                                     void *stream);

/*
 * csa2_topk_merge -- context-parallel decode, the global top-k from the
 * shards' candidates. G shards own increasing, disjoint position ranges of
 * the same sequences; shard g's csa2_indexer_topk_scores output for its k_shard
 * best positions (as global positions, ascending, -1 padded) is candidate
 * list g. Because a shard's own top-k holds every one of its positions that
 * belongs to the global top-k, the k best candidates by (score desc, position
 * asc) are the top-k of the whole context, the same rule as
 * csa2_indexer_topk.
 *
 *   cand_scores device float [G][R][k_shard]   (R = B * Sq query rows)
 *   cand_idx    device int32 [G][R][k_shard]   global positions, ascending per
 *               list, shards in position order; a descending pair sets
 *               CSA2_ERR_DEVICE_BOUNDS
 *   k           entries to select; 1 <= G * k_shard <= 32768
 *   out_idx     device int32 [R][k] the global top-k, ascending, -1 padded
 *               (may be NULL)
 *   out_local   device int32 [R][k] the same list with the entries in
 *               [shard_lo, shard_hi) given as local positions (minus
 *               shard_lo) and every other entry -1: the indices a shard
 *               attends with over its own cache (may be NULL; not both NULL)
 * No workspace.
 */
csa2_status csa2_topk_merge(const float *cand_scores, const int32_t *cand_idx, int n_shards, int R,
                            int k_shard, int k, int32_t shard_lo, int32_t shard_hi,
                            int32_t *out_idx, int32_t *out_local, void *stream);

/*
 * csa2_lse_merge -- context-parallel decode, one softmax over the union of
 * the shards' disjoint key sets from their normalised results:
 *     L = log sum_p exp(lse_p),  out = sum_p exp(lse_p - L) * o_p,  lse = L
 * A part with lse = -inf (no key) weighs 0; with no key anywhere out = 0 and
 * lse = -inf. Natural-log lse as csa2_sparse_attn_decode writes it.
 *
 *   o_parts     device float [n_parts][R][16][576], 16-byte aligned
 *   lse_parts   device float [n_parts][R][16]
 *   out, lse    device float [R][16][576] and [R][16]
 */
csa2_status csa2_lse_merge(const float *o_parts, const float *lse_parts, int n_parts, int R,
                           float *out, float *lse, void *stream);

/*
 * csa2_indexer_pool_topk -- Reindex under the hierarchical sparse indexer
 * ([NEO part 2]: later indexing layers filter only within the candidate pool
 * built by the first Full layer, so their cost does not grow with the
 * context).
 *
 * For query row (b, j), scores only the tokens of pool[b][j] with the same
 * formula as csa2_indexer_topk (this layer's q_idx and w, the owner's indexer
 * keys and sigma) and writes to out_idx[b][j] the k best by (score desc,
 * token index asc), in ascending token order, -1 padded when the pool holds
 * fewer than k valid entries. The pool is typically the Full layer's
 * csa2_indexer_topk output for k = pool_size (its top-C); with this layer's
 * own q and w over its own pool the call returns exactly its top-k.
 *
 *   q_idx, w, cache, page_table, seq_lens, max_pages: as csa2_indexer_topk
 *   pool        device int32 [B][Sq][pool_size]: token indices in ascending
 *               order, -1 entries skipped; an entry after the query's
 *               position seq_lens[b] - Sq + j (causal bound), a bad
 *               page-table entry or a descending pair sets
 *               CSA2_ERR_DEVICE_BOUNDS (the entry is skipped)
 *   pool_size   1 <= pool_size <= 32768 (CSA2_ERR_UNSUPPORTED above)
 *   k           k >= 1
 *   out_idx     device int32 [B][Sq][k]
 * No workspace. Limits: 4 indexer heads x 64 channels, B * Sq <= 65535.
 */
csa2_status csa2_indexer_pool_topk(const void *q_idx, const float *w, int B, int Sq,
                                   int idx_heads, int idx_dim,
                                   const csa2_paged_cache *cache,
                                   const int32_t *page_table, int max_pages,
                                   const int32_t *seq_lens, const int32_t *pool,
                                   int pool_size, int k, int32_t *out_idx,
                                   void *stream);

/*
 * csa2_sparse_attn_decode -- all modes: attention over the selected FP4
 * entries plus the sliding window ([NEO part 2]; [ZUL section 4]).
 *
 * For query token j of sequence b (position pos = seq_lens[b] - Sq + j) and
 * head h, the keys are the dequantized cache entries topk_idx[b][j][i] >= 0
 * together with the window rows j .. j+W-1 of swa[b] (row r holds position
 * seq_lens[b] - (W + Sq - 1) + r; rows at negative positions are skipped).
 * The same vectors are the values. One softmax over their union:
 *     out[b][j][h] = sum_i softmax_i(scale * <q, key_i>) * key_i
 *     lse[b][j][h] = log sum_i exp(scale * <q, key_i>)
 * With no key at all out = 0 and lse = -inf. Dequantized FP4 entries are
 * exact in f16. q is carried in f16 under a power-of-two exponent per query
 * row, and the window rows under one per 64-row tile (each chosen from the
 * values: none when the largest magnitude lies in [2^-4, 2^15)), so rows
 * whose largest magnitude lies between about 2^-50 and 2^70 keep f16
 * precision; probabilities are rounded to f16; all sums accumulate in fp32.
 * Logits must stay within fp32 range.
 *
 *   q_bf16      device bf16 [B][Sq][16][576]
 *   cache       host pointer; reads kv_fp4 and kv_scale of the owner's cache
 *   page_table  device int32 [B][max_pages];   seq_lens device int32 [B]
 *   topk_idx    device int32 [B][Sq][k] (k may be 0: window only); an index
 *               after its query's position, past the sequence or on a bad
 *               page sets CSA2_ERR_DEVICE_BOUNDS and is skipped
 *   swa_bf16    device bf16 [B][W + Sq - 1][576]; W must be 128, or 0 for no
 *               window rows at all (swa_bf16 may then be NULL; a
 *               context-parallel shard that does not hold the newest tokens).
 *               W = 0 with k = 0 is CSA2_ERR_INVALID_ARG.
 *   out         device float [B][Sq][16][576];  lse device float [B][Sq][16]
 *   ws          device workspace of csa2_sparse_attn_workspace_bytes() bytes,
 *               256-byte aligned (partials of rows split into runs, one per
 *               CTA, 37 KB each; rows are split only while all the runs fit
 *               one wave of CTAs, so at most 2 x SMs partials); clobbered.
 *               The size returned for (B, Sq, k) also covers W = 0; it is 0
 *               when no row is split.
 */
size_t csa2_sparse_attn_workspace_bytes(int B, int Sq, int k);
csa2_status csa2_sparse_attn_decode(const void *q_bf16, int B, int Sq, int H,
                                    int D, const csa2_paged_cache *cache,
                                    const int32_t *page_table, int max_pages,
                                    const int32_t *seq_lens,
                                    const int32_t *topk_idx, int k,
                                    const void *swa_bf16, int W,
                                    float softmax_scale, float *out, float *lse,
                                    void *ws, size_t ws_bytes, void *stream);

/*
 * csa2_sparse_attn_decode_noalloc -- csa2_sparse_attn_decode for callers that
 * cannot allocate device memory. The pages describe no such variant; it is a
 * convenience of this library.
 *
 * Who needs it: code that is handed only its input and output buffers by a
 * host framework and has no allocator to call (for example a plugin whose
 * enqueue hook receives no workspace), and decode loops that must not call
 * cudaMalloc because it can synchronise the device and stall the stream.
 *
 * Same arguments and results as csa2_sparse_attn_decode, minus the workspace:
 * the split-k partials live in one library-owned device array of
 * CSA2_NOALLOC_SCRATCH_BYTES (32 MiB), which every GPU that loads the library
 * keeps until process exit. The call allocates nothing and never calls
 * cudaMalloc / cudaFree. Its first call on a device looks up the device
 * address of that array with the device current; make that first call before
 * any stream capture. When the partials of a call would need more than
 * CSA2_NOALLOC_SCRATCH_BYTES (csa2_sparse_attn_workspace_bytes() larger than
 * the limit) it returns CSA2_ERR_WORKSPACE and enqueues nothing. Every call on
 * a device shares the one array: two calls whose kernels can overlap on the
 * GPU (different streams without ordering between them) race on it and give
 * wrong results; calls ordered on one stream are safe. Nothing in the array
 * needs to start at zero (each call writes every partial it reads).
 */
#define CSA2_NOALLOC_SCRATCH_BYTES (32u << 20)
csa2_status csa2_sparse_attn_decode_noalloc(const void *q_bf16, int B, int Sq,
                                            int H, int D,
                                            const csa2_paged_cache *cache,
                                            const int32_t *page_table,
                                            int max_pages,
                                            const int32_t *seq_lens,
                                            const int32_t *topk_idx, int k,
                                            const void *swa_bf16, int W,
                                            float softmax_scale, float *out,
                                            float *lse, void *stream);

/*
 * csa2_swa_replay_attn -- window attention of L consecutive query tokens:
 * the SWA bounded replay ([ZUL section 5], [INF section 2]: the last 128
 * tokens are recomputed instead of persisted) and the window part of a
 * Full-mode prefill. Query j of sequence b sits at position
 * seq_lens[b] - L + j and attends to the window rows j .. j + 127 of swa[b]
 * (row r holds position seq_lens[b] - (W + L - 1) + r; rows at negative
 * positions are skipped), one softmax per (query, head):
 *     out[b][j][h] = sum_r softmax_r(scale * <q, row_r>) * row_r
 * This is csa2_sparse_attn_decode with k = 0 and Sq = L, computed with the
 * queries tiled 8 at a time over one staged copy of their window band. The
 * scores use the exact bf16 inputs (fp32 accumulation); the window rows
 * enter the value product in f16 under a power-of-two exponent per tile and
 * the probabilities are rounded to f16.
 *
 *   q_bf16      device bf16 [B][L][16][576]
 *   swa_bf16    device bf16 [B][W + L - 1][576], W must be 128
 *   seq_lens    device int32 [B]; seq_lens[b] >= L (else CSA2_ERR_DEVICE_BOUNDS
 *               and that sequence's outputs are left unwritten)
 *   out         device float [B][L][16][576];  lse device float [B][L][16]
 * No workspace. Limits: B <= 65535, L <= 2^24.
 */
csa2_status csa2_swa_replay_attn(const void *q_bf16, int B, int L, int H, int D,
                                 const void *swa_bf16, int W, const int32_t *seq_lens,
                                 float softmax_scale, float *out, float *lse, void *stream);

/*
 * csa2_plan -- ownership bookkeeping for a group of layers ([ZUL section 3]:
 * KV owner layer -> consumer layers; [NEO part 2]: KV, indexer keys and top-K
 * indices shared across layers). Host-only, no device work.
 *
 * Fills, for each layer i, kv_owner[i] = the Full layer whose cache it reads
 * (itself for a Full layer, else the nearest Full layer before it) and
 * index_src[i] = the layer whose top-k indices it attends with (itself for
 * Full and Reindex; the nearest Full layer before it for Reuse). Returns
 * CSA2_ERR_BAD_PLAN when a Reindex or Reuse layer has no Full layer before
 * it or a mode is unknown, CSA2_ERR_INVALID_ARG for null pointers.
 */
csa2_status csa2_plan(const int *modes, int n_layers, int *kv_owner,
                      int *index_src);

/*
 * csa2_last_device_error -- synchronises `stream`, then reads and clears the
 * sticky device status word of the current device. Returns CSA2_OK,
 * CSA2_ERR_DEVICE_BOUNDS or CSA2_ERR_TIMEOUT (the first set, in that order of
 * precedence: timeout first), or CSA2_ERR_CUDA if the synchronisation failed.
 * A diagnostic call: it blocks the host.
 */
csa2_status csa2_last_device_error(void *stream);

/* Human-readable name of a status code (static storage). */
const char *csa2_status_string(csa2_status s);

/* Number of kernels this library has launched in this process. */
uint64_t csa2_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */
