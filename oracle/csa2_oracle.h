/*
 * csa2_oracle.h -- CPU oracle for the CSA2 FP4 sparse-decode path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library includes,
 * links or calls this. Only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py load it. It shares no code, header, table or
 * constant with the CUDA library.
 *
 * Citation tags used in this directory:
 *   [INF]  page "DeepSeek V4.1 Flash 模型架構與推論優化技術規格剖析"
 *          (infernews.com): section 2 "線性 KV 快取投影與滑動窗口重播"
 *          and the section-4 specification table (row "CSA 2").
 *   [NEO]  page "DeepSeek 首次公开 V4.1-Flash 技术报告：552B 骨干参数与
 *          CED 架构亮相，KV 缓存压至 890 字节" (neodrop.ai): architecture
 *          part 2 "压缩稀疏注意力 2（CSA2）与跨层索引复用" and part 3
 *          "FP4 主 KV 缓存与 SWA Bounded Replay".
 *   [ZUL]  page "DeepSeek V4 1-Flash 架构拆解：CED、CSA2、Engram、mHC 与 DSp"
 *          (blog.zulogic.cn): section 3 (CSA2 mode table and the KV-owner
 *          state graph) and section 4 (global KV + sliding window).
 *
 * Arithmetic: fp64 and exact integers. Every function is single-threaded
 * and written for clarity, not speed.
 */
#ifndef CSA2_ORACLE_H
#define CSA2_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- number formats ---------------------------------------------------- */

/* bf16 bit pattern -> exact double. */
double orc_bf16_value(uint16_t bits);

/* FP4 E2M1 code (low 4 bits) -> exact value. [NEO part 3] */
double orc_e2m1_value(uint8_t code);

/* FP8 E4M3FN byte -> exact value (NaN for the two NaN codes). [NEO part 3] */
double orc_e4m3_value(uint8_t byte);

/* ---- quantizer ([NEO part 3]: E2M1 data, one E4M3 scale per 16 channels) */

/* Scale byte for a 16-channel group whose largest magnitude is `amax`:
 * the E4M3FN value nearest to amax/6 (ties to even mantissa), saturated
 * to 448. */
uint8_t orc_group_scale(double amax);

/* E2M1 code of x under scale value s: nearest magnitude on the E2M1 grid
 * to |x|/s with ties to even, saturated to 6, sign in bit 3, canonical +0.
 * s == 0 gives code 0. */
uint8_t orc_e2m1_code(double x, double s);

/* Element-wise array forms of the two functions above (for exhaustive
 * checks): out[i] = orc_group_scale(amax[i]) and out[i] =
 * orc_e2m1_code(x[i], s[i]). */
void orc_group_scale_n(const double *amax, int64_t n, uint8_t *out);
void orc_e2m1_code_n(const double *x, const double *s, int64_t n, uint8_t *out);

/* Quantize n tokens of `dim` bf16 channels (dim % 16 == 0).
 * codes: [n][dim/2], byte j = code(2j) | code(2j+1) << 4.
 * scales: [n][dim/16]. */
void orc_quant_fp4(const uint16_t *x_bf16, int64_t n, int dim,
                   uint8_t *codes, uint8_t *scales);

/* Dequantize n tokens back to doubles: out[n][dim]. */
void orc_dequant_fp4(const uint8_t *codes, const uint8_t *scales, int64_t n,
                     int dim, double *out);

/* ---- indexer FP8 quantiser ([ZUL section 3] "indexer K / scale") ------- */

/* E4M3FN code of the exact quotient x / sigma (sigma > 0 binary32): nearest
 * grid value, ties to even mantissa, saturating at +-448, canonical +0. */
uint8_t orc_e4m3_code_quotient(double x, float sigma);

/* n_rows rows of `dim` bf16 channels -> codes [n_rows][dim] (E4M3FN) and one
 * binary32 scale per row: sigma = binary32 nearest to amax / 448 and
 * code = orc_e4m3_code_quotient(x, sigma); an all-zero row gives sigma = 0
 * and zero codes. */
void orc_quant_index_fp8(const uint16_t *x_bf16, int64_t n_rows, int dim,
                         uint8_t *codes, float *sigma);

/* ---- lightweight indexer ([NEO part 2], [ZUL section 3]) --------------- */

/* Scores for one query token over n cached tokens:
 *   s_t = sum_h w_h * relu(sigma_t * <q_h, k_t>)   (relu optional)
 * q: [n_heads][idim] E4M3FN, w: [n_heads], k: [n][idim] E4M3FN,
 * sigma: [n]. Output s: [n] doubles. */
void orc_indexer_scores(const uint8_t *q, const float *w, int n_heads,
                        int idim, const uint8_t *k, const float *sigma,
                        int64_t n, int relu, double *s);

/* Top-k of the first n_valid scores: the k largest by (score desc,
 * index asc), emitted in ascending index order; -1 padding when
 * n_valid < k. Returns the number of valid indices written. */
int orc_topk(const double *s, int64_t n_valid, int k, int32_t *out);

/* Top-k inside a candidate pool (hierarchical sparse indexer, [NEO part 2]):
 * pool: [n_pool] token indices (-1 skipped), s: [n_pool] their scores. The k
 * best by (score desc, token index asc), ascending, -1 padded. Returns the
 * number of valid indices written. */
int orc_pool_topk(const double *s, const int32_t *pool, int n_pool, int k,
                  int32_t *out);

/* ---- sparse attention over FP4 entries plus the SWA window -------------
 * ([NEO part 2]: attention over the top-k selected entries; [ZUL section 4]:
 * a per-layer sliding window of recent tokens kept beside the global KV.)
 *
 * One query token, n_heads heads of dim channels (bf16 bits).
 * Keys = { dequant(cache row idx[i]) : idx[i] >= 0 }  U  { swa rows }.
 * Values are the same vectors as the keys. One softmax over the union.
 * o: [n_heads][dim], lse: [n_heads] (natural log). With no keys at all,
 * o = 0 and lse = -inf. */
void orc_sparse_attn(const uint16_t *q, int n_heads, int dim,
                     const uint8_t *codes, const uint8_t *scales,
                     int64_t n_cache, const int32_t *idx, int k,
                     const uint16_t *swa, int n_swa, double softmax_scale,
                     double *o, double *lse);

/* ---- per-layer static mode and ownership ([ZUL section 3], [NEO part 2])
 * modes: 0 = Full, 1 = Reindex, 2 = Reuse. Fills kv_owner[i] (the layer
 * whose KV and indexer keys layer i reads) and index_src[i] (the layer whose
 * top-k indices layer i uses). Returns 0, or -1 - i for the first layer i
 * that has no Full layer before it. */
int orc_plan(const int *modes, int n_layers, int *kv_owner, int *index_src);

#ifdef __cplusplus
}
#endif
#endif
