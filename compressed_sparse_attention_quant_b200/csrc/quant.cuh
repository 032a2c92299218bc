// quant.cuh -- K1: FP4 (E2M1 + E4M3 per 16 channels) quantize-and-append of
// the global KV latent into the paged cache. Page "DeepSeek 首次公开
// V4.1-Flash 技术报告…" (neodrop.ai), architecture part 3: the main KV cache
// is E2M1 with one E4M3 scale for every 16 channels.
//
// One thread per (token, 16-channel group): two 16-byte loads of bf16, the
// group max by compares, the scale by IEEE division and the hardware
// round-to-nearest-even satfinite FP8 conversion, the codes by exact
// compares against the scaled E2M1 midpoints, one 8-byte store of packed
// codes and one scale byte. HBM-bound: 32 B read + 9 B written per group.
#pragma once

#include "common.cuh"

namespace csa2 {

constexpr int kQuantThreads = 256;

__global__ void __launch_bounds__(kQuantThreads)
quant_kv_fp4_kernel(const uint4 *__restrict__ x, int64_t n_tok, const int32_t *__restrict__ slots,
                    const uint4 *__restrict__ kidx_in, const float *__restrict__ ksig_in,
                    uint8_t *__restrict__ kv_fp4, uint8_t *__restrict__ kv_scale,
                    uint8_t *__restrict__ kidx, float *__restrict__ kidx_scale, int64_t n_slots) {
    constexpr int kGroups = kDim / kGroup;  // 36
    pdl_wait();
    pdl_trigger();
    const int64_t gid = static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x;
    const int64_t tok = gid / kGroups;
    const int g = static_cast<int>(gid - tok * kGroups);
    if (tok >= n_tok) return;
    // 16 bf16 channels = two 16-byte vectors, loaded together with the slot
    // id (the input rows exist for every token, padding included).
    const uint4 v0 = x[(tok * kGroups + g) * 2 + 0];
    const uint4 v1 = x[(tok * kGroups + g) * 2 + 1];
    const bool key_part = kidx_in != nullptr && g < 4;          // threads 0..3 of a token move its indexer key
    const uint4 kin = key_part ? kidx_in[tok * 4 + g] : make_uint4(0u, 0u, 0u, 0u);
    const float ksig = (key_part && g == 0) ? ksig_in[tok] : 0.0f;
    const int32_t slot = slots[tok];
    if (slot < 0) return;                       // padding token: nothing to append
    if (static_cast<int64_t>(slot) >= n_slots) {
        if (g == 0) flag_status(kStatusBounds);
        return;
    }
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float f[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));

    // Scale: E4M3FN nearest to amax/6. The fp32 quotient is correctly rounded
    // and cannot cross an E4M3 midpoint (amax has 8 significant bits, 6 x a
    // midpoint at most 7), so RNE of the fp32 quotient is RNE of the exact one.
    const float t = __fdiv_rn(amax, 6.0f);
    const __nv_fp8_storage_t sb = __nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3);
    const float s = __half2float(__half(__nv_cvt_fp8_to_halfraw(sb, __NV_E4M3)));

    // Codes: count the E2M1 midpoints below |x|/s, comparing |x| with s * mu
    // (exact in fp32). Ties go to the even code: strict '>' at midpoints that
    // sit above an even code, '>=' at those above an odd code.
    const float m0 = s * 0.25f, m1 = s * 0.75f, m2 = s * 1.25f, m3 = s * 1.75f;
    const float m4 = s * 2.5f, m5 = s * 3.5f, m6 = s * 5.0f;
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float a = fabsf(f[i]);
        uint32_t c = (a > m0) + (a >= m1) + (a > m2) + (a >= m3) + (a > m4) + (a >= m5) + (a > m6);
        if (s == 0.0f) c = 0u;
        if (c != 0u && f[i] < 0.0f) c |= 8u;
        packed[i >> 3] |= c << (4 * (i & 7));
    }
    const int64_t sl = slot;
    *reinterpret_cast<uint2 *>(kv_fp4 + sl * kFp4Bytes + g * 8) = make_uint2(packed[0], packed[1]);
    kv_scale[sl * kScaleBytes + g] = sb;

    // Indexer key and scale of the token, in the page's core-matrix order.
    if (key_part) {
        const int64_t page = sl / kPage;
        const int r = static_cast<int>(sl % kPage);
        uint8_t *dst = kidx + page * kKidxPageBytes + (r >> 3) * 512 + g * 128 + (r & 7) * 16;
        *reinterpret_cast<uint4 *>(dst) = kin;
        if (g == 0) kidx_scale[sl] = ksig;
    }
}

inline cudaError_t launch_quant_kv_fp4(const void *x, int64_t n_tok, const int32_t *slots,
                                       const void *kidx_in, const float *ksig_in,
                                       const csa2_paged_cache &c, cudaStream_t stream) {
    const int64_t threads = n_tok * (kDim / kGroup);
    const int64_t blocks = (threads + kQuantThreads - 1) / kQuantThreads;
    return launch_pdl(quant_kv_fp4_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kQuantThreads), 0, stream,
                      static_cast<const uint4 *>(x), n_tok, slots, static_cast<const uint4 *>(kidx_in), ksig_in,
                      static_cast<uint8_t *>(c.kv_fp4), static_cast<uint8_t *>(c.kv_scale),
                      static_cast<uint8_t *>(c.kidx), c.kidx_scale, c.num_pages * kPage);
}

// K1b: indexer key / query quantiser, bf16 -> E4M3FN with one fp32 scale per
// 64-channel row. Page "DeepSeek V4 1-Flash 架构拆解…" (blog.zulogic.cn),
// section 3: the KV owner hands "indexer K / scale" to its consumer layers;
// page "DeepSeek 首次公开 V4.1-Flash 技术报告…" (neodrop.ai), architecture
// part 2: the indexer scores with FP8 operands. The pages give no scale rule;
// the one taken is sigma = binary32 nearest to amax / 448 and code = the E4M3FN
// value nearest to the exact quotient x / sigma (one rounding, ties to even,
// saturating, canonical +0), all codes 0 (and sigma 0) for an all-zero row.
//
// Exact rounding without a division per channel: p = RN(|x| * RN(1 / sigma))
// is within 2 binary32 ulps of the exact quotient, so the hardware RNE
// conversion of p can differ from the exact decision only when an E4M3
// midpoint lies within those ulps of p. Such channels (the low 20 bits of p
// within 3 of a midpoint's pattern, or p in the E4M3 subnormal range) take a
// fix-up that decides the side by the sign of fma(midpoint, sigma, -|x|): the
// product is exact in the fma and a single rounding keeps the sign. Rows with
// sigma < 2^-100 are first scaled by 2^64 (exact), so no product of the
// fix-up underflows.
//
// Eight threads per row, each with 8 channels; a thread runs kIdxQuantRows
// rows per pass with all their 16-byte loads issued first, so more bytes are
// in flight per warp. HBM-bound: 128 B read + 68 B written per row.
constexpr int kIdxQuantThreads = 256;
constexpr int kIdxQuantRows = 4;                                   // rows per thread per pass
constexpr int kIdxQuantRowsPerBlock = kIdxQuantThreads / 8 * kIdxQuantRows;

// E4M3FN magnitude code of the exact quotient a / s (a >= 0, s > 0 binary32,
// s >= 2^-100), given p = a * RN(1 / s) rounded once.
__device__ __forceinline__ uint32_t e4m3_quotient_fixup(float a, float s, float p) {
    if (p >= 448.0f) return 0x7Eu;
    if (p < 0.015625f) {                                           // E4M3 subnormal range: steps of 2^-9
        const float n = floorf(p * 512.0f);
        const float d = __fmaf_rn((n + 0.5f) * 0.001953125f, s, -a);
        const uint32_t k = static_cast<uint32_t>(n);
        return d > 0.0f ? k : d < 0.0f ? k + 1u : k + (k & 1u);    // codes 0..8 are k itself
    }
    const uint32_t lo = __float_as_uint(p) & ~0xFFFFFu;            // grid value just below the midpoint
    const float d = __fmaf_rn(__uint_as_float(lo | 0x80000u), s, -a);
    const uint32_t clo = (((lo >> 23) - 120u) << 3) | ((lo >> 20) & 7u);   // exponent bias 127 -> 7
    const uint32_t chi = min(clo + 1u, 0x7Eu);
    return d > 0.0f ? clo : d < 0.0f ? chi : ((clo & 1u) ? chi : clo);
}

// Whether RNE(p) may differ from the exact decision (see above).
__device__ __forceinline__ bool e4m3_quotient_near(float p) {
    const uint32_t b = __float_as_uint(p);
    const bool mid = ((b - 0x7FFFDu) & 0xFFFFFu) <= 6u;            // within 3 ulps of an E4M3 midpoint
    const bool sub = b - 0x3A000000u < 0x3C800000u - 0x3A000000u;  // p in [2^-11, 2^-6)
    return mid || sub;
}

__global__ void __launch_bounds__(kIdxQuantThreads, 4)
quant_index_fp8_kernel(const uint4 *__restrict__ x, int64_t n_rows, uint2 *__restrict__ codes,
                       float *__restrict__ sigma) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31, part = threadIdx.x & 7;
    const unsigned gmask = 0xffu << (lane & 24);        // the 8 lanes of this row
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kIdxQuantRowsPerBlock;
    for (int64_t row0 = static_cast<int64_t>(blockIdx.x) * kIdxQuantRowsPerBlock + (threadIdx.x >> 3);
         row0 < n_rows; row0 += stride) {
        uint4 v[kIdxQuantRows];
#pragma unroll
        for (int r = 0; r < kIdxQuantRows; ++r) {
            const int64_t row = row0 + r * (kIdxQuantThreads / 8);
            v[r] = row < n_rows ? x[row * 8 + part] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int r = 0; r < kIdxQuantRows; ++r) {
            const int64_t row = row0 + r * (kIdxQuantThreads / 8);
            const uint32_t w[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
            float f[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                f[2 * i] = __uint_as_float(w[i] << 16);
                f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
            for (int off = 1; off < 8; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, off));
            const float sg = __fdiv_rn(amax, 448.0f);
            // Scaled domain for tiny sigma (exact power-of-two scaling).
            const float scl = sg < 0x1p-100f ? 0x1p64f : 1.0f;
            const float s2 = sg * scl;
            const float inv = __frcp_rn(s2);
            float a[8], p[8];
            uint32_t near = 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                a[i] = fabsf(f[i]) * scl;
                p[i] = a[i] * inv;
                near |= e4m3_quotient_near(p[i]) ? (1u << i) : 0u;
            }
            uint32_t mag[8];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const uint32_t c2 = __nv_cvt_float2_to_fp8x2(make_float2(p[i], p[i + 1]), __NV_SATFINITE, __NV_E4M3);
                mag[i] = c2 & 0x7Fu;
                mag[i + 1] = (c2 >> 8) & 0x7Fu;
            }
            if (__any_sync(0xffffffffu, near != 0u)) {                 // rare: exact fix-up of close calls
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (near & (1u << i)) mag[i] = e4m3_quotient_fixup(a[i], s2, p[i]);
            }
            uint32_t packed[2] = {0u, 0u};
            if (sg != 0.0f) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t c = mag[i] | ((mag[i] != 0u && f[i] < 0.0f) ? 0x80u : 0u);   // canonical +0
                    packed[i >> 2] |= c << (8 * (i & 3));
                }
            }
            if (row < n_rows) {
                codes[row * 8 + part] = make_uint2(packed[0], packed[1]);
                if (part == 0) sigma[row] = sg;
            }
        }
    }
}

// Grid: one wave of resident blocks (grid-stride loop), or fewer when the
// rows run out.
inline cudaError_t launch_quant_index_fp8(const void *x, int64_t n_rows, void *codes, float *sigma, int resident,
                                          cudaStream_t stream) {
    const int64_t need = (n_rows + kIdxQuantRowsPerBlock - 1) / kIdxQuantRowsPerBlock;
    const int64_t blocks = std::min<int64_t>(need, resident);
    return launch_pdl(quant_index_fp8_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kIdxQuantThreads), 0, stream,
                      static_cast<const uint4 *>(x), n_rows, static_cast<uint2 *>(codes), sigma);
}

}  // namespace csa2
