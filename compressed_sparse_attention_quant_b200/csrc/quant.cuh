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
// Exact rounding without a division per channel: p = RN(|x| * r), r an
// approximation of 1 / sigma to ~1 ulp, lies within 2^-22 (relative) of the
// exact quotient q. The codes of lo = RN(p (1 - 2^-21)) < q and
// hi = RN(p (1 + 2^-21)) > q are taken by the hardware RNE satfinite E4M3
// conversion; rounding is monotone, so when they agree that code is the
// exact decision for q. When they differ (an E4M3 midpoint lies between them:
// a fraction of a percent of the channels) a fix-up decides the side by the
// sign of fma(midpoint, sigma, -|x|), which is exact. Rows with
// sigma < 2^-100 are first scaled by 2^64 (exact), so no product of the
// fix-up underflows.
//
// Four threads per row; thread t of a row takes channels 8t .. 8t + 7 and
// 32 + 8t .. 32 + 8t + 7 (two 16-byte loads, each warp load covering whole
// 64-byte runs of its 8 rows); each thread keeps kIdxQuantStages rows in
// flight (cp.async into its own shared-memory slots). The
// codes are packed four at a time: magnitudes from the paired conversions,
// signs from the high bytes of the bf16 inputs, and a sign only on a nonzero
// magnitude (canonical +0). 128 B read + 68 B written per row; as built the
// per-row chain (maximum, shuffles, scale, reciprocal, conversions) bounds
// it at about half of the copy bandwidth, not the HBM.
constexpr int kIdxQuantThreads = 256;
constexpr int kIdxQuantStages = 4;                                 // rows per thread in flight
constexpr int kIdxQuantTpr = 4;                                    // threads per row
constexpr int kIdxQuantRowsPerBlock = kIdxQuantThreads / kIdxQuantTpr;

// E4M3FN magnitude code of the exact quotient a / s (a >= 0, s > 0 binary32,
// s >= 2^-100), given p = a * r rounded once with r within a few ulps of 1 / s.
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

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Two E4M3FN codes (RNE, satfinite) of a pair of non-negative floats, low
// byte first, in the low 16 bits.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
    return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

__global__ void __launch_bounds__(kIdxQuantThreads, 3)
quant_index_fp8_kernel(const uint4 *__restrict__ x, int64_t n_rows, uint2 *__restrict__ codes,
                       float *__restrict__ sigma) {
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31, part = threadIdx.x & (kIdxQuantTpr - 1);
    const unsigned gmask = 0xfu << (lane & 28);         // the 4 lanes of this row
    // Each thread keeps its next kIdxQuantStages rows in flight with cp.async
    // into its own shared-memory slots (no registers held, no barrier: a
    // thread reads only what it copied).
    __shared__ __align__(16) uint4 stage[kIdxQuantStages][kIdxQuantThreads][2];
    const int64_t stride = static_cast<int64_t>(gridDim.x) * (kIdxQuantThreads / kIdxQuantTpr);
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * (kIdxQuantThreads / kIdxQuantTpr) + threadIdx.x / kIdxQuantTpr;
    auto fetch = [&](int64_t k) {                       // row row0 + k * stride into stage k % kIdxQuantStages
        const int64_t row = row0 + k * stride;
        const bool ok = row < n_rows;
        const uint4 *src = ok ? x + row * 8 + part : x;
#pragma unroll
        for (int h = 0; h < 2; ++h)
            cp_async16(&stage[k % kIdxQuantStages][threadIdx.x][h], src + 4 * h, ok ? 16u : 0u);
    };
#pragma unroll
    for (int k = 0; k < kIdxQuantStages - 1; ++k) {
        fetch(k);
        cp_async_commit();
    }
    for (int64_t k = 0; row0 + k * stride < n_rows; ++k) {
        fetch(k + kIdxQuantStages - 1);
        cp_async_commit();
        cp_async_wait<kIdxQuantStages - 1>();           // row k has landed
        {
            const int64_t row = row0 + k * stride;
            const uint4 va = stage[k % kIdxQuantStages][threadIdx.x][0];
            const uint4 vb = stage[k % kIdxQuantStages][threadIdx.x][1];
            const uint32_t w[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
            float f[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                f[2 * i] = __uint_as_float(w[i] << 16);
                f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
            amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, 2));
            // sigma = RN(amax / 448): one rounded product and one fma
            // correction (equal to the IEEE quotient for every finite bf16
            // amax, checked exhaustively on the host).
            const float q0 = __fmul_rn(amax, 1.0f / 448.0f);
            const float sg = __fmaf_rn(__fmaf_rn(-q0, 448.0f, amax), 1.0f / 448.0f, q0);
            // Scaled domain for tiny sigma (exact power-of-two scaling): a =
            // |x| scl, s2 = sigma scl, p = a / s2 through inv = scl / s2;
            // below 2^-120 the inputs themselves are scaled (inv would overflow).
            const float scl = sg < 0x1p-100f ? 0x1p64f : 1.0f;
            const float s2 = sg * scl;
            float inv = rcp_approx(s2) * scl, ascl = scl;
            if (sg < 0x1p-120f) {
#pragma unroll
                for (int i = 0; i < 16; ++i) f[i] *= scl;
                inv = rcp_approx(s2);
                ascl = 1.0f;
            }
            uint32_t mag[8];                                    // code pairs (2i, 2i + 1)
            uint32_t near = 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float p0 = fabsf(f[2 * i]) * inv, p1 = fabsf(f[2 * i + 1]) * inv;
                const uint32_t lo = e4m3x2(p0 * 0.99999952316284180f, p1 * 0.99999952316284180f);   // 1 - 2^-21
                const uint32_t hi = e4m3x2(p0 * 1.00000047683715820f, p1 * 1.00000047683715820f);   // 1 + 2^-21
                mag[i] = lo;
                near |= lo != hi ? (1u << i) : 0u;
            }
            if (__any_sync(0xffffffffu, near != 0u)) {          // rare: exact fix-up of close calls
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (near & (1u << i)) {
                        const float a0 = fabsf(f[2 * i]) * ascl, a1 = fabsf(f[2 * i + 1]) * ascl;
                        const float p0 = fabsf(f[2 * i]) * inv, p1 = fabsf(f[2 * i + 1]) * inv;
                        mag[i] = e4m3_quotient_fixup(a0, s2, p0) | (e4m3_quotient_fixup(a1, s2, p1) << 8);
                    }
                }
            }
            uint32_t o[4] = {0u, 0u, 0u, 0u};
            if (sg != 0.0f) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t m4 = __byte_perm(mag[2 * j], mag[2 * j + 1], 0x5410);     // 4 magnitudes
                    const uint32_t sgn = __byte_perm(w[2 * j], w[2 * j + 1], 0x7531) & 0x80808080u;
                    o[j] = m4 | (sgn & __vcmpne4(m4, 0u));                                  // canonical +0
                }
            }
            if (row < n_rows) {
                codes[row * 8 + part] = make_uint2(o[0], o[1]);           // channels 8t .. 8t + 7
                codes[row * 8 + 4 + part] = make_uint2(o[2], o[3]);       // channels 32 + 8t ..
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
