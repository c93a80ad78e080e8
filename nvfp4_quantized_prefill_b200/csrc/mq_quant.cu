// mq_quant.cu -- NVFP4 quantization of BF16 matrices on sm_100a.
//
// Method: the Mix-Quant pages (gist.science technical summary, section 2
// "Hybrid Precision Strategy") quantize prefill weights and activations to
// NVFP4: a local scale per group of 16 elements plus a tensor-level scale,
// plain round-to-nearest.  Encoding used: E2M1 codes, E4M3 block scales,
// FP32 tensor scale s_enc = 2688 / amax (1 for an all-zero tensor),
// round-to-nearest-even:
//   sb = E4M3_satfinite(fp32(fp32(amax_b / 6) * s_enc))
//   f  = dec(sb) == 0 ? 0 : fp32(s_enc / dec(sb))
//   q  = E2M1_satfinite(fp32(x * f)), sign taken from x.
//
// Both kernels are HBM-streaming: 16-byte vector loads, coalesced across the
// warp, grids sized in multiples of the SM count.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_fp16.h>

#include "mq_internal.h"

namespace mq {

namespace {

constexpr int kThreads = 256;
constexpr int kAmaxUnroll = 4;

__device__ __forceinline__ uint4 ldg_v4(const uint4 *p) { return __ldg(p); }

// max of |bf16| over the 8 values of a 16-byte vector, as 16-bit magnitude bits
// (non-negative bf16 values order like their bit patterns).
__device__ __forceinline__ uint32_t absmax8_bits(uint4 v) {
    const uint32_t m = 0x7FFF7FFFu;
    uint32_t a = __vmaxu2(__vmaxu2(v.x & m, v.y & m), __vmaxu2(v.z & m, v.w & m));
    return max(a & 0xFFFFu, a >> 16);
}

__device__ __forceinline__ float block_max(float v, float *red) {
    // non-negative floats: max of the bit patterns is the bit pattern of the max
    uint32_t b = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(v));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = __uint_as_float(b);
    __syncthreads();
    float r = 0.0f;
    for (int i = 0; i < kThreads / 32; ++i) r = fmaxf(r, red[i]);
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kThreads) amax_kernel(const uint4 *__restrict__ x, uint32_t M,
                                                        uint32_t vpr, uint64_t ldv,
                                                        float *__restrict__ partials) {
    __shared__ float red[kThreads / 32];
    const uint32_t total = M * vpr;
    const uint32_t stride = gridDim.x * kThreads;
    uint32_t i = blockIdx.x * kThreads + threadIdx.x;
    uint32_t mx = 0;
    for (; i + (kAmaxUnroll - 1) * stride < total; i += kAmaxUnroll * stride) {
        uint4 v[kAmaxUnroll];
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) {
            uint32_t idx = i + u * stride;
            uint32_t r = idx / vpr, c = idx - r * vpr;
            v[u] = ldg_v4(x + r * ldv + c);
        }
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) mx = max(mx, absmax8_bits(v[u]));
    }
    for (; i < total; i += stride) {
        uint32_t r = i / vpr, c = i - r * vpr;
        mx = max(mx, absmax8_bits(ldg_v4(x + r * ldv + c)));
    }
    float m = block_max(__uint_as_float(mx << 16), red);
    if (threadIdx.x == 0) partials[blockIdx.x] = m;
}

// E4M3 byte -> float (exact).
__device__ __forceinline__ float e4m3_to_float(uint32_t b) {
    __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(b), __NV_E4M3);
    return __half2float(__half(h));
}

// Byte offset of the 4 scales (r, 4*cq .. 4*cq+3) in the swizzled layout.
__device__ __forceinline__ uint64_t sf_word_offset(uint32_t r, uint32_t cq, uint32_t ctiles) {
    return (static_cast<uint64_t>(r >> 7) * ctiles + cq) * 512u + (r & 31u) * 16u +
           ((r >> 5) & 3u) * 4u;
}

#ifndef MQ_QUANT_HW_SIGN
#define MQ_QUANT_HW_SIGN 1
#endif
constexpr int kQuantUnroll = 2;

// fp32(a / 6) for a non-negative finite BF16 value a, in three operations:
// q0 = RN(a * RN(1/6)), r = RN(a - 6 q0) (exact by FMA), q = RN(r * RN(1/6) + q0).
// Checked exhaustively against IEEE division for all 32640 non-negative finite
// BF16 inputs.
__device__ __forceinline__ float div6_bf16(float a) {
    const float inv6 = 0.16666667163372039794921875f;  // RN(1/6)
    const float q0 = __fmul_rn(a, inv6);
    const float r = __fmaf_rn(-q0, 6.0f, a);
    return __fmaf_rn(r, inv6, q0);
}

// Two E2M1 codes (lo in bits 3:0, hi in bits 7:4) of x * f, round-to-nearest-even,
// saturating at 6, sign from x (the conversion keeps the sign of a product
// that rounds to zero).
__device__ __forceinline__ uint32_t e2m1x2_signed(float lo, float hi) {
    uint32_t out;
    asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %2, %1;\n\tcvt.u32.u8 %0, b;\n\t}"
        : "=r"(out)
        : "f"(lo), "f"(hi));
    return out;
}

// One lane quantizes one 16-element block held in w[0..7] (two BF16 per word,
// element 2j in the low half of w[j]).  ftab[b] = s_enc / dec(b) for every
// non-negative E4M3 byte b (0 for b = 0).  Returns the 8 code bytes in (lo, hi)
// and the block scale byte in *sb_out.
__device__ __forceinline__ void quantize_block16(const uint32_t (&w)[8], float s_enc,
                                                 const float *ftab, uint32_t &lo, uint32_t &hi,
                                                 uint32_t &sb_out) {
    const uint32_t m = 0x7FFF7FFFu;
    uint32_t a = __vmaxu2(__vmaxu2(w[0] & m, w[1] & m), __vmaxu2(w[2] & m, w[3] & m));
    a = __vmaxu2(a, __vmaxu2(__vmaxu2(w[4] & m, w[5] & m), __vmaxu2(w[6] & m, w[7] & m)));
    const float amax_b = __uint_as_float(max(a & 0xFFFFu, a >> 16) << 16);
    const float sbf = __fmul_rn(div6_bf16(amax_b), s_enc);
    const uint32_t sb = __nv_cvt_float_to_fp8(sbf, __NV_SATFINITE, __NV_E4M3);
    const float f = ftab[sb];  // = dec(sb) == 0 ? 0 : fp32(s_enc / dec(sb))
    uint32_t byte[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float x0 = __uint_as_float(w[j] << 16);
        const float x1 = __uint_as_float(w[j] & 0xFFFF0000u);
#if MQ_QUANT_HW_SIGN
        byte[j] = e2m1x2_signed(__fmul_rn(x0, f), __fmul_rn(x1, f));
#else
        byte[j] = e2m1x2_signed(fabsf(__fmul_rn(x0, f)), fabsf(__fmul_rn(x1, f))) |
                  ((w[j] >> 12) & 0x8u) | ((w[j] >> 24) & 0x80u);
#endif
    }
    lo = byte[0] | (byte[1] << 8) | (byte[2] << 16) | (byte[3] << 24);
    hi = byte[4] | (byte[5] << 8) | (byte[6] << 16) | (byte[7] << 24);
    sb_out = sb;
}

// Each warp quantizes 512-element row segments (lane l: 16-block l of the
// segment, two 16-byte loads), kQuantUnroll segments per iteration with all
// loads issued first.  Lanes 4t..4t+3 hold the 4 scales of one swizzled
// 32-bit scale word.
__global__ void __launch_bounds__(kThreads) quantize_kernel(
    const uint4 *__restrict__ x, uint32_t M, uint32_t K, uint64_t ldv,
    const float *__restrict__ partials, int n_partials, uint2 *__restrict__ codes,
    uint8_t *__restrict__ sf, float *__restrict__ s_enc_out, uint32_t Mpad) {
    __shared__ float red[kThreads / 32];
    __shared__ float ftab[128];
    float amx = 0.0f;
    for (int i = threadIdx.x; i < n_partials; i += kThreads) amx = fmaxf(amx, partials[i]);
    const float amax = block_max(amx, red);
    float s_enc = __fdiv_rn(2688.0f, amax);
    if (amax == 0.0f || !isfinite(s_enc)) s_enc = 1.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0) *s_enc_out = s_enc;
    if (threadIdx.x < 128) {
        const float dec = e4m3_to_float(threadIdx.x);
        ftab[threadIdx.x] = dec == 0.0f ? 0.0f : __fdiv_rn(s_enc, dec);
    }
    __syncthreads();

    const uint32_t ctiles = K / 64u;
    const uint32_t kblocks = K / 16u;
    const uint32_t segs = (K + 511u) / 512u;
    const uint32_t total = M * segs;
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t nwarps = gridDim.x * (kThreads / 32);
    const uint32_t warp_id = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    for (uint32_t base = warp_id; base < total; base += nwarps * kQuantUnroll) {
        uint32_t w[kQuantUnroll][8];
        uint32_t rr[kQuantUnroll], bb[kQuantUnroll];
        bool act[kQuantUnroll];
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            const uint32_t seg = base + u * nwarps;
            const uint32_t r = seg / segs, sg = seg - r * segs;
            rr[u] = r;
            bb[u] = sg * 32u + lane;  // block index within the row
            act[u] = seg < total && bb[u] < kblocks;
            uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
            if (act[u]) {
                const uint4 *px = x + r * ldv + bb[u] * 2u;
                v0 = ldg_v4(px);
                v1 = ldg_v4(px + 1);
            }
            w[u][0] = v0.x; w[u][1] = v0.y; w[u][2] = v0.z; w[u][3] = v0.w;
            w[u][4] = v1.x; w[u][5] = v1.y; w[u][6] = v1.z; w[u][7] = v1.w;
        }
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            uint32_t lo, hi, sb;
            quantize_block16(w[u], s_enc, ftab, lo, hi, sb);
            const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sb, 1);
            const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sb, 2);
            const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sb, 3);
            if (act[u]) {
                codes[static_cast<uint64_t>(rr[u]) * kblocks + bb[u]] = make_uint2(lo, hi);
                if ((lane & 3u) == 0)
                    *reinterpret_cast<uint32_t *>(sf + sf_word_offset(rr[u], bb[u] / 4u, ctiles)) =
                        sb | (s1 << 8) | (s2 << 16) | (s3 << 24);
            }
        }
    }
    // zero the scale bytes of the padding rows [M, Mpad)
    const uint32_t pad_words = (Mpad - M) * ctiles;
    for (uint32_t i = blockIdx.x * kThreads + threadIdx.x; i < pad_words;
         i += gridDim.x * kThreads) {
        const uint32_t r = M + i / ctiles, cq = i % ctiles;
        *reinterpret_cast<uint32_t *>(sf + sf_word_offset(r, cq, ctiles)) = 0u;
    }
}

}  // namespace

int amax_grid(int64_t M, int64_t K, int num_sms) {
    const int64_t vecs = M * (K / 8);
    int64_t g = (vecs + kThreads * kAmaxUnroll - 1) / (kThreads * kAmaxUnroll);
    const int64_t cap = 4LL * num_sms;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    return static_cast<int>(g);
}

cudaError_t launch_amax(const void *x, int64_t M, int64_t K, int64_t ldx, float *partials,
                        int grid, cudaStream_t s) {
    amax_kernel<<<grid, kThreads, 0, s>>>(static_cast<const uint4 *>(x),
                                          static_cast<uint32_t>(M),
                                          static_cast<uint32_t>(K / 8),
                                          static_cast<uint64_t>(ldx / 8), partials);
    return cudaGetLastError();
}

cudaError_t launch_quantize(const void *x, int64_t M, int64_t K, int64_t ldx,
                            const float *partials, int n_partials, uint8_t *codes,
                            uint8_t *sf_swizzled, float *s_enc, int num_sms, cudaStream_t s) {
    const int64_t segs = M * ((K + 511) / 512);
    int64_t g = (segs + (kThreads / 32) - 1) / (kThreads / 32);
    const int64_t cap = 8LL * num_sms;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    const int64_t Mpad = (M + 127) / 128 * 128;
    quantize_kernel<<<static_cast<int>(g), kThreads, 0, s>>>(
        static_cast<const uint4 *>(x), static_cast<uint32_t>(M), static_cast<uint32_t>(K),
        static_cast<uint64_t>(ldx / 8), partials, n_partials, reinterpret_cast<uint2 *>(codes),
        sf_swizzled, s_enc, static_cast<uint32_t>(Mpad));
    return cudaGetLastError();
}

}  // namespace mq
