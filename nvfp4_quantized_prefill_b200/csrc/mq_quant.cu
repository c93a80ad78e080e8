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

// Four pairs of non-negative floats -> 4 bytes of E2M1x2 (second of each pair
// in the high nibble), round-to-nearest-even, saturating at 6.
__device__ __forceinline__ uint32_t e2m1x8(const float (&a)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(a[0]), "f"(a[1]), "f"(a[2]), "f"(a[3]), "f"(a[4]), "f"(a[5]), "f"(a[6]),
          "f"(a[7]));
    return out;
}

// Byte offset of the 4 scales (r, 4*cq .. 4*cq+3) in the swizzled layout.
__device__ __forceinline__ uint64_t sf_word_offset(uint32_t r, uint32_t cq, uint32_t ctiles) {
    return (static_cast<uint64_t>(r >> 7) * ctiles + cq) * 512u + (r & 31u) * 16u +
           ((r >> 5) & 3u) * 4u;
}

// One warp quantizes one 256-element segment of a row per iteration: lane l
// owns elements [8l, 8l+8), lanes 2j and 2j+1 form 16-block j.
__global__ void __launch_bounds__(kThreads) quantize_kernel(
    const uint4 *__restrict__ x, uint32_t M, uint32_t K, uint64_t ldv,
    const float *__restrict__ partials, int n_partials, uint32_t *__restrict__ codes,
    uint8_t *__restrict__ sf, float *__restrict__ s_enc_out, uint32_t Mpad) {
    __shared__ float red[kThreads / 32];
    float a = 0.0f;
    for (int i = threadIdx.x; i < n_partials; i += kThreads) a = fmaxf(a, partials[i]);
    const float amax = block_max(a, red);
    float s_enc = __fdiv_rn(2688.0f, amax);
    if (amax == 0.0f || !isfinite(s_enc)) s_enc = 1.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0) *s_enc_out = s_enc;

    const uint32_t ctiles = K / 64u;
    const uint32_t segs = (K + 255u) / 256u;
    const uint32_t total = M * segs;
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t nwarps = gridDim.x * (kThreads / 32);
    for (uint32_t seg = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); seg < total;
         seg += nwarps) {
        const uint32_t r = seg / segs, s = seg - r * segs;
        const uint32_t k0 = s * 256u + lane * 8u;
        const bool active = k0 < K;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (active) v = ldg_v4(x + r * ldv + k0 / 8u);
        uint32_t mb = absmax8_bits(v);
        mb = max(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, 1));
        const float amax_b = __uint_as_float(mb << 16);
        const float sbf = __fmul_rn(__fdiv_rn(amax_b, 6.0f), s_enc);
        const uint32_t sb = __nv_cvt_float_to_fp8(sbf, __NV_SATFINITE, __NV_E4M3);
        const float dec = e4m3_to_float(sb);
        const float f = dec == 0.0f ? 0.0f : __fdiv_rn(s_enc, dec);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float mag[8];
        uint32_t signs = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t bits = (w[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu;
            mag[e] = fabsf(__fmul_rn(__uint_as_float(bits << 16), f));
            signs |= (bits >> 15) << (4 * e + 3);
        }
        const uint32_t word = e2m1x8(mag) | signs;
        // scales of 4 consecutive blocks: lanes 8t, 8t+2, 8t+4, 8t+6
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sb, 2);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sb, 4);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sb, 6);
        if (active) {
            codes[(static_cast<uint64_t>(r) * K + k0) / 8u] = word;
            if ((lane & 7u) == 0) {
                const uint32_t cq = k0 / 64u;
                *reinterpret_cast<uint32_t *>(sf + sf_word_offset(r, cq, ctiles)) =
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
    const int64_t segs = M * ((K + 255) / 256);
    int64_t g = (segs + (kThreads / 32) - 1) / (kThreads / 32);
    const int64_t cap = 8LL * num_sms;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    const int64_t Mpad = (M + 127) / 128 * 128;
    quantize_kernel<<<static_cast<int>(g), kThreads, 0, s>>>(
        static_cast<const uint4 *>(x), static_cast<uint32_t>(M), static_cast<uint32_t>(K),
        static_cast<uint64_t>(ldx / 8), partials, n_partials, reinterpret_cast<uint32_t *>(codes),
        sf_swizzled, s_enc, static_cast<uint32_t>(Mpad));
    return cudaGetLastError();
}

}  // namespace mq
