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
// warp, grids sized in multiples of the SM count.  amax keeps 8 independent
// 16-byte loads per thread in flight (HBM latency x bandwidth needs ~64 KB in
// flight per SM); quantize runs one resident wave of CTAs and walks the matrix
// from its end back to its start, so that it first reads the rows that amax
// read last -- the ones most likely still in L2.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_fp16.h>

#include "mq_internal.h"

namespace mq {

namespace {

// Tuning constants (compile-time overridable for sweeps).
#ifndef MQ_AMAX_UNROLL
#define MQ_AMAX_UNROLL 4
#endif
#ifndef MQ_AMAX_BLOCKS_PER_SM
#define MQ_AMAX_BLOCKS_PER_SM 8
#endif
#ifndef MQ_AMAX_NO_ALLOCATE
#define MQ_AMAX_NO_ALLOCATE 0
#endif
#ifndef MQ_QUANT_UNROLL
#define MQ_QUANT_UNROLL 2
#endif
#ifndef MQ_QUANT_BLOCKS_PER_SM
#define MQ_QUANT_BLOCKS_PER_SM 6
#endif

constexpr int kThreads = 256;
constexpr int kAmaxUnroll = MQ_AMAX_UNROLL;
constexpr int kAmaxBlocksPerSm = MQ_AMAX_BLOCKS_PER_SM;

__device__ __forceinline__ uint4 ldg_v4(const uint4 *p) { return __ldg(p); }

// streaming read that does not allocate in L1 (each byte is read once)
__device__ __forceinline__ uint4 ldg_v4_stream(const uint4 *p) {
#if MQ_AMAX_NO_ALLOCATE
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
#else
    return __ldg(p);
#endif
}

// max of |bf16| over the 8 values of a 16-byte vector, as 16-bit magnitude bits
// (non-negative bf16 values order like their bit patterns).
__device__ __forceinline__ uint32_t absmax8_bits(uint4 v) {
    uint32_t a, b;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(v.x), "r"(v.y));
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(b) : "r"(v.z), "r"(v.w));
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(a), "r"(b));
    a &= 0x7FFF7FFFu;
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

// Grid-stride over the [M, vpr] matrix of 16-byte vectors (row stride ldv
// vectors); each round issues kAmaxUnroll loads before reducing them.
__global__ void __launch_bounds__(kThreads, kAmaxBlocksPerSm)
    amax_kernel(const uint4 *__restrict__ x, uint32_t M, uint32_t vpr, uint64_t ldv,
                float *__restrict__ partials) {
    __shared__ float red[kThreads / 32];
    griddep_wait();
    griddep_launch_dependents();
    const uint32_t total = M * vpr;
    const uint32_t stride = gridDim.x * kThreads;
    const bool dense = ldv == vpr;
    uint32_t mx = 0;
    for (uint32_t i = blockIdx.x * kThreads + threadIdx.x; i < total; i += kAmaxUnroll * stride) {
        uint4 v[kAmaxUnroll];
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) {
            const uint32_t idx = i + u * stride;
            v[u] = make_uint4(0, 0, 0, 0);
            if (idx < total) {
                uint64_t off = idx;
                if (!dense) {
                    const uint32_t r = idx / vpr;
                    off = r * ldv + (idx - r * vpr);
                }
                v[u] = ldg_v4_stream(x + off);
            }
        }
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) mx = max(mx, absmax8_bits(v[u]));
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

constexpr int kQuantUnroll = MQ_QUANT_UNROLL;
constexpr int kQuantBlocksPerSm = MQ_QUANT_BLOCKS_PER_SM;

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

// max(|a|, |b|) per BF16 half, sign bits = sign(a) ^ sign(b) (mask them off
// to read the magnitudes).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Eight BF16 values (two per word, element 2j in the low half of word j)
// times f, each product rounded to FP32 (packed f32x2 multiplies) and then to
// E2M1 (round-to-nearest-even, saturating at 6, the sign of x kept even when
// the code is zero); returns the four code bytes, element 2j in the low
// nibble of byte j.
__device__ __forceinline__ uint32_t e2m1x8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                           float f) {
    uint32_t out;
    asm("{\n\t"
        ".reg .b8 c0, c1, c2, c3;\n\t"
        ".reg .b64 f2, x0, x1, x2, x3;\n\t"
        ".reg .b32 l0, h0, l1, h1, l2, h2, l3, h3;\n\t"
        "mov.b64 f2, {%5, %5};\n\t"
        "shl.b32 l0, %1, 16;\n\tand.b32 h0, %1, 0xFFFF0000;\n\t"
        "shl.b32 l1, %2, 16;\n\tand.b32 h1, %2, 0xFFFF0000;\n\t"
        "shl.b32 l2, %3, 16;\n\tand.b32 h2, %3, 0xFFFF0000;\n\t"
        "shl.b32 l3, %4, 16;\n\tand.b32 h3, %4, 0xFFFF0000;\n\t"
        "mov.b64 x0, {l0, h0};\n\tmov.b64 x1, {l1, h1};\n\t"
        "mov.b64 x2, {l2, h2};\n\tmov.b64 x3, {l3, h3};\n\t"
        "mul.rn.f32x2 x0, x0, f2;\n\tmul.rn.f32x2 x1, x1, f2;\n\t"
        "mul.rn.f32x2 x2, x2, f2;\n\tmul.rn.f32x2 x3, x3, f2;\n\t"
        "mov.b64 {l0, h0}, x0;\n\tmov.b64 {l1, h1}, x1;\n\t"
        "mov.b64 {l2, h2}, x2;\n\tmov.b64 {l3, h3}, x3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c0, h0, l0;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c1, h1, l1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c2, h2, l2;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c3, h3, l3;\n\t"
        "mov.b32 %0, {c0, c1, c2, c3};\n\t"
        "}"
        : "=r"(out)
        : "r"(w0), "r"(w1), "r"(w2), "r"(w3), "f"(f));
    return out;
}

// One lane quantizes one 16-element block held in w[0..7] (two BF16 per word,
// element 2j in the low half of w[j]).  ftab[b] = s_enc / dec(b) for every
// non-negative E4M3 byte b (0 for b = 0).  Returns the 8 code bytes in (lo, hi)
// and the block scale byte in *sb_out.
__device__ __forceinline__ void quantize_block16(const uint32_t (&w)[8], float s_enc,
                                                 const float *ftab, uint32_t &lo, uint32_t &hi,
                                                 uint32_t &sb_out) {
    uint32_t a = absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(w[0], w[1]), absmax_bf16x2(w[2], w[3])),
                               absmax_bf16x2(absmax_bf16x2(w[4], w[5]), absmax_bf16x2(w[6], w[7])));
    a &= 0x7FFF7FFFu;
    const float amax_b = __uint_as_float(max(a & 0xFFFFu, a >> 16) << 16);
    const float sbf = __fmul_rn(div6_bf16(amax_b), s_enc);
    const uint32_t sb = __nv_cvt_float_to_fp8(sbf, __NV_SATFINITE, __NV_E4M3);
    const float f = ftab[sb];  // = dec(sb) == 0 ? 0 : fp32(s_enc / dec(sb))
    lo = e2m1x8(w[0], w[1], w[2], w[3], f);
    hi = e2m1x8(w[4], w[5], w[6], w[7], f);
    sb_out = sb;
}

// Each warp quantizes 512-element row segments (lane l: 16-block l of the
// segment, two 16-byte loads), kQuantUnroll segments per iteration with all
// loads issued first; segments are taken from the last one backwards.  Lanes
// 4t..4t+3 hold the 4 scales of one swizzled 32-bit scale word.
__global__ void __launch_bounds__(kThreads, kQuantBlocksPerSm) quantize_kernel(
    const uint4 *__restrict__ x, uint32_t M, uint32_t K, uint64_t ldv,
    const float *__restrict__ partials, int n_partials, uint2 *__restrict__ codes,
    uint8_t *__restrict__ sf, float *__restrict__ s_enc_out, uint32_t Mpad) {
    __shared__ float red[kThreads / 32];
    __shared__ float ftab[128];
    griddep_wait();
    griddep_launch_dependents();
    float amx = 0.0f;
#pragma unroll 4
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
    // Segment seg = total - 1 - pos for pos = warp_id, warp_id + nwarps, ...;
    // (row, segment-in-row) of the current seg is stepped back by nwarps
    // segments at a time: dq rows and dr segments.
    const uint32_t dq = nwarps / segs, dr = nwarps - (nwarps / segs) * segs;
    uint32_t r0 = 0, s0 = 0;
    if (warp_id < total) {
        const uint32_t seg = total - 1u - warp_id;
        r0 = seg / segs;
        s0 = seg - r0 * segs;
    }
    auto step_back = [&](uint32_t &r, uint32_t &sg) {
        if (sg >= dr) {
            sg -= dr;
            r -= dq;
        } else {
            sg += segs - dr;
            r -= dq + 1u;
        }
    };
    for (uint32_t base = warp_id; base < total; base += nwarps * kQuantUnroll) {
        uint32_t w[kQuantUnroll][8];
        uint32_t rr[kQuantUnroll], bb[kQuantUnroll];
        bool act[kQuantUnroll];
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            rr[u] = r0;
            bb[u] = s0 * 32u + lane;  // block index within the row
            act[u] = base + u * nwarps < total && bb[u] < kblocks;
            uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
            if (act[u]) {
                const uint4 *px = x + r0 * ldv + bb[u] * 2u;
                v0 = ldg_v4(px);
                v1 = ldg_v4(px + 1);
            }
            w[u][0] = v0.x; w[u][1] = v0.y; w[u][2] = v0.z; w[u][3] = v0.w;
            w[u][4] = v1.x; w[u][5] = v1.y; w[u][6] = v1.z; w[u][7] = v1.w;
            step_back(r0, s0);
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
    const int64_t cap = static_cast<int64_t>(kAmaxBlocksPerSm) * num_sms;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    return static_cast<int>(g);
}

cudaError_t launch_amax(const void *x, int64_t M, int64_t K, int64_t ldx, float *partials,
                        int grid, cudaStream_t s) {
    return launch_pdl(amax_kernel, dim3(grid), dim3(kThreads), 0, s, static_cast<const uint4 *>(x),
                      static_cast<uint32_t>(M), static_cast<uint32_t>(K / 8),
                      static_cast<uint64_t>(ldx / 8), partials);
}

cudaError_t launch_quantize(const void *x, int64_t M, int64_t K, int64_t ldx,
                            const float *partials, int n_partials, uint8_t *codes,
                            uint8_t *sf_swizzled, float *s_enc, int num_sms, cudaStream_t s) {
    // one resident wave: every CTA pays the scale-table prologue once
    static int resident = 0;
    if (resident == 0) {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, quantize_kernel, kThreads, 0) !=
                cudaSuccess ||
            b < 1)
            b = 1;
        resident = b;
    }
    const int64_t segs = M * ((K + 511) / 512);
    int64_t g = (segs + (kThreads / 32) - 1) / (kThreads / 32);
    const int64_t cap = static_cast<int64_t>(resident) * num_sms;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    const int64_t Mpad = (M + 127) / 128 * 128;
    return launch_pdl(quantize_kernel, dim3(static_cast<unsigned>(g)), dim3(kThreads), 0, s,
                      static_cast<const uint4 *>(x), static_cast<uint32_t>(M),
                      static_cast<uint32_t>(K), static_cast<uint64_t>(ldx / 8), partials,
                      n_partials, reinterpret_cast<uint2 *>(codes), sf_swizzled, s_enc,
                      static_cast<uint32_t>(Mpad));
}

}  // namespace mq
