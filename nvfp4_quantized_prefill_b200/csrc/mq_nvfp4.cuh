// mq_nvfp4.cuh -- device routines of the NVFP4 encoding shared by the
// activation quantizer and the W4A4 decode (which quantizes its tokens
// in-kernel): one 16-element block of BF16 values -> E4M3 block scale and
// E2M1 codes, exactly as the quantize kernel defines them.
//
// Encoding (Mix-Quant pages: NVFP4 with a per-16 local scale and a tensor
// scale, round-to-nearest; gist.science technical summary, section 2 "Hybrid
// Precision Strategy"): s_enc = 2688 / amax (1 for an all-zero tensor),
//   sb = E4M3_satfinite(fp32(fp32(amax_b / 6) * s_enc))
//   f  = dec(sb) == 0 ? 0 : fp32(s_enc / dec(sb))
//   q  = E2M1_satfinite(fp32(x * f)), sign taken from x.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace mq {

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

// E4M3 byte -> float (exact).
__device__ __forceinline__ float e4m3_to_float(uint32_t b) {
    __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(b), __NV_E4M3);
    return __half2float(__half(h));
}

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
// times f, each product rounded to FP32 and then to E2M1 (round-to-nearest-
// even, saturating at 6, the sign of x kept even when the code is zero);
// returns the four code bytes, element 2j in the low nibble of byte j.  The
// products are scalar FP32 multiplies: the packed f32x2 form measured ~12%
// slower in the quantizer.  kToMemory: the bytes are packed with one vector
// mov of the four 8-bit results (the quantizer, whose codes go to memory).
// Otherwise they are widened and combined with integer arithmetic: a packed
// word that was unpacked again into 8-bit registers in the same kernel,
// without passing through memory, was observed to lose its top byte.
template <bool kToMemory>
__device__ __forceinline__ uint32_t e2m1x8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                           float f) {
    uint32_t out;
    if (kToMemory) {
        asm("{\n\t"
            ".reg .b8 c0, c1, c2, c3;\n\t"
            ".reg .b32 l0, h0, l1, h1, l2, h2, l3, h3;\n\t"
            "shl.b32 l0, %1, 16;\n\tand.b32 h0, %1, 0xFFFF0000;\n\t"
            "shl.b32 l1, %2, 16;\n\tand.b32 h1, %2, 0xFFFF0000;\n\t"
            "shl.b32 l2, %3, 16;\n\tand.b32 h2, %3, 0xFFFF0000;\n\t"
            "shl.b32 l3, %4, 16;\n\tand.b32 h3, %4, 0xFFFF0000;\n\t"
            "mul.rn.f32 l0, l0, %5;\n\tmul.rn.f32 h0, h0, %5;\n\t"
            "mul.rn.f32 l1, l1, %5;\n\tmul.rn.f32 h1, h1, %5;\n\t"
            "mul.rn.f32 l2, l2, %5;\n\tmul.rn.f32 h2, h2, %5;\n\t"
            "mul.rn.f32 l3, l3, %5;\n\tmul.rn.f32 h3, h3, %5;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 c0, h0, l0;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 c1, h1, l1;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 c2, h2, l2;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 c3, h3, l3;\n\t"
            "mov.b32 %0, {c0, c1, c2, c3};\n\t"
            "}"
            : "=r"(out)
            : "r"(w0), "r"(w1), "r"(w2), "r"(w3), "f"(f));
    } else {
        asm("{\n\t"
            ".reg .b8 c0, c1, c2, c3;\n\t"
            ".reg .b32 l0, h0, l1, h1, l2, h2, l3, h3;\n\t"
            "shl.b32 l0, %1, 16;\n\tand.b32 h0, %1, 0xFFFF0000;\n\t"
            "shl.b32 l1, %2, 16;\n\tand.b32 h1, %2, 0xFFFF0000;\n\t"
            "shl.b32 l2, %3, 16;\n\tand.b32 h2, %3, 0xFFFF0000;\n\t"
            "shl.b32 l3, %4, 16;\n\tand.b32 h3, %4, 0xFFFF0000;\n\t"
            "mul.rn.f32 l0, l0, %5;\n\tmul.rn.f32 h0, h0, %5;\n\t"
            "mul.rn.f32 l1, l1, %5;\n\tmul.rn.f32 h1, h1, %5;\n\t"
            "mul.rn.f32 l2, l2, %5;\n\tmul.rn.f32 h2, h2, %5;\n\t"
            "mul.rn.f32 l3, l3, %5;\n\tmul.rn.f32 h3, h3, %5;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 c0, h0, l0;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 c1, h1, l1;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 c2, h2, l2;\n\t"
            "cvt.rn.satfinite.e2m1x2.f32 c3, h3, l3;\n\t"
            "cvt.u32.u8 l0, c0;\n\tcvt.u32.u8 l1, c1;\n\t"
            "cvt.u32.u8 l2, c2;\n\tcvt.u32.u8 l3, c3;\n\t"
            "mad.lo.u32 l0, l1, 256, l0;\n\tmad.lo.u32 l2, l3, 256, l2;\n\t"
            "mad.lo.u32 %0, l2, 65536, l0;\n\t"
            "}"
            : "=r"(out)
            : "r"(w0), "r"(w1), "r"(w2), "r"(w3), "f"(f));
    }
    return out;
}

// One lane quantizes one 16-element block held in w[0..7] (two BF16 per word,
// element 2j in the low half of w[j]).  ftab[b] = s_enc / dec(b) for every
// non-negative E4M3 byte b (0 for b = 0).  Returns the 8 code bytes in (lo, hi)
// and the block scale byte in *sb_out (kToMemory: see e2m1x8).
template <bool kToMemory>
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
    lo = e2m1x8<kToMemory>(w[0], w[1], w[2], w[3], f);
    hi = e2m1x8<kToMemory>(w[4], w[5], w[6], w[7], f);
    sb_out = sb;
}

// s_enc from the tensor amax, as the quantizer defines it.
__device__ __forceinline__ float nvfp4_tensor_scale(float amax) {
    float s_enc = __fdiv_rn(2688.0f, amax);
    if (amax == 0.0f || !isfinite(s_enc)) s_enc = 1.0f;
    return s_enc;
}

// ftab[b] = s_enc / dec(b) (0 for dec(b) = 0) for the 128 non-negative E4M3
// bytes, written by threads tid = 0 .. nthreads - 1 (by default threads
// 0..127 of the block, one entry each).
__device__ __forceinline__ void nvfp4_scale_table(float s_enc, float *ftab, uint32_t tid,
                                                  uint32_t nthreads) {
    for (uint32_t b = tid; b < 128u; b += nthreads) {
        const float dec = e4m3_to_float(b);
        ftab[b] = dec == 0.0f ? 0.0f : __fdiv_rn(s_enc, dec);
    }
}
__device__ __forceinline__ void nvfp4_scale_table(float s_enc, float *ftab) {
    if (threadIdx.x < 128) nvfp4_scale_table(s_enc, ftab, threadIdx.x, 128u);
}

}  // namespace mq
