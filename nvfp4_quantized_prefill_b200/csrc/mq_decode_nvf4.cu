// mq_decode_nvf4.cu -- decode linear with NVFP4 weights and NVFP4 activations
// (W4A4) for a handful of tokens: Y = bf16(alpha * sum_k deq(x) deq(w)).
//
// Method: the Mix-Quant pages contrast their phase-aware scheme (NVFP4 prefill,
// BF16 decode) with uniform NVFP4 quantization of both phases (gist.science
// technical summary, section 1 "Problem Statement" and section 4
// "Experimental Results"); this is the decode half of that uniform variant,
// on the same weight handle's NVFP4 copy.  The activations are quantized with
// the prefill recipe (one tensor scale per call): for up to 8 tokens inside
// this kernel (every CTA takes the tokens' amax and quantizes the blocks it
// needs), for more tokens by the quantize kernels beforehand.
//
// The op streams the NVFP4 weight once (0.5625 byte per parameter).  Work
// unit: 16 weight rows x one K slice; a CTA (8 warps) owns one unit and its
// warps split the slice into steps of 64 K-elements (4 scale blocks).  Per
// step, lane (g, t) takes 8 code bytes of rows g and g + 8 (its 16 elements,
// scale block 4 step + t) and the matching 8 code bytes of token g, turns them
// into FP16 with the hardware E2M1 -> FP16 conversion and multiplies by the
// block scale in FP16 -- both exact: an E2M1 value (2 significant bits) times
// an E4M3 scale (4 significant bits) has at most 6 significant bits and lies
// in [2^-10, 2688] -- and feeds four m16n8k16 FP16 MMAs (FP32 accumulate)
// with W rows as M and up to 8 tokens as N.  Both fragments take the same K
// permutation (a thread's byte p of W pairs with its byte p of X), so no
// staging is needed.  K is split into S slices when there are few row groups;
// the last CTA of a group (atomic counter, reset by that CTA) adds the slices
// in order and writes BF16.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "mq_internal.h"
#include "mq_nvfp4.cuh"

namespace mq {

namespace {

constexpr int kWarps = 8;
constexpr int kRows = 16;
constexpr int kUnroll = 4;

// Byte offset of scale (r, c) in the swizzled layout (512-byte tiles of 128
// rows x 4 scale columns, column tiles fastest).
__device__ __forceinline__ uint64_t sf_offset(uint32_t r, uint32_t c, uint32_t ctiles) {
    return (static_cast<uint64_t>(r >> 7) * ctiles + (c >> 2)) * 512u + (r & 31u) * 16u +
           ((r >> 5) & 3u) * 4u + (c & 3u);
}

// Four code bytes (8 E2M1 values, element 2j in the low nibble of byte j) to
// four FP16x2 words, each multiplied by the block scale s (an FP16x2 pair).
__device__ __forceinline__ void dequant8(uint32_t codes, uint32_t s, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        ".reg .b32 e0, e1, e2, e3;\n\t"
        "shr.b32 e1, %4, 8;\n\tshr.b32 e2, %4, 16;\n\tshr.b32 e3, %4, 24;\n\t"
        "cvt.u8.u32 b0, %4;\n\tcvt.u8.u32 b1, e1;\n\t"
        "cvt.u8.u32 b2, e2;\n\tcvt.u8.u32 b3, e3;\n\t"
        "cvt.rn.f16x2.e2m1x2 e0, b0;\n\tcvt.rn.f16x2.e2m1x2 e1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 e2, b2;\n\tcvt.rn.f16x2.e2m1x2 e3, b3;\n\t"
        "mul.rn.f16x2 %0, e0, %5;\n\tmul.rn.f16x2 %1, e1, %5;\n\t"
        "mul.rn.f16x2 %2, e2, %5;\n\tmul.rn.f16x2 %3, e3, %5;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(codes), "r"(s));
}

// E4M3 scale byte -> the FP16x2 pair (dec(b), dec(b)); exact.
__device__ __forceinline__ uint32_t scale_f16x2(uint32_t b) {
    uint32_t s;
    asm("{\n\t.reg .b16 h;\n\tcvt.u16.u32 h, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, h;\n\t}"
        : "=r"(s)
        : "r"(b * 0x101u));
    return s;
}

__device__ __forceinline__ void mma_f16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32"
        " {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct Step {
    uint2 wa, wb, xv;       // code bytes: row g, row g + 8, token g
    uint32_t sa, sb, sx;    // their scale bytes
    uint4 x0, x1;           // kQuantX: token g's 16 BF16 values of the block
};

// kQuantX = false: x given as NVFP4 codes + swizzled scales (+ tensor scale).
// kQuantX = true (M <= 8): x given in BF16 [M, K]; every CTA takes the
// tokens' amax (a few KB from L2), and each lane quantizes its own 16-element
// block of token g per step with the quantizer's routine -- the codes and
// scales are the ones mq_quantize_nvfp4 would write.
template <bool kQuantX>
__global__ void __launch_bounds__(kWarps * 32) decode_nvf4_kernel(
    const uint8_t *__restrict__ xc, const uint8_t *__restrict__ xsf, uint32_t xrow0, int M,
    const float *__restrict__ s_enc_x, const __nv_bfloat16 *__restrict__ xb,
    const uint8_t *__restrict__ wc, const uint8_t *__restrict__ wsf,
    const float *__restrict__ s_enc_w, int N, int K, int S, __nv_bfloat16 *__restrict__ y,
    float *__restrict__ partials, unsigned *__restrict__ counters) {
    __shared__ float part[kWarps][128];
    __shared__ int last;
    __shared__ float ftab[128];
    __shared__ float red[kWarps];
    griddep_wait();
    griddep_launch_dependents();
    float sx_enc = 0.0f;
    if (kQuantX) {
        // tensor amax of the M x K tokens, then the scale table
        const uint32_t vecs = static_cast<uint32_t>(M) * static_cast<uint32_t>(K / 8);
        const uint4 *xv = reinterpret_cast<const uint4 *>(xb);
        uint32_t mx = 0;
#pragma unroll 4
        for (uint32_t i = threadIdx.x; i < vecs; i += kWarps * 32) mx = max(mx, absmax8_bits(__ldg(xv + i)));
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = __uint_as_float(mx << 16);
        __syncthreads();
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < kWarps; ++i) amax = fmaxf(amax, red[i]);
        sx_enc = nvfp4_tensor_scale(amax);
        nvfp4_scale_table(sx_enc, ftab);
        __syncthreads();
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int group = blockIdx.x / S, slice = blockIdx.x - group * S;
    const int n0 = group * kRows;
    const uint32_t rowb = static_cast<uint32_t>(K / 2);  // code bytes per row
    const uint32_t ctiles = static_cast<uint32_t>(K / 64);
    const int steps = K / 64;
    const int sl0 = static_cast<int>(static_cast<int64_t>(steps) * slice / S);
    const int sl1 = static_cast<int>(static_cast<int64_t>(steps) * (slice + 1) / S);
    const int s0 = sl0 + (sl1 - sl0) * warp / kWarps;
    const int s1 = sl0 + (sl1 - sl0) * (warp + 1) / kWarps;
    const bool ra = n0 + g < N, rb = n0 + g + 8 < N, rx = g < M;
    const uint32_t rA = ra ? n0 + g : 0, rB = rb ? n0 + g + 8 : 0, rX = xrow0 + (rx ? g : 0);
    const uint8_t *pa = wc + static_cast<uint64_t>(rA) * rowb + 8 * t;
    const uint8_t *pb = wc + static_cast<uint64_t>(rB) * rowb + 8 * t;
    const uint8_t *px = xc + static_cast<uint64_t>(rX) * rowb + 8 * t;
    const uint4 *pxb =
        kQuantX ? reinterpret_cast<const uint4 *>(xb) +
                      (static_cast<uint64_t>(rX) * static_cast<uint32_t>(K) + 16u * t) / 8u
                : nullptr;
    const uint2 z2 = make_uint2(0, 0);
    float c[4] = {0.f, 0.f, 0.f, 0.f};

    auto load = [&](int s, Step &d) {
        const uint32_t cb = 4u * static_cast<uint32_t>(s) + static_cast<uint32_t>(t);  // scale block
        d.wa = ra ? __ldg(reinterpret_cast<const uint2 *>(pa + 32 * s)) : z2;
        d.wb = rb ? __ldg(reinterpret_cast<const uint2 *>(pb + 32 * s)) : z2;
        d.sa = ra ? __ldg(wsf + sf_offset(rA, cb, ctiles)) : 0u;
        d.sb = rb ? __ldg(wsf + sf_offset(rB, cb, ctiles)) : 0u;
        if (kQuantX) {
            const uint4 z4 = make_uint4(0, 0, 0, 0);
            d.x0 = rx ? __ldg(pxb + 8 * s) : z4;       // 64 K-elements = 8 vectors per step
            d.x1 = rx ? __ldg(pxb + 8 * s + 1) : z4;
        } else {
            d.xv = rx ? __ldg(reinterpret_cast<const uint2 *>(px + 32 * s)) : z2;
            d.sx = rx ? __ldg(xsf + sf_offset(rX, cb, ctiles)) : 0u;
        }
    };
    auto compute = [&](Step &d) {
        if (kQuantX) {
            const uint32_t w8[8] = {d.x0.x, d.x0.y, d.x0.z, d.x0.w, d.x1.x, d.x1.y, d.x1.z, d.x1.w};
            uint32_t lo, hi, sb;
            quantize_block16<false>(w8, sx_enc, ftab, lo, hi, sb);
            d.xv = make_uint2(lo, hi);
            d.sx = sb;
        }
        uint32_t a0[4], a1[4], b0[4], b1[4], x0[4], x1[4];
        const uint32_t fa = scale_f16x2(d.sa), fb = scale_f16x2(d.sb), fx = scale_f16x2(d.sx);
        dequant8(d.wa.x, fa, a0);
        dequant8(d.wa.y, fa, a1);
        dequant8(d.wb.x, fb, b0);
        dequant8(d.wb.y, fb, b1);
        dequant8(d.xv.x, fx, x0);
        dequant8(d.xv.y, fx, x1);
        // MMA j: this thread's pairs 2j and 2j + 1 of rows g, g + 8 and token g
        mma_f16_16816(c, a0[0], b0[0], a0[1], b0[1], x0[0], x0[1]);
        mma_f16_16816(c, a0[2], b0[2], a0[3], b0[3], x0[2], x0[3]);
        mma_f16_16816(c, a1[0], b1[0], a1[1], b1[1], x1[0], x1[1]);
        mma_f16_16816(c, a1[2], b1[2], a1[3], b1[3], x1[2], x1[3]);
    };
    int s = s0;
    for (; s + kUnroll <= s1; s += kUnroll) {
        Step d[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) load(s + u, d[u]);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) compute(d[u]);
    }
    for (; s < s1; ++s) {
        Step d;
        load(s, d);
        compute(d);
    }
    const float alpha = __frcp_rn(__fmul_rn(kQuantX ? sx_enc : *s_enc_x, *s_enc_w));
#pragma unroll
    for (int i = 0; i < 4; ++i) part[warp][lane * 4 + i] = c[i];
    __syncthreads();
    // accumulator element q = 4 * lane' + i': W row g' (+8 for i' >= 2), token 2 t' + (i' & 1)
    const int q = threadIdx.x;
    if (q >= 128) return;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) acc += part[i][q];
    const int lq = q >> 2, iq = q & 3;
    const int wrow = n0 + (lq >> 2) + ((iq >> 1) << 3);
    const int m = 2 * (lq & 3) + (iq & 1);
    if (S == 1) {
        if (m < M && wrow < N)
            y[static_cast<int64_t>(m) * N + wrow] = __float2bfloat16_rn(__fmul_rn(alpha, acc));
        return;
    }
    float *mine = partials + (static_cast<int64_t>(group) * S + slice) * 128;
    mine[q] = acc;
    __threadfence();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (threadIdx.x == 0) last = (atomicAdd(&counters[group], 1u) == static_cast<unsigned>(S - 1));
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (!last) return;
    __threadfence();
    float sum = 0.f;
    for (int k = 0; k < S; ++k)
        sum += __ldcg(partials + (static_cast<int64_t>(group) * S + k) * 128 + q);
    if (m < M && wrow < N)
        y[static_cast<int64_t>(m) * N + wrow] = __float2bfloat16_rn(__fmul_rn(alpha, sum));
    if (threadIdx.x == 0) counters[group] = 0u;  // ready for the next call
}

}  // namespace

int decode_nvf4_slices(int64_t N, int64_t K, int num_sms) {
    const int64_t groups = (N + kRows - 1) / kRows;
    if (groups >= 2LL * num_sms) return 1;
    int64_t S = (2LL * num_sms + groups - 1) / groups;
    const int64_t max_s = K / 1024 > 0 ? K / 1024 : 1;   // keep >= 16 steps per slice
    if (S > max_s) S = max_s;
    if (S > 16) S = 16;
    if (S < 1) S = 1;
    return static_cast<int>(S);
}

cudaError_t launch_decode_nvf4(const uint8_t *x_codes, const uint8_t *x_sf, const float *s_enc_x,
                               const void *x_bf16, int64_t M, const uint8_t *w_codes,
                               const uint8_t *w_sf, const float *s_enc_w, int64_t N, int64_t K,
                               void *y, void *scratch, int num_sms, cudaStream_t s) {
    const int S = decode_nvf4_slices(N, K, num_sms);
    const int64_t groups = (N + kRows - 1) / kRows;
    unsigned *counters = static_cast<unsigned *>(scratch);
    float *partials = reinterpret_cast<float *>(static_cast<uint8_t *>(scratch) +
                                                decode_counter_bytes(N));
    const int grid = static_cast<int>(groups * S);
    if (x_bf16) {  // M <= 8: tokens quantized in the kernel
        cudaError_t e = launch_pdl(decode_nvf4_kernel<true>, dim3(grid), dim3(kWarps * 32), 0, s,
                                   x_codes, x_sf, 0u, static_cast<int>(M), s_enc_x,
                                   static_cast<const __nv_bfloat16 *>(x_bf16), w_codes, w_sf, s_enc_w,
                                   static_cast<int>(N), static_cast<int>(K), S,
                                   static_cast<__nv_bfloat16 *>(y), partials, counters);
        return e == cudaSuccess ? cudaGetLastError() : e;
    }
    for (int64_t m0 = 0; m0 < M; m0 += 8) {
        const int mg = static_cast<int>(M - m0 < 8 ? M - m0 : 8);
        cudaError_t e = launch_pdl(decode_nvf4_kernel<false>, dim3(grid), dim3(kWarps * 32), 0, s,
                                   x_codes, x_sf, static_cast<uint32_t>(m0), mg, s_enc_x,
                                   static_cast<const __nv_bfloat16 *>(nullptr), w_codes, w_sf,
                                   s_enc_w, static_cast<int>(N), static_cast<int>(K), S,
                                   static_cast<__nv_bfloat16 *>(y) + m0 * N, partials, counters);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace mq
