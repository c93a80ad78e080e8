// mq_decode_gemv4.cu -- uniform-NVFP4 (W4A4) decode linear for 1 to 4
// tokens on the CUDA cores: Y = bf16(alpha * sum_k deq(x) deq(w)).
//
// Method: the Mix-Quant pages contrast their scheme (NVFP4 prefill, BF16
// decode) with quantizing both phases to NVFP4 (gist.science technical
// summary, section 1 "Problem Statement" and section 4 "Experimental
// Results"); this is the decode half of that uniform variant on the weight
// handle's NVFP4 copy, the tokens quantized with the prefill recipe (one
// tensor scale for the call, E4M3 scale per 16, E2M1 codes).
//
// A few tokens read each weight byte once and do a few operations with it,
// so the kernel is a stream: every warp walks its rows K step by K step (a
// step = 1024 K-elements: lane l takes 16 code bytes = 32 elements = two
// scale blocks), with eight steps' loads in flight per lane, issued before
// the wait on the preceding kernel (the weight is constant; packing ends with
// a memory set, so the kernel before a decode never writes it).  Per element:
// the hardware E2M1 -> FP16 conversion (shared by the tokens), a multiply by
// the block scale in FP16 -- exact: an E2M1 value (2 significant bits) times
// an E4M3 scale (4 bits) lies in [2^-10, 2688] with at most 6 bits -- and one
// FP16 x FP16 -> FP32 fused multiply-add per token against the token's
// dequantized value (also exact in FP16), so every product is exact and only
// the FP32 sums round.  Each CTA quantizes the tokens into shared memory first
// (the quantizer's own block routine: codes, scales and tensor scale equal
// mq_quantize_nvfp4's), stored so that a step's 32 lanes read consecutive
// 16-byte chunks.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "mq_internal.h"
#include "mq_nvfp4.cuh"

namespace mq {

namespace {

constexpr int kGWarps = 8;
constexpr int kGThreads = 32 * kGWarps;
constexpr int kRing = 8;                  // steps in flight per lane
constexpr int kStepElems = 1024;          // K-elements per warp step (32 per lane)

struct GemvParams {
    const uint4 *w;          // codes [N, K/2] bytes as 16-byte words (K/32 a row)
    const uint8_t *w_sf;     // swizzled E4M3 scales of the weight
    const float *s_enc_w;
    const __nv_bfloat16 *x;  // [M, K]
    __nv_bfloat16 *y;        // [M, N]
    int N, K, steps;         // steps = ceil(K / 1024)
};

// E4M3 scale byte -> the FP16x2 pair (dec(b), dec(b)); exact.
__device__ __forceinline__ uint32_t scale_pair(uint32_t b) {
    uint32_t s;
    asm("{\n\t.reg .b16 h;\n\tcvt.u16.u32 h, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, h;\n\t}"
        : "=r"(s)
        : "r"(b * 0x101u));
    return s;
}

// Four code bytes (8 E2M1 values; element 2j in the low nibble of byte j) read
// from memory -> four FP16x2 words, each times the scale pair s (exact).
__device__ __forceinline__ void dequant8(uint32_t codes, uint32_t s, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        ".reg .b32 e0, e1, e2, e3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 e0, b0;\n\tcvt.rn.f16x2.e2m1x2 e1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 e2, b2;\n\tcvt.rn.f16x2.e2m1x2 e3, b3;\n\t"
        "mul.rn.f16x2 %0, e0, %5;\n\tmul.rn.f16x2 %1, e1, %5;\n\t"
        "mul.rn.f16x2 %2, e2, %5;\n\tmul.rn.f16x2 %3, e3, %5;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(codes), "r"(s));
}

// Four code bytes read from memory -> four FP16x2 words of the E2M1 values.
__device__ __forceinline__ void e2m1x8_f16(uint32_t codes, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(codes));
}

// acc_lo += lo(a) lo(b), acc_hi += hi(a) hi(b): FP16 x FP16 products (exact
// in FP32) added in FP32.
__device__ __forceinline__ void fma2_f16_f32(uint32_t a, uint32_t b, float &acc_lo, float &acc_hi) {
    asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\t"
        "mov.b32 {a0, a1}, %2;\n\tmov.b32 {b0, b1}, %3;\n\t"
        "fma.rn.f32.f16 %0, a0, b0, %0;\n\t"
        "fma.rn.f32.f16 %1, a1, b1, %1;\n\t}"
        : "+f"(acc_lo), "+f"(acc_hi)
        : "r"(a), "r"(b));
}

__device__ __forceinline__ uint32_t sf_word_off(uint32_t r, uint32_t cq, uint32_t ctiles) {
    return ((r >> 7) * ctiles + cq) * 512u + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u;
}

__device__ __forceinline__ void st_shared_v4_(uint32_t addr, const uint32_t (&v)[4]) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]),
                 "r"(v[3])
                 : "memory");
}

__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t (&v)[4]) {
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                 : "r"(addr));
}

template <int kM>
__global__ void __launch_bounds__(kGThreads, 2) decode_nvf4_gemv_kernel(const GemvParams p) {
    extern __shared__ __align__(16) uint8_t xs_raw[];   // [kM][steps][4][32][16 B]
    __shared__ float ftab[128];
    __shared__ float red[kGWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t K = static_cast<uint32_t>(p.K);
    const uint32_t row_words = K / 32u;          // 16-byte code words per weight row
    const uint32_t ctiles = K / 64u;
    const int steps = p.steps;
    const int gw = blockIdx.x * kGWarps + warp, nw = gridDim.x * kGWarps;
    const int my_rows = gw < p.N ? (p.N - 1 - gw) / nw + 1 : 0;
    const int total = my_rows * steps;         // this warp's (row, step) sequence

    // ---- the first kRing steps' weight loads, before the wait: the weight is
    // constant (see the file comment)
    uint4 ring[kRing];
    uint32_t sring[kRing];
    // issue position: row index in this warp's rows, step, and the lane's
    // code word / scale addresses, advanced by constant strides within a row
    int irow = 0, istep = 0;
    const uint4 *wp = nullptr;
    const unsigned short *sp = nullptr;
    auto row_start = [&]() {
        const uint32_t r = static_cast<uint32_t>(gw + irow * nw);
        wp = p.w + static_cast<uint64_t>(r) * row_words + lane;
        // scale blocks 2 lane, 2 lane + 1 of step 0: word (lane / 2), bytes 2 (lane % 2) ..
        sp = reinterpret_cast<const unsigned short *>(p.w_sf + sf_word_off(r, lane >> 1, ctiles) +
                                                      2u * (lane & 1u));
    };
    if (my_rows > 0) row_start();
    auto issue = [&](uint4 &c, uint32_t &sc) {
        c = make_uint4(0, 0, 0, 0);
        sc = 0;
        if (irow < my_rows) {
            if (static_cast<uint32_t>(istep) * 32u + lane < row_words) {
                c = __ldg(wp);
                sc = __ldg(sp);
            }
            wp += 32;            // the next 1024 K-elements of the row
            sp += 16 * 512 / 2;  // 64 scale blocks = 16 scale tiles of 512 bytes further
            if (++istep == steps) {
                istep = 0;
                if (++irow < my_rows) row_start();
            }
        }
    };
#pragma unroll
    for (int u = 0; u < kRing; ++u) issue(ring[u], sring[u]);

    griddep_wait();            // the tokens come from the preceding kernel
    griddep_launch_dependents();

    // ---- quantize the tokens (tensor amax over all of them, then 16-blocks)
    const uint32_t n_vec = kM * K / 8u;
    uint32_t mx = 0;
    for (uint32_t i = threadIdx.x; i < n_vec; i += kGThreads)
        mx = max(mx, absmax8_bits(__ldg(reinterpret_cast<const uint4 *>(p.x) + i)));
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (lane == 0) red[warp] = __uint_as_float(mx << 16);
    __syncthreads();
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kGWarps; ++i) amax = fmaxf(amax, red[i]);
    const float s_enc_x = nvfp4_tensor_scale(amax);
    nvfp4_scale_table(s_enc_x, ftab);
    __syncthreads();
    const uint32_t xs0 = static_cast<uint32_t>(__cvta_generic_to_shared(xs_raw));
    const uint32_t kblocks = K / 16u;
    for (uint32_t b = threadIdx.x; b < kM * kblocks; b += kGThreads) {
        const uint32_t t = b / kblocks, kb = b - t * kblocks;
        const uint4 *src = reinterpret_cast<const uint4 *>(p.x) + (t * K + kb * 16u) / 8u;
        const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
        const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t lo, hi, sb;
        quantize_block16<false>(w8, s_enc_x, ftab, lo, hi, sb);
        uint32_t h0[4], h1[4];
        const uint32_t s2 = scale_pair(sb);
        dequant8(lo, s2, h0);
        dequant8(hi, s2, h1);
        // block kb = elements 16 kb ..: step kb / 64, lane (kb % 64) / 2,
        // 16-byte chunks 2 (kb % 2) and 2 (kb % 2) + 1 of that lane's 64 bytes
        const uint32_t step = kb / 64u, ln = (kb % 64u) / 2u, j0 = (kb % 2u) * 2u;
        const uint32_t base = xs0 + t * static_cast<uint32_t>(steps) * 2048u + step * 2048u;
        st_shared_v4_(base + ((j0 * 32u + ln) * 16u), h0);
        st_shared_v4_(base + (((j0 + 1u) * 32u + ln) * 16u), h1);
    }
    __syncthreads();
    const float alpha = __frcp_rn(__fmul_rn(s_enc_x, *p.s_enc_w));

    // ---- the stream: consume the oldest step, issue the one kRing ahead
    float acc[kM][2];
#pragma unroll
    for (int t = 0; t < kM; ++t) acc[t][0] = acc[t][1] = 0.0f;
    int crow = 0, cstep = 0;
    for (int s = 0; s < total; s += kRing) {
#pragma unroll
        for (int u = 0; u < kRing; ++u) {
            if (s + u < total) {       // warp-uniform
                const uint32_t word = static_cast<uint32_t>(cstep) * 32u + lane;
                if (word < row_words) {
                    // the two blocks' sums of e2m1(w) x deq(x) (exact products,
                    // FP32 sums), then each times its E4M3 scale
                    const float sc_lo = e4m3_to_float(sring[u] & 0xFFu);
                    const float sc_hi = e4m3_to_float(sring[u] >> 8);
                    const uint32_t cw[4] = {ring[u].x, ring[u].y, ring[u].z, ring[u].w};
                    const uint32_t xb = xs0 + static_cast<uint32_t>(cstep) * 2048u + lane * 16u;
                    float bs[kM][2][2];
#pragma unroll
                    for (int t = 0; t < kM; ++t) bs[t][0][0] = bs[t][0][1] = bs[t][1][0] = bs[t][1][1] = 0.0f;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t wd[4];
                        e2m1x8_f16(cw[q], wd);
#pragma unroll
                        for (int t = 0; t < kM; ++t) {
                            uint32_t xv[4];
                            ld_shared_v4(xb + t * static_cast<uint32_t>(steps) * 2048u + q * 512u, xv);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                fma2_f16_f32(wd[e], xv[e], bs[t][q >> 1][0], bs[t][q >> 1][1]);
                        }
                    }
#pragma unroll
                    for (int t = 0; t < kM; ++t) {
                        acc[t][0] = fmaf(bs[t][0][0] + bs[t][0][1], sc_lo, acc[t][0]);
                        acc[t][1] = fmaf(bs[t][1][0] + bs[t][1][1], sc_hi, acc[t][1]);
                    }
                }
                issue(ring[u], sring[u]);
                if (++cstep == steps) {
                    // the row is complete: reduce over the warp and store
                    const int r = gw + crow * nw;
#pragma unroll
                    for (int t = 0; t < kM; ++t) {
                        float v = acc[t][0] + acc[t][1];
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                        if (lane == 0)
                            p.y[static_cast<int64_t>(t) * p.N + r] = __float2bfloat16_rn(__fmul_rn(v, alpha));
                        acc[t][0] = acc[t][1] = 0.0f;
                    }
                    cstep = 0;
                    ++crow;
                }
            }
        }
    }
}

template <int kM>
cudaError_t launch_gemv(const GemvParams &p, int num_sms, cudaStream_t s) {
    const size_t smem = static_cast<size_t>(kM) * p.steps * 2048u;
    cudaError_t e = cudaFuncSetAttribute(decode_nvf4_gemv_kernel<kM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    // two resident CTAs per SM, or one warp per weight row when there are fewer
    int grid = 2 * num_sms;
    if (grid * kGWarps > p.N) grid = (p.N + kGWarps - 1) / kGWarps;
    if (grid < 1) grid = 1;
    return launch_pdl(decode_nvf4_gemv_kernel<kM>, dim3(grid), dim3(kGThreads), smem, s, p);
}

}  // namespace

bool decode_nvf4_gemv_fits(int64_t M, int64_t K) {
    return M >= 1 && M <= 4 && static_cast<int64_t>(M) * ((K + kStepElems - 1) / kStepElems) * 2048 <=
                                   kDecodeGemvTokenSmem;
}

cudaError_t launch_decode_nvf4_gemv(const uint8_t *w_codes, const uint8_t *w_sf, const float *s_enc_w,
                                    int64_t N, int64_t K, const void *x_bf16, int64_t M, void *y,
                                    int num_sms, cudaStream_t s) {
    GemvParams p;
    p.w = reinterpret_cast<const uint4 *>(w_codes);
    p.w_sf = w_sf;
    p.s_enc_w = s_enc_w;
    p.x = static_cast<const __nv_bfloat16 *>(x_bf16);
    p.y = static_cast<__nv_bfloat16 *>(y);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.steps = static_cast<int>((K + kStepElems - 1) / kStepElems);
    switch (M) {
        case 1: return launch_gemv<1>(p, num_sms, s);
        case 2: return launch_gemv<2>(p, num_sms, s);
        case 3: return launch_gemv<3>(p, num_sms, s);
        default: return launch_gemv<4>(p, num_sms, s);
    }
}

}  // namespace mq
