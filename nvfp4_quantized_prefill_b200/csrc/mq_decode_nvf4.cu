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

// Four code bytes (8 E2M1 values, element 2j in the low nibble of byte j;
// read from memory) to four FP16x2 words, each multiplied by the block scale
// s (an FP16x2 pair).
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

// Byte offset of the scale of (row r, block 4 * step + t) minus 512 * step:
// the offset of step s is this + 512 s (one 512-byte scale tile per 64 K).
__device__ __forceinline__ uint32_t sf_row_base(uint32_t r, uint32_t t, uint32_t ctiles) {
    return (r >> 7) * ctiles * 512u + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + t;
}

struct Step {
    uint2 wa, wb, xv;       // code bytes: row g, row g + 8, token g
    uint32_t sa, sb, sx;    // their scale bytes
};

// x given as NVFP4 codes + swizzled scales (+ tensor scale) in global memory
// (more than 8 tokens, quantized by the quantize kernels first): one CTA of
// 8 warps per (16 weight rows, K slice) unit, the warps splitting the slice.
__global__ void __launch_bounds__(kWarps * 32) decode_nvf4_kernel(
    const uint8_t *__restrict__ xc, const uint8_t *__restrict__ xsf, uint32_t xrow0, int M,
    const float *__restrict__ s_enc_x, const uint8_t *__restrict__ wc,
    const uint8_t *__restrict__ wsf, const float *__restrict__ s_enc_w, int N, int K, int S,
    __nv_bfloat16 *__restrict__ y, float *__restrict__ partials, unsigned *__restrict__ counters) {
    __shared__ float part[kWarps][128];
    __shared__ int last;
    griddep_wait();
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int group = blockIdx.x / S, slice = blockIdx.x - group * S;
    const int n0 = group * kRows;
    const uint32_t rowb = static_cast<uint32_t>(K / 2);  // code bytes per row
    const uint32_t ctiles = static_cast<uint32_t>(K / 64);
    const int steps = K / 64;
    const int sl0 = static_cast<int>(static_cast<int64_t>(steps) * slice / S);
    const int sl1 = static_cast<int>(static_cast<int64_t>(steps) * (slice + 1) / S);
    const uint32_t nsl = static_cast<uint32_t>(sl1 - sl0);   // steps in this CTA's slice
    const int s0 = sl0 + static_cast<int>(nsl) * warp / kWarps;
    const int s1 = sl0 + static_cast<int>(nsl) * (warp + 1) / kWarps;
    const bool ra = n0 + g < N, rb = n0 + g + 8 < N, rx = g < M;
    const uint32_t rA = ra ? n0 + g : 0, rB = rb ? n0 + g + 8 : 0, rX = xrow0 + (rx ? g : 0);
    const uint8_t *pa = wc + static_cast<uint64_t>(rA) * rowb + 8 * t;
    const uint8_t *pb = wc + static_cast<uint64_t>(rB) * rowb + 8 * t;
    const uint8_t *wsa = wsf + sf_row_base(rA, t, ctiles);
    const uint8_t *wsb = wsf + sf_row_base(rB, t, ctiles);
    const uint8_t *px = xc + static_cast<uint64_t>(rX) * rowb + 8 * t;
    const uint8_t *pxs = xsf + sf_row_base(rX, t, ctiles);
    const uint2 z2 = make_uint2(0, 0);
    float c[4] = {0.f, 0.f, 0.f, 0.f};

    auto load = [&](int s, Step &d) {
        d.wa = ra ? __ldg(reinterpret_cast<const uint2 *>(pa + 32 * s)) : z2;
        d.wb = rb ? __ldg(reinterpret_cast<const uint2 *>(pb + 32 * s)) : z2;
        d.sa = ra ? __ldg(wsa + 512u * s) : 0u;
        d.sb = rb ? __ldg(wsb + 512u * s) : 0u;
        d.xv = rx ? __ldg(reinterpret_cast<const uint2 *>(px + 32 * s)) : z2;
        d.sx = rx ? __ldg(pxs + 512u * s) : 0u;
    };
    auto compute = [&](const Step &d) {
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
    const float alpha = __frcp_rn(__fmul_rn(*s_enc_x, *s_enc_w));
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

// Persistent form for M <= 8 tokens given in BF16: one CTA of kPWarps warps
// per SM takes the tokens' amax and quantizes all of x into shared memory once
// (codes [M][K / 2], scales [M][K / 16], the quantizer's block routine); then
// every warp owns whole work units -- 16 weight rows x one of S K-slices --
// taken with a stride of the total warp count, and accumulates a unit in
// registers.  A unit's 16 x 8 result goes straight to y when S = 1; else to
// partials[group][slice], and the last warp to finish a group (atomic counter,
// reset by that warp) adds the S slices in order.
constexpr int kPWarps = 24;
constexpr size_t kPersistMaxSmem = kDecodeNvf4TokenSmem;

__global__ void __launch_bounds__(kPWarps * 32, 1) decode_nvf4_persist_kernel(
    const __nv_bfloat16 *__restrict__ xb, int M, const uint8_t *__restrict__ wc,
    const uint8_t *__restrict__ wsf, const float *__restrict__ s_enc_w, int N, int K, int S,
    __nv_bfloat16 *__restrict__ y, float *__restrict__ partials, unsigned *__restrict__ counters) {
    extern __shared__ __align__(16) uint8_t xsm[];   // codes [M][K/2], then scales [M][K/16]
    __shared__ float ftab[128];
    __shared__ float red[kPWarps];
    __shared__ float s_enc_sh;
    griddep_wait();
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t rowb = static_cast<uint32_t>(K / 2);
    const uint32_t ctiles = static_cast<uint32_t>(K / 64);
    const uint32_t kblk = static_cast<uint32_t>(K / 16);
    // tensor amax of the tokens, the scale table, then all of x quantized
    {
        const uint32_t vecs = static_cast<uint32_t>(M) * static_cast<uint32_t>(K / 8);
        const uint4 *xv = reinterpret_cast<const uint4 *>(xb);
        uint32_t mx = 0;
        // 8 loads in flight per thread (X comes from L2 in every CTA)
        for (uint32_t i0 = threadIdx.x; i0 < vecs; i0 += 8u * kPWarps * 32) {
            uint4 v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t i = i0 + k * kPWarps * 32;
                v[k] = i < vecs ? __ldg(xv + i) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) mx = max(mx, absmax8_bits(v[k]));
        }
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        if (lane == 0) red[warp] = __uint_as_float(mx << 16);
        __syncthreads();
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < kPWarps; ++i) amax = fmaxf(amax, red[i]);
        const float s = nvfp4_tensor_scale(amax);
        nvfp4_scale_table(s, ftab);
        if (threadIdx.x == 0) s_enc_sh = s;   // read back below, after the barrier
        __syncthreads();
        const uint32_t nblk = static_cast<uint32_t>(M) * kblk;
        uint8_t *scl = xsm + static_cast<uint32_t>(M) * rowb;
        // four blocks' loads issued before their quantization
        for (uint32_t i0 = threadIdx.x; i0 < nblk; i0 += 4u * kPWarps * 32) {
            uint4 v[4][2];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t i = i0 + k * kPWarps * 32;
                v[k][0] = v[k][1] = make_uint4(0, 0, 0, 0);
                if (i < nblk) {
                    const uint4 *src = xv + static_cast<uint64_t>(i) * 2u;  // block i = 16 elements
                    v[k][0] = __ldg(src);
                    v[k][1] = __ldg(src + 1);
                }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t i = i0 + k * kPWarps * 32;
                if (i >= nblk) break;
                const uint32_t w8[8] = {v[k][0].x, v[k][0].y, v[k][0].z, v[k][0].w,
                                        v[k][1].x, v[k][1].y, v[k][1].z, v[k][1].w};
                uint32_t lo, hi, sb;
                quantize_block16<true>(w8, s, ftab, lo, hi, sb);
                *reinterpret_cast<uint2 *>(xsm + i * 8u) = make_uint2(lo, hi);
                scl[i] = static_cast<uint8_t>(sb);
            }
        }
        __syncthreads();
    }
    const float alpha = __frcp_rn(__fmul_rn(s_enc_sh, *s_enc_w));
    const bool rx = g < M;
    const uint32_t xg = static_cast<uint32_t>(rx ? g : 0);
    const uint8_t *px = xsm + xg * rowb + 8u * t;                                 // + 32 s
    const uint8_t *pxs = xsm + static_cast<uint32_t>(M) * rowb + xg * kblk + t;  // + 4 s
    const int steps = K / 64;
    const int groups = (N + kRows - 1) / kRows;
    const int units = groups * S;
    const int nwarps = gridDim.x * kPWarps;
    const uint2 z2 = make_uint2(0, 0);
    // units interleaved across CTAs first, so every SM gets work
    for (int u = warp * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x); u < units;
         u += nwarps) {
        const int group = u / S, slice = u - group * S;
        const int n0 = group * kRows;
        const int s0 = static_cast<int>(static_cast<int64_t>(steps) * slice / S);
        const int s1 = static_cast<int>(static_cast<int64_t>(steps) * (slice + 1) / S);
        const bool ra = n0 + g < N, rb = n0 + g + 8 < N;
        const uint32_t rA = ra ? n0 + g : 0, rB = rb ? n0 + g + 8 : 0;
        const uint8_t *pa = wc + static_cast<uint64_t>(rA) * rowb + 8 * t;
        const uint8_t *pb = wc + static_cast<uint64_t>(rB) * rowb + 8 * t;
        const uint8_t *wsa = wsf + sf_row_base(rA, t, ctiles);
        const uint8_t *wsb = wsf + sf_row_base(rB, t, ctiles);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        auto load = [&](int s, Step &d) {
            d.wa = ra ? __ldg(reinterpret_cast<const uint2 *>(pa + 32 * s)) : z2;
            d.wb = rb ? __ldg(reinterpret_cast<const uint2 *>(pb + 32 * s)) : z2;
            d.sa = ra ? __ldg(wsa + 512u * s) : 0u;
            d.sb = rb ? __ldg(wsb + 512u * s) : 0u;
            d.xv = rx ? *reinterpret_cast<const uint2 *>(px + 32 * s) : z2;
            d.sx = rx ? pxs[4 * s] : 0u;
        };
        auto compute = [&](const Step &d) {
            uint32_t a0[4], a1[4], b0[4], b1[4], x0[4], x1[4];
            const uint32_t fa = scale_f16x2(d.sa), fb = scale_f16x2(d.sb), fx = scale_f16x2(d.sx);
            dequant8(d.wa.x, fa, a0);
            dequant8(d.wa.y, fa, a1);
            dequant8(d.wb.x, fb, b0);
            dequant8(d.wb.y, fb, b1);
            dequant8(d.xv.x, fx, x0);
            dequant8(d.xv.y, fx, x1);
            mma_f16_16816(c, a0[0], b0[0], a0[1], b0[1], x0[0], x0[1]);
            mma_f16_16816(c, a0[2], b0[2], a0[3], b0[3], x0[2], x0[3]);
            mma_f16_16816(c, a1[0], b1[0], a1[1], b1[1], x1[0], x1[1]);
            mma_f16_16816(c, a1[2], b1[2], a1[3], b1[3], x1[2], x1[3]);
        };
        int s = s0;
        for (; s + kUnroll <= s1; s += kUnroll) {
            Step d[kUnroll];
#pragma unroll
            for (int v = 0; v < kUnroll; ++v) load(s + v, d[v]);
#pragma unroll
            for (int v = 0; v < kUnroll; ++v) compute(d[v]);
        }
        for (; s < s1; ++s) {
            Step d;
            load(s, d);
            compute(d);
        }
        // c[i]: W row g (+8 for i >= 2), token 2 t + (i & 1)
        if (S == 1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int wrow = n0 + g + ((i >> 1) << 3), m = 2 * t + (i & 1);
                if (m < M && wrow < N)
                    y[static_cast<int64_t>(m) * N + wrow] = __float2bfloat16_rn(__fmul_rn(alpha, c[i]));
            }
            continue;
        }
        float *mine = partials + (static_cast<int64_t>(group) * S + slice) * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) mine[lane * 4 + i] = c[i];
        __threadfence();
        __syncwarp();
        unsigned was = 0;
        if (lane == 0) was = atomicAdd(&counters[group], 1u);
        was = __shfl_sync(0xFFFFFFFFu, was, 0);
        if (was != static_cast<unsigned>(S - 1)) continue;
        __threadfence();
        float sum[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k = 0; k < S; ++k) {
            const float *pk = partials + (static_cast<int64_t>(group) * S + k) * 128 + lane * 4;
#pragma unroll
            for (int i = 0; i < 4; ++i) sum[i] += __ldcg(pk + i);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int wrow = n0 + g + ((i >> 1) << 3), m = 2 * t + (i & 1);
            if (m < M && wrow < N)
                y[static_cast<int64_t>(m) * N + wrow] = __float2bfloat16_rn(__fmul_rn(alpha, sum[i]));
        }
        if (lane == 0) counters[group] = 0u;  // ready for the next call
    }
}

}  // namespace

int decode_nvf4_slices(int64_t N, int64_t K, int num_sms) {
    // enough (16-row group, K slice) units for every warp of the persistent
    // grid (num_sms x 16 warps) to get about one, with >= 8 steps per slice
    const int64_t groups = (N + kRows - 1) / kRows;
    const int64_t target = static_cast<int64_t>(num_sms) * kPWarps;
    if (groups >= target) return 1;
    int64_t S = target / groups;   // at most one unit per warp
    const int64_t max_s = K / 512 > 0 ? K / 512 : 1;
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
    if (x_bf16) {  // M <= 8: tokens quantized in the kernel, persistent warps
        const size_t smem = static_cast<size_t>(M) * static_cast<size_t>(K) * 9u / 16u;  // K/2 + K/16
        if (smem > kPersistMaxSmem) return cudaErrorInvalidValue;
        // always the same (largest allowed) value: calls from several host
        // threads cannot undo each other's setting
        cudaError_t e = cudaFuncSetAttribute(decode_nvf4_persist_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kPersistMaxSmem));
        if (e != cudaSuccess) return e;
        const int64_t units = groups * S;
        const int64_t pgrid = units < num_sms ? units : num_sms;   // one CTA per SM
        e = launch_pdl(decode_nvf4_persist_kernel, dim3(static_cast<unsigned>(pgrid)),
                       dim3(kPWarps * 32), smem, s, static_cast<const __nv_bfloat16 *>(x_bf16),
                       static_cast<int>(M), w_codes, w_sf, s_enc_w, static_cast<int>(N),
                       static_cast<int>(K), S, static_cast<__nv_bfloat16 *>(y), partials, counters);
        return e == cudaSuccess ? cudaGetLastError() : e;
    }
    for (int64_t m0 = 0; m0 < M; m0 += 8) {
        const int mg = static_cast<int>(M - m0 < 8 ? M - m0 : 8);
        cudaError_t e = launch_pdl(decode_nvf4_kernel, dim3(grid), dim3(kWarps * 32), 0, s,
                                   x_codes, x_sf, static_cast<uint32_t>(m0), mg, s_enc_x, w_codes, w_sf,
                                   s_enc_w, static_cast<int>(N), static_cast<int>(K), S,
                                   static_cast<__nv_bfloat16 *>(y) + m0 * N, partials, counters);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace mq
