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
#include "mq_nvfp4.cuh"

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
    // total < 2^32 - 1 (checked on the host); the loop steps only while the
    // next start is still below total, so no index ever wraps around 2^32
    const uint32_t total = M * vpr;
    const uint32_t stride = gridDim.x * kThreads;
    const uint32_t step = kAmaxUnroll * stride;
    const bool dense = ldv == vpr;
    uint32_t mx = 0;
    for (uint32_t i = blockIdx.x * kThreads + threadIdx.x; i < total;
         i = (total - i > step) ? i + step : total) {
        uint4 v[kAmaxUnroll];
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) {
            // idx is used only when it is below total (no wrap-around)
            const uint32_t idx = i + u * stride;
            v[u] = make_uint4(0, 0, 0, 0);
            if (total - i > static_cast<uint32_t>(u) * stride) {
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

// Byte offset of the 4 scales (r, 4*cq .. 4*cq+3) in the swizzled layout.
__device__ __forceinline__ uint64_t sf_word_offset(uint32_t r, uint32_t cq, uint32_t ctiles) {
    return (static_cast<uint64_t>(r >> 7) * ctiles + cq) * 512u + (r & 31u) * 16u +
           ((r >> 5) & 3u) * 4u;
}

constexpr int kQuantUnroll = MQ_QUANT_UNROLL;
constexpr int kQuantBlocksPerSm = MQ_QUANT_BLOCKS_PER_SM;

// Each warp quantizes 512-element row segments (lane l: 16-block l of the
// segment, two 16-byte loads), kQuantUnroll segments per iteration with all
// loads issued first; segments are taken from the last one backwards.  Each
// lane stores its own scale byte (lanes 4t..4t+3 fill one swizzled 32-bit
// scale word).  Issuing the first iteration's loads ahead of the CTA's
// prologue (partial maxima, scale table) measured 15% slower.
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
    const float s_enc = nvfp4_tensor_scale(amax);
    if (blockIdx.x == 0 && threadIdx.x == 0) *s_enc_out = s_enc;
    nvfp4_scale_table(s_enc, ftab);
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
            quantize_block16<true>(w[u], s_enc, ftab, lo, hi, sb);
            if (act[u]) {
                codes[static_cast<uint64_t>(rr[u]) * kblocks + bb[u]] = make_uint2(lo, hi);
                // byte (bb & 3) of the swizzled scale word; the four bytes of
                // a word come from lanes 4t .. 4t+3 and merge in L2
                sf[sf_word_offset(rr[u], bb[u] / 4u, ctiles) + (bb[u] & 3u)] = static_cast<uint8_t>(sb);
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

// max(partials[0 .. n)) into out[0]: the tensor amax as one float, e.g. to be
// combined across token shards (max is exact and order-free).
__global__ void __launch_bounds__(kThreads) amax_combine_kernel(const float *__restrict__ partials,
                                                                int n, float *__restrict__ out) {
    __shared__ float red[kThreads / 32];
    griddep_wait();
    griddep_launch_dependents();
    float m = 0.0f;
    for (int i = threadIdx.x; i < n; i += kThreads) m = fmaxf(m, partials[i]);
    m = block_max(m, red);
    if (threadIdx.x == 0) out[0] = m;
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
    // one resident wave: every CTA pays the scale-table prologue once (the
    // occupancy is a property of the kernel on sm_100; computed once,
    // thread-safely)
    static const int resident = []() {
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, quantize_kernel, kThreads, 0) !=
                cudaSuccess ||
            b < 1)
            b = 1;
        return b;
    }();
    const int64_t segs = M * ((K + 511) / 512);
    int64_t g = (segs + (kThreads / 32) - 1) / (kThreads / 32);
    const int64_t cap = static_cast<int64_t>(resident) * num_sms;
    if (g > cap) g = cap;
    const int64_t Mpad = (M + 127) / 128 * 128;
    // enough CTAs for the padding rows' scale words too (about 8 per thread):
    // a handful of tokens would otherwise leave ~8000 words to one CTA
    const int64_t gpad = ((Mpad - M) * (K / 64) + kThreads * 8 - 1) / (kThreads * 8);
    if (g < gpad) g = gpad < cap ? gpad : cap;
    if (g < 1) g = 1;
    return launch_pdl(quantize_kernel, dim3(static_cast<unsigned>(g)), dim3(kThreads), 0, s,
                      static_cast<const uint4 *>(x), static_cast<uint32_t>(M),
                      static_cast<uint32_t>(K), static_cast<uint64_t>(ldx / 8), partials,
                      n_partials, reinterpret_cast<uint2 *>(codes), sf_swizzled, s_enc,
                      static_cast<uint32_t>(Mpad));
}

cudaError_t launch_amax_combine(const float *partials, int n, float *out, cudaStream_t s) {
    return launch_pdl(amax_combine_kernel, dim3(1), dim3(kThreads), 0, s, partials, n, out);
}

}  // namespace mq
