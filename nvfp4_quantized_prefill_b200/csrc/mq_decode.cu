// mq_decode.cu -- BF16 decode linear Y = X * W^T for a handful of tokens.
//
// Method: Mix-Quant keeps decoding in BF16 on the original weights
// (gist.science technical summary, section 2 "Hybrid Precision Strategy");
// the same weight handle that feeds the NVFP4 prefill GEMM keeps a BF16 copy
// for this path, so the phase switch costs nothing.
//
// The op is bound by streaming W from HBM once (2 N K bytes).  Work unit: 16
// rows of W x one K slice.  A CTA (8 warps) owns one unit and its warps split
// the slice; per step a warp reads 64 contiguous bytes of each of its 16 rows
// (16-byte vector loads) plus the matching 64 bytes of each X row and feeds
// two m16n8k16 BF16 MMAs (FP32 accumulate) with W rows as the M dimension and
// up to 8 X rows as N.  Both fragments take the same K permutation (the 8
// elements a thread loads), so no shuffles or staging are needed; for 8 tokens
// the tensor core does the 8 FMAs per weight element that would otherwise
// load the FP32 pipes.  A CTA's unit is 16 whole consecutive rows when there
// are enough row groups (one contiguous block of W).  The weight loads of
// eight steps are issued together, before their MMAs (8 KB in flight per
// warp).  With fewer row groups than SMs, K is split into S slices so that
// every SM gets two to three CTAs, all resident at once (the register budget
// allows three per SM); the last CTA of a row group to finish (an atomic
// counter, reset by that CTA) adds the S partial sums in slice order --
// deterministically -- and writes BF16.
// Scratch (per weight): one counter per row group first, then the partial
// sums.
#include <cuda_bf16.h>

#include "mq_internal.h"

namespace mq {

namespace {

constexpr int kWarps = 8;
constexpr int kRows = 16;
constexpr int kUnroll = 8;
constexpr int kCtasPerSm = 3;   // register budget: the grid of a split K is resident at once

// W is streamed once: the loads are issued as written (all of a batch before
// its MMAs), not sunk towards their use.
__device__ __forceinline__ uint4 ld_w(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32"
        " {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kWarps * 32, kCtasPerSm)
    decode_kernel(const uint4 *__restrict__ x, int M, const uint4 *__restrict__ w, int N, int K,
                  int S, __nv_bfloat16 *__restrict__ y, float *__restrict__ partials,
                  unsigned *__restrict__ counters) {
    __shared__ float part[kWarps][128];
    __shared__ int last;
    griddep_wait();
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int group = blockIdx.x / S, slice = blockIdx.x - group * S;
    const int n0 = group * kRows;
    const int vpr = K / 8;                       // 16-byte vectors per row
    const int steps = K / 32;                    // 32 K-elements per step (2 MMAs)
    const int sl0 = static_cast<int>(static_cast<int64_t>(steps) * slice / S);
    const int sl1 = static_cast<int>(static_cast<int64_t>(steps) * (slice + 1) / S);
    const int s0 = sl0 + (sl1 - sl0) * warp / kWarps;
    const int s1 = sl0 + (sl1 - sl0) * (warp + 1) / kWarps;
    // rows past N read row N - 1 and tokens past M read token 0: those
    // accumulator entries are never written out
    const int ra = n0 + g < N ? n0 + g : N - 1, rb = n0 + g + 8 < N ? n0 + g + 8 : N - 1;
    const uint4 *wa = w + static_cast<int64_t>(ra) * vpr + t4;
    const uint4 *wb = w + static_cast<int64_t>(rb) * vpr + t4;
    const uint4 *xr = x + static_cast<int64_t>(g < M ? g : 0) * vpr + t4;
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    int s = s0;
    for (; s + kUnroll <= s1; s += kUnroll) {
        uint4 va[kUnroll], vb[kUnroll], vx[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            va[u] = ld_w(wa + (s + u) * 4);
            vb[u] = ld_w(wb + (s + u) * 4);
            vx[u] = __ldg(xr + (s + u) * 4);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            mma_bf16_16816(c, va[u].x, vb[u].x, va[u].y, vb[u].y, vx[u].x, vx[u].y);
            mma_bf16_16816(c, va[u].z, vb[u].z, va[u].w, vb[u].w, vx[u].z, vx[u].w);
        }
    }
    for (; s < s1; ++s) {
        const uint4 va = ld_w(wa + s * 4);
        const uint4 vb = ld_w(wb + s * 4);
        const uint4 vx = __ldg(xr + s * 4);
        mma_bf16_16816(c, va.x, vb.x, va.y, vb.y, vx.x, vx.y);
        mma_bf16_16816(c, va.z, vb.z, va.w, vb.w, vx.z, vx.w);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) part[warp][lane * 4 + i] = c[i];
    __syncthreads();
    // accumulator element q = 4 * lane' + i': W row g' (+8 for i' >= 2), X row 2 t4' + (i' & 1)
    const int q = threadIdx.x;  // one accumulator element per thread (first 128)
    if (q >= 128) return;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) acc += part[i][q];
    const int lq = q >> 2, iq = q & 3;
    const int wrow = n0 + (lq >> 2) + ((iq >> 1) << 3);
    const int m = 2 * (lq & 3) + (iq & 1);
    if (S == 1) {
        if (m < M && wrow < N) y[static_cast<int64_t>(m) * N + wrow] = __float2bfloat16_rn(acc);
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
    if (m < M && wrow < N) y[static_cast<int64_t>(m) * N + wrow] = __float2bfloat16_rn(sum);
    if (threadIdx.x == 0) counters[group] = 0u;  // ready for the next call
}

}  // namespace

int decode_slices(int64_t N, int64_t K, int num_sms) {
    const int64_t groups = (N + kRows - 1) / kRows;
    if (groups >= num_sms) return 1;   // whole rows: no partial sums, one block of W a CTA
    int64_t S = (2LL * num_sms + groups - 1) / groups;   // >= 2 CTAs per SM
    const int64_t max_s = K / 512 > 0 ? K / 512 : 1;     // keep >= 16 steps per slice
    if (S > max_s) S = max_s;
    if (S > 16) S = 16;
    if (S < 1) S = 1;
    return static_cast<int>(S);
}

size_t decode_counter_bytes(int64_t N) {
    const int64_t groups = (N + kRows - 1) / kRows;
    return (static_cast<size_t>(groups) * sizeof(unsigned) + 255) / 256 * 256;
}

size_t decode_scratch_bytes(int64_t N, int64_t K, int num_sms) {
    int S = decode_slices(N, K, num_sms);
    const int S4 = decode_nvf4_slices(N, K, num_sms);
    if (S4 > S) S = S4;
    const int64_t groups = (N + kRows - 1) / kRows;
    size_t floats = static_cast<size_t>(groups) * S * 128;
    const size_t tc = decode_tc_partial_floats(N, K, num_sms);
    if (tc > floats) floats = tc;
    return decode_counter_bytes(N) + floats * sizeof(float);
}

cudaError_t launch_decode(const void *x, int64_t M, const void *w, int64_t N, int64_t K, void *y,
                          void *scratch, int num_sms, cudaStream_t s) {
    const int S = decode_slices(N, K, num_sms);
    const int64_t groups = (N + kRows - 1) / kRows;
    unsigned *counters = static_cast<unsigned *>(scratch);
    float *partials = reinterpret_cast<float *>(static_cast<uint8_t *>(scratch) +
                                                decode_counter_bytes(N));
    const int grid = static_cast<int>(groups * S);
    for (int64_t m0 = 0; m0 < M; m0 += 8) {
        const int mg = static_cast<int>(M - m0 < 8 ? M - m0 : 8);
        cudaError_t e = launch_pdl(
            decode_kernel, dim3(grid), dim3(kWarps * 32), 0, s,
            static_cast<const uint4 *>(x) + m0 * (K / 8), mg, static_cast<const uint4 *>(w),
            static_cast<int>(N), static_cast<int>(K), S, static_cast<__nv_bfloat16 *>(y) + m0 * N,
            partials, counters);
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace mq
