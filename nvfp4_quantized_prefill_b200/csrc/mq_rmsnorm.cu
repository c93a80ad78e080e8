// mq_rmsnorm.cu -- RMSNorm in front of a prefill linear, emitting the amax of
// its output for the NVFP4 quantizer.
//
// Method: Mix-Quant converts activations to NVFP4 at the phase boundary
// (zingnex.cn forum thread, section "动态精度切换"), with one tensor-level
// scale from the tensor's absolute maximum (gist.science technical summary,
// section 2 "Hybrid Precision Strategy").  In a transformer layer the QKV and
// gate/up inputs come out of an RMSNorm, so the kernel that writes them can
// take that maximum on the way out -- the quantizer then skips its own pass
// over the activations.  RMSNorm (the pages do not define it; the Llama
// family's is used):
//   r   = RN(1 / sqrt(RN(sum_k x_k^2 / K) + eps))   (binary32)
//   t_k = bf16_RNE(x_k * r),  y_k = bf16_RNE(gamma_k * t_k).
// The sum of squares is taken in binary32 in a fixed order (lane-strided
// partial sums, then a butterfly), so the result is deterministic; it can
// differ from the binary64 definition by an ulp of r, which moves a t_k by
// one BF16 step in rare cases.
//
// Rows of up to 8192 elements: a CTA per row, the row held in registers
// (2-4 vectors a thread) with the next rows in flight; longer rows: one warp
// per row, persistent over rows, a first pass over the row's 16-byte vectors
// summing the squares and a second reading the row again (L1 / L2).  Either
// writes y, keeps max|y| and writes one partial maximum per CTA.
#include <cuda_bf16.h>

#include "mq_internal.h"

namespace mq {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ float lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// y pair from an x pair and a gamma pair: bf16(gamma * bf16(x * r)) each half;
// returns the packed BF16 pair.
__device__ __forceinline__ uint32_t norm_pair(uint32_t xw, uint32_t gw, float r) {
    const float t0 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(lo_f(xw), r)));
    const float t1 = __bfloat162float(__float2bfloat16_rn(__fmul_rn(hi_f(xw), r)));
    const __nv_bfloat162 y = __floats2bfloat162_rn(__fmul_rn(lo_f(gw), t0), __fmul_rn(hi_f(gw), t1));
    return *reinterpret_cast<const uint32_t *>(&y);
}

__global__ void __launch_bounds__(kThreads) rmsnorm_amax_kernel(
    const uint4 *__restrict__ x, uint32_t M, uint32_t vpr, uint64_t ldv,
    const uint4 *__restrict__ gamma, float eps, uint4 *__restrict__ y,
    float *__restrict__ partials) {
    __shared__ float red[kWarps];
    griddep_wait();
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t nwarps = gridDim.x * kWarps;
    const float kf = static_cast<float>(vpr * 8u);
    uint32_t mx = 0;  // max |y| as BF16 magnitude bits
    auto sumsq = [&](const uint4 &q, float ss) {
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            ss = __fmaf_rn(lo_f(w[j]), lo_f(w[j]), ss);
            ss = __fmaf_rn(hi_f(w[j]), hi_f(w[j]), ss);
        }
        return ss;
    };
    // writes the y vector, returns its max |y| as BF16 magnitude bits
    auto emit = [&](const uint4 &q, uint32_t v, float r, uint4 *yr) -> uint32_t {
        const uint4 g = __ldg(gamma + v);
        uint4 o;
        o.x = norm_pair(q.x, g.x, r);
        o.y = norm_pair(q.y, g.y, r);
        o.z = norm_pair(q.z, g.z, r);
        o.w = norm_pair(q.w, g.w, r);
        yr[v] = o;
        const uint32_t m4 = 0x7FFF7FFFu;
        uint32_t a = __vmaxu2(__vmaxu2(o.x & m4, o.y & m4), __vmaxu2(o.z & m4, o.w & m4));
        a = __vmaxu2(a, a >> 16);
        return a & 0xFFFFu;
    };
    for (uint32_t row = blockIdx.x * kWarps + warp; row < M; row += nwarps) {
        const uint4 *xr = x + row * ldv;
        uint4 *yr = y + static_cast<uint64_t>(row) * vpr;
        float ss = 0.0f;
#pragma unroll 8
        for (uint32_t v = lane; v < vpr; v += 32) ss = sumsq(__ldg(xr + v), ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
        const float r = __frsqrt_rn(__fadd_rn(__fdiv_rn(ss, kf), eps));
#pragma unroll 4
        for (uint32_t v = lane; v < vpr; v += 32) mx = max(mx, emit(__ldg(xr + v), v, r, yr));
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (lane == 0) red[warp] = __uint_as_float(mx << 16);
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.0f;
        for (int i = 0; i < kWarps; ++i) m = fmaxf(m, red[i]);
        partials[blockIdx.x] = m;
    }
}

// A CTA per row, for rows of up to kThreads x 4 16-byte vectors (K <= 8192):
// each thread holds its V vectors of the row in registers between the sum of
// squares and the normalisation, keeps its gamma vectors in registers for
// every row, and has the next D rows of its CTA in flight while it works on
// the current one (V x D = 4 vectors, 64 bytes a thread).  The sum of squares
// is taken in a fixed order (a thread's vectors, a warp butterfly, the 8 warp
// sums in order), so the result is deterministic; one __syncthreads per row
// (the warp sums alternate between two buffers).
template <int V, int D, int kMinBlocks>
__global__ void __launch_bounds__(kThreads, kMinBlocks) rmsnorm_amax_rows_kernel(
    const uint4 *__restrict__ x, uint32_t M, uint32_t vpr, uint64_t ldv,
    const uint4 *__restrict__ gamma, float eps, uint4 *__restrict__ y,
    float *__restrict__ partials) {
    __shared__ float wsum[2][kWarps];
    __shared__ float red[kWarps];
    griddep_wait();
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float kf = static_cast<float>(vpr * 8u);
    const uint4 z = make_uint4(0, 0, 0, 0);
    uint4 g[V], buf[D + 1][V];
#pragma unroll
    for (int j = 0; j < V; ++j) {
        const uint32_t v = threadIdx.x + j * kThreads;
        g[j] = v < vpr ? __ldg(gamma + v) : z;
    }
    auto load_row = [&](uint32_t r, uint4 (&d)[V]) {
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint32_t v = threadIdx.x + j * kThreads;
            d[j] = (r < M && v < vpr) ? __ldg(x + static_cast<uint64_t>(r) * ldv + v) : z;
        }
    };
    uint32_t row = blockIdx.x;
#pragma unroll
    for (int d = 0; d < D; ++d) load_row(row + d * gridDim.x, buf[d]);
    uint32_t mx = 0;   // max |y| as BF16 magnitude bits
    for (int it = 0; row < M; ++it, row += gridDim.x) {
        load_row(row + D * gridDim.x, buf[D]);   // D rows ahead
        float ss = 0.0f;
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint32_t w[4] = {buf[0][j].x, buf[0][j].y, buf[0][j].z, buf[0][j].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                ss = __fmaf_rn(lo_f(w[k]), lo_f(w[k]), ss);
                ss = __fmaf_rn(hi_f(w[k]), hi_f(w[k]), ss);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xFFFFFFFFu, ss, o));
        if (lane == 0) wsum[it & 1][warp] = ss;
        __syncthreads();
        float tot = 0.0f;
#pragma unroll
        for (int i = 0; i < kWarps; ++i) tot = __fadd_rn(tot, wsum[it & 1][i]);
        const float r = __frsqrt_rn(__fadd_rn(__fdiv_rn(tot, kf), eps));
        uint4 *yr = y + static_cast<uint64_t>(row) * vpr;
#pragma unroll
        for (int j = 0; j < V; ++j) {
            const uint32_t v = threadIdx.x + j * kThreads;
            if (v < vpr) {
                uint4 o;
                o.x = norm_pair(buf[0][j].x, g[j].x, r);
                o.y = norm_pair(buf[0][j].y, g[j].y, r);
                o.z = norm_pair(buf[0][j].z, g[j].z, r);
                o.w = norm_pair(buf[0][j].w, g[j].w, r);
                yr[v] = o;
                const uint32_t m4 = 0x7FFF7FFFu;
                uint32_t a = __vmaxu2(__vmaxu2(o.x & m4, o.y & m4), __vmaxu2(o.z & m4, o.w & m4));
                a = __vmaxu2(a, a >> 16);
                mx = max(mx, a & 0xFFFFu);
            }
        }
#pragma unroll
        for (int d = 0; d < D; ++d)
#pragma unroll
            for (int j = 0; j < V; ++j) buf[d][j] = buf[d + 1][j];
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (lane == 0) red[warp] = __uint_as_float(mx << 16);
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.0f;
        for (int i = 0; i < kWarps; ++i) m = fmaxf(m, red[i]);
        partials[blockIdx.x] = m;
    }
}

}  // namespace

int rmsnorm_grid(int64_t M, int64_t K, int num_sms) {
    int64_t g;
    if (K / 8 <= 4LL * kThreads) {
        g = M;   // a CTA per row, persistent: one wave (4 or 3 resident CTAs per SM)
        const int64_t cap = (K / 8 <= 2LL * kThreads ? 4LL : 3LL) * num_sms;
        if (g > cap) g = cap;
    } else {
        g = (M + kWarps - 1) / kWarps;   // a warp per row
        const int64_t cap = 4LL * num_sms;   // (8 per SM measured slower)
        if (g > cap) g = cap;
    }
    if (g < 1) g = 1;
    return static_cast<int>(g);
}

cudaError_t launch_rmsnorm_amax(const void *x, int64_t M, int64_t K, int64_t ldx, const void *gamma,
                                float eps, void *y, float *partials, int grid, cudaStream_t s) {
    const int64_t vpr = K / 8;
    auto kernel = vpr <= 2LL * kThreads   ? rmsnorm_amax_rows_kernel<2, 2, 4>
                  : vpr <= 4LL * kThreads ? rmsnorm_amax_rows_kernel<4, 1, 3>
                                          : rmsnorm_amax_kernel;
    return launch_pdl(kernel, dim3(grid), dim3(kThreads), 0, s,
                      static_cast<const uint4 *>(x), static_cast<uint32_t>(M),
                      static_cast<uint32_t>(vpr), static_cast<uint64_t>(ldx / 8),
                      static_cast<const uint4 *>(gamma), eps, static_cast<uint4 *>(y), partials);
}

}  // namespace mq
