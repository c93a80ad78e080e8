// mq_attention.cu -- the attention of the prefill layer (causal, grouped KV
// heads, BF16 in, FP32 softmax and accumulation, BF16 out) on the sm_100a
// tcgen05 tensor cores, writing the BF16 KV cache that the decode step reads,
// and the decode step's attention over that cache.
//
// Method: Mix-Quant's prefill builds the KV cache that decoding then consumes
// (gist.science technical summary, section 2 "System-Level Deployment"; the
// zingnex.cn forum thread, section "动态精度切换", on the cache across the
// two precisions).  Here the prefill's projections run in NVFP4 and the
// attention in BF16; the cache is BF16 and the decode step keeps BF16
// throughout.  The pages do not define the attention; the Llama family's
// causal softmax attention with grouped KV heads is used, without positional
// rotation:  o_i = sum_{j <= i} softmax_j(q_i . k_j / sqrt(D)) v_j.
//
// Prefill kernel: one CTA per (128-query tile, query head), heaviest tiles
// first.  Warp 0 loads Q once and K / V tiles (TMA, 128-byte swizzle) into a
// 2-stage ring; warp 1 issues S = Q K^T (kind::f16, M = 128, N = 128, K = 16
// per instruction) into one of two 128-column FP32 buffers in tensor memory,
// and O += P V with P read from tensor memory; warps 2-5 (one query row per
// thread) take the row maximum, raise the running maximum only when it grows
// by more than 2^8 (then O is rescaled in place; otherwise the stale maximum
// keeps every weight below 2^8 and the final division by the same-based sum is
// exact), write P as BF16 over the S buffer, and finally divide O by the row
// sum, store it and keep max |o| for the O projection's quantizer.  The first
// query head of each KV group writes its diagonal K / V tile to the cache.
#include <cuda_bf16.h>

#include <cstring>

#include "mq_internal.h"
#include "mq_ptx.cuh"

namespace mq {

namespace {

constexpr int kD = 128;                   // head dimension
constexpr int kTile = 128;                // query rows per CTA, keys per KV tile
constexpr uint32_t kHalfBytes = kTile * 128;       // 128 rows x 64 BF16 (one swizzle atom column)
constexpr uint32_t kTileBytes = 2 * kHalfBytes;    // 128 rows x 128 BF16
constexpr int kStages = 2;
constexpr uint32_t kQOff = 0;
constexpr uint32_t kKOff = kTileBytes;                       // K stages
constexpr uint32_t kVOff = kKOff + kStages * kTileBytes;     // V stages
constexpr uint32_t kBarOff = kVOff + kStages * kTileBytes;
constexpr uint32_t kSmemBytes = kBarOff + 256 + 1024;
constexpr int kThreads = 192;             // producer, MMA, 4 softmax warps
constexpr uint32_t kTmemCols = 512;       // S0 [0,128), S1 [128,256), O [256,384)
constexpr uint32_t kOCol = 256;
// log2(e) / sqrt(128): scores in the base-2 exponent domain
constexpr float kScaleLog2 = 0.12751743082459868f;
constexpr float kRescaleThreshold = 8.0f;  // raise the running max past 2^8 growth only

struct PrefillParams {
    int M, H, Hkv, n_qt;
    int write_cache;          // 1: the group's first head writes K / V tiles to the cache
    __nv_bfloat16 *o;         // [M, H * 128]
    float *amax_partials;     // one per CTA, or atomically maxed slots (see below)
    int partial_slots;        // > 0: atomicMax into amax_partials[cta % slots]
    unsigned *err;
};

// Bounded wait on an mbarrier phase (all lanes poll); false after the limit.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_timer_ns() - t0 > kWaitLimitNs) return false;
    return true;
}

__global__ void __launch_bounds__(kThreads, 1)
    attention_prefill_kernel(const __grid_constant__ CUtensorMap tmap_qkv,
                             const __grid_constant__ CUtensorMap tmap_kc,
                             const __grid_constant__ CUtensorMap tmap_vc, const PrefillParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t s0 = smem_u32(smem);
    const uint32_t bar = s0 + kBarOff;
    const uint32_t q_full = bar;
    const uint32_t k_full = bar + 8;          // [2]
    const uint32_t v_full = bar + 24;         // [2]
    const uint32_t kv_empty = bar + 40;       // [2]
    const uint32_t s_full = bar + 56;         // [2]
    const uint32_t p_full = bar + 72;         // [2]
    const uint32_t o_done = bar + 88;
    const uint32_t drain = bar + 96;          // every MMA issued has completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kBarOff + 112);
    float *red = reinterpret_cast<float *>(smem + kBarOff + 128);   // 4 floats

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int group = p.H / p.Hkv;
    const int qt = p.n_qt - 1 - static_cast<int>(blockIdx.x) / p.H;   // heaviest first
    const int h = static_cast<int>(blockIdx.x) % p.H;
    const int g = h / group;
    const int nkv = qt + 1;                   // causal: KV tiles 0..qt
    const int qkv_cols_q = h * kD;
    const int qkv_cols_k = p.H * kD + g * kD;
    const int qkv_cols_v = (p.H + p.Hkv) * kD + g * kD;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(k_full + 8 * i, 1);
            mbar_init(v_full + 8 * i, 1);
            mbar_init(kv_empty + 8 * i, 1);
            mbar_init(s_full + 8 * i, 1);
            mbar_init(p_full + 8 * i, 4);     // one arrival per softmax warp
        }
        mbar_init(o_done, 1);
        mbar_init(drain, 1);
        fence_barrier_init();
        prefetch_tmap(&tmap_qkv);
        if (p.write_cache) {
            prefetch_tmap(&tmap_kc);
            prefetch_tmap(&tmap_vc);
        }
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_wait();            // qkv comes from the preceding kernel
    griddep_launch_dependents();
    bool ok = true;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, kTileBytes);
            tma_load_2d(s0 + kQOff, &tmap_qkv, qkv_cols_q, qt * kTile, q_full);
            tma_load_2d(s0 + kQOff + kHalfBytes, &tmap_qkv, qkv_cols_q + 64, qt * kTile, q_full);
            const bool writer = p.write_cache && (h % group) == 0;
            bool stored[kStages] = {false, false};
            for (int j = 0; j < nkv && ok; ++j) {
                const int st = j & 1;
                if (j >= kStages) {
                    if (!wait_bar(kv_empty + 8 * st, ((j - kStages) >> 1) & 1)) ok = false;
                    if (stored[st]) {
                        bulk_wait_group_read0();   // the cache store has read the stage
                        stored[st] = false;
                    }
                }
                const uint32_t ks = s0 + kKOff + st * kTileBytes;
                const uint32_t vs = s0 + kVOff + st * kTileBytes;
                mbar_arrive_expect_tx(k_full + 8 * st, kTileBytes);
                tma_load_2d(ks, &tmap_qkv, qkv_cols_k, j * kTile, k_full + 8 * st);
                tma_load_2d(ks + kHalfBytes, &tmap_qkv, qkv_cols_k + 64, j * kTile, k_full + 8 * st);
                mbar_arrive_expect_tx(v_full + 8 * st, kTileBytes);
                tma_load_2d(vs, &tmap_qkv, qkv_cols_v, j * kTile, v_full + 8 * st);
                tma_load_2d(vs + kHalfBytes, &tmap_qkv, qkv_cols_v + 64, j * kTile, v_full + 8 * st);
                if (writer && j == qt) {
                    // the diagonal tile: this head's group writes keys / values
                    // qt*128 .. to the cache (rows past M are clipped by S_max
                    // or rewritten by later decode steps)
                    if (!wait_bar(k_full + 8 * st, (j >> 1) & 1)) ok = false;
                    if (!wait_bar(v_full + 8 * st, (j >> 1) & 1)) ok = false;
                    tma_store_3d(&tmap_kc, 0, j * kTile, g, ks);
                    tma_store_3d(&tmap_kc, 64, j * kTile, g, ks + kHalfBytes);
                    tma_store_3d(&tmap_vc, 0, j * kTile, g, vs);
                    tma_store_3d(&tmap_vc, 64, j * kTile, g, vs + kHalfBytes);
                    bulk_commit_group();
                    stored[st] = true;
                }
            }
            // the loads of the last tile of each stage have landed (they have on
            // the normal path; after a timeout, before the CTA may exit)
            for (int j = nkv - 1; j >= 0 && j >= nkv - kStages; --j) {
                wait_bar(k_full + 8 * (j & 1), (j >> 1) & 1);
                wait_bar(v_full + 8 * (j & 1), (j >> 1) & 1);
            }
            bulk_wait_group0();   // cache stores complete before the CTA exits
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(128, 128, 0, 0);   // Q, K both K-major
            constexpr uint32_t idesc_o = idesc_bf16(128, 128, 0, 1);   // V MN-major
            if (!wait_bar(q_full, 0)) ok = false;
            tc_fence_after();
            for (int j = 0; j <= nkv && ok; ++j) {
                if (j < nkv) {
                    const int st = j & 1;
                    if (!wait_bar(k_full + 8 * st, (j >> 1) & 1)) ok = false;
                    // S buffer st last held P_{j-2}: its PV must have completed
                    if (j >= 2 && !wait_bar(o_done, (j - 2) & 1)) ok = false;
                    tc_fence_after();
                    const uint32_t ks = s0 + kKOff + st * kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32u;
                        tc_mma_bf16_ss(tmem + st * 128u, sdesc_kmajor_sw128(s0 + kQOff + off),
                                       sdesc_kmajor_sw128(ks + off), idesc_s, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(s_full + 8 * st);
                }
                if (j >= 1) {
                    const int jj = j - 1, st = jj & 1;
                    if (!wait_bar(p_full + 8 * st, (jj >> 1) & 1)) ok = false;
                    if (!wait_bar(v_full + 8 * st, (jj >> 1) & 1)) ok = false;
                    tc_fence_after();
                    const uint32_t vs = s0 + kVOff + st * kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk) {
                        // keys 16 kk .. 16 kk + 15: two 8-row groups of the V tile
                        tc_mma_bf16_ts(tmem + kOCol, tmem + st * 128u + kk * 8u,
                                       sdesc_mnmajor_sw128(vs + kk * 2048u, kHalfBytes), idesc_o,
                                       (jj > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(o_done);
                    tc_commit(kv_empty + 8 * st);
                }
            }
            // every MMA this thread issued completes before TMEM is freed
            tc_commit(drain);
            wait_bar(drain, 0);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- softmax
        const int quarter = warp & 3;             // TMEM lane group of this warp
        const int r = quarter * 32 + lane;        // query row in the tile
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        float m_run = -INFINITY, l = 0.0f;
        for (int j = 0; j < nkv && ok; ++j) {
            const int st = j & 1;
            ok = __all_sync(0xFFFFFFFFu, wait_bar(s_full + 8 * st, (j >> 1) & 1)) && ok;
            tc_fence_after();
            uint32_t sr[kTile];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_ld32(tmem + lane_off + st * 128u + c * 32u, *reinterpret_cast<uint32_t (*)[32]>(&sr[c * 32]));
            tmem_ld_wait();
            float s[kTile];
            float mx = -INFINITY;
            const bool diag = (j == qt);
#pragma unroll
            for (int c = 0; c < kTile; ++c) {
                float x = __uint_as_float(sr[c]) * kScaleLog2;
                if (diag && c > r) x = -INFINITY;
                s[c] = x;
                mx = fmaxf(mx, x);
            }
            // raise the running maximum only for a growth beyond 2^8 (or at
            // the first tile); O then needs the factor 2^(m_old - m_new)
            const bool need = mx > m_run + kRescaleThreshold;
            const float m_new = need ? mx : m_run;
            const float f = need ? exp2f(m_run - m_new) : 1.0f;   // 0 at the first tile
            if (__any_sync(0xFFFFFFFFu, need) && j > 0) {
                ok = __all_sync(0xFFFFFFFFu, wait_bar(o_done, (j - 1) & 1)) && ok;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(tmem + lane_off + kOCol + c * 32u, ov);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
                    tmem_st32(tmem + lane_off + kOCol + c * 32u, ov);
                }
                tmem_st_wait();
            }
            l *= f;
            m_run = m_new;
            uint32_t pk[kTile / 2];
#pragma unroll
            for (int c = 0; c < kTile / 2; ++c) {
                const __nv_bfloat162 pb =
                    __floats2bfloat162_rn(exp2f(s[2 * c] - m_run), exp2f(s[2 * c + 1] - m_run));
                // the row sum of the BF16 weights the PV product uses
                l += __bfloat162float(pb.x) + __bfloat162float(pb.y);
                pk[c] = *reinterpret_cast<const uint32_t *>(&pb);
            }
            tmem_st32(tmem + lane_off + st * 128u, *reinterpret_cast<uint32_t (*)[32]>(&pk[0]));
            tmem_st32(tmem + lane_off + st * 128u + 32u, *reinterpret_cast<uint32_t (*)[32]>(&pk[32]));
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full + 8 * st);
        }
        // epilogue: O / l -> BF16, and max |o| of the tile
        ok = __all_sync(0xFFFFFFFFu, wait_bar(o_done, (nkv - 1) & 1)) && ok;
        tc_fence_after();
        const float inv = 1.0f / l;
        const int row = qt * kTile + r;
        float omax = 0.0f;
        __nv_bfloat16 *orow = p.o + static_cast<int64_t>(row) * (p.H * kD) + h * kD;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t ov[32];
            tmem_ld32(tmem + lane_off + kOCol + c * 32u, ov);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(ov[2 * e]) * inv,
                                                               __uint_as_float(ov[2 * e + 1]) * inv);
                omax = fmaxf(omax, fmaxf(fabsf(__bfloat162float(b.x)), fabsf(__bfloat162float(b.y))));
                pk[e] = *reinterpret_cast<const uint32_t *>(&b);
            }
            if (row < p.M) {
                uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
            }
        }
        if (row >= p.M) omax = 0.0f;
        const uint32_t b = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(omax));
        if (lane == 0) red[warp - 2] = __uint_as_float(b);
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (warp == 2 && lane == 0) {
            const float m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
            if (p.partial_slots > 0)
                atomicMax(reinterpret_cast<unsigned *>(p.amax_partials) + blockIdx.x % p.partial_slots,
                          __float_as_uint(m));   // non-negative floats order like their bits
            else
                p.amax_partials[blockIdx.x] = m;
        }
    }
    if (!__all_sync(0xFFFFFFFFu, ok) && lane == 0) atomicOr(p.err, kDevErrTimeout);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                              const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                              const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
    static const EncodeFn fn = []() -> EncodeFn {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !ptr)
            return nullptr;
        return reinterpret_cast<EncodeFn>(ptr);
    }();
    return fn;
}

// ---------------------------------------------------------------------------
// Decode step: m new tokens at positions pos0 .. pos0 + m - 1.  Their K / V
// rows are appended to the cache, then each query attends over keys
// 0 .. pos0 + t of the cache.  Memory-bound (the cache is read once): the
// keys are split into 128-key chunks across CTAs (one CTA per chunk and KV
// head, all of the group's query rows at once), each CTA leaves (max, sum,
// unnormalised o) per query row, and a combine pass merges the chunks.
// FP32 throughout (scores, weights, accumulation); BF16 output.

constexpr int kDecChunk = 128;            // keys per CTA
constexpr int kDecThreads = 256;
constexpr int kDecMaxRows = 64;           // query rows per KV head (group size x tokens)
constexpr int kKPad = kD + 2;             // padded K row in shared memory (conflict-free dot products)
constexpr uint32_t kDecSmem = kDecChunk * kKPad * 2 + kDecChunk * kD * 2 +
                              kDecMaxRows * kD * 4 + kDecMaxRows * kDecChunk * 4;

struct DecodeParams {
    const __nv_bfloat16 *qkv;   // [m, (H + 2 Hkv) * 128]
    __nv_bfloat16 *k_cache;     // [Hkv, S_max, 128]
    __nv_bfloat16 *v_cache;
    __nv_bfloat16 *o;           // [m, H * 128]
    float *part;                // [Hkv, n_chunks, rows, 2 + 128]
    int m, pos0, H, Hkv, S_max, n_chunks, rows;
};

// Copies the new tokens' K and V rows into the cache (grid m x Hkv, 32 threads).
__global__ void __launch_bounds__(32) kv_append_kernel(const DecodeParams p) {
    griddep_wait();
    griddep_launch_dependents();
    const int t = blockIdx.x, g = blockIdx.y, lane = threadIdx.x;
    const int cols = (p.H + 2 * p.Hkv) * kD;
    const uint4 *src_k = reinterpret_cast<const uint4 *>(p.qkv + static_cast<int64_t>(t) * cols +
                                                         (p.H + g) * kD);
    const uint4 *src_v = reinterpret_cast<const uint4 *>(p.qkv + static_cast<int64_t>(t) * cols +
                                                         (p.H + p.Hkv + g) * kD);
    const int64_t dst = (static_cast<int64_t>(g) * p.S_max + p.pos0 + t) * kD;
    if (lane < 16)
        reinterpret_cast<uint4 *>(p.k_cache + dst)[lane] = src_k[lane];
    else
        reinterpret_cast<uint4 *>(p.v_cache + dst)[lane - 16] = src_v[lane - 16];
}

__global__ void __launch_bounds__(kDecThreads) attention_decode_kernel(const DecodeParams p) {
    extern __shared__ __align__(16) uint8_t dsm[];
    __nv_bfloat16 *ks = reinterpret_cast<__nv_bfloat16 *>(dsm);                       // [128][130]
    __nv_bfloat16 *vs = ks + kDecChunk * kKPad;                                          // [128][128]
    float *qs = reinterpret_cast<float *>(vs + kDecChunk * kD);                          // [rows][128]
    float *ss = qs + kDecMaxRows * kD;                                                   // [rows][128]
    const int c = blockIdx.x, g = blockIdx.y, tid = threadIdx.x;
    const int group = p.H / p.Hkv;
    const int n_keys = p.pos0 + p.m;
    const int key0 = c * kDecChunk;
    const int nk = min(kDecChunk, n_keys - key0);
    const int cols = (p.H + 2 * p.Hkv) * kD;
    griddep_wait();            // the appended rows and the queries are in place
    griddep_launch_dependents();
    // the chunk's keys and values (rows past the chunk read as zero)
    for (int i = tid; i < kDecChunk * (kD / 8); i += kDecThreads) {
        const int k = i / (kD / 8), d8 = (i % (kD / 8)) * 8;
        uint4 kv = make_uint4(0, 0, 0, 0), vv = kv;
        if (k < nk) {
            const int64_t off = (static_cast<int64_t>(g) * p.S_max + key0 + k) * kD + d8;
            kv = *reinterpret_cast<const uint4 *>(p.k_cache + off);
            vv = *reinterpret_cast<const uint4 *>(p.v_cache + off);
        }
        const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)   // the padded K rows are only 4-byte aligned
            *reinterpret_cast<uint32_t *>(ks + k * kKPad + d8 + 2 * e) = w[e];
        *reinterpret_cast<uint4 *>(vs + k * kD + d8) = vv;
    }
    // the group's query rows: row rr = hh * m + t (head g * group + hh, token t)
    for (int i = tid; i < p.rows * kD; i += kDecThreads) {
        const int rr = i / kD, d = i % kD, hh = rr / p.m, t = rr % p.m;
        qs[rr * kD + d] = __bfloat162float(p.qkv[static_cast<int64_t>(t) * cols + (g * group + hh) * kD + d]);
    }
    __syncthreads();
    // scores: thread -> one key, every other row
    {
        const int k = tid & (kDecChunk - 1), half = tid >> 7;
        float kr[kD];
#pragma unroll
        for (int d = 0; d < kD; d += 2) {
            const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(ks + k * kKPad + d);
            kr[d] = __bfloat162float(b.x);
            kr[d + 1] = __bfloat162float(b.y);
        }
        const int pos = key0 + k;
        for (int rr = half; rr < p.rows; rr += 2) {
            const float *q = qs + rr * kD;
            float acc = 0.0f;
#pragma unroll
            for (int d = 0; d < kD; d += 4) {
                const float4 qv = *reinterpret_cast<const float4 *>(q + d);
                acc = fmaf(qv.x, kr[d], acc);
                acc = fmaf(qv.y, kr[d + 1], acc);
                acc = fmaf(qv.z, kr[d + 2], acc);
                acc = fmaf(qv.w, kr[d + 3], acc);
            }
            const int t = rr % p.m;
            ss[rr * kDecChunk + k] = (k < nk && pos <= p.pos0 + t) ? acc * kScaleLog2 : -INFINITY;
        }
    }
    __syncthreads();
    // per row: chunk max, weights 2^(x - max), their sum (a warp per row)
    const int warp = tid >> 5, lane = tid & 31;
    float *part = p.part + (static_cast<int64_t>(g) * p.n_chunks + c) * p.rows * (2 + kD);
    for (int rr = warp; rr < p.rows; rr += kDecThreads / 32) {
        float x[4], mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            x[e] = ss[rr * kDecChunk + lane + 32 * e];
            mx = fmaxf(mx, x[e]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        float sum = 0.0f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float w = mx == -INFINITY ? 0.0f : exp2f(x[e] - mx);
            ss[rr * kDecChunk + lane + 32 * e] = w;
            sum += w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        if (lane == 0) {
            part[rr * (2 + kD)] = mx;
            part[rr * (2 + kD) + 1] = sum;
        }
    }
    __syncthreads();
    // unnormalised o: thread -> one dimension, every other row
    {
        const int d = tid & (kD - 1), half = tid >> 7;
        for (int rr = half; rr < p.rows; rr += 2) {
            const float *w = ss + rr * kDecChunk;
            float acc = 0.0f;
            for (int k = 0; k < nk; ++k) acc = fmaf(w[k], __bfloat162float(vs[k * kD + d]), acc);
            part[rr * (2 + kD) + 2 + d] = acc;
        }
    }
}

// Merges the chunks of one query row (a CTA of 128 threads, one per dimension).
__global__ void __launch_bounds__(kD) attention_combine_kernel(const DecodeParams p) {
    griddep_wait();
    griddep_launch_dependents();
    const int rr = blockIdx.x, g = blockIdx.y, d = threadIdx.x;
    const int group = p.H / p.Hkv, hh = rr / p.m, t = rr % p.m;
    const float *base = p.part + static_cast<int64_t>(g) * p.n_chunks * p.rows * (2 + kD) + rr * (2 + kD);
    const int64_t step = static_cast<int64_t>(p.rows) * (2 + kD);
    float mx = -INFINITY;
    for (int c = 0; c < p.n_chunks; ++c) mx = fmaxf(mx, base[c * step]);
    float l = 0.0f, acc = 0.0f;
    for (int c = 0; c < p.n_chunks; ++c) {
        const float mc = base[c * step];
        if (mc == -INFINITY) continue;   // no visible key in this chunk
        const float f = exp2f(mc - mx);
        l = fmaf(base[c * step + 1], f, l);
        acc = fmaf(base[c * step + 2 + d], f, acc);
    }
    p.o[static_cast<int64_t>(t) * (p.H * kD) + (g * group + hh) * kD + d] = __float2bfloat16_rn(acc / l);
}

}  // namespace

size_t attention_decode_workspace_bytes(int64_t m, int64_t pos0, int64_t H, int64_t Hkv) {
    const int64_t n_chunks = (pos0 + m + kDecChunk - 1) / kDecChunk;
    const int64_t rows = H / Hkv * m;
    return static_cast<size_t>(Hkv * n_chunks * rows * (2 + kD)) * sizeof(float);
}

int attention_decode_max_rows() { return kDecMaxRows; }

cudaError_t launch_attention_decode(const void *qkv, int64_t m, int64_t pos0, int64_t H, int64_t Hkv,
                                    void *k_cache, void *v_cache, int64_t S_max, void *o, void *ws,
                                    cudaStream_t s) {
    DecodeParams p;
    p.qkv = static_cast<const __nv_bfloat16 *>(qkv);
    p.k_cache = static_cast<__nv_bfloat16 *>(k_cache);
    p.v_cache = static_cast<__nv_bfloat16 *>(v_cache);
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.part = static_cast<float *>(ws);
    p.m = static_cast<int>(m);
    p.pos0 = static_cast<int>(pos0);
    p.H = static_cast<int>(H);
    p.Hkv = static_cast<int>(Hkv);
    p.S_max = static_cast<int>(S_max);
    p.n_chunks = static_cast<int>((pos0 + m + kDecChunk - 1) / kDecChunk);
    p.rows = static_cast<int>(H / Hkv * m);
    cudaError_t e = launch_pdl(kv_append_kernel, dim3(p.m, p.Hkv), dim3(32), 0, s, p);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attention_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kDecSmem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(attention_decode_kernel, dim3(p.n_chunks, p.Hkv), dim3(kDecThreads), kDecSmem, s, p);
    if (e != cudaSuccess) return e;
    e = launch_pdl(attention_combine_kernel, dim3(p.rows, p.Hkv), dim3(kD), 0, s, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

int attention_prefill_grid(int64_t M, int64_t H) { return static_cast<int>((M + kTile - 1) / kTile * H); }

cudaError_t launch_attention_prefill(const void *qkv, int64_t M, int64_t H, int64_t Hkv,
                                     void *k_cache, void *v_cache, int64_t S_max, void *o,
                                     float *amax_partials, int partial_slots, unsigned *err,
                                     cudaStream_t s) {
    EncodeFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    CUtensorMap tq, tk, tv;
    std::memset(&tk, 0, sizeof(tk));
    std::memset(&tv, 0, sizeof(tv));
    const int64_t cols = (H + 2 * Hkv) * kD;
    {
        // qkv [M, cols] BF16; boxes of 128 rows x 64 columns, 128-byte swizzle;
        // rows past M read as zeros
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(M)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * 2)};
        const cuuint32_t box[2] = {64, kTile};
        const cuuint32_t estr[2] = {1, 1};
        if (fn(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(qkv), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const int write_cache = (k_cache && v_cache) ? 1 : 0;
    if (write_cache) {
        // cache [Hkv, S_max, 128] BF16 as 3-D maps; a store is clipped at S_max
        const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(S_max),
                                    static_cast<cuuint64_t>(Hkv)};
        const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD * 2),
                                       static_cast<cuuint64_t>(S_max * kD * 2)};
        const cuuint32_t box[3] = {64, kTile, 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (fn(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k_cache, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
            fn(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v_cache, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    PrefillParams p;
    p.M = static_cast<int>(M);
    p.H = static_cast<int>(H);
    p.Hkv = static_cast<int>(Hkv);
    p.n_qt = static_cast<int>((M + kTile - 1) / kTile);
    p.write_cache = write_cache;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.amax_partials = amax_partials;
    p.partial_slots = partial_slots;
    p.err = err;
    cudaError_t e = cudaFuncSetAttribute(attention_prefill_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    e = launch_pdl(attention_prefill_kernel, dim3(static_cast<unsigned>(p.n_qt * p.H)), dim3(kThreads),
                   kSmemBytes, s, tq, tk, tv, p);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace mq
