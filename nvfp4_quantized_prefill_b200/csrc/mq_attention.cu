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
// 2-stage ring, K and V released separately; warp 1 issues S = Q K^T
// (kind::f16, M = 128, N = 128, K = 16 per instruction) into one of three
// 128-column FP32 buffers in tensor memory; warp 2 issues O += P V with P
// read from tensor memory; warps 3-6 (one thread per query row, all 128
// columns of its S row: no exchange between threads) take the row maximum,
// raise the running maximum only when it grows by more than 2^8 (then O is
// rescaled in place; otherwise the stale maximum keeps every weight below 2^8
// and the final division by the same-based sum is exact), write P as BF16
// over the S buffer, and finally divide O by the row sum, store it and keep
// max |o| for the O projection's quantizer.  The first query head of each KV
// group writes its diagonal K / V tile to the cache.
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
#ifndef MQ_ATT_COL_GROUPS
#define MQ_ATT_COL_GROUPS 1
#endif
// softmax warpgroups, each a column range of every row: one (a thread owns
// its whole S row) measured 4% faster on the 8B shape than two (half rows,
// row maxima exchanged through shared memory and a named barrier per tile)
constexpr int kColGroups = MQ_ATT_COL_GROUPS;
constexpr int kCols = 128 / kColGroups;          // S columns per softmax thread
constexpr uint32_t kXchgOff = kBarOff + 256;     // row maxima, 2 tiles x kColGroups x 128
constexpr uint32_t kLsumOff = kXchgOff + 2 * kColGroups * 128 * 4;   // row sums, kColGroups x 128
constexpr uint32_t kSmemBytes = kLsumOff + kColGroups * 128 * 4 + 1024;
constexpr int kSoftmaxWarps = 4 * kColGroups;
static_assert(kCols % 32 == 0, "whole 32-column TMEM loads per thread");
constexpr int kSoftWarp0 = 3;             // warps 0-2: producer, S issuer, PV issuer
constexpr int kThreads = 32 * (kSoftWarp0 + kSoftmaxWarps);
constexpr int kSBufs = 3;                 // S / P buffers in tensor memory
constexpr uint32_t kTmemCols = 512;       // S0, S1, S2 at 0, 128, 256; O at 384
constexpr uint32_t kOCol = 128 * kSBufs;
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

// 2^x by the hardware approximation (relative error about 2^-22, subnormal
// results flushed to zero): the weights it feeds are rounded to BF16.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// a * b + c on two FP32 lanes at once (packed pairs: element 0 in the low word)
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
__device__ __forceinline__ void unpack_f32x2(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// acc + both BF16 halves of w, each widened exactly to FP32 by the mixed-type FMA
__device__ __forceinline__ float add_bf16x2_f32(float acc, uint32_t w) {
    asm("{\n\t.reg .b16 lo, hi, one;\n\tmov.b32 {lo, hi}, %1;\n\tmov.b16 one, 0x3F80;\n\t"
        "fma.rn.f32.bf16 %0, lo, one, %0;\n\tfma.rn.f32.bf16 %0, hi, one, %0;\n\t}"
        : "+f"(acc)
        : "r"(w));
    return acc;
}

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
    const uint32_t k_full = bar + 8;          // [2] per K/V stage
    const uint32_t v_full = bar + 24;         // [2]
    const uint32_t k_empty = bar + 40;        // [2] S of that stage's K tile has completed
    const uint32_t v_empty = bar + 232;       // [2] PV of that stage's V tile has completed
    const uint32_t s_full = bar + 56;         // [3] per S buffer
    const uint32_t p_full = bar + 80;         // [3]
    const uint32_t pv_done = bar + 104;       // [3] the PV product that read P of that buffer
    const uint32_t drain = bar + 128;         // every MMA issued has completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kBarOff + 136);
    float *red = reinterpret_cast<float *>(smem + kBarOff + 160);   // one float per softmax warp
    float *xchg = reinterpret_cast<float *>(smem + kXchgOff);      // [2][kColGroups][128]
    float *lsum = reinterpret_cast<float *>(smem + kLsumOff);      // [kColGroups][128]

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
            mbar_init(k_empty + 8 * i, 1);
            mbar_init(v_empty + 8 * i, 1);
        }
        for (int i = 0; i < kSBufs; ++i) {
            mbar_init(s_full + 8 * i, 1);
            mbar_init(p_full + 8 * i, kSoftmaxWarps);   // one arrival per softmax warp
            mbar_init(pv_done + 8 * i, 1);
        }
        mbar_init(drain, 2);                       // one commit per MMA-issuing warp
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
            int last_k = -1, last_v = -1;   // the last tiles whose K / V loads were issued
            for (int j = 0; j < nkv && ok; ++j) {
                const int st = j & 1;
                // K and V tiles are released separately (K once S has read it,
                // V once PV has), so the next K tile does not wait for a softmax;
                // a barrier is re-armed only after its previous phase completed
                if (j >= kStages && !wait_bar(k_empty + 8 * st, ((j - kStages) >> 1) & 1)) {
                    ok = false;
                    break;
                }
                if (stored[st]) {
                    bulk_wait_group_read0();   // the cache store has read the stage
                    stored[st] = false;
                }
                const uint32_t ks = s0 + kKOff + st * kTileBytes;
                const uint32_t vs = s0 + kVOff + st * kTileBytes;
                mbar_arrive_expect_tx(k_full + 8 * st, kTileBytes);
                tma_load_2d(ks, &tmap_qkv, qkv_cols_k, j * kTile, k_full + 8 * st);
                tma_load_2d(ks + kHalfBytes, &tmap_qkv, qkv_cols_k + 64, j * kTile, k_full + 8 * st);
                if (j >= kStages && !wait_bar(v_empty + 8 * st, ((j - kStages) >> 1) & 1)) {
                    ok = false;
                    last_k = j;
                    break;
                }
                last_k = last_v = j;
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
            // the loads of the last tiles of each stage have landed (they have
            // on the normal path; after a timeout, before the CTA may exit)
            for (int j = last_k; j >= 0 && j > last_k - kStages; --j) wait_bar(k_full + 8 * (j & 1), (j >> 1) & 1);
            for (int j = last_v; j >= 0 && j > last_v - kStages; --j) wait_bar(v_full + 8 * (j & 1), (j >> 1) & 1);
            bulk_wait_group0();   // cache stores complete before the CTA exits
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------- S = Q K^T issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16(128, 128, 0, 0);   // Q, K both K-major
            if (!wait_bar(q_full, 0)) ok = false;
            tc_fence_after();
            for (int j = 0; j < nkv && ok; ++j) {
                const int st = j & 1, sb = j % kSBufs;
                if (!wait_bar(k_full + 8 * st, (j >> 1) & 1)) ok = false;
                // S buffer sb last held P_{j-3}: its PV must have completed
                if (j >= kSBufs && !wait_bar(pv_done + 8 * sb, ((j - kSBufs) / kSBufs) & 1)) ok = false;
                if (!ok) break;
                tc_fence_after();
                tc_mma8_bf16_ss_commit2(tmem + sb * 128u, sdesc_kmajor_sw128(s0 + kQOff),
                                        sdesc_kmajor_sw128(s0 + kKOff + st * kTileBytes), idesc_s, 0u,
                                        s_full + 8 * sb, k_empty + 8 * st);
            }
            // every MMA this thread issued completes before TMEM is freed
            tc_commit(drain);
            wait_bar(drain, 0);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ---------------------------------------------------------- O += P V issuer
        // (its own warp: the two products of a tile go to different TMEM
        // regions and are ordered only through the barriers, so S of later
        // tiles is issued while this warp waits for a softmax)
        if (lane == 0) {
            constexpr uint32_t idesc_o = idesc_bf16(128, 128, 0, 1);   // V MN-major
            for (int jj = 0; jj < nkv && ok; ++jj) {
                const int st = jj & 1, sb = jj % kSBufs;
                if (!wait_bar(p_full + 8 * sb, (jj / kSBufs) & 1)) ok = false;
                if (!wait_bar(v_full + 8 * st, (jj >> 1) & 1)) ok = false;
                if (!ok) break;
                tc_fence_after();
                // keys 16 kk .. 16 kk + 15: two 8-row groups of the V tile
                tc_mma8_bf16_ts_commit2(tmem + kOCol, tmem + sb * 128u,
                                        sdesc_mnmajor_sw128(s0 + kVOff + st * kTileBytes, kHalfBytes),
                                        idesc_o, jj > 0 ? 1u : 0u, pv_done + 8 * sb, v_empty + 8 * st);
            }
            tc_commit(drain);
            wait_bar(drain, 0);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------- softmax
        // warpgroup wg holds columns [kCols wg, kCols wg + kCols) of every row
        // (all of them with one group); with several groups the threads of a
        // row agree on the row maximum through shared memory (one named
        // barrier a tile, double-buffered by tile parity) and keep their own
        // share of the row sum
        const int wg = (warp - kSoftWarp0) >> 2;
        const int quarter = warp & 3;             // TMEM lane group of this warp
        const int r = quarter * 32 + lane;        // query row in the tile
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const int col0 = wg * kCols;
        float m_run = -INFINITY, l = 0.0f;
        for (int j = 0; j < nkv; ++j) {
            const int st = j & 1, sb = j % kSBufs;
            ok = __all_sync(0xFFFFFFFFu, wait_bar(s_full + 8 * sb, (j / kSBufs) & 1)) && ok;
            tc_fence_after();
            uint32_t sr[kCols];
#pragma unroll
            for (int h = 0; h < kCols / 32; ++h)
                tmem_ld32(tmem + lane_off + sb * 128u + col0 + 32u * h,
                          *reinterpret_cast<uint32_t (*)[32]>(&sr[32 * h]));
            tmem_ld_wait();
            // raw scores (the base-2 scale is applied inside the exponent);
            // keys after the row's own position masked on the diagonal tile
            float s[kCols];
#pragma unroll
            for (int c = 0; c < kCols; ++c) s[c] = __uint_as_float(sr[c]);
            if (j == qt) {
#pragma unroll
                for (int c = 0; c < kCols; ++c)
                    if (col0 + c > r) s[c] = -INFINITY;
            }
            // eight chains of three-input maxima
            float mp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mp[e] = fmaxf(s[e], s[8 + e]);
#pragma unroll
            for (int c = 16; c < kCols; c += 16)
#pragma unroll
                for (int e = 0; e < 8; ++e) mp[e] = fmax3(mp[e], s[c + e], s[c + 8 + e]);
            // the scale is positive: the maximum of the scaled scores
            float mx = fmaxf(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], fmax3(mp[5], mp[6], mp[7]))) *
                       kScaleLog2;
            if constexpr (kColGroups > 1) {
                xchg[(st * kColGroups + wg) * 128 + r] = mx;
                // the barrier's AND also carries "every softmax warp saw S":
                // after a timed-out wait all softmax warps leave the loop
                // together (none may be left waiting here for the others); it
                // also orders every thread's S loads before any thread's P
                // stores over the buffer
                uint32_t all_ok;
                asm volatile(
                    "{\n\t.reg .pred p, q;\n\t"
                    "setp.ne.u32 p, %1, 0;\n\t"
                    "bar.red.and.pred q, 2, %2, p;\n\t"
                    "selp.u32 %0, 1, 0, q;\n\t}"
                    : "=r"(all_ok)
                    : "r"(ok ? 1u : 0u), "n"(32 * kSoftmaxWarps)
                    : "memory");
                if (!all_ok) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int w2 = 0; w2 < kColGroups; ++w2)
                    if (w2 != wg) mx = fmaxf(mx, xchg[(st * kColGroups + w2) * 128 + r]);
            } else {
                // one thread per row: the row maximum is the thread's own, and
                // a warp overwrites S only in its own TMEM lanes; a timed-out
                // warp leaves on its own (the others run into their own
                // bounded waits and meet it at the epilogue's barriers)
                if (!ok) break;
            }
            // raise the running maximum only for a growth beyond 2^8 (or at
            // the first tile); O then needs the factor 2^(m_old - m_new)
            const bool need = mx > m_run + kRescaleThreshold;
            const float m_new = need ? mx : m_run;
            const float f = need ? exp2f(m_run - m_new) : 1.0f;   // 0 at the first tile
            if (__any_sync(0xFFFFFFFFu, need) && j > 0) {
                // (a timeout here is seen by the other warps at the next
                // tile's barrier)
                ok = __all_sync(0xFFFFFFFFu,
                                wait_bar(pv_done + 8 * ((j - 1) % kSBufs), ((j - 1) / kSBufs) & 1)) && ok;
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < kCols / 32; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(tmem + lane_off + kOCol + col0 + c * 32u, ov);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
                    tmem_st32(tmem + lane_off + kOCol + col0 + c * 32u, ov);
                }
                tmem_st_wait();
            }
            l *= f;
            m_run = m_new;
            // exponents two at a time (packed FMA), the weights rounded to
            // BF16 pairs, and their row sum taken over the rounded values
            const uint64_t sc2 = pack_f32x2(kScaleLog2, kScaleLog2);
            const uint64_t nm2 = pack_f32x2(-m_run, -m_run);
            float lp[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int h = 0; h < kCols / 32; ++h) {
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const int cc = 16 * h + c;
                    float x0, x1;
                    unpack_f32x2(ffma2(pack_f32x2(s[2 * cc], s[2 * cc + 1]), sc2, nm2), x0, x1);
                    const __nv_bfloat162 pb = __floats2bfloat162_rn(ex2_approx(x0), ex2_approx(x1));
                    pk[c] = *reinterpret_cast<const uint32_t *>(&pb);
                    lp[c & 3] = add_bf16x2_f32(lp[c & 3], pk[c]);
                }
                // P (BF16 pairs) over the S buffer's first 64 columns
                tmem_st16(tmem + lane_off + sb * 128u + static_cast<uint32_t>(col0 / 2 + 16 * h), pk);
            }
            l += (lp[0] + lp[1]) + (lp[2] + lp[3]);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full + 8 * sb);
        }
        // epilogue: O / l -> BF16 (this group's kCols columns), and max |o|
        if constexpr (kColGroups > 1) {
            lsum[wg * 128 + r] = l;
            asm volatile("bar.sync 3, %0;" ::"n"(32 * kSoftmaxWarps) : "memory");
            l = 0.0f;
#pragma unroll
            for (int w2 = 0; w2 < kColGroups; ++w2) l += lsum[w2 * 128 + r];
        }
        ok = __all_sync(0xFFFFFFFFu,
                        wait_bar(pv_done + 8 * ((nkv - 1) % kSBufs), ((nkv - 1) / kSBufs) & 1)) && ok;
        tc_fence_after();
        const float inv = 1.0f / l;
        const int row = qt * kTile + r;
        float omax = 0.0f;
        __nv_bfloat16 *orow = p.o + static_cast<int64_t>(row) * (p.H * kD) + h * kD + col0;
#pragma unroll
        for (int c = 0; c < kCols / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(tmem + lane_off + kOCol + col0 + c * 32u, ov);
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
        if (lane == 0) red[warp - kSoftWarp0] = __uint_as_float(b);
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kSoftmaxWarps) : "memory");
        if (warp == kSoftWarp0 && lane == 0) {
            float m = 0.0f;
            for (int i = 0; i < kSoftmaxWarps; ++i) m = fmaxf(m, red[i]);
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
// keys are split into spans across CTAs (one CTA per span and KV head, all of
// the group's query rows at once, so each K / V byte crosses HBM once per
// step); a CTA streams its span in 64-key blocks, double-buffered in shared
// memory by cp.async, computes S = Q K^T and O += P V with BF16 m16n8k16
// tensor-core MMAs (FP32 accumulation; P rounded to BF16 and the row sums
// taken over the rounded weights, as in the prefill kernel), and leaves
// (max, sum, unnormalised o) per query row; a combine pass merges the spans.

constexpr int kDecKeys = 64;              // keys per block
constexpr int kDecThreads = 128;          // 4 warps: 16 keys each for S, 32 dimensions each for P.V
constexpr int kDecMaxRows = 64;           // query rows per KV head (group size x tokens)
#ifndef MQ_DEC_MAX_CTAS
#define MQ_DEC_MAX_CTAS 256
#endif
constexpr int kDecMaxCtas = MQ_DEC_MAX_CTAS;  // spans x KV heads stay at or below this
constexpr uint32_t kDecTileBytes = kDecKeys * kD * 2;      // one K or V block, 16 KB
constexpr int kDecQPitch = kD + 8;                          // BF16 per Q row (bank-conflict-free)
constexpr int kDecPPitch = kDecKeys + 8;                    // BF16 per P row
// shared memory: K and V blocks (two each), then Q, P and the per-warp row
// maxima / sums for kNT row tiles of 8
template <int kNT>
constexpr uint32_t dec_smem_bytes() {
    return 4 * kDecTileBytes + 8 * kNT * (kDecQPitch * 2 + kDecPPitch * 2 + 2 * 4 * 4);
}

// 64-key blocks per span: as few as keep spans x KV heads within kDecMaxCtas
__host__ __device__ constexpr int64_t dec_span_blocks(int64_t n_keys, int64_t Hkv) {
    const int64_t blocks = (n_keys + kDecKeys - 1) / kDecKeys;
    const int64_t sb = (blocks * Hkv + kDecMaxCtas - 1) / kDecMaxCtas;
    return sb < 1 ? 1 : sb;
}

struct DecodeParams {
    const __nv_bfloat16 *qkv;   // [m, (H + 2 Hkv) * 128]
    __nv_bfloat16 *k_cache;     // [Hkv, S_max, 128]
    __nv_bfloat16 *v_cache;
    __nv_bfloat16 *o;           // [m, H * 128]
    float *part;                // [Hkv, n_chunks, rows, 2 + 128]
    int m, pos0, H, Hkv, S_max, n_chunks, rows;
    int span_blocks;            // 64-key blocks per CTA
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

// 16 bytes global -> shared, asynchronously; src_bytes = 0 fills zeros
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// D (16x8 FP32) += A (16x16 BF16, row-major) * B (16x8 BF16, column-major)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// byte offset of (key, 8-element chunk c) in a [64][128] BF16 block whose
// 16-byte chunks are XOR-swizzled by the key's low three bits
__device__ __forceinline__ uint32_t dec_tile_off(int key, int c) {
    return static_cast<uint32_t>(key * 256 + ((c ^ (key & 7)) << 4));
}

// kNT: 8-row tiles of query rows this instance serves (rows <= 8 kNT)
template <int kNT>
__global__ void __launch_bounds__(kDecThreads) attention_decode_kernel(const DecodeParams p) {
    extern __shared__ __align__(128) uint8_t dsm[];
    const uint32_t kv0 = smem_u32(dsm);                     // K[2], V[2]: 4 x 16 KB
    __nv_bfloat16 *qs = reinterpret_cast<__nv_bfloat16 *>(dsm + 4 * kDecTileBytes);   // [8 kNT][136]
    __nv_bfloat16 *ps = qs + 8 * kNT * kDecQPitch;                                     // [8 kNT][72]
    float *red_max = reinterpret_cast<float *>(ps + 8 * kNT * kDecPPitch);             // [4][8 kNT]
    float *red_sum = red_max + 4 * 8 * kNT;                                             // [4][8 kNT]
    __shared__ float m_run[kDecMaxRows], l_run[kDecMaxRows], alpha[kDecMaxRows];
    const int c = blockIdx.x, g = blockIdx.y, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
    const int group = p.H / p.Hkv;
    const int n_keys = p.pos0 + p.m;
    const int cols = (p.H + 2 * p.Hkv) * kD;
    const __nv_bfloat16 *kbase = p.k_cache + static_cast<int64_t>(g) * p.S_max * kD;
    const __nv_bfloat16 *vbase = p.v_cache + static_cast<int64_t>(g) * p.S_max * kD;
    const int key_begin = c * p.span_blocks * kDecKeys;
    const int nb = min(p.span_blocks, (n_keys - key_begin + kDecKeys - 1) / kDecKeys);
    // block b of the span into buffer b & 1 (K at kv0 + buf 16 KB, V two buffers on)
    auto load_block = [&](int b) {
        const int key0 = key_begin + b * kDecKeys;
        const uint32_t kdst = kv0 + static_cast<uint32_t>(b & 1) * kDecTileBytes;
        const uint32_t vdst = kdst + 2 * kDecTileBytes;
        for (int i = tid; i < kDecKeys * (kD / 8); i += kDecThreads) {
            const int k = i >> 4, ch = i & 15;
            const bool in = key0 + k < n_keys;
            const int64_t off = static_cast<int64_t>(in ? key0 + k : key0) * kD + ch * 8;
            cp_async16(kdst + dec_tile_off(k, ch), kbase + off, in ? 16u : 0u);
            cp_async16(vdst + dec_tile_off(k, ch), vbase + off, in ? 16u : 0u);
        }
        cp_async_commit();
    };
    griddep_wait();            // the appended rows and the queries are in place
    griddep_launch_dependents();
    load_block(0);
    // the group's query rows (row rr = hh * m + t: head g * group + hh, token t), zeros past p.rows
    for (int i = tid; i < 8 * kNT * (kD / 2); i += kDecThreads) {
        const int rr = i / (kD / 2), d2 = (i % (kD / 2)) * 2;
        uint32_t v = 0;
        if (rr < p.rows) {
            const int hh = rr / p.m, t = rr % p.m;
            v = *reinterpret_cast<const uint32_t *>(p.qkv + static_cast<int64_t>(t) * cols + (g * group + hh) * kD + d2);
        }
        *reinterpret_cast<uint32_t *>(qs + rr * kDecQPitch + d2) = v;
    }
    for (int rr = tid; rr < kDecMaxRows; rr += kDecThreads) {
        m_run[rr] = -INFINITY;
        l_run[rr] = 0.0f;
    }
    // P.V accumulators: dims 32 warp + 16 i + gq (+ 8), rows 8 j + 2 tq (+ 1)
    float acc[2][kNT][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < kNT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.0f;
    for (int b = 0; b < nb; ++b) {
        if (b + 1 < nb) {
            load_block(b + 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();           // block b (and, the first time, Q) is in shared memory
        const int key0 = key_begin + b * kDecKeys;
        const uint32_t kt = kv0 + static_cast<uint32_t>(b & 1) * kDecTileBytes;
        const uint32_t vt = kt + 2 * kDecTileBytes;
        // S^T (keys 16 warp .. of the block x rows) = K Q^T
        float sc[kNT][4];
#pragma unroll
        for (int j = 0; j < kNT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[j][e] = 0.0f;
#pragma unroll
        for (int s = 0; s < kD / 16; ++s) {
            uint32_t a[4];
            ldsm_x4(kt + dec_tile_off(16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * s + (lane >> 4)), a);
#pragma unroll
            for (int j = 0; j < kNT; ++j) {
                const __nv_bfloat16 *qr = qs + (8 * j + gq) * kDecQPitch + 16 * s + 2 * tq;
                mma_bf16_16816(sc[j], a, *reinterpret_cast<const uint32_t *>(qr),
                               *reinterpret_cast<const uint32_t *>(qr + 8));
            }
        }
        // scale, mask (past the cache, after the row's own position, padding
        // rows), and the block maximum of each row over this warp's keys
        float mx[kNT][2];
#pragma unroll
        for (int j = 0; j < kNT; ++j) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int row = 8 * j + 2 * tq + (e & 1);
                const int pos = key0 + 16 * warp + gq + (e >> 1) * 8;
                const bool ok = row < p.rows && pos < n_keys && pos <= p.pos0 + row % p.m;
                sc[j][e] = ok ? sc[j][e] * kScaleLog2 : -INFINITY;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float v = fmaxf(sc[j][h], sc[j][h + 2]);
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
                mx[j][h] = v;
            }
            if (gq == 0) {
                red_max[warp * 8 * kNT + 8 * j + 2 * tq] = mx[j][0];
                red_max[warp * 8 * kNT + 8 * j + 2 * tq + 1] = mx[j][1];
            }
        }
        __syncthreads();
        // weights 2^(s - m_new) rounded to BF16 (the P.V operand), and their row sums
#pragma unroll
        for (int j = 0; j < kNT; ++j) {
            float mnew[2], sum[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = 8 * j + 2 * tq + h;
                float v = m_run[row];
#pragma unroll
                for (int w = 0; w < 4; ++w) v = fmaxf(v, red_max[w * 8 * kNT + row]);
                mnew[h] = v;
                sum[h] = 0.0f;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h = e & 1;
                const float w = mnew[h] == -INFINITY ? 0.0f : exp2f(sc[j][e] - mnew[h]);
                const __nv_bfloat16 wb = __float2bfloat16_rn(w);
                sum[h] += __bfloat162float(wb);
                ps[(8 * j + 2 * tq + h) * kDecPPitch + 16 * warp + gq + (e >> 1) * 8] = wb;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float v = sum[h];
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                if (gq == 0) red_sum[warp * 8 * kNT + 8 * j + 2 * tq + h] = v;
            }
        }
        __syncthreads();
        // running maximum and sum per row
        for (int row = tid; row < 8 * kNT; row += kDecThreads) {
            float v = m_run[row];
#pragma unroll
            for (int w = 0; w < 4; ++w) v = fmaxf(v, red_max[w * 8 * kNT + row]);
            const float m_old = m_run[row];
            const float a = m_old == -INFINITY ? 0.0f : exp2f(m_old - v);
            float l = 0.0f;
#pragma unroll
            for (int w = 0; w < 4; ++w) l += red_sum[w * 8 * kNT + row];
            alpha[row] = a;
            l_run[row] = l_run[row] * a + l;
            m_run[row] = v;
        }
        __syncthreads();
        // O^T (dims x rows) = alpha O^T + V^T P^T over the block's 64 keys
#pragma unroll
        for (int j = 0; j < kNT; ++j) {
            const float a0 = alpha[8 * j + 2 * tq], a1 = alpha[8 * j + 2 * tq + 1];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                acc[i][j][0] *= a0;
                acc[i][j][1] *= a1;
                acc[i][j][2] *= a0;
                acc[i][j][3] *= a1;
            }
        }
#pragma unroll
        for (int s = 0; s < kDecKeys / 16; ++s) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                uint32_t a[4];
                const int mi = lane >> 3;
                ldsm_x4_trans(vt + dec_tile_off(16 * s + (lane & 7) + (mi >> 1) * 8, 4 * warp + 2 * i + (mi & 1)), a);
#pragma unroll
                for (int j = 0; j < kNT; ++j) {
                    const __nv_bfloat16 *pr = ps + (8 * j + gq) * kDecPPitch + 16 * s + 2 * tq;
                    mma_bf16_16816(acc[i][j], a, *reinterpret_cast<const uint32_t *>(pr),
                                   *reinterpret_cast<const uint32_t *>(pr + 8));
                }
            }
        }
        __syncthreads();           // buffers b & 1, P and the row partials may be overwritten
    }
    float *part = p.part + (static_cast<int64_t>(g) * p.n_chunks + c) * p.rows * (2 + kD);
    for (int rr = tid; rr < p.rows; rr += kDecThreads) {
        part[rr * (2 + kD)] = m_run[rr];
        part[rr * (2 + kD) + 1] = l_run[rr];
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < kNT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int row = 8 * j + 2 * tq + (e & 1);
                const int d = 32 * warp + 16 * i + gq + (e >> 1) * 8;
                if (row < p.rows) part[row * (2 + kD) + 2 + d] = acc[i][j][e];
            }
}

// Up to 8 query rows (one or two new tokens of a grouped head): each warp
// keeps its own running maximum, sum and o over its 16 keys of every block
// (S, the softmax and P.V need no cross-warp exchange: one block barrier per
// 64 keys, for the double buffer), and the four warps' partials are merged
// once at the end of the span.  Three K / V blocks per CTA: two loads stay in
// flight while a block is computed.
constexpr int kDecWarpPPitch = 24;    // BF16 per row of a warp's P transpose area
constexpr int kDecWarpStages = 3;    // K / V blocks in flight or in use per CTA
constexpr uint32_t kDecWarpSmem = 2 * kDecWarpStages * kDecTileBytes + 8 * kDecQPitch * 2 + 4 * 8 * kDecWarpPPitch * 2;

__global__ void __launch_bounds__(kDecThreads) attention_decode_warp_kernel(const DecodeParams p) {
    extern __shared__ __align__(128) uint8_t dsm[];
    const uint32_t kv0 = smem_u32(dsm);                     // K[3], V[3]: 6 x 16 KB
    __nv_bfloat16 *qs = reinterpret_cast<__nv_bfloat16 *>(dsm + 2 * kDecWarpStages * kDecTileBytes);   // [8][136]
    __nv_bfloat16 *pw = qs + 8 * kDecQPitch;                                           // [4][8][24]
    const int c = blockIdx.x, g = blockIdx.y, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
    const int group = p.H / p.Hkv;
    const int n_keys = p.pos0 + p.m;
    const int cols = (p.H + 2 * p.Hkv) * kD;
    const __nv_bfloat16 *kbase = p.k_cache + static_cast<int64_t>(g) * p.S_max * kD;
    const __nv_bfloat16 *vbase = p.v_cache + static_cast<int64_t>(g) * p.S_max * kD;
    const int key_begin = c * p.span_blocks * kDecKeys;
    const int nb = min(p.span_blocks, (n_keys - key_begin + kDecKeys - 1) / kDecKeys);
    auto load_block = [&](int b) {
        const int key0 = key_begin + b * kDecKeys;
        const uint32_t kdst = kv0 + static_cast<uint32_t>(b % kDecWarpStages) * kDecTileBytes;
        const uint32_t vdst = kdst + kDecWarpStages * kDecTileBytes;
        for (int i = tid; i < kDecKeys * (kD / 8); i += kDecThreads) {
            const int k = i >> 4, ch = i & 15;
            const bool in = key0 + k < n_keys;
            const int64_t off = static_cast<int64_t>(in ? key0 + k : key0) * kD + ch * 8;
            cp_async16(kdst + dec_tile_off(k, ch), kbase + off, in ? 16u : 0u);
            cp_async16(vdst + dec_tile_off(k, ch), vbase + off, in ? 16u : 0u);
        }
        cp_async_commit();
    };
    griddep_wait();            // the appended rows and the queries are in place
    griddep_launch_dependents();
    load_block(0);
    if (nb > 1) load_block(1);
    for (int i = tid; i < 8 * (kD / 2); i += kDecThreads) {
        const int rr = i / (kD / 2), d2 = (i % (kD / 2)) * 2;
        uint32_t v = 0;
        if (rr < p.rows) {
            const int hh = rr / p.m, t = rr % p.m;
            v = *reinterpret_cast<const uint32_t *>(p.qkv + static_cast<int64_t>(t) * cols + (g * group + hh) * kD + d2);
        }
        *reinterpret_cast<uint32_t *>(qs + rr * kDecQPitch + d2) = v;
    }
    // this warp's running state for rows 2 tq, 2 tq + 1 (the C-fragment
    // columns) and its O^T: dims 16 i + gq (+ 8), rows 2 tq (+ 1)
    float m_w[2] = {-INFINITY, -INFINITY}, l_w[2] = {0.0f, 0.0f};
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][e] = 0.0f;
    __nv_bfloat16 *pwt = pw + warp * 8 * kDecWarpPPitch;
    for (int b = 0; b < nb; ++b) {
        // block b landed (block b + 1 may still be in flight)
        if (b + 1 < nb)
            cp_async_wait<1>();
        else
            cp_async_wait<0>();
        __syncthreads();           // ... for every thread's copies; every warp is done with block b - 1
        if (b + 2 < nb) load_block(b + 2);   // into the buffer block b - 1 used
        const int key0 = key_begin + b * kDecKeys;
        const uint32_t kt = kv0 + static_cast<uint32_t>(b % kDecWarpStages) * kDecTileBytes;
        const uint32_t vt = kt + kDecWarpStages * kDecTileBytes;
        float sc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int s = 0; s < kD / 16; ++s) {
            uint32_t a[4];
            ldsm_x4(kt + dec_tile_off(16 * warp + (lane & 7) + ((lane >> 3) & 1) * 8, 2 * s + (lane >> 4)), a);
            const __nv_bfloat16 *qr = qs + gq * kDecQPitch + 16 * s + 2 * tq;
            mma_bf16_16816(sc, a, *reinterpret_cast<const uint32_t *>(qr),
                           *reinterpret_cast<const uint32_t *>(qr + 8));
        }
        float mx[2];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int row = 2 * tq + (e & 1);
            const int pos = key0 + 16 * warp + gq + (e >> 1) * 8;
            const bool ok = row < p.rows && pos < n_keys && pos <= p.pos0 + row % p.m;
            sc[e] = ok ? sc[e] * kScaleLog2 : -INFINITY;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float v = fmaxf(sc[h], sc[h + 2]);
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
            mx[h] = v;
        }
        float sum[2] = {0.0f, 0.0f}, alpha[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float m_new = fmaxf(m_w[h], mx[h]);
            alpha[h] = m_w[h] == -INFINITY ? 0.0f : exp2f(m_w[h] - m_new);
            m_w[h] = m_new;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int h = e & 1;
            const float w = m_w[h] == -INFINITY ? 0.0f : exp2f(sc[e] - m_w[h]);
            const __nv_bfloat16 wb = __float2bfloat16_rn(w);
            sum[h] += __bfloat162float(wb);
            pwt[(2 * tq + h) * kDecWarpPPitch + gq + (e >> 1) * 8] = wb;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float v = sum[h];
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
            l_w[h] = l_w[h] * alpha[h] + v;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            acc[i][0] *= alpha[0];
            acc[i][1] *= alpha[1];
            acc[i][2] *= alpha[0];
            acc[i][3] *= alpha[1];
        }
        __syncwarp();              // this warp's P transpose is complete
        const uint32_t b0 = *reinterpret_cast<const uint32_t *>(pwt + gq * kDecWarpPPitch + 2 * tq);
        const uint32_t b1 = *reinterpret_cast<const uint32_t *>(pwt + gq * kDecWarpPPitch + 2 * tq + 8);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t a[4];
            const int mi = lane >> 3;
            ldsm_x4_trans(vt + dec_tile_off(16 * warp + (lane & 7) + (mi >> 1) * 8, 2 * i + (mi & 1)), a);
            mma_bf16_16816(acc[i], a, b0, b1);
        }
        __syncwarp();              // P reads done before the next block's P is written
    }
    __syncthreads();               // the K / V buffers are free for the merge
    // merge the four warps: per warp m and l of the 8 rows and O[8][128]
    float *mw = reinterpret_cast<float *>(dsm);              // [4][8]
    float *lw = mw + 32;                                      // [4][8]
    float *ow = lw + 32;                                      // [4][8][128]
    if (gq == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mw[warp * 8 + 2 * tq + h] = m_w[h];
            lw[warp * 8 + 2 * tq + h] = l_w[h];
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e)
            ow[(warp * 8 + 2 * tq + (e & 1)) * kD + 16 * i + gq + (e >> 1) * 8] = acc[i][e];
    __syncthreads();
    float *part = p.part + (static_cast<int64_t>(g) * p.n_chunks + c) * p.rows * (2 + kD);
    for (int rr = 0; rr < p.rows; ++rr) {
        float mm = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) mm = fmaxf(mm, mw[w * 8 + rr]);
        float l = 0.0f, o = 0.0f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float f = mw[w * 8 + rr] == -INFINITY ? 0.0f : exp2f(mw[w * 8 + rr] - mm);
            l = fmaf(lw[w * 8 + rr], f, l);
            o = fmaf(ow[(w * 8 + rr) * kD + tid], f, o);
        }
        if (tid == 0) {
            part[rr * (2 + kD)] = mm;
            part[rr * (2 + kD) + 1] = l;
        }
        part[rr * (2 + kD) + 2 + tid] = o;
    }
}

template <int kNT>
cudaError_t launch_decode_rows(const DecodeParams &p, cudaStream_t s) {
    constexpr uint32_t smem = dec_smem_bytes<kNT>();
    cudaError_t e = cudaFuncSetAttribute(attention_decode_kernel<kNT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(attention_decode_kernel<kNT>, dim3(p.n_chunks, p.Hkv), dim3(kDecThreads), smem, s, p);
}

// Merges the spans of one query row: 512 threads, four groups of 128 (one
// thread per dimension) taking every fourth span, then a shared-memory sum.
constexpr int kCombineGroups = 4;
__global__ void __launch_bounds__(kD * kCombineGroups) attention_combine_kernel(const DecodeParams p) {
    __shared__ float red[kD * kCombineGroups / 32];
    __shared__ float part_acc[kCombineGroups - 1][kD];
    __shared__ float part_l[kCombineGroups - 1];
    griddep_wait();
    griddep_launch_dependents();
    const int rr = blockIdx.x, g = blockIdx.y, tid = threadIdx.x;
    const int d = tid & (kD - 1), q = tid / kD;
    const int group = p.H / p.Hkv, hh = rr / p.m, t = rr % p.m;
    const float *base = p.part + static_cast<int64_t>(g) * p.n_chunks * p.rows * (2 + kD) + rr * (2 + kD);
    const int64_t step = static_cast<int64_t>(p.rows) * (2 + kD);
    // the largest span maximum, over all 512 threads
    float mx = -INFINITY;
    for (int c = tid; c < p.n_chunks; c += kD * kCombineGroups) mx = fmaxf(mx, base[c * step]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if ((tid & 31) == 0) red[tid >> 5] = mx;
    __syncthreads();
    mx = red[0];
#pragma unroll
    for (int w = 1; w < kD * kCombineGroups / 32; ++w) mx = fmaxf(mx, red[w]);
    float l = 0.0f, acc = 0.0f;
#pragma unroll 8
    for (int c = q; c < p.n_chunks; c += kCombineGroups) {
        const float mc = base[c * step];
        // a span with no visible key (maximum -inf) adds nothing
        const float f = mc == -INFINITY ? 0.0f : exp2f(mc - mx);
        l = fmaf(base[c * step + 1], f, l);
        acc = fmaf(base[c * step + 2 + d], f, acc);
    }
    if (q > 0) {
        part_acc[q - 1][d] = acc;
        if (d == 0) part_l[q - 1] = l;
    }
    __syncthreads();
    if (q == 0) {
#pragma unroll
        for (int i = 0; i < kCombineGroups - 1; ++i) {
            acc += part_acc[i][d];
            l += part_l[i];
        }
        p.o[static_cast<int64_t>(t) * (p.H * kD) + (g * group + hh) * kD + d] = __float2bfloat16_rn(acc / l);
    }
}

}  // namespace

size_t attention_decode_workspace_bytes(int64_t m, int64_t pos0, int64_t H, int64_t Hkv) {
    const int64_t rows = H / Hkv * m;
    const int64_t span = kDecKeys * dec_span_blocks(pos0 + m, Hkv);
    const int64_t n_chunks = (pos0 + m + span - 1) / span;
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
    p.rows = static_cast<int>(H / Hkv * m);
    p.span_blocks = static_cast<int>(dec_span_blocks(pos0 + m, Hkv));
    const int64_t span = static_cast<int64_t>(kDecKeys) * p.span_blocks;
    p.n_chunks = static_cast<int>((pos0 + m + span - 1) / span);
    cudaError_t e = launch_pdl(kv_append_kernel, dim3(p.m, p.Hkv), dim3(32), 0, s, p);
    if (e != cudaSuccess) return e;
    if (p.rows <= 8) {
        e = cudaFuncSetAttribute(attention_decode_warp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kDecWarpSmem);
        if (e == cudaSuccess)
            e = launch_pdl(attention_decode_warp_kernel, dim3(p.n_chunks, p.Hkv), dim3(kDecThreads),
                           kDecWarpSmem, s, p);
    } else {
        e = p.rows <= 32 ? launch_decode_rows<4>(p, s) : launch_decode_rows<kDecMaxRows / 8>(p, s);
    }
    if (e != cudaSuccess) return e;
    e = launch_pdl(attention_combine_kernel, dim3(p.rows, p.Hkv), dim3(kD * kCombineGroups), 0, s, p);
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
