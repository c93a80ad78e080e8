// mq_gemm.cu -- block-scaled NVFP4 x NVFP4 GEMM on the sm_100a tcgen05 tensor
// cores, FP32 accumulation in tensor memory, BF16 output, with an optional
// fused SwiGLU epilogue.
//
// Method: Mix-Quant's prefill linear runs both weights and activations in
// NVFP4 ("W4A4", gist.science technical summary, section 2 "System-Level
// Deployment"); decoding keeps BF16.  Y = bf16(acc / (s_enc_a * s_enc_b)),
// acc = sum_k e2m1(a) dec(sa) e2m1(b) dec(sb), one E4M3 scale per 16 K.
//
// Kernel shape: CTA pairs (clusters of 2, one CTA per SM, persistent), each
// pair computing 256 x 256 output tiles with the paired MMA
// (tcgen05.mma.cta_group::2, M = 256 split 128 rows per CTA, N = 256):
//   warp 0       (both CTAs) TMA producer: this CTA's 128 A rows and 128 B
//                rows of a 256-wide K step (128-byte swizzle), its A scale
//                tiles and both B scale halves, into a 5-stage ring; every
//                load completes on the even CTA's stage barriers (scale tiles
//                on their own, so their TMEM copies overlap the operand loads).
//   warp 1       (even CTA) MMA issuer: one wait per stage, then 4 paired
//                MMAs (K = 64 each) and the stage's commit from one issue
//                block, into a 128 x 256 FP32 accumulator in each CTA's TMEM.
//   warps 2-3    (even CTA) scale copiers: tcgen05.cp of the stage's scale
//                tiles into both CTAs' TMEM (6 copies per copier per stage in
//                one issue block), from their own threads -- a thread's
//                tcgen05 instructions run in order, so copies issued by the
//                MMA thread would queue ahead of its MMAs; a copier commits
//                the stage's sf_full only after the operand barrier too.
//                Each tcgen05 instruction, barrier wait and commit costs the
//                issuing warp ~80-100 cycles, against ~550 cycles of tensor
//                work per stage: the issue paths are trimmed to stay below.
//   warps 4-11   (both CTAs) epilogue: drain the CTA's accumulator half with
//                tcgen05.ld, meet on a named barrier, and release it with one
//                arrive per CTA (CTA-scope release: the cluster-scope form
//                stalls the arriving thread for ~0.7 us, all of it on the
//                tensor pipe's idle time between tiles); then store while the
//                next tile's main loop runs.  The SwiGLU variant computes
//                SiLU(gate) * up only after the release.  Warpgroup 0 hands
//                registers to the epilogue warpgroups (setmaxnreg).
// Every mbarrier wait is bounded (about two seconds); on a timeout the kernel
// latches an error bit, stops issuing work, lets issued copies and MMAs land,
// frees its tensor memory and exits.
#include <cuda_bf16.h>

#include <cstring>

#include "mq_internal.h"
#include "mq_ptx.cuh"

namespace mq {

namespace {

#ifndef MQ_GEMM_STAGES
#define MQ_GEMM_STAGES 5
#endif
#ifndef MQ_GEMM_GROUP_M
#define MQ_GEMM_GROUP_M 8
#endif



constexpr int kStages = MQ_GEMM_STAGES;
constexpr uint32_t kABytes = 128 * 128;          // this CTA's 128 A rows x 128 B (256 fp4)
constexpr uint32_t kBBytes = 128 * 128;          // this CTA's 128 B rows
constexpr uint32_t kSfaBytes = 4 * 512;          // 4 scale tiles (K = 256) of the A rows
constexpr uint32_t kSfbBytes = 2 * 4 * 512;      // both 128-row halves of the B tile
constexpr uint32_t kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;  // 38912
constexpr uint32_t kPairTxAB = 2 * (kABytes + kBBytes);                      // both CTAs
constexpr uint32_t kPairTxSF = 2 * (kSfaBytes + kSfbBytes);
constexpr uint32_t kStageTileBytes = 32 * 128;    // epilogue staging: 32 rows x 64 bf16
constexpr uint32_t kStagingBytes = 8 * kStageTileBytes;  // one per epilogue warp
constexpr uint32_t kBarBytes = 256;
constexpr uint32_t kSmemBytes = kStages * kStageBytes + kStagingBytes + kBarBytes + 1024;
constexpr int kCopiers = 2;                      // scale-copy warps
constexpr int kEpiWarp0 = 2 + kCopiers;          // first of 8 epilogue warps
constexpr int kThreads = 32 * (kEpiWarp0 + 8);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol = 256;                 // scale columns follow the accumulator
constexpr uint32_t kSfColsPerStage = 48;         // 16 for A + 32 for B
constexpr int kGroupM = MQ_GEMM_GROUP_M;         // tile raster: M-tiles per group
constexpr uint16_t kPairMask = 0x3;

constexpr int kRegsLaunch = 168;                 // per thread, from __launch_bounds__(kThreads, 1)
constexpr int kRegsLow = 56;                     // warpgroup 0 after setmaxnreg.dec
constexpr int kRegsHigh = 224;                   // epilogue warpgroups after setmaxnreg.inc
static_assert(kEpiWarp0 == 4, "warpgroup 0 = producer, MMA, copiers; 1-2 = epilogue");
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kRegsLaunch, "register split");
static_assert(kThreads * kRegsLaunch <= 65536, "launch register file");
static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
static_assert(kSfCol + kStages * kSfColsPerStage <= kTmemCols, "TMEM budget");
static_assert((4 * kStages + 4) * 8 + 48 <= kBarBytes, "barrier area");

struct Params {
    const float *s_enc_a;
    const float *s_enc_b;
    __nv_bfloat16 *y;
    int64_t ldy;
    int M, N, K;
    int tiles_m, tiles_n, k_tiles, sf_ktiles, n_half;
    float *amax_partials;
    unsigned *err;
    int tma_store;        // 1: outputs leave through TMA stores via shared memory
    unsigned long long wait_ns;   // bound of every wait (kWaitLimitNs outside tests)
    int withhold_release;         // test only: the first stage is never released
};

__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int &tm, int &tn) {
    const int per_group = kGroupM * tiles_n;
    const int g = t / per_group;
    const int first = g * kGroupM;
    const int gs = min(tiles_m - first, kGroupM);
    const int local = t - g * per_group;
    tm = first + local % gs;
    tn = local / gs;
}

// Waits (time-bounded, ignoring the abort flag) so that in-flight asynchronous
// work signalling `bar` has landed before the CTA exits.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, unsigned *err,
                                           unsigned long long limit_ns) {
    unsigned long long t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) {
            atomicOr(err, kDevErrTimeout);
            return;
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float bf16_round(float v) {
    return __bfloat162float(__float2bfloat16_rn(v));
}

template <int kCols>
__device__ __forceinline__ void store_row(__nv_bfloat16 *dst, const uint32_t *packed, int ncols_valid,
                                          bool vec_ok) {
    if (vec_ok && ncols_valid >= kCols) {
        uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
        for (int i = 0; i < kCols / 8; ++i)
            d[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
    } else {
#pragma unroll
        for (int i = 0; i < kCols / 2; ++i) {
            if (2 * i < ncols_valid)
                reinterpret_cast<unsigned short *>(dst)[2 * i] =
                    static_cast<unsigned short>(packed[i] & 0xFFFFu);
            if (2 * i + 1 < ncols_valid)
                reinterpret_cast<unsigned short *>(dst)[2 * i + 1] =
                    static_cast<unsigned short>(packed[i] >> 16);
        }
    }
}

template <bool kSwiglu>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_sfa,
                     const __grid_constant__ CUtensorMap tmap_sfb,
                     const __grid_constant__ CUtensorMap tmap_y, const Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes + kStagingBytes);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * kStages + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *red = reinterpret_cast<float *>(tmem_slot + 2);  // 8 floats

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();         // 0: the pair's issuing CTA
    const uint32_t bar0 = smem_u32(bars);             // full[s]  = bar0 + 8 s
    const uint32_t empty0 = bar0 + 8u * kStages;      // empty[s]
    const uint32_t sf_full0 = bar0 + 16u * kStages;   // sf_full[s]
    const uint32_t sfd_full0 = bar0 + 24u * kStages;  // scale tiles landed[s]
    const uint32_t acc_full = bar0 + 32u * kStages;
    const uint32_t acc_empty = acc_full + 8u;
    const uint32_t drain_bar = acc_full + 16u;
    const uint32_t sf_drain_bar = acc_full + 24u;
    const uint32_t smem0 = smem_u32(smem);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar0 + 8u * s, 1);             // arrive.expect_tx of the even CTA
            mbar_init(empty0 + 8u * s, 1);           // MMA commit (to both CTAs)
            mbar_init(sf_full0 + 8u * s, kCopiers);  // one commit per copier
            mbar_init(sfd_full0 + 8u * s, 1);        // arrive.expect_tx of the even CTA
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2);                     // one arrive per CTA's epilogue
        mbar_init(drain_bar, 1);
        mbar_init(sf_drain_bar, kCopiers);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
        prefetch_tmap(&tmap_sfa);
        prefetch_tmap(&tmap_sfb);
        if (p.tma_store) prefetch_tmap(&tmap_y);
    }
    if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the peer's barriers exist before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the set-up above overlaps the previous kernel's tail; operands and
    // outputs are touched only after it has completed
    griddep_wait();
    griddep_launch_dependents();
    const int num_tiles = p.tiles_m * p.tiles_n;
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int npairs = static_cast<int>(gridDim.x >> 1);

    // The producer, MMA and copier roles run their loops on all 32 lanes with
    // warp-uniform state; one elected lane issues each TMA / tcgen05
    // instruction (see the warp_* wrappers).
    // Registers: warpgroup 0 (producer, MMA, copiers) gives most of its share
    // to the two epilogue warpgroups, which hold a whole 128-column
    // accumulator row slice: 128 x 56 + 256 x 224 = 384 x 168 (the launch).
    if (warp < kEpiWarp0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int stage = 0;
        uint32_t phase = 0;
        uint32_t armed = 0, armed_parity = 0;
        bool ok = true;
        for (int t = pair; t < num_tiles && ok; t += npairs) {
            int tm, tn;
            tile_coords(t, p.tiles_m, p.tiles_n, tm, tn);
            // B rows of this CTA and the two 128-row scale blocks of the tile
            int b_row, rb0, rb1;
            if (kSwiglu) {
                rb0 = tn;                            // gate rows 128 tn ..
                rb1 = p.n_half / 128 + tn;           // matching up rows
                b_row = (rank == 0 ? rb0 : rb1) * 128;
            } else {
                rb0 = 2 * tn;
                rb1 = 2 * tn + 1;
                b_row = tn * 256 + static_cast<int>(rank) * 128;
            }
            const int a_row = tm * 256 + static_cast<int>(rank) * 128;
            const int a_sf = (2 * tm + static_cast<int>(rank)) * p.sf_ktiles;
            for (int kt = 0; kt < p.k_tiles; ++kt) {
                if (!warp_mbar_wait(empty0 + 8u * stage, phase ^ 1u, abort_flag, p.err, p.wait_ns)) {
                    ok = false;
                    break;
                }
                const uint32_t full_local = bar0 + 8u * stage;
                const uint32_t full_pair = mapa_shared(full_local, 0);
                const uint32_t sfd_local = sfd_full0 + 8u * stage;
                const uint32_t sfd_pair = mapa_shared(sfd_local, 0);
                if (rank == 0) {
                    warp_arrive_expect_tx(sfd_local, kPairTxSF);
                    warp_arrive_expect_tx(full_local, kPairTxAB);
                    armed |= 1u << stage;
                    armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                }
                const uint32_t sA = smem0 + stage * kStageBytes;
                const uint32_t sB = sA + kABytes;
                const uint32_t sSFA = sB + kBBytes;
                const uint32_t sSFB = sSFA + kSfaBytes;
                // the small scale tiles first, on their own barrier, so the
                // scale copies into TMEM can start before the operands land
                warp_tma_load_2d_pair(sSFA, &tmap_sfa, 0, a_sf + kt * 4, sfd_pair);
                warp_tma_load_2d_pair(sSFB, &tmap_sfb, 0, rb0 * p.sf_ktiles + kt * 4, sfd_pair);
                warp_tma_load_2d_pair(sSFB + 4u * 512u, &tmap_sfb, 0, rb1 * p.sf_ktiles + kt * 4,
                                      sfd_pair);
                warp_tma_load_2d_pair(sA, &tmap_a, kt * 128, a_row, full_pair);
                warp_tma_load_2d_pair(sB, &tmap_b, kt * 128, b_row, full_pair);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // both CTAs' loads of every armed stage land before the pair may exit
        for (int s2 = 0; s2 < kStages; ++s2)
            if (armed & (1u << s2)) {
                drain_wait(sfd_full0 + 8u * s2, (armed_parity >> s2) & 1u, p.err, p.wait_ns);
                drain_wait(bar0 + 8u * s2, (armed_parity >> s2) & 1u, p.err, p.wait_ns);
            }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (rank == 0) {
            constexpr uint32_t idesc = idesc_nvf4(256, 256);
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += npairs) {
                if (!warp_mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag, p.err, p.wait_ns)) break;
                tc_fence_after();
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    // the stage's scales are in TMEM and both CTAs' operands
                    // landed: the copiers commit sf_full only after seeing the
                    // operand barrier, so this is the one wait per stage
                    if (!warp_mbar_wait(sf_full0 + 8u * stage, phase, abort_flag, p.err, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int natoms = min(4, p.sf_ktiles - kt * 4);
                    const uint32_t sA = smem0 + stage * kStageBytes;
                    const uint32_t sB = sA + kABytes;
                    const uint32_t tsfa = tmem + kSfCol + stage * kSfColsPerStage;
                    const uint32_t tsfb = tsfa + 16u;
                    if (p.withhold_release && t == pair && kt == 0) {
                        // test only: the stage's MMAs without the commit that
                        // frees it, so the producer's next wait on it runs out
                        for (int kb = 0; kb < natoms; ++kb)
                            warp_mma_nvf4_pair(tmem, sdesc_kmajor_sw128(sA + 32u * kb),
                                               sdesc_kmajor_sw128(sB + 32u * kb), idesc, tsfa + 4u * kb,
                                               tsfb + 8u * kb, kb != 0 ? 1u : 0u);
                    } else if (natoms == 4) {
                        warp_mma4_commit_pair(tmem, sdesc_kmajor_sw128(sA), sdesc_kmajor_sw128(sB), idesc,
                                              tsfa, tsfb, kt != 0 ? 1u : 0u, empty0 + 8u * stage,
                                              kPairMask);
                    } else {
                        for (int kb = 0; kb < natoms; ++kb) {
                            warp_mma_nvf4_pair(tmem, sdesc_kmajor_sw128(sA + 32u * kb),
                                               sdesc_kmajor_sw128(sB + 32u * kb), idesc, tsfa + 4u * kb,
                                               tsfb + 8u * kb, (kt | kb) != 0 ? 1u : 0u);
                        }
                        warp_commit_pair_mc(empty0 + 8u * stage, kPairMask);  // frees both CTAs' stage
                    }
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                warp_commit_pair_mc(acc_full, kPairMask);
                acc_phase ^= 1u;
            }
            // every MMA issued by this warp completes before TMEM is freed
            warp_commit_pair(drain_bar);
            drain_wait(drain_bar, 0, p.err, p.wait_ns);
        }
    } else {
        // ------------------------------------------------------------ scale copiers
        // Copier c copies k-blocks c, c + kCopiers, ... of each stage: the A
        // scale tile (each CTA its own rows) and both B halves, into the
        // stage's TMEM scale slot of both CTAs, then arrives on sf_full[stage].
        const int cid = warp - 2;
        if (rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += npairs) {
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    if (!warp_mbar_wait(sfd_full0 + 8u * stage, phase, abort_flag, p.err, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int natoms = min(4, p.sf_ktiles - kt * 4);
                    const uint32_t sSFA = smem0 + stage * kStageBytes + kABytes + kBBytes;
                    const uint32_t sSFB = sSFA + kSfaBytes;
                    const uint32_t tsfa = tmem + kSfCol + stage * kSfColsPerStage;
                    const uint32_t tsfb = tsfa + 16u;
                    if (natoms == 4) {
                        const uint32_t a = static_cast<uint32_t>(cid);
                        warp_cp6_pair(tsfa + 4u * a, tsfb + 8u * a, sdesc_sf_tile(sSFA + 512u * a),
                                      sdesc_sf_tile(sSFB + 512u * a),
                                      sdesc_sf_tile(sSFB + 4u * 512u + 512u * a));
                    } else {
                        for (int a = cid; a < natoms; a += kCopiers) {
                            warp_cp_sf_pair(tsfa + 4u * a, sdesc_sf_tile(sSFA + 512u * a));
                            warp_cp_sf_pair(tsfb + 8u * a, sdesc_sf_tile(sSFB + 512u * a));
                            warp_cp_sf_pair(tsfb + 8u * a + 4u,
                                            sdesc_sf_tile(sSFB + 4u * 512u + 512u * a));
                        }
                    }
                    // the operands too have landed when sf_full completes, so
                    // the MMA thread waits on one barrier per stage
                    if (!warp_mbar_wait(bar0 + 8u * stage, phase, abort_flag, p.err, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    warp_commit_pair(sf_full0 + 8u * stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            warp_commit_pair(sf_drain_bar);
            drain_wait(sf_drain_bar, 0, p.err, p.wait_ns);
        }
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
        // ------------------------------------------------------------ epilogue
        const int ew = warp - kEpiWarp0;  // 0..7
        const int sub = warp & 3;         // TMEM lane group this warp may read
        const int half = ew >> 2;         // column half of the tile
        const float alpha = __frcp_rn(__fmul_rn(*p.s_enc_a, *p.s_enc_b));
        const bool vec_ok = (p.ldy % 8) == 0;
        const uint32_t acc_empty_pair = mapa_shared(acc_empty, 0);
        // The accumulator may be overwritten once all 8 epilogue warps of both
        // CTAs have their tcgen05.ld data in registers: the warps meet on a
        // named barrier and one thread per CTA arrives on the MMA thread's
        // acc_empty (count 2).
        // `got`: this warp saw the accumulator complete (false after an
        // abort); the barrier's AND keeps the 8 warps leaving together.
        auto release_acc = [&](bool got) -> bool {
            tc_fence_before();
            uint32_t all;
            asm volatile(
                "{\n\t.reg .pred p, q;\n\t"
                "setp.ne.u32 p, %1, 0;\n\t"
                "bar.red.and.pred q, 2, 256, p;\n\t"
                "selp.u32 %0, 1, 0, q;\n\t}"
                : "=r"(all)
                : "r"(got ? 1u : 0u)
                : "memory");
            if (!all) return false;
            if (ew == 0 && lane == 0) {
                if (rank == 0)
                    mbar_arrive(acc_empty);
                else
                    mbar_arrive_remote(acc_empty_pair);
            }
            return true;
        };
        // this warp's staging tile: 32 rows of 128 bytes, 128-byte swizzled
        // (16-byte chunk j of row r at r * 128 + ((j ^ (r % 8)) * 16)), the
        // layout the output tensor map's SWIZZLE_128B store reads
        const uint32_t stg = smem0 + kStages * kStageBytes + ew * kStageTileBytes;
        const uint32_t stg_row = stg + lane * 128u;
        uint32_t acc_phase = 0;
        float hmax = 0.0f;
        // Stages 32 rows x 64 columns (this lane's row: 32 packed bf16 pairs)
        // and stores them at output (col0, row0) with one TMA store.
        auto tma_store_chunk = [&](const uint32_t *q, int col0, int row0) {
            if (lane == 0) bulk_wait_group_read0();  // staging free again
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                st_shared_v4(stg_row + ((static_cast<uint32_t>(j) ^ (lane & 7u)) << 4), q[4 * j],
                             q[4 * j + 1], q[4 * j + 2], q[4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(&tmap_y, col0, row0, stg);
                bulk_commit_group();
            }
        };
        for (int t = pair; t < num_tiles; t += npairs) {
            int tm, tn;
            tile_coords(t, p.tiles_m, p.tiles_n, tm, tn);
            // warp-uniform decision: the TMEM loads below are .sync.aligned
            const bool got = __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, acc_phase, abort_flag, p.err, p.wait_ns));
            if (got) tc_fence_after();
            const int row0 = tm * 256 + static_cast<int>(rank) * 128 + sub * 32;
            const int row = row0 + lane;
            const uint32_t tbase = tmem + (static_cast<uint32_t>(sub * 32) << 16);
            if (!kSwiglu) {
                // two rounds of 64 columns: load, scale and round; then release
                // (measured faster than loading all 128 before the release)
                uint32_t packed[64];
                if (got) {
#pragma unroll
                    for (int c = 0; c < 4; c += 2) {
                        uint32_t r0[32], r1[32];
                        tmem_ld32(tbase + half * 128 + c * 32, r0);
                        tmem_ld32(tbase + half * 128 + (c + 1) * 32, r1);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            packed[c * 16 + j] = pack_bf16x2(__fmul_rn(alpha, __uint_as_float(r0[2 * j])),
                                                             __fmul_rn(alpha, __uint_as_float(r0[2 * j + 1])));
                            packed[(c + 1) * 16 + j] =
                                pack_bf16x2(__fmul_rn(alpha, __uint_as_float(r1[2 * j])),
                                            __fmul_rn(alpha, __uint_as_float(r1[2 * j + 1])));
                        }
                    }
                }
                if (!release_acc(got)) break;
                const int n0 = tn * 256 + half * 128;
                if (p.tma_store) {
                    if (row0 < p.M && n0 < p.N) {
                        tma_store_chunk(packed, n0, row0);
                        if (n0 + 64 < p.N) tma_store_chunk(packed + 32, n0 + 64, row0);
                    }
                } else if (row < p.M && n0 < p.N) {
                    store_row<128>(p.y + static_cast<int64_t>(row) * p.ldy + n0, packed, p.N - n0,
                                   vec_ok);
                }
            } else {
                // gate columns [64 half, +64) and the matching up columns
                // (128 + ...) into registers, release, then SwiGLU
                uint32_t rg[2][32], ru[2][32];
                if (got) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        tmem_ld32(tbase + half * 64 + c * 32, rg[c]);
                        tmem_ld32(tbase + 128 + half * 64 + c * 32, ru[c]);
                    }
                    tmem_ld_wait();
                }
                if (!release_acc(got)) break;
                uint32_t packed[32];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float hv[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const float g = bf16_round(__fmul_rn(alpha, __uint_as_float(rg[c][2 * j + e])));
                            const float u = bf16_round(__fmul_rn(alpha, __uint_as_float(ru[c][2 * j + e])));
                            const float silu = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
                            hv[e] = __fmul_rn(silu, u);
                        }
                        packed[c * 16 + j] = pack_bf16x2(hv[0], hv[1]);
                    }
                }
                const int n0 = tn * 128 + half * 64;
                if (row < p.M) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&packed[i]);
                        hmax = fmaxf(hmax, fmaxf(fabsf(__bfloat162float(v.x)),
                                                 fabsf(__bfloat162float(v.y))));
                    }
                }
                if (p.tma_store) {
                    if (row0 < p.M) tma_store_chunk(packed, n0, row0);
                } else if (row < p.M) {
                    store_row<64>(p.y + static_cast<int64_t>(row) * p.ldy + n0, packed, 64, true);
                }
            }
            acc_phase ^= 1u;
        }
        if (lane == 0) bulk_wait_group0();  // this warp's output stores have completed
        __syncwarp();
        if (kSwiglu) {
            const uint32_t b = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(hmax));
            if (lane == 0) red[ew] = __uint_as_float(b);
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (ew == 0 && lane == 0) {
                float m = 0.0f;
                for (int i = 0; i < 8; ++i) m = fmaxf(m, red[i]);
                p.amax_partials[blockIdx.x] = m;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // after a timeout, give copies this CTA issued toward the peer's
        // barriers time to land before the pair tears down
        const unsigned long long t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 1000000ull) {
        }
    }
    cluster_sync();  // no peer signal or paired MMA can still target this CTA
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                              const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                              const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
    // resolved once; the initialization of a function-local static is
    // thread-safe
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

}  // namespace

bool encode_codes_tmap(CUtensorMap *map, const void *codes, int64_t rows, int64_t K) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    const cuuint32_t box[2] = {128, 128};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(codes), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_sf_tmap(CUtensorMap *map, const void *sf, int64_t rows, int64_t K) {
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    // the swizzled scales as an array of 512-byte tiles (128 words each); a box
    // is the 4 consecutive tiles of one K step
    const int64_t tiles = (rows + 127) / 128 * (K / 64);
    const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(tiles)};
    const cuuint64_t strides[1] = {512};
    const cuuint32_t box[2] = {128, 4};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(sf), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_out_tmap(CUtensorMap *map, const void *y, int64_t rows, int64_t cols, int64_t ld) {
    EncodeFn fn = encode_fn();
    if (!fn || ld % 8 != 0 || (reinterpret_cast<uintptr_t>(y) & 15u)) return false;
    // BF16 [rows, cols] with leading dimension ld; a box is 32 rows x 64 columns
    // (128 bytes, 128-byte swizzled in shared memory)
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
    const cuuint32_t box[2] = {64, 32};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(y), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_gemm_nvf4(const CUtensorMap &tmap_a, const CUtensorMap &tmap_b,
                             const CUtensorMap &tmap_sfa, const CUtensorMap &tmap_sfb,
                             const GemmArgs &a, bool swiglu, int num_sms, int *grid_out,
                             cudaStream_t s) {
    Params p;
    CUtensorMap tmap_y;
    std::memset(&tmap_y, 0, sizeof(tmap_y));
    const int64_t out_cols = swiglu ? a.N / 2 : a.N;
    p.tma_store = encode_out_tmap(&tmap_y, a.y, a.M, out_cols, a.ldy) ? 1 : 0;
    p.s_enc_a = a.s_enc_a;
    p.s_enc_b = a.s_enc_b;
    p.y = static_cast<__nv_bfloat16 *>(a.y);
    p.ldy = a.ldy;
    p.M = a.M;
    p.N = a.N;
    p.K = a.K;
    p.tiles_m = (a.M + 255) / 256;
    p.n_half = a.N / 2;
    p.tiles_n = swiglu ? p.n_half / 128 : (a.N + 255) / 256;
    p.sf_ktiles = a.K / 64;
    p.k_tiles = (p.sf_ktiles + 3) / 4;
    p.amax_partials = a.amax_partials;
    p.err = a.err;
    p.wait_ns = a.wait_ns ? a.wait_ns : kWaitLimitNs;
    p.withhold_release = a.withhold_release;
    const int tiles = p.tiles_m * p.tiles_n;
    const int max_pairs = num_sms / 2;
    int pairs = tiles < max_pairs ? tiles : max_pairs;
    if (pairs < 1) pairs = 1;
    const int grid = 2 * pairs;
    if (grid_out) *grid_out = grid;
    cudaError_t e;
    if (swiglu) {
        e = cudaFuncSetAttribute(gemm_nvf4_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes);
        if (e != cudaSuccess) return e;
        e = launch_pdl(gemm_nvf4_kernel<true>, dim3(grid), dim3(kThreads), kSmemBytes, s, tmap_a,
                       tmap_b, tmap_sfa, tmap_sfb, tmap_y, p);
    } else {
        e = cudaFuncSetAttribute(gemm_nvf4_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes);
        if (e != cudaSuccess) return e;
        e = launch_pdl(gemm_nvf4_kernel<false>, dim3(grid), dim3(kThreads), kSmemBytes, s, tmap_a,
                       tmap_b, tmap_sfa, tmap_sfb, tmap_y, p);
    }
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace mq
