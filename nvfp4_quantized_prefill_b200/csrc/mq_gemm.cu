// mq_gemm.cu -- block-scaled NVFP4 x NVFP4 GEMM on the sm_100a tcgen05 tensor
// cores, FP32 accumulation in tensor memory, BF16 output, with an optional
// fused SwiGLU epilogue.
//
// Method: Mix-Quant's prefill linear runs both weights and activations in
// NVFP4 ("W4A4", gist.science technical summary, section 2 "System-Level
// Deployment"); decoding keeps BF16.  Y = bf16(acc / (s_enc_a * s_enc_b)),
// acc = sum_k e2m1(a) dec(sa) e2m1(b) dec(sb), one E4M3 scale per 16 K.
//
// Kernel shape (one persistent CTA per SM, 10 warps):
//   warp 0     TMA producer: A tile [128 x 256 fp4], B tile [256 x 256 fp4]
//              (two 128-row boxes, 128-byte swizzle) and the matching 512-byte
//              scale-factor tiles (plain bulk copies) into a 4-stage ring.
//   warp 1     MMA issuer: copies the scale tiles into TMEM (tcgen05.cp) and
//              issues tcgen05.mma kind::mxf4nvf4 block16, M=128 N=256 K=64,
//              into one 128 x 256 FP32 accumulator in TMEM.
//   warps 2-9  epilogue: drain the accumulator (tcgen05.ld), release it to
//              the MMA warp, then scale, round to BF16 and store -- the stores
//              overlap the next tile's main loop.
// Every mbarrier wait is bounded (about two seconds); on a timeout the kernel
// latches an error bit, stops issuing work, lets in-flight copies and MMAs
// land, frees its tensor memory and exits.
#include <cuda_bf16.h>

#include "mq_internal.h"
#include "mq_ptx.cuh"

namespace mq {

namespace {

constexpr int kStages = 4;
constexpr uint32_t kABytes = 128 * 128;          // 128 rows x 128 B (256 fp4)
constexpr uint32_t kBBytes = 256 * 128;          // 256 rows x 128 B
constexpr uint32_t kSfaBytes = 4 * 512;          // 4 scale tiles (K = 256)
constexpr uint32_t kSfbBytes = 2 * 4 * 512;      // two 128-row halves
constexpr uint32_t kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;  // 55296
constexpr uint32_t kBarBytes = 256;
constexpr uint32_t kSmemBytes = kStages * kStageBytes + kBarBytes + 1024;
#ifndef MQ_GEMM_COPIERS
#define MQ_GEMM_COPIERS 2
#endif
constexpr int kCopiers = MQ_GEMM_COPIERS;        // scale-copy warps
constexpr int kEpiWarp0 = 2 + kCopiers;          // first of 8 epilogue warps
constexpr int kThreads = 32 * (kEpiWarp0 + 8);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol = 256;                 // scale columns follow the accumulator
constexpr uint32_t kSfColsPerStage = 48;         // 16 for A + 32 for B
constexpr int kGroupM = 16;                      // tile raster: 16 M-tiles per group

static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
static_assert(kSfCol + kStages * kSfColsPerStage <= kTmemCols, "TMEM budget");

struct Params {
    const uint8_t *sfa;
    const uint8_t *sfb;
    const float *s_enc_a;
    const float *s_enc_b;
    __nv_bfloat16 *y;
    int64_t ldy;
    int M, N, K;
    int tiles_m, tiles_n, k_tiles, sf_ktiles, sf_rowblocks_b, n_half;
    float *amax_partials;
    unsigned *err;
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

// B rows / scale row-blocks of N-tile tn: plain mode covers weight rows
// [256 tn, 256 tn + 256); SwiGLU mode covers gate rows [128 tn, +128) and the
// matching up rows [n_half + 128 tn, +128).
__device__ __forceinline__ void b_rows(const Params &p, int tn, bool swiglu, int &row0, int &row1,
                                       int &rb0, int &rb1) {
    if (swiglu) {
        row0 = tn * 128;
        row1 = p.n_half + tn * 128;
    } else {
        row0 = tn * 256;
        row1 = tn * 256 + 128;
    }
    rb0 = row0 / 128;
    rb1 = row1 / 128;
}

// Waits (time-bounded, ignoring the abort flag) so that in-flight asynchronous
// work signalling `bar` has landed before the CTA exits.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, unsigned *err) {
    unsigned long long t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) {
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
__global__ void __launch_bounds__(kThreads, 1)
    gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b, const Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * kStages + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *red = reinterpret_cast<float *>(tmem_slot + 2);  // 8 floats

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_u32(bars);
    const uint32_t acc_full = bar0 + 8u * (2 * kStages);
    const uint32_t acc_empty = acc_full + 8u;
    const uint32_t drain_bar = acc_full + 16u;
    const uint32_t sf_drain_bar = acc_full + 24u;
    const uint32_t sf_full0 = acc_full + 32u;     // sf_full[s] = sf_full0 + 8 s
    const uint32_t smem0 = smem_u32(smem);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(bar0 + 8u * s, 1);               // full[s]
            mbar_init(bar0 + 8u * (kStages + s), 1);   // empty[s]
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 8);
        mbar_init(drain_bar, 1);
        mbar_init(sf_drain_bar, kCopiers);
        for (int s = 0; s < kStages; ++s) mbar_init(sf_full0 + 8u * s, kCopiers);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int num_tiles = p.tiles_m * p.tiles_n;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_parity = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                int tm, tn, row0, row1, rb0, rb1;
                tile_coords(t, p.tiles_m, p.tiles_n, tm, tn);
                b_rows(p, tn, kSwiglu, row0, row1, rb0, rb1);
                const bool rb1_ok = rb1 < p.sf_rowblocks_b;
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    const uint32_t full = bar0 + 8u * stage;
                    if (!mbar_wait(bar0 + 8u * (kStages + stage), phase ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    const int natoms = min(4, p.sf_ktiles - kt * 4);
                    const uint32_t sf_bytes = static_cast<uint32_t>(natoms) * 512u;
                    const uint32_t bytes =
                        kABytes + kBBytes + sf_bytes * (rb1_ok ? 3u : 2u);
                    mbar_arrive_expect_tx(full, bytes);
                    armed |= 1u << stage;
                    armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                    const uint32_t sA = smem0 + stage * kStageBytes;
                    const uint32_t sB = sA + kABytes;
                    const uint32_t sSFA = sB + kBBytes;
                    const uint32_t sSFB = sSFA + kSfaBytes;
                    tma_load_2d(sA, &tmap_a, kt * 128, tm * 128, full);
                    tma_load_2d(sB, &tmap_b, kt * 128, row0, full);
                    tma_load_2d(sB + 128u * 128u, &tmap_b, kt * 128, row1, full);
                    bulk_load(sSFA, p.sfa + (static_cast<int64_t>(tm) * p.sf_ktiles + kt * 4) * 512,
                              sf_bytes, full);
                    bulk_load(sSFB, p.sfb + (static_cast<int64_t>(rb0) * p.sf_ktiles + kt * 4) * 512,
                              sf_bytes, full);
                    if (rb1_ok)
                        bulk_load(sSFB + 4u * 512u,
                                  p.sfb + (static_cast<int64_t>(rb1) * p.sf_ktiles + kt * 4) * 512,
                                  sf_bytes, full);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // let every issued copy land before the CTA may exit
            for (int s = 0; s < kStages; ++s)
                if (armed & (1u << s)) drain_wait(bar0 + 8u * s, (armed_parity >> s) & 1u, p.err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_nvf4(128, 256);
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                if (!mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag, p.err)) break;
                tc_fence_after();
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    // operands landed and this stage's scales are in TMEM
                    if (!mbar_wait(sf_full0 + 8u * stage, phase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int natoms = min(4, p.sf_ktiles - kt * 4);
                    const uint32_t sA = smem0 + stage * kStageBytes;
                    const uint32_t sB = sA + kABytes;
                    const uint32_t tsfa = tmem + kSfCol + stage * kSfColsPerStage;
                    const uint32_t tsfb = tsfa + 16u;
                    for (int kb = 0; kb < natoms; ++kb) {
                        tc_mma_nvf4(tmem, sdesc_kmajor_sw128(sA + 32u * kb),
                                    sdesc_kmajor_sw128(sB + 32u * kb), idesc, tsfa + 4u * kb,
                                    tsfb + 8u * kb, (kt | kb) != 0 ? 1u : 0u);
                    }
                    tc_commit(bar0 + 8u * (kStages + stage));  // frees the smem stage
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(acc_full);
                acc_phase ^= 1u;
            }
            // every MMA / copy issued by this thread completes before TMEM is freed
            tc_commit(drain_bar);
            drain_wait(drain_bar, 0, p.err);
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------------ scale copiers
        // Each copier warp copies its share of a stage's scale tiles (k-blocks
        // c, c + kCopiers, ...) smem -> TMEM with tcgen05.cp from its own
        // thread: a thread's tcgen05 instructions run in order, so copies
        // issued by the MMA thread would queue in front of its MMAs.  Each
        // copier arrives on sf_full[stage] once its copies have landed.
        const int cid = warp - 2;
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    if (!mbar_wait(bar0 + 8u * stage, phase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int natoms = min(4, p.sf_ktiles - kt * 4);
                    const uint32_t sSFA = smem0 + stage * kStageBytes + kABytes + kBBytes;
                    const uint32_t sSFB = sSFA + kSfaBytes;
                    const uint32_t tsfa = tmem + kSfCol + stage * kSfColsPerStage;
                    const uint32_t tsfb = tsfa + 16u;
                    for (int a = cid; a < natoms; a += kCopiers) {
                        tc_cp_sf(tsfa + 4u * a, sdesc_sf_tile(sSFA + 512u * a));
                        tc_cp_sf(tsfb + 8u * a, sdesc_sf_tile(sSFB + 512u * a));
                        tc_cp_sf(tsfb + 8u * a + 4u, sdesc_sf_tile(sSFB + 4u * 512u + 512u * a));
                    }
                    tc_commit(sf_full0 + 8u * stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            tc_commit(sf_drain_bar);
            drain_wait(sf_drain_bar, 0, p.err);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - kEpiWarp0; // 0..7
        const int sub = warp & 3;        // TMEM lane group this warp may read
        const int half = ew >> 2;        // column half of the tile
        const float alpha = __frcp_rn(__fmul_rn(*p.s_enc_a, *p.s_enc_b));
        const bool vec_ok = (p.ldy % 8) == 0;
        uint32_t acc_phase = 0;
        float hmax = 0.0f;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
            int tm, tn;
            tile_coords(t, p.tiles_m, p.tiles_n, tm, tn);
            // warp-uniform decision: the TMEM loads below are .sync.aligned
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(acc_full, acc_phase, abort_flag, p.err))) break;
            tc_fence_after();
            const int row = tm * 128 + sub * 32 + lane;
            const uint32_t tbase = tmem + (static_cast<uint32_t>(sub * 32) << 16);
            if (!kSwiglu) {
                uint32_t packed[64];
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
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
                const int n0 = tn * 256 + half * 128;
                if (row < p.M && n0 < p.N)
                    store_row<128>(p.y + static_cast<int64_t>(row) * p.ldy + n0, packed, p.N - n0,
                                   vec_ok);
            } else {
                uint32_t packed[32];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t rg[32], ru[32];
                    tmem_ld32(tbase + half * 64 + c * 32, rg);
                    tmem_ld32(tbase + 128 + half * 64 + c * 32, ru);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float hv[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const float g = bf16_round(__fmul_rn(alpha, __uint_as_float(rg[2 * j + e])));
                            const float u = bf16_round(__fmul_rn(alpha, __uint_as_float(ru[2 * j + e])));
                            const float silu = __fdiv_rn(g, __fadd_rn(1.0f, expf(-g)));
                            hv[e] = __fmul_rn(silu, u);
                        }
                        packed[c * 16 + j] = pack_bf16x2(hv[0], hv[1]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
                const int n0 = tn * 128 + half * 64;
                if (row < p.M) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&packed[i]);
                        hmax = fmaxf(hmax, fmaxf(fabsf(__bfloat162float(v.x)),
                                                 fabsf(__bfloat162float(v.y))));
                    }
                    store_row<64>(p.y + static_cast<int64_t>(row) * p.ldy + n0, packed, 64, true);
                }
            }
            acc_phase ^= 1u;
        }
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
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool encode_codes_tmap(CUtensorMap *map, const void *codes, int64_t rows, int64_t K) {
    using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !ptr)
            return false;
        fn = reinterpret_cast<EncodeFn>(ptr);
    }
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    const cuuint32_t box[2] = {128, 128};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(codes), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_gemm_nvf4(const CUtensorMap &tmap_a, const CUtensorMap &tmap_b,
                             const GemmArgs &a, bool swiglu, int num_sms, int *grid_out,
                             cudaStream_t s) {
    Params p;
    p.sfa = a.sfa;
    p.sfb = a.sfb;
    p.s_enc_a = a.s_enc_a;
    p.s_enc_b = a.s_enc_b;
    p.y = static_cast<__nv_bfloat16 *>(a.y);
    p.ldy = a.ldy;
    p.M = a.M;
    p.N = a.N;
    p.K = a.K;
    p.tiles_m = (a.M + 127) / 128;
    p.n_half = a.N / 2;
    p.tiles_n = swiglu ? p.n_half / 128 : (a.N + 255) / 256;
    p.sf_ktiles = a.K / 64;
    p.k_tiles = (p.sf_ktiles + 3) / 4;
    p.sf_rowblocks_b = (a.N + 127) / 128;
    p.amax_partials = a.amax_partials;
    p.err = a.err;
    const int tiles = p.tiles_m * p.tiles_n;
    int grid = tiles < num_sms ? tiles : num_sms;
    if (grid < 1) grid = 1;
    if (grid_out) *grid_out = grid;
    cudaError_t e;
    if (swiglu) {
        e = cudaFuncSetAttribute(gemm_nvf4_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes);
        if (e != cudaSuccess) return e;
        gemm_nvf4_kernel<true><<<grid, kThreads, kSmemBytes, s>>>(tmap_a, tmap_b, p);
    } else {
        e = cudaFuncSetAttribute(gemm_nvf4_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes);
        if (e != cudaSuccess) return e;
        gemm_nvf4_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(tmap_a, tmap_b, p);
    }
    return cudaGetLastError();
}

}  // namespace mq
