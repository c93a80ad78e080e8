// mq_decode_tc.cu -- W4A4 decode linear for up to 16 tokens on the tcgen05
// tensor cores: the tokens X [M, K] (BF16) are quantized to NVFP4 inside the
// kernel with the prefill recipe (one tensor scale s_enc_x from max |X|,
// E4M3 scales per 16, E2M1 codes), then
// Y = bf16(alpha * sum_k e2m1(x) dec(sx) e2m1(w) dec(sw)),
// alpha = 1 / (s_enc_x * s_enc_w).
//
// Method: the decode half of uniform NVFP4 quantization, which the Mix-Quant
// pages set against their phase-aware scheme (gist.science technical summary,
// section 1 "Problem Statement" and section 4 "Experimental Results"), on
// the same weight handle's NVFP4 copy.
//
// The op streams the NVFP4 weight once (0.5625 byte per parameter); the
// tensor core does the E2M1 decoding and the block scaling that an FP16 MMA
// path spends most of its instructions on.  Each CTA quantizes the tokens
// only over the K stages its units cover, and that NVFP4 form must fit in
// shared memory (M x stages x 144 bytes <= kDecodeTcTokenSmem).  The weight is the
// MMA's A operand (M = 128 weight rows) and the tokens its B operand (N = 16;
// token rows past M stay zero), K = 64 per instruction with one UE4M3 scale
// per 16 K.  Work unit: one 128-row weight tile x one 256-wide K stage; the
// flattened (tile, stage) sequence is split into equal contiguous ranges, one
// per CTA (one CTA per SM), so every SM streams the same bytes.  Each CTA's
// few stages are short next to its fixed path (set-up, the first TMA round
// trip, the token quantization, the accumulator hand-off and the cross-CTA
// reduction), so the library uses it for up to 4 tokens and for 9 to 16; for
// 5 to 8 the FP16-MMA kernel is used.
//
// CTA roles (9 warps):
//   warp 0     TMA producer: weight codes [128 x 128 B] (128-byte swizzle)
//              and the 512-byte weight scale tiles (bulk copies) into an
//              8-stage ring.  The weight is constant for the call, so this
//              warp starts before the wait for the preceding kernel.
//   warps 2-5, 7-8  first, together: max |X| over all tokens (every CTA
//              computes it), the scale table, and X quantized into shared
//              memory over the K stages of this CTA's units (codes, then
//              scales, stage-major per token row), while the weight streams in.
//   warps 7-8  then per stage: the token codes copied into the swizzled image
//              the MMA reads and the token scales into their 512-byte tiles.
//   warp 6     scale copier: copies a stage's scale tiles into tensor memory
//              (tcgen05.cp) and signals them with a tcgen05 commit.
//   warp 1     MMA issuer: the stage's MMAs into one of two 128 x 16 FP32
//              accumulators; after the last stage of a tile in its range it
//              hands the accumulator to the epilogue and continues in the
//              other one.
//   warps 2-5  epilogue: one TMEM lane quarter (32 weight rows) each.  A tile
//              covered by one CTA is written directly; otherwise each covering
//              CTA stores its partial sums in the tile's slot for it and the
//              last CTA to arrive (atomic counter, reset by it) adds the slots
//              in CTA order -- deterministically -- and writes BF16.
// Every mbarrier wait is bounded; on a timeout the kernel latches an error
// bit, stops issuing work, lets in-flight copies and MMAs land, frees its
// tensor memory and exits.
#include <cuda_bf16.h>

#include "mq_internal.h"
#include "mq_nvfp4.cuh"
#include "mq_ptx.cuh"

namespace mq {

namespace {

constexpr int kStages = 8;
constexpr int kTokens = 16;                       // the MMA's N
constexpr uint32_t kABytes = 128 * 128;           // 128 weight rows x 128 B (256 fp4)
constexpr uint32_t kBBytes = kTokens * 128;       // 16 token rows x 128 B
constexpr uint32_t kSfBytes = 4 * 512;            // 4 scale tiles (K = 256)
constexpr uint32_t kStageBytes = kABytes + kBBytes + 2 * kSfBytes;   // 22528
constexpr uint32_t kBarBytes = 512;
constexpr uint32_t kTabBytes = 128 * 4 + 64;      // scale table + reduction scratch
constexpr uint32_t kTokOff = kStages * kStageBytes + kBarBytes + kTabBytes;   // quantized tokens
constexpr uint32_t kSmemFixed = kTokOff + 1024;   // + the tokens' bytes (decode_tc_token_bytes)
constexpr uint32_t kSmemMax = kSmemFixed + static_cast<uint32_t>(kDecodeTcTokenSmem);
constexpr int kProducer = 0, kMma = 1, kEpi0 = 2, kCopier = 6, kQuant0 = 7;
constexpr int kThreads = 9 * 32;
constexpr int kQuantThreads = 64;
constexpr int kPrologueThreads = 192;             // epilogue + quantizer warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 32;                 // two accumulators at columns 0 and 32
constexpr uint32_t kSfCol = 2 * kAccCols;         // per-stage scale slots follow
constexpr uint32_t kSfColsPerStage = 32;          // 16 for the weight, 16 for the tokens
// named barriers (id 0 is __syncthreads)
constexpr uint32_t kBarEpi = 1;                   // the 128 epilogue threads
constexpr uint32_t kBarTok = 2;                   // the 192 threads quantizing the tokens

static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
static_assert(kTokOff % 16 == 0, "token buffer alignment");
static_assert(kSmemMax <= 227 * 1024, "shared memory budget");
static_assert(kSfCol + kStages * kSfColsPerStage <= kTmemCols, "TMEM budget");

struct TcParams {
    const uint4 *x;            // [M, K] BF16 tokens
    const uint8_t *w_sf;       // swizzled weight scales
    const float *s_enc_w;
    __nv_bfloat16 *y;          // [M, N]
    float *partials;           // [tiles][slots][16 tokens][128 rows]
    unsigned *counters;        // one per tile, zero between calls
    unsigned *err;
    int M, N, K;
    int kst;                   // K stages of 256
    int sf_ktiles;             // K / 64
    int slots;
    int64_t total;             // tiles x kst
};

// 32 TMEM lanes x 16 consecutive 32-bit columns: thread t of the warp gets
// lane (the warp's lane quarter base + t), columns [col, col + 16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// A whole 256-wide K stage from one thread in one issue block: four such MMAs
// (K = 64 each: descriptors 32 bytes = 2 units apart, scale columns 4 apart),
// the first accumulating only if `accumulate`, then a commit to `bar`.
__device__ __forceinline__ void tc_mma4_nvf4_commit(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                    uint32_t idesc, uint32_t sfa_tmem,
                                                    uint32_t sfb_tmem, uint32_t accumulate,
                                                    uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred p, t;\n\t"
        ".reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
        ".reg .b32 sa1, sa2, sa3, sb1, sb2, sb3;\n\t"
        "setp.ne.b32 p, %4, 0;\n\tsetp.eq.b32 t, 0, 0;\n\t"
        "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"
        "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
        "add.u32 sa1, %5, 4;\n\tadd.u32 sa2, %5, 8;\n\tadd.u32 sa3, %5, 12;\n\t"
        "add.u32 sb1, %6, 4;\n\tadd.u32 sb2, %6, 8;\n\tadd.u32 sb3, %6, 12;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], a1, b1, %3, [sa1], [sb1], t;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], a2, b2, %3, [sa2], [sb2], t;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], a3, b3, %3, [sa3], [sb3], t;\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%7];\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem), "r"(bar)
        : "memory");
}

// The four A and four B scale tiles of a 256-wide K stage (512-byte tiles,
// 32 descriptor units apart) into TMEM columns 4 apart, then a commit to
// `bar`, from one thread in one issue block.
__device__ __forceinline__ void tc_cp8_sf_commit(uint32_t tsa, uint32_t tsb, uint64_t da, uint64_t db,
                                                 uint32_t bar) {
    asm volatile(
        "{\n\t.reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
        ".reg .b32 ta1, ta2, ta3, tb1, tb2, tb3;\n\t"
        "add.s64 a1, %2, 32;\n\tadd.s64 a2, %2, 64;\n\tadd.s64 a3, %2, 96;\n\t"
        "add.s64 b1, %3, 32;\n\tadd.s64 b2, %3, 64;\n\tadd.s64 b3, %3, 96;\n\t"
        "add.u32 ta1, %0, 4;\n\tadd.u32 ta2, %0, 8;\n\tadd.u32 ta3, %0, 12;\n\t"
        "add.u32 tb1, %1, 4;\n\tadd.u32 tb2, %1, 8;\n\tadd.u32 tb3, %1, 12;\n\t"
        "tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %2;\n\t"
        "tcgen05.cp.cta_group::1.32x128b.warpx4 [%1], %3;\n\t"
        "tcgen05.cp.cta_group::1.32x128b.warpx4 [ta1], a1;\n\t"
        "tcgen05.cp.cta_group::1.32x128b.warpx4 [tb1], b1;\n\t"
        "tcgen05.cp.cta_group::1.32x128b.warpx4 [ta2], a2;\n\t"
        "tcgen05.cp.cta_group::1.32x128b.warpx4 [tb2], b2;\n\t"
        "tcgen05.cp.cta_group::1.32x128b.warpx4 [ta3], a3;\n\t"
        "tcgen05.cp.cta_group::1.32x128b.warpx4 [tb3], b3;\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%4];\n\t}" ::"r"(tsa),
        "r"(tsb), "l"(da), "l"(db), "r"(bar)
        : "memory");
}

// CTA that owns flattened unit u when `total` units are split over `g` CTAs,
// CTA c taking [floor(total c / g), floor(total (c + 1) / g)).
__device__ __forceinline__ int64_t owner_cta(int64_t u, int64_t total, int64_t g) {
    return ((u + 1) * g - 1) / total;
}

// Named barrier over `n` threads, and the same returning the AND of `pred`
// over them.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool named_bar_and(uint32_t id, uint32_t n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred a, b;\n\tsetp.ne.b32 a, %1, 0;\n\t"
        "bar.red.and.pred b, %2, %3, a;\n\tselp.u32 %0, 1, 0, b;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// Time-bounded wait that ignores the abort flag: lets in-flight asynchronous
// work signalling `bar` land before the CTA exits.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, unsigned *err) {
    const unsigned long long t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            atomicOr(err, kDevErrTimeout);
            return;
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    decode_nvf4_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, const TcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
    // barriers: full[s] (weight bytes), xq[s] (token operands written),
    // sf_full[s] (scales in TMEM), empty[s] (MMAs done), acc_full[2], acc_empty[2], drain x2
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * kStages + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *last_flag = reinterpret_cast<volatile int *>(tmem_slot + 2);
    float *ftab = reinterpret_cast<float *>(smem + kStages * kStageBytes + kBarBytes);
    float *red = ftab + 128;   // 6 floats
    uint8_t *xs = smem + kTokOff;   // this CTA's K stages of the tokens: codes, then scales

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t full0 = smem_u32(bars);                 // full[s]      = full0 + 8 s
    const uint32_t xq0 = full0 + 8u * kStages;             // xq[s]
    const uint32_t sff0 = xq0 + 8u * kStages;              // sf_full[s]
    const uint32_t empty0 = sff0 + 8u * kStages;           // empty[s]
    const uint32_t accf0 = empty0 + 8u * kStages;          // acc_full[b]  = accf0 + 8 b
    const uint32_t acce0 = accf0 + 16u;                    // acc_empty[b] = acce0 + 8 b
    const uint32_t drain_mma = acce0 + 16u;
    const uint32_t drain_cp = drain_mma + 8u;
    const uint32_t smem0 = smem_u32(smem);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full0 + 8u * s, 1);
            mbar_init(xq0 + 8u * s, 2);      // the two quantizer warps
            mbar_init(sff0 + 8u * s, 1);
            mbar_init(empty0 + 8u * s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(accf0 + 8u * b, 1);
            mbar_init(acce0 + 8u * b, 4);    // the four epilogue warps
        }
        mbar_init(drain_mma, 1);
        mbar_init(drain_cp, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&tmap_w);
    }
    if (warp == kMma) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_launch_dependents();

    const int64_t G = gridDim.x, cta = blockIdx.x;
    const int64_t u0 = p.total * cta / G, u1 = p.total * (cta + 1) / G;

    if (warp == kProducer) {
        // ------------------------------------------------------------ producer
        // reads only the weight, which no kernel writes: no wait on the
        // preceding kernel
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_parity = 0;
            for (int64_t u = u0; u < u1; ++u) {
                const int tile = static_cast<int>(u / p.kst);
                const int ks = static_cast<int>(u - static_cast<int64_t>(tile) * p.kst);
                if (!mbar_wait(empty0 + 8u * stage, phase ^ 1u, abort_flag, p.err)) break;
                const int natoms = min(4, p.sf_ktiles - 4 * ks);
                const uint32_t sf_bytes = static_cast<uint32_t>(natoms) * 512u;
                const uint32_t full = full0 + 8u * stage;
                mbar_arrive_expect_tx(full, kABytes + sf_bytes);
                armed |= 1u << stage;
                armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                const uint32_t sA = smem0 + static_cast<uint32_t>(stage) * kStageBytes;
                const uint32_t sSA = sA + kABytes + kBBytes;
                tma_load_2d(sA, &tmap_w, ks * 128, tile * 128, full);
                bulk_load(sSA, p.w_sf + (static_cast<int64_t>(tile) * p.sf_ktiles + 4 * ks) * 512,
                          sf_bytes, full);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            // every issued copy lands before the CTA may exit
            for (int s = 0; s < kStages; ++s)
                if (armed & (1u << s)) drain_wait(full0 + 8u * s, (armed_parity >> s) & 1u, p.err);
        }
    } else if (warp == kCopier) {
        // ------------------------------------------------------------ scale copier
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int64_t u = u0; u < u1; ++u) {
                const int tile = static_cast<int>(u / p.kst);
                const int ks = static_cast<int>(u - static_cast<int64_t>(tile) * p.kst);
                if (!mbar_wait(full0 + 8u * stage, phase, abort_flag, p.err)) break;
                if (!mbar_wait(xq0 + 8u * stage, phase, abort_flag, p.err)) break;
                tc_fence_after();
                const int natoms = min(4, p.sf_ktiles - 4 * ks);
                const uint32_t sSA = smem0 + static_cast<uint32_t>(stage) * kStageBytes + kABytes + kBBytes;
                const uint32_t sSB = sSA + kSfBytes;
                const uint32_t tsa = tmem + kSfCol + static_cast<uint32_t>(stage) * kSfColsPerStage;
                const uint32_t tsb = tsa + 16u;
                if (natoms == 4) {
                    tc_cp8_sf_commit(tsa, tsb, sdesc_sf_tile(sSA), sdesc_sf_tile(sSB), sff0 + 8u * stage);
                } else {
                    for (int kb = 0; kb < natoms; ++kb) {
                        tc_cp_sf(tsa + 4u * kb, sdesc_sf_tile(sSA + 512u * kb));
                        tc_cp_sf(tsb + 4u * kb, sdesc_sf_tile(sSB + 512u * kb));
                    }
                    tc_commit(sff0 + 8u * stage);
                }
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            tc_commit(drain_cp);
            drain_wait(drain_cp, 0, p.err);
        }
    } else if (warp == kMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_nvf4(128, kTokens);
            int stage = 0;
            uint32_t phase = 0, buf = 0, use_par = 0;
            bool ok = true;
            int64_t u = u0;
            while (u < u1 && ok) {
                const int64_t tile = u / p.kst;
                const int64_t seg_end = u1 < (tile + 1) * p.kst ? u1 : (tile + 1) * p.kst;
                // the epilogue has read this accumulator's previous tile
                if (!mbar_wait(acce0 + 8u * buf, ((use_par >> buf) & 1u) ^ 1u, abort_flag, p.err)) break;
                tc_fence_after();
                const uint32_t dacc = tmem + buf * kAccCols;
                uint32_t accumulate = 0;
                for (; u < seg_end; ++u) {
                    // operands in shared memory and scales in TMEM (the copier
                    // waited for the operands before copying)
                    if (!mbar_wait(sff0 + 8u * stage, phase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int ks = static_cast<int>(u - tile * p.kst);
                    const int natoms = min(4, p.sf_ktiles - 4 * ks);
                    const uint32_t sA = smem0 + static_cast<uint32_t>(stage) * kStageBytes;
                    const uint32_t sB = sA + kABytes;
                    const uint32_t tsa = tmem + kSfCol + static_cast<uint32_t>(stage) * kSfColsPerStage;
                    const uint32_t tsb = tsa + 16u;
                    if (natoms == 4) {   // the stage's MMAs and the commit that frees it
                        tc_mma4_nvf4_commit(dacc, sdesc_kmajor_sw128(sA), sdesc_kmajor_sw128(sB), idesc, tsa, tsb,
                                            accumulate, empty0 + 8u * stage);
                        accumulate = 1;
                    } else {
                        for (int kb = 0; kb < natoms; ++kb) {
                            tc_mma_nvf4(dacc, sdesc_kmajor_sw128(sA + 32u * kb),
                                        sdesc_kmajor_sw128(sB + 32u * kb), idesc, tsa + 4u * kb,
                                        tsb + 4u * kb, accumulate);
                            accumulate = 1;
                        }
                        tc_commit(empty0 + 8u * stage);   // frees the stage
                    }
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(accf0 + 8u * buf);
                use_par ^= 1u << buf;
                buf ^= 1u;
            }
            // every MMA issued by this thread completes before TMEM is freed
            tc_commit(drain_mma);
            drain_wait(drain_mma, 0, p.err);
        }
    } else {
        // ------------------------------------------------------------ tokens
        // The four epilogue and the two quantizer warps quantize all M x K
        // tokens into shared memory first (prefill recipe: tensor amax over
        // X, scale table, 16-element blocks), while the producer already
        // streams the weight.
        const int j = warp >= kQuant0 ? 128 + (threadIdx.x - kQuant0 * 32) : threadIdx.x - kEpi0 * 32;
        griddep_wait();   // X comes from the preceding kernel; y and the scratch may be in use
        // token rows M .. 15 of every stage's operands stay zero
        for (int s = 0; s < kStages; ++s) {
            uint8_t *sB = smem + s * kStageBytes + kABytes;
            for (uint32_t i = j * 16u; i < kBBytes + 2 * kSfBytes; i += kPrologueThreads * 16u)
                if (i < kBBytes || i >= kBBytes + kSfBytes)   // skip the weight scale slot
                    *reinterpret_cast<uint4 *>(sB + i) = make_uint4(0, 0, 0, 0);
        }
        // max |X| over all tokens: every CTA reads all of X (from L2), 16
        // loads in flight per thread (with 4, 8 tokens x K = 14336 took ~19
        // dependent rounds of L2 latency)
        const uint32_t vecs = static_cast<uint32_t>(p.M) * static_cast<uint32_t>(p.K / 8);
        uint32_t mx = 0;
        for (uint32_t i0 = j; i0 < vecs; i0 += 16u * kPrologueThreads) {
            uint4 v[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint32_t i = i0 + k * kPrologueThreads;
                v[k] = i < vecs ? __ldg(p.x + i) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int k = 0; k < 16; ++k) mx = max(mx, absmax8_bits(v[k]));
        }
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        if (lane == 0) red[j >> 5] = __uint_as_float(mx << 16);
        named_bar_sync(kBarTok, kPrologueThreads);
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < kPrologueThreads / 32; ++k) amax = fmaxf(amax, red[k]);
        const float s_enc = nvfp4_tensor_scale(amax);
        nvfp4_scale_table(s_enc, ftab, static_cast<uint32_t>(j), kPrologueThreads);
        named_bar_sync(kBarTok, kPrologueThreads);   // table complete
        // Only the K stages this CTA's units cover are quantized (all of them
        // once the range spans a whole tile), into a compact buffer: stage ks
        // at slot so = (ks - ks0) mod kst, token row m holding n_st stages.
        // Entry i = (m n_st + so) 16 + bb is 16-block bb of that stage:
        // codes at 8 i, scale byte at xs_sf + i.
        const uint32_t kb16 = static_cast<uint32_t>(p.K / 16);   // 16-blocks per token row
        const int64_t nu = u1 - u0;
        const int n_st = nu >= p.kst ? p.kst : static_cast<int>(nu);
        const int ks0 = nu >= p.kst ? 0 : static_cast<int>(u0 % p.kst);
        const uint32_t per_row = static_cast<uint32_t>(n_st) * 16u;   // blocks per token row
        const uint32_t nblk = static_cast<uint32_t>(p.M) * per_row;
        uint8_t *xs_sf = xs + 8u * nblk;
        // every stage, and whole stages of 16 blocks: entry i is block i of X
        // (the loop without the compact index arithmetic, which measured
        // ~0.6 us slower on the 8B gate/up weight at one token)
        const bool whole = n_st == p.kst && per_row == kb16;
        auto quant_entry = [&](uint32_t i, const uint4 &a0, const uint4 &a1) {
            const uint32_t w8[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            uint32_t lo, hi, sb;
            quantize_block16<true>(w8, s_enc, ftab, lo, hi, sb);
            *reinterpret_cast<uint2 *>(xs + 8u * i) = make_uint2(lo, hi);
            xs_sf[i] = static_cast<uint8_t>(sb);
        };
        if (whole) {
            for (uint32_t i0 = j; i0 < nblk; i0 += 4u * kPrologueThreads) {
                uint4 v[4][2];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t i = i0 + k * kPrologueThreads;
                    v[k][0] = v[k][1] = make_uint4(0, 0, 0, 0);
                    if (i < nblk) {
                        v[k][0] = __ldg(p.x + 2u * i);
                        v[k][1] = __ldg(p.x + 2u * i + 1u);
                    }
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t i = i0 + k * kPrologueThreads;
                    if (i >= nblk) break;
                    quant_entry(i, v[k][0], v[k][1]);
                }
            }
        } else {
            for (uint32_t i0 = j; i0 < nblk; i0 += 4u * kPrologueThreads) {
                uint4 v[4][2];
                bool valid[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t i = i0 + k * kPrologueThreads;
                    v[k][0] = v[k][1] = make_uint4(0, 0, 0, 0);
                    valid[k] = false;
                    if (i < nblk) {
                        const uint32_t m = i / per_row, rem = i - m * per_row;
                        int ks = ks0 + static_cast<int>(rem >> 4);
                        if (ks >= p.kst) ks -= p.kst;
                        const uint32_t b = static_cast<uint32_t>(ks) * 16u + (rem & 15u);
                        if (b < kb16) {   // a partial last K stage has fewer blocks
                            const uint32_t gi = m * kb16 + b;   // block of X, row-major
                            v[k][0] = __ldg(p.x + 2u * gi);
                            v[k][1] = __ldg(p.x + 2u * gi + 1u);
                            valid[k] = true;
                        }
                    }
                }
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (valid[k]) quant_entry(i0 + k * kPrologueThreads, v[k][0], v[k][1]);
            }
        }
        named_bar_sync(kBarTok, kPrologueThreads);   // tokens quantized

        if (warp >= kQuant0) {
            // -------------------------------------------------------- quantizers:
            // each stage's token operands from the quantized tokens: codes into
            // the swizzled image the MMA reads (16-byte chunks of a 128-byte
            // row XORed with the row index mod 8), scales into the 512-byte tiles
            const int qt = threadIdx.x - kQuant0 * 32;   // 0 .. 63
            const uint32_t rowc = per_row * 8u;   // code bytes per token row in the buffer
            int stage = 0;
            uint32_t phase = 0;
            for (int64_t u = u0; u < u1; ++u) {
                const int tile = static_cast<int>(u / p.kst);
                const int ks = static_cast<int>(u - static_cast<int64_t>(tile) * p.kst);
                if (!warp_mbar_wait(empty0 + 8u * stage, phase ^ 1u, abort_flag, p.err)) break;
                const int natoms = min(4, p.sf_ktiles - 4 * ks);
                const int so = ks >= ks0 ? ks - ks0 : ks - ks0 + p.kst;   // slot in the buffer
                uint8_t *sB = smem + stage * kStageBytes + kABytes;
                uint8_t *sSB = sB + kBBytes + kSfBytes;
                const int chunks = natoms * 2;   // 16-byte code chunks per token row
                for (int it = qt; it < p.M * chunks; it += kQuantThreads) {
                    const int m = it / chunks, c = it - m * chunks;
                    const uint4 v = *reinterpret_cast<const uint4 *>(xs + m * rowc + so * 128 + c * 16);
                    *reinterpret_cast<uint4 *>(sB + m * 128 + ((c ^ (m & 7)) * 16)) = v;
                }
                for (int it = qt; it < p.M * natoms; it += kQuantThreads) {
                    const int m = it / natoms, t4 = it - m * natoms;
                    // scales of blocks 4 t4 .. 4 t4 + 3 of the stage, row m < 32
                    *reinterpret_cast<uint32_t *>(sSB + t4 * 512 + m * 16) =
                        *reinterpret_cast<const uint32_t *>(xs_sf + m * per_row + so * 16 + t4 * 4);
                }
                fence_proxy_async_smem();   // the writes above are read by the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(xq0 + 8u * stage);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                  // TMEM lanes 32 q .. 32 q + 31
        const int t = threadIdx.x - kEpi0 * 32;  // 0 .. 127 over the four warps
        const float alpha = __frcp_rn(__fmul_rn(s_enc, *p.s_enc_w));
        uint32_t buf = 0, use_par = 0;
        int64_t u = u0;
        while (u < u1) {
            const int64_t tile = u / p.kst;
            u = u1 < (tile + 1) * p.kst ? u1 : (tile + 1) * p.kst;
            // the four warps agree on going on (the barriers below need all of them)
            const bool ok = warp_mbar_wait(accf0 + 8u * buf, (use_par >> buf) & 1u, abort_flag, p.err);
            if (!named_bar_and(kBarEpi, 128, ok)) break;
            tc_fence_after();
            uint32_t r[kTokens];   // r[m]: row 128 tile + 32 q + lane, token m
            tmem_ld16(tmem + (static_cast<uint32_t>(32 * q) << 16) + buf * kAccCols, r);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce0 + 8u * buf);
            use_par ^= 1u << buf;
            buf ^= 1u;
            const int64_t cf = owner_cta(tile * p.kst, p.total, G);
            const int nw = static_cast<int>(owner_cta(tile * p.kst + p.kst - 1, p.total, G) - cf + 1);
            const int row = static_cast<int>(tile) * 128 + 32 * q + lane;
            if (nw == 1) {
#pragma unroll
                for (int m = 0; m < kTokens; ++m)
                    if (m < p.M && row < p.N)
                        p.y[static_cast<int64_t>(m) * p.N + row] =
                            __float2bfloat16_rn(__fmul_rn(alpha, __uint_as_float(r[m])));
                continue;
            }
            float *grp = p.partials + tile * p.slots * (kTokens * 128);
            float *mine = grp + (cta - cf) * (kTokens * 128) + 32 * q + lane;
#pragma unroll
            for (int m = 0; m < kTokens; ++m)
                if (m < p.M) mine[m * 128] = __uint_as_float(r[m]);
            __threadfence();
            named_bar_sync(kBarEpi, 128);
            if (t == 0) *last_flag = atomicAdd(p.counters + tile, 1u) == static_cast<unsigned>(nw - 1);
            named_bar_sync(kBarEpi, 128);
            if (!*last_flag) continue;
            // the last of the nw CTAs covering the tile: thread t adds row t of
            // the nw slots in CTA order
            __threadfence();
            const int rr = static_cast<int>(tile) * 128 + t;
            for (int m = 0; m < p.M; ++m) {
                const float *src = grp + m * 128 + t;
                float sum = 0.0f;
#pragma unroll 4
                for (int k = 0; k < nw; ++k) sum += __ldcg(src + k * (kTokens * 128));
                if (rr < p.N)
                    p.y[static_cast<int64_t>(m) * p.N + rr] = __float2bfloat16_rn(__fmul_rn(alpha, sum));
            }
            if (t == 0) p.counters[tile] = 0u;   // ready for the next call
        }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

namespace {

struct TcSplit {
    int64_t tiles, total;
    int kst, sf_ktiles, ctas, slots;
};

TcSplit tc_split(int64_t N, int64_t K, int num_sms) {
    TcSplit d;
    d.tiles = (N + 127) / 128;
    d.sf_ktiles = static_cast<int>(K / 64);
    d.kst = (d.sf_ktiles + 3) / 4;
    d.total = d.tiles * d.kst;
    const int64_t g = d.total < num_sms ? d.total : num_sms;
    d.ctas = static_cast<int>(g);
    // ranges hold r = floor(total / g) >= 1 units or one more; the kst units
    // of a tile meet at most ceil(kst / r) + 1 of them
    const int64_t r = d.total / g;
    int64_t slots = (d.kst + r - 1) / r + 1;
    if (slots > d.kst) slots = d.kst;
    d.slots = static_cast<int>(slots);
    return d;
}

}  // namespace

size_t decode_tc_token_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
    // a CTA's range holds floor(total / ctas) units or one more, so it meets
    // at most that many K stages (or all kst of them); 144 bytes per token
    // and K stage (128 of codes, 16 of scales)
    const TcSplit d = tc_split(N, K, num_sms);
    int64_t n_st = d.total / d.ctas + 1;
    if (n_st > d.kst) n_st = d.kst;
    return static_cast<size_t>((M * n_st * 144 + 15) / 16 * 16);
}

size_t decode_tc_partial_floats(int64_t N, int64_t K, int num_sms) {
    const TcSplit d = tc_split(N, K, num_sms);
    return static_cast<size_t>(d.tiles) * d.slots * kTokens * 128;
}

cudaError_t launch_decode_nvf4_tc(const CUtensorMap &tmap_w, const uint8_t *w_sf,
                                  const float *s_enc_w, int64_t N, int64_t K, const void *x_bf16,
                                  int64_t M, void *y, void *scratch, unsigned *err, int num_sms,
                                  cudaStream_t s) {
    const size_t tok = decode_tc_token_bytes(M, N, K, num_sms);
    if (M < 1 || M > kDecodeTcTokens || tok > kDecodeTcTokenSmem) return cudaErrorInvalidValue;
    const TcSplit d = tc_split(N, K, num_sms);
    TcParams p;
    p.x = static_cast<const uint4 *>(x_bf16);
    p.w_sf = w_sf;
    p.s_enc_w = s_enc_w;
    p.y = static_cast<__nv_bfloat16 *>(y);
    p.counters = static_cast<unsigned *>(scratch);
    p.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(scratch) + decode_counter_bytes(N));
    p.err = err;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.kst = d.kst;
    p.sf_ktiles = d.sf_ktiles;
    p.slots = d.slots;
    p.total = d.total;
    // the same value on every call: concurrent callers cannot undo each other
    cudaError_t e = cudaFuncSetAttribute(decode_nvf4_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemMax));
    if (e != cudaSuccess) return e;
    e = launch_pdl(decode_nvf4_tc_kernel, dim3(d.ctas), dim3(kThreads), kSmemFixed + tok, s, tmap_w,
                   p);
    return e == cudaSuccess ? cudaGetLastError() : e;
}

}  // namespace mq
