/*
 * mq.h -- C ABI of libmq, the B200 (sm_100a) library for the prefill-phase
 * NVFP4 linear layer of Mix-Quant and the BF16 decode linear on the same
 * weights.
 *
 * Method (pages describing "Mix-Quant: Quantized Prefilling, Precise Decoding
 * for Agentic LLMs", arXiv 2605.20315):
 *   - gist.science technical summary, section 2 "Hybrid Precision Strategy":
 *     prefill runs NVFP4 for weights and activations (local scale per group of
 *     16 elements plus a tensor-level scale, round-to-nearest quantization);
 *     decoding keeps BF16.
 *   - same section, "System-Level Deployment": the prefill path is W4A4.
 *   - zingnex.cn forum post, section "动态精度切换" (dynamic precision
 *     switch): weights are stored in a quickly convertible form; activations
 *     are converted at the phase boundary.  Here one weight handle holds both
 *     the BF16 and the NVFP4 copy, and every prefill call quantizes its BF16
 *     activations on the fly.
 * Encoding (the pages name NVFP4 but not its fields): E2M1 elements, one E4M3
 * block scale per 16 contiguous K-elements, one FP32 tensor scale,
 * round-to-nearest-even.  Tensor scale s_enc = 2688 / amax (1 when amax is 0);
 * block scale sb = E4M3(amax_b / 6 * s_enc); element code = E2M1(x * s_enc /
 * dec(sb)); the GEMM output is Y = bf16(acc / (s_enc_x * s_enc_w)).
 *
 * Conventions for every entry point:
 *   - Matrices are row-major with K contiguous: X [M, K], W [N, K],
 *     Y = X * W^T [M, N].  BF16 values are passed as raw 16-bit storage.
 *   - Pointers marked "device" are CUDA device pointers on the current device,
 *     owned by the caller, 16-byte aligned (else MQ_ERR_ALIGNMENT).
 *   - All work is queued on `stream` (0 = legacy default stream); no call
 *     synchronizes except mq_check, mq_weight_free and mq_weight_pack's
 *     allocation.  Launch failures return MQ_ERR_CUDA.
 *   - K must be a multiple of 64 (MQ_ERR_SHAPE); M, N >= 1.
 *   - The current device must be compute capability 10.0 (B200 class), else
 *     MQ_ERR_UNSUPPORTED_DEVICE.
 *   - Inputs must be finite; NaN / Inf inputs give unspecified codes.
 *   - Kernels that wait on on-chip barriers give up after about two seconds,
 *     latch MQ_ERR_TIMEOUT in a per-device error word and exit; mq_check
 *     reports and clears it.
 */
#ifndef MQ_H
#define MQ_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mq_status {
    MQ_OK = 0,
    MQ_ERR_INVALID_ARG = 1,        /* null pointer, bad size, workspace too small */
    MQ_ERR_SHAPE = 2,              /* K % 64 != 0, M or N < 1, mismatched weights */
    MQ_ERR_ALIGNMENT = 3,          /* a pointer or leading dimension is misaligned */
    MQ_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not sm_100 */
    MQ_ERR_OOM = 5,                /* mq_weight_pack could not allocate */
    MQ_ERR_CUDA = 6,               /* a CUDA runtime / launch error */
    MQ_ERR_TIMEOUT = 7             /* a kernel's bounded on-chip wait ran out */
} mq_status;

/* Opaque, library-owned dual-precision weight (BF16 copy + NVFP4 copy). */
typedef struct mq_weight mq_weight;

/* Maximum number of partial maxima accepted by mq_quantize_nvfp4. */
#define MQ_AMAX_PARTIALS_MAX 4096

/* Human-readable name of a status code (static string). */
const char *mq_status_string(mq_status s);

/* Synchronizes `stream`, then reads and clears the current device's latched
 * kernel error word: MQ_ERR_TIMEOUT if a bounded wait ran out since the last
 * check, MQ_ERR_CUDA on a CUDA error, else MQ_OK. */
mq_status mq_check(cudaStream_t stream);

/* Diagnostic of the failure-detection path (no counterpart on the pages):
 * queues one tiny kernel that waits, for at most limit_us microseconds
 * (1 .. 2000000), on a barrier phase that nothing completes, then latches
 * the same timeout bit the kernels latch when one of their bounded waits runs
 * out.  The next mq_check on the stream returns MQ_ERR_TIMEOUT (and clears
 * the bit); the device stays usable.  Never faults or hangs the GPU. */
mq_status mq_selftest_bounded_wait(uint32_t limit_us, cudaStream_t stream);

/* ---- weights (zingnex "动态精度切换": store weights convertible) ---------- */

/* Builds a weight handle from a BF16 device matrix w_bf16 [N, K] (copied; the
 * caller keeps ownership of w_bf16).  The handle owns one device allocation
 * holding: the BF16 copy, NVFP4 codes [N, K/2] (element 2j in bits 3:0 of
 * byte j), the E4M3 block scales in the swizzled layout (see
 * mq_quantize_nvfp4) and the FP32 tensor scale.  The quantization runs on
 * `stream`; the handle may be used on that stream immediately.
 * Errors: MQ_ERR_INVALID_ARG, MQ_ERR_SHAPE, MQ_ERR_ALIGNMENT, MQ_ERR_OOM,
 * MQ_ERR_CUDA. */
mq_status mq_weight_pack(const void *w_bf16, int64_t N, int64_t K, cudaStream_t stream,
                         mq_weight **out);

/* Releases the handle's device memory (synchronizes the device).  NULL is
 * accepted. */
mq_status mq_weight_free(mq_weight *w);

/* Read-only device views into a handle (for parity checks and for callers
 * that drive mq_gemm_nvfp4 themselves).  Any output pointer may be NULL. */
mq_status mq_weight_views(const mq_weight *w, int64_t *N, int64_t *K, const void **bf16,
                          const uint8_t **codes, const uint8_t **sf_swizzled,
                          const float **s_enc_dev);

/* ---- activation quantization (gist.science §2: groups of 16 + tensor scale,
 *      round to nearest) ------------------------------------------------- */

/* Size in bytes of the swizzled block-scale buffer for a [rows, K] operand:
 * rows padded to a multiple of 128, K/16 scales padded to a multiple of 4. */
size_t mq_sf_bytes(int64_t rows, int64_t K);

/* Per-tensor absolute maximum of a BF16 device matrix x [M, K] (leading
 * dimension ldx elements, ldx % 8 == 0, ldx >= K).  Writes `n_partials`
 * partial maxima to amax_partials (device, MQ_AMAX_PARTIALS_MAX floats are
 * always enough) -- the tensor maximum is their max.  *n_partials is set on
 * the host before any kernel runs.  K % 8 == 0 suffices here. */
mq_status mq_tensor_amax(const void *x_bf16, int64_t M, int64_t K, int64_t ldx,
                         float *amax_partials, int *n_partials, cudaStream_t stream);

/* amax_out[0] = max(amax_partials[0 .. n_partials)) on the device (one
 * kernel): the tensor amax as one float, for instance to take its max over
 * the token shards of a batch split across GPUs, so that every shard is
 * quantized with the scale of the whole batch (then pass amax_out with
 * n_partials = 1 to mq_quantize_nvfp4).  Both pointers device, 4-byte
 * aligned; 1 <= n_partials <= MQ_AMAX_PARTIALS_MAX. */
mq_status mq_amax_combine(const float *amax_partials, int n_partials, float *amax_out,
                          cudaStream_t stream);

/* NVFP4-quantizes a BF16 device matrix x [M, K] (ldx as above, K % 64 == 0).
 *   amax_partials / n_partials: device array of partial maxima whose max is
 *     the tensor amax (from mq_tensor_amax or a fused epilogue); pass NULL to
 *     have the amax computed here (then `workspace` must hold
 *     MQ_AMAX_PARTIALS_MAX floats; otherwise workspace may be NULL).
 *   codes [M, K/2] (device): byte j of row r = element 2j (bits 3:0) and
 *     element 2j+1 (bits 7:4).
 *   sf_swizzled (device, mq_sf_bytes(M, K) bytes): scale of row r, 16-block c
 *     at ((r/128) * ceil(K/64) + c/4) * 512 + (r%32)*16 + ((r/32)%4)*4 + c%4;
 *     padding bytes are written as 0.
 *   s_enc_dev (device, 1 float): receives the tensor encode scale. */
mq_status mq_quantize_nvfp4(const void *x_bf16, int64_t M, int64_t K, int64_t ldx,
                            uint8_t *codes, uint8_t *sf_swizzled, float *s_enc_dev,
                            const float *amax_partials, int n_partials, void *workspace,
                            size_t ws_bytes, cudaStream_t stream);

/* ---- prefill GEMM (gist.science §2 "System-Level Deployment": W4A4) ------- */

/* Block-scaled FP4 x FP4 GEMM on the tcgen05 tensor cores with FP32
 * accumulation: y[m, n] = bf16( sum_k deq(a)[m,k] * deq(w)[n,k] ) where the
 * activation operand is (a_codes [M, K/2], a_sf_swizzled, *a_s_enc_dev) as
 * written by mq_quantize_nvfp4 and the weight operand is the handle's NVFP4
 * copy.  y (device) is BF16 [M, N] with leading dimension ldy >= N. */
mq_status mq_gemm_nvfp4(const uint8_t *a_codes, const uint8_t *a_sf_swizzled,
                        const float *a_s_enc_dev, int64_t M, const mq_weight *w, void *y_bf16,
                        int64_t ldy, cudaStream_t stream);

/* Gate/up GEMM with the SwiGLU epilogue fused: the handle holds the fused
 * [gate; up] weight (rows 0..N/2-1 gate, N/2..N-1 up; N/2 % 128 == 0), and
 * h[m, j] = bf16( SiLU(g) * u ) with g = bf16(Y[m, j]), u = bf16(Y[m, N/2+j])
 * evaluated in FP32.  h (device) is BF16 [M, N/2] (leading dimension N/2).
 * The maximum |h| is written as *n_partials partial maxima to h_amax_partials
 * (device, MQ_AMAX_PARTIALS_MAX floats), ready for mq_quantize_nvfp4. */
mq_status mq_gemm_nvfp4_swiglu(const uint8_t *a_codes, const uint8_t *a_sf_swizzled,
                               const float *a_s_enc_dev, int64_t M, const mq_weight *w_gate_up,
                               void *h_bf16, float *h_amax_partials, int *n_partials,
                               cudaStream_t stream);

/* Workspace bytes needed by mq_prefill_linear_nvfp4 for an [M, K] activation:
 * codes, swizzled scales, amax partials and the tensor scale. */
size_t mq_workspace_bytes(int64_t M, int64_t K);

/* The prefill linear layer: amax(x) -> NVFP4 quantize(x) -> block-scaled GEMM
 * with the handle's NVFP4 weight.  x (device) BF16 [M, K] contiguous, K = the
 * handle's K; y (device) BF16 [M, N] contiguous.  workspace (device, 256-byte
 * aligned) of at least mq_workspace_bytes(M, K) bytes. */
mq_status mq_prefill_linear_nvfp4(const mq_weight *w, const void *x_bf16, int64_t M,
                                  void *y_bf16, void *workspace, size_t ws_bytes,
                                  cudaStream_t stream);

/* Workspace bytes for mq_prefill_mlp_swiglu_nvfp4 with M tokens, hidden K and
 * intermediate size I (the gate+up weight has 2*I rows). */
size_t mq_mlp_workspace_bytes(int64_t M, int64_t K, int64_t I);

/* SwiGLU MLP prefill: quantize(x) -> gate/up GEMM with the fused SwiGLU
 * epilogue -> quantize(h) with the amax from that epilogue -> down GEMM.
 * x [M, K], y [M, K_out] where K_out = w_down's N; w_gate_up is [2I, K],
 * w_down is [K_out, I].  If h_bf16 is not NULL the intermediate h [M, I] is
 * written there, else into the workspace. */
mq_status mq_prefill_mlp_swiglu_nvfp4(const mq_weight *w_gate_up, const mq_weight *w_down,
                                      const void *x_bf16, int64_t M, void *y_bf16,
                                      void *h_bf16, void *workspace, size_t ws_bytes,
                                      cudaStream_t stream);

/* Size of the fixed device scratch used by mq_prefill_linear_nvfp4_noalloc. */
#define MQ_NOALLOC_SCRATCH_BYTES ((size_t)48 << 20)

/* The prefill linear layer without any device allocation, for callers that
 * cannot allocate device memory at all: a plugin or host program that is
 * handed only its input and output buffers and owns no allocator, or code on
 * a latency-critical path where the implicit device synchronization of
 * cudaMalloc / cudaFree is not acceptable.  The method's pages have no
 * counterpart to this call; it is a deployment convenience.
 *
 * Same computation and arguments as mq_prefill_linear_nvfp4 minus the
 * workspace: the quantized activation (codes, scales, amax partials, tensor
 * scale) lives in one fixed array of MQ_NOALLOC_SCRATCH_BYTES (48 MiB) in the
 * library's device memory, which every GPU that loads libmq keeps until the
 * process exits.  Requests whose workspace would exceed it --
 * mq_workspace_bytes(M, K) > MQ_NOALLOC_SCRATCH_BYTES, e.g. more than about
 * 21800 tokens at K = 4096 -- return MQ_ERR_SHAPE before any work is queued.
 * Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and keeps it for that device's context; the first call
 * after a cudaDeviceReset looks it up again, since the new context may place
 * the library's device memory elsewhere.  Make each such first call before
 * any stream capture begins; a lookup that fails returns MQ_ERR_CUDA and
 * queues no work.
 * All calls on a device share the one array and it keeps the last call's
 * contents (every byte a call reads is written earlier in the same call, so
 * nothing needs clearing).  Calls whose work overlaps on the GPU -- on two
 * streams without ordering, or from two host threads -- race on the array and
 * corrupt each other's results; serialize them. */
mq_status mq_prefill_linear_nvfp4_noalloc(const mq_weight *w, const void *x_bf16, int64_t M,
                                          void *y_bf16, cudaStream_t stream);

/* ---- RMSNorm in front of a prefill linear ----------------------------------
 * Mix-Quant converts activations to NVFP4 at the phase boundary (zingnex.cn
 * forum thread, section "动态精度切换") with one tensor scale from the
 * tensor's amax (gist.science technical summary, section 2 "Hybrid Precision
 * Strategy").  The QKV and gate/up inputs of a transformer layer come out of
 * an RMSNorm; the pages do not define it, the Llama family's is used:
 *   y = bf16( gamma * bf16( x / sqrt(mean(x^2) + eps) ) ) per row (binary32
 *   sum of squares in a fixed order, correctly rounded reciprocal root).
 * Emitting the amax of y on the way out removes the quantizer's own amax pass
 * over the activations. */

/* x (device) BF16 [M, K] (leading dimension ldx, ldx % 8 == 0, K % 8 == 0),
 * gamma (device) BF16 [K], eps >= 0.  Writes y (device, BF16 [M, K]
 * contiguous) and *n_partials partial maxima of |y| to amax_partials (device,
 * MQ_AMAX_PARTIALS_MAX floats are always enough), ready for
 * mq_quantize_nvfp4.  *n_partials is set on the host at once. */
mq_status mq_rmsnorm_amax(const void *x_bf16, const void *gamma_bf16, float eps, int64_t M,
                          int64_t K, int64_t ldx, void *y_bf16, float *amax_partials,
                          int *n_partials, cudaStream_t stream);

/* Prefill linear fed by an RMSNorm: xn = RMSNorm(r) * gamma (written to xn,
 * device BF16 [M, K] contiguous, K = the handle's K) with its amax, NVFP4
 * quantization of xn, block-scaled GEMM with the handle's NVFP4 weight into
 * y (device, BF16 [M, N] contiguous).  r (device) BF16 [M, K] contiguous,
 * gamma (device) BF16 [K].  workspace (device, 256-byte aligned) of at least
 * mq_workspace_bytes(M, K) bytes. */
mq_status mq_prefill_linear_rmsnorm_nvfp4(const mq_weight *w, const void *r_bf16,
                                          const void *gamma_bf16, float eps, int64_t M,
                                          void *xn_bf16, void *y_bf16, void *workspace,
                                          size_t ws_bytes, cudaStream_t stream);

/* ---- decode (gist.science §2: decoding keeps BF16) ----------------------- */

/* BF16 decode linear on the handle's BF16 copy: y[m, n] = bf16( sum_k x[m,k]
 * w[n,k] ) with FP32 accumulation.  x (device) BF16 [M, K] contiguous, y
 * (device) BF16 [M, N] contiguous.  Any M >= 1; meant for M <= 8.  For small
 * N the K range is split across CTAs whose partial sums live in scratch inside
 * the handle, so decode calls on the same handle must not overlap on the GPU
 * (same stream, or ordered streams). */
mq_status mq_decode_linear_bf16(const mq_weight *w, const void *x_bf16, int64_t M, void *y_bf16,
                                cudaStream_t stream);

/* Uniform-NVFP4 decode linear (W4A4), the decode half of quantizing both
 * phases, which the Mix-Quant pages compare their scheme against
 * (gist.science technical summary, section 1 "Problem Statement" and section
 * 4 "Experimental Results"): x is quantized with the prefill recipe (one tensor
 * scale for the call, E4M3 scale per 16, E2M1 codes), then
 * y[m, n] = bf16( sum_k deq(xq)[m,k] deq(wq)[n,k] / (s_enc_x s_enc_w) ) on the
 * handle's NVFP4 copy, FP32 accumulation -- the same arithmetic as
 * mq_prefill_linear_nvfp4, streaming 0.5625 byte per weight instead of 2.
 * x (device) BF16 [M, K] contiguous, y (device) BF16 [M, N] contiguous; any
 * M >= 1, meant for M <= 16.  Up to 4 tokens, and 9 to 16, whose quantized
 * form (M K 9/16 bytes) fits in 40 KB run as one tensor-core kernel that
 * quantizes them in shared memory; up to 8 tokens otherwise as one FP16-MMA
 * kernel that does the same; else x is quantized into `workspace` first.
 * workspace (device, 256-byte aligned) of at least mq_workspace_bytes(M, K)
 * bytes in every case.  Shares the handle's split-K scratch with
 * mq_decode_linear_bf16: decode calls on one handle must not overlap on the
 * GPU. */
mq_status mq_decode_linear_nvfp4(const mq_weight *w, const void *x_bf16, int64_t M, void *y_bf16,
                                 void *workspace, size_t ws_bytes, cudaStream_t stream);

/* ---- attention of the prefill layer and the KV cache the decode step reads --
 * Mix-Quant's prefill builds the KV cache that decoding consumes
 * (gist.science technical summary, section 2 "System-Level Deployment"; the
 * zingnex.cn forum thread, section "动态精度切换", on the cache kept across
 * the two precisions).  The pages do not define the attention; the Llama
 * family's causal softmax attention with grouped KV heads is used, without
 * positional rotation:
 *   o[i, h, :] = sum_{j <= pos(i)} softmax_j( q[i,h,:] . k[j,g,:] / sqrt(D) ) v[j,g,:],
 *   g = h / (H / Hkv).
 * Head dimension D = 128.  The activations use the QKV projection's output
 * layout: qkv (device) BF16 [rows, (H + 2 Hkv) * 128], query heads first, then
 * the Hkv key heads, then the Hkv value heads.  The KV cache is two device
 * BF16 arrays [Hkv, S_max, 128] (key / value of head g at position j at
 * (g * S_max + j) * 128), owned by the caller. */

/* Prefill attention over M tokens (positions 0 .. M-1) on the tensor cores
 * (BF16 products, FP32 softmax and accumulation): writes o (device, BF16
 * [M, H * 128], the O projection's input), keys and values of positions
 * 0 .. M-1 into the cache (k_cache / v_cache may both be NULL to skip it;
 * otherwise M <= S_max), and *n_partials partial maxima of |o| to
 * o_amax_partials (device, MQ_AMAX_PARTIALS_MAX floats), so the O
 * projection's quantizer (mq_quantize_nvfp4 with these partials) skips its
 * amax pass.  *n_partials is set on the host at once.  Requirements: D == 128,
 * H % Hkv == 0, all pointers 16-byte aligned.  Bounded waits: a timeout is
 * latched and reported by mq_check. */
mq_status mq_attention_prefill_bf16(const void *qkv_bf16, int64_t M, int64_t H, int64_t Hkv,
                                    int64_t D, void *k_cache, void *v_cache, int64_t S_max,
                                    void *o_bf16, float *o_amax_partials, int *n_partials,
                                    cudaStream_t stream);

/* Scratch bytes mq_attention_decode_bf16 needs for m new tokens after pos0
 * cached ones (0 for invalid sizes). */
size_t mq_attention_decode_workspace_bytes(int64_t m, int64_t pos0, int64_t H, int64_t Hkv,
                                           int64_t D);

/* Decode-step attention (BF16 cache, FP32 arithmetic) for m new tokens at
 * positions pos0 .. pos0 + m - 1: appends their keys and values (from qkv,
 * device BF16 [m, (H + 2 Hkv) * 128], the BF16 decode QKV projection's
 * output) to the cache, then token t attends over positions 0 .. pos0 + t.
 * Writes o (device, BF16 [m, H * 128]).  Requirements: D == 128,
 * H % Hkv == 0, (H / Hkv) * m <= 64, pos0 + m <= S_max, pointers 16-byte
 * aligned, workspace (device, 16-byte aligned) of at least
 * mq_attention_decode_workspace_bytes(m, pos0, H, Hkv, D) bytes. */
mq_status mq_attention_decode_bf16(const void *qkv_bf16, int64_t m, int64_t pos0, int64_t H,
                                   int64_t Hkv, int64_t D, void *k_cache, void *v_cache,
                                   int64_t S_max, void *o_bf16, void *workspace, size_t ws_bytes,
                                   cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MQ_H */
