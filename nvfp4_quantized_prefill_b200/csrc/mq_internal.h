// mq_internal.h -- launchers shared between the kernel translation units and
// the C-ABI layer.  Not part of the public interface.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <utility>

namespace mq {

// ---- programmatic dependent launch -------------------------------------------
//
// Every kernel of this library is launched with programmatic stream
// serialization: it may start while the previous kernel in the stream is
// finishing (its prologue overlaps that kernel's tail), and it calls
// griddep_wait() before its first access to global memory that an earlier
// kernel may write or read.  griddep_wait() returns once the previous grid has
// completed and its memory is visible; because every kernel waits before its
// own accesses, the ordering carries down the whole stream.  Each kernel
// also allows its successor to launch early (griddep_launch_dependents()).
// Both are no-ops for a kernel launched without the attribute.
#ifdef __CUDACC__
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
#endif

// ---- activation / weight quantization (mq_quant.cu) ------------------------

// Number of CTAs (= partial maxima) the amax kernel uses for an [M, K] input.
int amax_grid(int64_t M, int64_t K, int num_sms);

// Writes `grid` partial maxima of |x| (x: BF16 [M, K], leading dimension ldx).
cudaError_t launch_amax(const void *x, int64_t M, int64_t K, int64_t ldx, float *partials,
                        int grid, cudaStream_t s);

// out[0] = max(partials[0..n)) (one CTA).
cudaError_t launch_amax_combine(const float *partials, int n, float *out, cudaStream_t s);

// NVFP4 quantization with the tensor amax = max(partials[0..n_partials)).
cudaError_t launch_quantize(const void *x, int64_t M, int64_t K, int64_t ldx,
                            const float *partials, int n_partials, uint8_t *codes,
                            uint8_t *sf_swizzled, float *s_enc, int num_sms, cudaStream_t s);

// ---- RMSNorm with the amax of its output (mq_rmsnorm.cu) ----------------------

// Number of CTAs (= partial maxima) the RMSNorm kernel uses for M rows.
int rmsnorm_grid(int64_t M, int64_t K, int num_sms);

// y = RMSNorm(x) * gamma (BF16 [M, K] contiguous) and `grid` partial maxima of
// |y|; x BF16 [M, K] with leading dimension ldx, gamma BF16 [K].
cudaError_t launch_rmsnorm_amax(const void *x, int64_t M, int64_t K, int64_t ldx, const void *gamma,
                                float eps, void *y, float *partials, int grid, cudaStream_t s);

// ---- block-scaled GEMM (mq_gemm.cu) ------------------------------------------

struct GemmArgs {
    const float *s_enc_a;     // device scalars
    const float *s_enc_b;
    void *y;                  // BF16 output
    int64_t ldy;              // output leading dimension (elements)
    int M, N, K;              // N = weight rows (gate+up rows with SwiGLU)
    float *amax_partials;     // SwiGLU: one max |h| per CTA
    unsigned *err;            // device error word
    unsigned long long wait_ns = 0;   // 0: the standard bound of every wait
    int withhold_release = 0;         // test only (mq_debug.h): never free the first stage
};

// Launches the tcgen05 GEMM; *grid_out receives the CTA count (the number of
// amax partials written in SwiGLU mode).
cudaError_t launch_gemm_nvf4(const CUtensorMap &tmap_a, const CUtensorMap &tmap_b,
                             const CUtensorMap &tmap_sfa, const CUtensorMap &tmap_sfb,
                             const GemmArgs &a, bool swiglu, int num_sms, int *grid_out,
                             cudaStream_t s);

// Host-side tensor map over an [rows, K/2]-byte code matrix, 128 x 128-byte
// boxes with 128-byte swizzle.
bool encode_codes_tmap(CUtensorMap *map, const void *codes, int64_t rows, int64_t K);

// Host-side tensor map over a swizzled scale buffer of an [rows, K] operand,
// seen as consecutive 512-byte scale tiles; one box = the 4 tiles of a
// 256-wide K step of one 128-row block.
bool encode_sf_tmap(CUtensorMap *map, const void *sf, int64_t rows, int64_t K);

// ---- attention (mq_attention.cu) ----------------------------------------------

// CTAs of the prefill attention over M tokens and H query heads (head dim 128).
int attention_prefill_grid(int64_t M, int64_t H);
// Prefill attention; k_cache / v_cache NULL: no cache write.  partial_slots 0:
// one amax partial per CTA; > 0: atomic max into that many (zeroed) slots.
cudaError_t launch_attention_prefill(const void *qkv, int64_t M, int64_t H, int64_t Hkv,
                                     void *k_cache, void *v_cache, int64_t S_max, void *o,
                                     float *amax_partials, int partial_slots, unsigned *err,
                                     cudaStream_t s);
size_t attention_decode_workspace_bytes(int64_t m, int64_t pos0, int64_t H, int64_t Hkv);
int attention_decode_max_rows();
// Appends the m new tokens' K / V to the cache, then the decode attention.
cudaError_t launch_attention_decode(const void *qkv, int64_t m, int64_t pos0, int64_t H, int64_t Hkv,
                                    void *k_cache, void *v_cache, int64_t S_max, void *o, void *ws,
                                    cudaStream_t s);

// ---- decode (mq_decode.cu: BF16; mq_decode_nvf4.cu: NVFP4 W4A4) ----------------

// Number of K slices the BF16 / NVFP4 (FP16-MMA) decode splits an [N, K]
// weight into, and the bytes of per-weight decode scratch: one counter per
// 16-row group (decode_counter_bytes, at the start; the counters must start
// at zero and are left at zero by every launch), then the FP32 partial sums
// of whichever decode kernel needs the most (S x 128 per 16-row group, or the
// tensor-core decode's decode_tc_partial_floats).
int decode_slices(int64_t N, int64_t K, int num_sms);
int decode_nvf4_slices(int64_t N, int64_t K, int num_sms);
size_t decode_counter_bytes(int64_t N);
size_t decode_scratch_bytes(int64_t N, int64_t K, int num_sms);

cudaError_t launch_decode(const void *x, int64_t M, const void *w, int64_t N, int64_t K,
                          void *y, void *scratch, int num_sms, cudaStream_t s);

// Largest M x K x 9 / 16 (bytes of the tokens' codes and scales in shared
// memory) for which the W4A4 decode quantizes up to 8 tokens itself.
constexpr size_t kDecodeNvf4TokenSmem = 160 * 1024;

// W4A4 decode, weights from the handle's NVFP4 copy.  With x_bf16 set (M <= 8,
// M x K x 9 / 16 <= kDecodeNvf4TokenSmem) the kernel quantizes the tokens
// itself; otherwise x is given quantized
// (codes, swizzled scales with rows padded to 128, tensor scale).
cudaError_t launch_decode_nvf4(const uint8_t *x_codes, const uint8_t *x_sf, const float *s_enc_x,
                               const void *x_bf16, int64_t M, const uint8_t *w_codes,
                               const uint8_t *w_sf, const float *s_enc_w, int64_t N, int64_t K,
                               void *y, void *scratch, int num_sms, cudaStream_t s);

// W4A4 decode on the CUDA cores for 1 to 4 tokens (mq_decode_gemv4.cu): a
// stream over the weight's NVFP4 bytes with the tokens quantized in shared
// memory (M x ceil(K / 1024) x 2 KB of it, at most kDecodeGemvTokenSmem).
constexpr int64_t kDecodeGemvTokenSmem = 96 * 1024;
bool decode_nvf4_gemv_fits(int64_t M, int64_t K);
cudaError_t launch_decode_nvf4_gemv(const uint8_t *w_codes, const uint8_t *w_sf, const float *s_enc_w,
                                    int64_t N, int64_t K, const void *x_bf16, int64_t M, void *y,
                                    int num_sms, cudaStream_t s);

// W4A4 decode on the tcgen05 tensor cores (mq_decode_tc.cu) for up to
// kDecodeTcTokens BF16 tokens x [M, K]; each CTA quantizes them itself over
// the K stages it covers, which must fit in kDecodeTcTokenSmem
// (decode_tc_token_bytes: bytes per CTA for M tokens on an [N, K] weight).  tmap_w is
// the weight codes' tensor map (encode_codes_tmap).  The weight is read
// before the wait on the preceding kernel: no kernel may write it just before
// (packing ends with a memory set).  decode_tc_partial_floats is the FP32
// partial-sum space it needs after the per-weight counters.
constexpr int64_t kDecodeTcTokens = 16;
constexpr size_t kDecodeTcTokenSmem = 40 * 1024;
size_t decode_tc_partial_floats(int64_t N, int64_t K, int num_sms);
size_t decode_tc_token_bytes(int64_t M, int64_t N, int64_t K, int num_sms);
cudaError_t launch_decode_nvf4_tc(const CUtensorMap &tmap_w, const uint8_t *w_sf,
                                  const float *s_enc_w, int64_t N, int64_t K, const void *x_bf16,
                                  int64_t M, void *y, void *scratch, unsigned *err, int num_sms,
                                  cudaStream_t s);

}  // namespace mq
