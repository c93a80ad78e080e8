// mq_capi.cu -- the C ABI of libmq (declared in include/mq.h): argument
// checks, the dual-precision weight handle, workspace carving and launches.
//
// The phase-aware scheme (Mix-Quant, zingnex.cn forum post, section
// "动态精度切换"; gist.science technical summary, section 2): weights are
// stored once in a form that serves both phases -- here a handle holding the
// BF16 matrix for decode and its NVFP4 copy for prefill -- and activations are
// converted (quantized) at the phase boundary on every prefill call.
#include <cmath>
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "mq.h"
#include "mq_debug.h"
#include "mq_internal.h"

// Per-device word in which kernels latch asynchronous errors (bounded waits
// that ran out).  Read and cleared by mq_check.
__device__ unsigned int g_mq_device_error;

struct mq_weight {
    int device;
    int64_t N, K;
    void *base;          // the one device allocation below
    void *bf16;          // [N, K] BF16
    uint8_t *codes;      // [N, K/2]
    uint8_t *sf;         // swizzled scales, mq_sf_bytes(N, K)
    float *s_enc;        // device scalar
    float *partials;     // MQ_AMAX_PARTIALS_MAX floats (pack-time scratch)
    void *decode_scratch; // K-slice partial sums + counters of the decode path
    CUtensorMap tmap;    // TMA map over the codes
    CUtensorMap tmap_sf; // TMA map over the swizzled scales
};

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool init = false;
    bool supported = false;
    int num_sms = 0;
    unsigned *err = nullptr;
    unsigned long long err_ctx = 0;  // context in which `err` was looked up
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Process-unique id of the calling thread's current CUDA context, or 0 if
// there is none.  A device's primary context made anew after cudaDeviceReset
// has a new id, and with it the library's device image (its __device__
// arrays) may sit at new addresses, so addresses looked up once per device
// are cached together with this id.
unsigned long long current_context_id() {
    struct Fns {
        CtxGetCurrentFn get = nullptr;
        CtxGetIdFn id = nullptr;
    };
    static const Fns fns = []() {
        Fns f;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f.get = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f.id = reinterpret_cast<CtxGetIdFn>(p);
        return f;
    }();
    CUcontext c = nullptr;
    if (!fns.get || !fns.id || fns.get(&c) != CUDA_SUCCESS || !c) return 0;
    unsigned long long id = 0;
    if (fns.id(c, &id) != CUDA_SUCCESS) return 0;
    return id;
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mq_status device_info(DeviceInfo **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.init) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MQ_ERR_CUDA;
        d.supported = (major == 10 && minor == 0);
        d.init = true;
    }
    if (!d.supported) return MQ_ERR_UNSUPPORTED_DEVICE;
    // the error word's device address, once per device context (looked up
    // again after the context was reset); the lookup itself makes the
    // context current if it was not
    const unsigned long long ctx = current_context_id();
    if (!d.err || ctx == 0 || ctx != d.err_ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_mq_device_error) != cudaSuccess || !p) return MQ_ERR_CUDA;
        d.err = static_cast<unsigned *>(p);
        d.err_ctx = current_context_id();
    }
    *out = &d;
    return MQ_OK;
}

mq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MQ_OK : MQ_ERR_CUDA; }

// Workspace carve for one [M, K] activation: codes | scales | partials | s_enc.
struct ActWs {
    uint8_t *codes;
    uint8_t *sf;
    float *partials;
    float *s_enc;
    size_t bytes;
};

size_t act_ws_bytes(int64_t M, int64_t K) {
    return align256(static_cast<size_t>(M) * static_cast<size_t>(K / 2)) +
           align256(mq_sf_bytes(M, K)) + align256(sizeof(float) * MQ_AMAX_PARTIALS_MAX) + 256;
}

ActWs carve_act(uint8_t *base, int64_t M, int64_t K) {
    ActWs w;
    size_t off = 0;
    w.codes = base + off;
    off += align256(static_cast<size_t>(M) * static_cast<size_t>(K / 2));
    w.sf = base + off;
    off += align256(mq_sf_bytes(M, K));
    w.partials = reinterpret_cast<float *>(base + off);
    off += align256(sizeof(float) * MQ_AMAX_PARTIALS_MAX);
    w.s_enc = reinterpret_cast<float *>(base + off);
    off += 256;
    w.bytes = off;
    return w;
}

// Shapes the kernels index with 32-bit arithmetic.
bool shape_fits(int64_t M, int64_t K) {
    return M >= 1 && K >= 64 && M <= (1LL << 30) && K <= (1LL << 24) &&
           M * (K / 8) < (1LL << 32) - 1;
}

mq_status quantize_impl(DeviceInfo *d, const void *x, int64_t M, int64_t K, int64_t ldx,
                        uint8_t *codes, uint8_t *sf, float *s_enc, const float *partials,
                        int n_partials, float *scratch_partials, cudaStream_t s) {
    if (!partials) {
        const int g = mq::amax_grid(M, K, d->num_sms);
        cudaError_t e = mq::launch_amax(x, M, K, ldx, scratch_partials, g, s);
        if (e != cudaSuccess) return MQ_ERR_CUDA;
        partials = scratch_partials;
        n_partials = g;
    }
    return cuda_status(
        mq::launch_quantize(x, M, K, ldx, partials, n_partials, codes, sf, s_enc, d->num_sms, s));
}

mq_status gemm_impl(DeviceInfo *d, const uint8_t *a_codes, const uint8_t *a_sf,
                    const float *a_s_enc, int64_t M, const mq_weight *w, void *y, int64_t ldy,
                    bool swiglu, float *amax_partials, int *n_partials, cudaStream_t s) {
    CUtensorMap ta, tsa;
    if (!mq::encode_codes_tmap(&ta, a_codes, M, w->K)) return MQ_ERR_CUDA;
    if (!mq::encode_sf_tmap(&tsa, a_sf, M, w->K)) return MQ_ERR_CUDA;
    mq::GemmArgs a;
    a.s_enc_a = a_s_enc;
    a.s_enc_b = w->s_enc;
    a.y = y;
    a.ldy = ldy;
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(w->N);
    a.K = static_cast<int>(w->K);
    a.amax_partials = amax_partials;
    a.err = d->err;
    int grid = 0;
    cudaError_t e = mq::launch_gemm_nvf4(ta, w->tmap, tsa, w->tmap_sf, a, swiglu, d->num_sms, &grid, s);
    if (n_partials) *n_partials = grid;
    return cuda_status(e);
}

mq_status check_weight(const mq_weight *w) {
    if (!w) return MQ_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MQ_ERR_CUDA;
    if (dev != w->device) return MQ_ERR_INVALID_ARG;
    return MQ_OK;
}

}  // namespace

extern "C" {

const char *mq_status_string(mq_status s) {
    switch (s) {
        case MQ_OK: return "MQ_OK";
        case MQ_ERR_INVALID_ARG: return "MQ_ERR_INVALID_ARG";
        case MQ_ERR_SHAPE: return "MQ_ERR_SHAPE";
        case MQ_ERR_ALIGNMENT: return "MQ_ERR_ALIGNMENT";
        case MQ_ERR_UNSUPPORTED_DEVICE: return "MQ_ERR_UNSUPPORTED_DEVICE";
        case MQ_ERR_OOM: return "MQ_ERR_OOM";
        case MQ_ERR_CUDA: return "MQ_ERR_CUDA";
        case MQ_ERR_TIMEOUT: return "MQ_ERR_TIMEOUT";
    }
    return "MQ_ERR_UNKNOWN";
}

mq_status mq_check(cudaStream_t stream) {
    DeviceInfo *d = nullptr;
    mq_status st = device_info(&d);
    if (st != MQ_OK) return st;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MQ_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, d->err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MQ_ERR_CUDA;
    if (v != 0) {
        const unsigned zero = 0;
        if (cudaMemcpy(d->err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
            return MQ_ERR_CUDA;
        return MQ_ERR_TIMEOUT;
    }
    return cudaGetLastError() == cudaSuccess ? MQ_OK : MQ_ERR_CUDA;
}

namespace {

// One CTA, one thread: an mbarrier that expects one arrival nobody makes, a
// wait on its first phase with the given time limit (%globaltimer), then the
// same timeout latch the kernels use.  Exits as soon as the limit passes.
__global__ void selftest_wait_kernel(unsigned long long limit_ns, unsigned *err) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(a) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    unsigned long long t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a)
            : "memory");
        if (done) return;  // not reachable: nothing arrives
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (t - t0 > limit_ns) {
            atomicOr(err, 1u);  // the timeout bit mq_check reports
            return;
        }
    }
}

}  // namespace

mq_status mq_selftest_bounded_wait(uint32_t limit_us, cudaStream_t stream) {
    if (limit_us < 1 || limit_us > 2000000u) return MQ_ERR_INVALID_ARG;
    DeviceInfo *d = nullptr;
    mq_status st = device_info(&d);
    if (st != MQ_OK) return st;
    selftest_wait_kernel<<<1, 1, 0, stream>>>(static_cast<unsigned long long>(limit_us) * 1000ull,
                                              d->err);
    return cudaGetLastError() == cudaSuccess ? MQ_OK : MQ_ERR_CUDA;
}

size_t mq_sf_bytes(int64_t rows, int64_t K) {
    if (rows < 1 || K < 16) return 0;
    const int64_t rp = (rows + 127) / 128 * 128;
    const int64_t cp = ((K / 16) + 3) / 4 * 4;
    return static_cast<size_t>(rp * cp);
}

size_t mq_workspace_bytes(int64_t M, int64_t K) {
    if (M < 1 || K < 64) return 0;
    return act_ws_bytes(M, K);
}

size_t mq_mlp_workspace_bytes(int64_t M, int64_t K, int64_t I) {
    if (M < 1 || K < 64 || I < 64) return 0;
    return act_ws_bytes(M, K) + align256(static_cast<size_t>(M) * static_cast<size_t>(I) * 2) +
           act_ws_bytes(M, I);
}

mq_status mq_weight_pack(const void *w_bf16, int64_t N, int64_t K, cudaStream_t stream,
                         mq_weight **out) {
    if (!w_bf16 || !out) return MQ_ERR_INVALID_ARG;
    *out = nullptr;
    if (N < 1 || K < 64 || K % 64 != 0 || !shape_fits(N, K)) return MQ_ERR_SHAPE;
    if (!aligned16(w_bf16)) return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    mq_status st = device_info(&d);
    if (st != MQ_OK) return st;
    mq_weight *w = new mq_weight();
    cudaGetDevice(&w->device);
    w->N = N;
    w->K = K;
    const size_t b_bf16 = align256(static_cast<size_t>(N) * K * 2);
    const size_t b_codes = align256(static_cast<size_t>(N) * (K / 2));
    const size_t b_sf = align256(mq_sf_bytes(N, K));
    const size_t b_part = align256(sizeof(float) * MQ_AMAX_PARTIALS_MAX);
    const size_t b_dec = align256(mq::decode_scratch_bytes(N, K, d->num_sms));
    const size_t total = b_bf16 + b_codes + b_sf + b_part + 256 + b_dec;
    if (cudaMalloc(&w->base, total) != cudaSuccess) {
        cudaGetLastError();
        delete w;
        return MQ_ERR_OOM;
    }
    uint8_t *p = static_cast<uint8_t *>(w->base);
    w->bf16 = p;
    w->codes = p + b_bf16;
    w->sf = w->codes + b_codes;
    w->partials = reinterpret_cast<float *>(w->sf + b_sf);
    w->s_enc = reinterpret_cast<float *>(w->sf + b_sf + b_part);
    w->decode_scratch = b_dec ? static_cast<void *>(w->sf + b_sf + b_part + 256) : nullptr;
    st = MQ_OK;
    if (cudaMemcpyAsync(w->bf16, w_bf16, static_cast<size_t>(N) * K * 2,
                        cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
        st = MQ_ERR_CUDA;
    if (st == MQ_OK)
        st = quantize_impl(d, w->bf16, N, K, K, w->codes, w->sf, w->s_enc, nullptr, 0, w->partials,
                           stream);
    // Last on the stream, and not a kernel: the tensor-core W4A4 decode reads
    // the weight before its wait on the preceding kernel (programmatic
    // dependent launch), so it must never directly follow the kernel that
    // writes the codes; a memory set in between orders it fully.  (b_dec is
    // never 0: the counters alone take 256 bytes.)
    if (st == MQ_OK && cudaMemsetAsync(w->decode_scratch, 0, b_dec, stream) != cudaSuccess)
        st = MQ_ERR_CUDA;
    if (st == MQ_OK && (!mq::encode_codes_tmap(&w->tmap, w->codes, N, K) ||
                        !mq::encode_sf_tmap(&w->tmap_sf, w->sf, N, K)))
        st = MQ_ERR_CUDA;
    if (st != MQ_OK) {
        cudaFree(w->base);
        delete w;
        return st;
    }
    *out = w;
    return MQ_OK;
}

mq_status mq_weight_free(mq_weight *w) {
    if (!w) return MQ_OK;
    cudaError_t e = cudaFree(w->base);
    delete w;
    return cuda_status(e);
}

mq_status mq_weight_views(const mq_weight *w, int64_t *N, int64_t *K, const void **bf16,
                          const uint8_t **codes, const uint8_t **sf_swizzled,
                          const float **s_enc_dev) {
    if (!w) return MQ_ERR_INVALID_ARG;
    if (N) *N = w->N;
    if (K) *K = w->K;
    if (bf16) *bf16 = w->bf16;
    if (codes) *codes = w->codes;
    if (sf_swizzled) *sf_swizzled = w->sf;
    if (s_enc_dev) *s_enc_dev = w->s_enc;
    return MQ_OK;
}

mq_status mq_tensor_amax(const void *x_bf16, int64_t M, int64_t K, int64_t ldx,
                         float *amax_partials, int *n_partials, cudaStream_t stream) {
    if (!x_bf16 || !amax_partials || !n_partials) return MQ_ERR_INVALID_ARG;
    if (M < 1 || K < 8 || K % 8 != 0 || ldx < K || !shape_fits(M, K < 64 ? 64 : K))
        return MQ_ERR_SHAPE;
    if (ldx % 8 != 0 || !aligned16(x_bf16) || !aligned16(amax_partials)) return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    mq_status st = device_info(&d);
    if (st != MQ_OK) return st;
    const int g = mq::amax_grid(M, K, d->num_sms);
    *n_partials = g;
    return cuda_status(mq::launch_amax(x_bf16, M, K, ldx, amax_partials, g, stream));
}

mq_status mq_amax_combine(const float *amax_partials, int n_partials, float *amax_out,
                          cudaStream_t stream) {
    if (!amax_partials || !amax_out) return MQ_ERR_INVALID_ARG;
    if (n_partials < 1 || n_partials > MQ_AMAX_PARTIALS_MAX) return MQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(amax_partials) & 3u) ||
        (reinterpret_cast<uintptr_t>(amax_out) & 3u))
        return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    mq_status st = device_info(&d);
    if (st != MQ_OK) return st;
    return cuda_status(mq::launch_amax_combine(amax_partials, n_partials, amax_out, stream));
}

mq_status mq_quantize_nvfp4(const void *x_bf16, int64_t M, int64_t K, int64_t ldx,
                            uint8_t *codes, uint8_t *sf_swizzled, float *s_enc_dev,
                            const float *amax_partials, int n_partials, void *workspace,
                            size_t ws_bytes, cudaStream_t stream) {
    if (!x_bf16 || !codes || !sf_swizzled || !s_enc_dev) return MQ_ERR_INVALID_ARG;
    if (M < 1 || K < 64 || K % 64 != 0 || ldx < K || !shape_fits(M, K)) return MQ_ERR_SHAPE;
    if (ldx % 8 != 0 || !aligned16(x_bf16) || !aligned16(codes) || !aligned16(sf_swizzled) ||
        (reinterpret_cast<uintptr_t>(s_enc_dev) & 3u))
        return MQ_ERR_ALIGNMENT;
    if (amax_partials) {
        if (n_partials < 1 || n_partials > MQ_AMAX_PARTIALS_MAX) return MQ_ERR_INVALID_ARG;
    } else {
        if (!workspace || ws_bytes < sizeof(float) * MQ_AMAX_PARTIALS_MAX)
            return MQ_ERR_INVALID_ARG;
        if (!aligned16(workspace)) return MQ_ERR_ALIGNMENT;
    }
    DeviceInfo *d = nullptr;
    mq_status st = device_info(&d);
    if (st != MQ_OK) return st;
    return quantize_impl(d, x_bf16, M, K, ldx, codes, sf_swizzled, s_enc_dev, amax_partials,
                         n_partials, static_cast<float *>(workspace), stream);
}

mq_status mq_gemm_nvfp4(const uint8_t *a_codes, const uint8_t *a_sf_swizzled,
                        const float *a_s_enc_dev, int64_t M, const mq_weight *w, void *y_bf16,
                        int64_t ldy, cudaStream_t stream) {
    if (!a_codes || !a_sf_swizzled || !a_s_enc_dev || !y_bf16) return MQ_ERR_INVALID_ARG;
    mq_status st = check_weight(w);
    if (st != MQ_OK) return st;
    if (M < 1 || ldy < w->N || !shape_fits(M, w->K) || (M + 127) / 128 * ((w->N + 255) / 256) > (1LL << 31) - 1)
        return MQ_ERR_SHAPE;
    if (!aligned16(a_codes) || !aligned16(a_sf_swizzled) || !aligned16(y_bf16))
        return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    st = device_info(&d);
    if (st != MQ_OK) return st;
    return gemm_impl(d, a_codes, a_sf_swizzled, a_s_enc_dev, M, w, y_bf16, ldy, false, nullptr,
                     nullptr, stream);
}

// Test-only entry point (include/mq_debug.h): the GEMM with every bounded
// wait limited to wait_limit_us and the first K stage of the first tile never
// released, so that the kernel's abort path runs: the producers' waits run out,
// the timeout bit is latched, every role stops, drains what it issued and the
// pair exits.  Not part of the public interface.
mq_status mq_debug_gemm_withhold_release(const uint8_t *a_codes, const uint8_t *a_sf_swizzled,
                                         const float *a_s_enc_dev, int64_t M, const mq_weight *w,
                                         void *y_bf16, int64_t ldy, uint32_t wait_limit_us,
                                         cudaStream_t stream) {
    if (!a_codes || !a_sf_swizzled || !a_s_enc_dev || !y_bf16) return MQ_ERR_INVALID_ARG;
    if (wait_limit_us < 1000 || wait_limit_us > 2000000u) return MQ_ERR_INVALID_ARG;
    mq_status st = check_weight(w);
    if (st != MQ_OK) return st;
    // at least one tile and more K steps than ring stages (the withheld
    // stage is waited for on the ring's second lap)
    if (M < 1 || ldy < w->N || !shape_fits(M, w->K) || w->K < 2048) return MQ_ERR_SHAPE;
    if (!aligned16(a_codes) || !aligned16(a_sf_swizzled) || !aligned16(y_bf16))
        return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    st = device_info(&d);
    if (st != MQ_OK) return st;
    CUtensorMap ta, tsa;
    if (!mq::encode_codes_tmap(&ta, a_codes, M, w->K)) return MQ_ERR_CUDA;
    if (!mq::encode_sf_tmap(&tsa, a_sf_swizzled, M, w->K)) return MQ_ERR_CUDA;
    mq::GemmArgs a;
    a.s_enc_a = a_s_enc_dev;
    a.s_enc_b = w->s_enc;
    a.y = y_bf16;
    a.ldy = ldy;
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(w->N);
    a.K = static_cast<int>(w->K);
    a.amax_partials = nullptr;
    a.err = d->err;
    a.wait_ns = static_cast<unsigned long long>(wait_limit_us) * 1000ull;
    a.withhold_release = 1;
    return cuda_status(mq::launch_gemm_nvf4(ta, w->tmap, tsa, w->tmap_sf, a, false, d->num_sms, nullptr,
                                            stream));
}

mq_status mq_gemm_nvfp4_swiglu(const uint8_t *a_codes, const uint8_t *a_sf_swizzled,
                               const float *a_s_enc_dev, int64_t M, const mq_weight *w_gate_up,
                               void *h_bf16, float *h_amax_partials, int *n_partials,
                               cudaStream_t stream) {
    if (!a_codes || !a_sf_swizzled || !a_s_enc_dev || !h_bf16 || !h_amax_partials || !n_partials)
        return MQ_ERR_INVALID_ARG;
    mq_status st = check_weight(w_gate_up);
    if (st != MQ_OK) return st;
    if (M < 1 || w_gate_up->N % 256 != 0 || !shape_fits(M, w_gate_up->K)) return MQ_ERR_SHAPE;
    if (!aligned16(a_codes) || !aligned16(a_sf_swizzled) || !aligned16(h_bf16) ||
        !aligned16(h_amax_partials))
        return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    st = device_info(&d);
    if (st != MQ_OK) return st;
    return gemm_impl(d, a_codes, a_sf_swizzled, a_s_enc_dev, M, w_gate_up, h_bf16,
                     w_gate_up->N / 2, true, h_amax_partials, n_partials, stream);
}

mq_status mq_prefill_linear_nvfp4(const mq_weight *w, const void *x_bf16, int64_t M,
                                  void *y_bf16, void *workspace, size_t ws_bytes,
                                  cudaStream_t stream) {
    if (!x_bf16 || !y_bf16 || !workspace) return MQ_ERR_INVALID_ARG;
    mq_status st = check_weight(w);
    if (st != MQ_OK) return st;
    if (M < 1 || !shape_fits(M, w->K)) return MQ_ERR_SHAPE;
    if (ws_bytes < act_ws_bytes(M, w->K)) return MQ_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(y_bf16) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    st = device_info(&d);
    if (st != MQ_OK) return st;
    ActWs a = carve_act(static_cast<uint8_t *>(workspace), M, w->K);
    st = quantize_impl(d, x_bf16, M, w->K, w->K, a.codes, a.sf, a.s_enc, nullptr, 0, a.partials,
                       stream);
    if (st != MQ_OK) return st;
    return gemm_impl(d, a.codes, a.sf, a.s_enc, M, w, y_bf16, w->N, false, nullptr, nullptr,
                     stream);
}

mq_status mq_rmsnorm_amax(const void *x_bf16, const void *gamma_bf16, float eps, int64_t M,
                          int64_t K, int64_t ldx, void *y_bf16, float *amax_partials,
                          int *n_partials, cudaStream_t stream) {
    if (!x_bf16 || !gamma_bf16 || !y_bf16 || !amax_partials || !n_partials)
        return MQ_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !isfinite(eps)) return MQ_ERR_INVALID_ARG;
    if (M < 1 || K < 8 || K % 8 != 0 || ldx < K || !shape_fits(M, K < 64 ? 64 : K))
        return MQ_ERR_SHAPE;
    if (ldx % 8 != 0 || !aligned16(x_bf16) || !aligned16(gamma_bf16) || !aligned16(y_bf16) ||
        !aligned16(amax_partials))
        return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    mq_status st = device_info(&d);
    if (st != MQ_OK) return st;
    const int g = mq::rmsnorm_grid(M, K, d->num_sms);
    *n_partials = g;
    return cuda_status(mq::launch_rmsnorm_amax(x_bf16, M, K, ldx, gamma_bf16, eps, y_bf16,
                                               amax_partials, g, stream));
}

mq_status mq_prefill_linear_rmsnorm_nvfp4(const mq_weight *w, const void *r_bf16,
                                          const void *gamma_bf16, float eps, int64_t M,
                                          void *xn_bf16, void *y_bf16, void *workspace,
                                          size_t ws_bytes, cudaStream_t stream) {
    if (!r_bf16 || !gamma_bf16 || !xn_bf16 || !y_bf16 || !workspace) return MQ_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !isfinite(eps)) return MQ_ERR_INVALID_ARG;
    mq_status st = check_weight(w);
    if (st != MQ_OK) return st;
    if (M < 1 || !shape_fits(M, w->K)) return MQ_ERR_SHAPE;
    if (ws_bytes < act_ws_bytes(M, w->K)) return MQ_ERR_INVALID_ARG;
    if (!aligned16(r_bf16) || !aligned16(gamma_bf16) || !aligned16(xn_bf16) || !aligned16(y_bf16) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    st = device_info(&d);
    if (st != MQ_OK) return st;
    ActWs a = carve_act(static_cast<uint8_t *>(workspace), M, w->K);
    const int g = mq::rmsnorm_grid(M, w->K, d->num_sms);
    cudaError_t e = mq::launch_rmsnorm_amax(r_bf16, M, w->K, w->K, gamma_bf16, eps, xn_bf16,
                                            a.partials, g, stream);
    if (e != cudaSuccess) return MQ_ERR_CUDA;
    st = quantize_impl(d, xn_bf16, M, w->K, w->K, a.codes, a.sf, a.s_enc, a.partials, g, nullptr,
                       stream);
    if (st != MQ_OK) return st;
    return gemm_impl(d, a.codes, a.sf, a.s_enc, M, w, y_bf16, w->N, false, nullptr, nullptr,
                     stream);
}

mq_status mq_prefill_mlp_swiglu_nvfp4(const mq_weight *w_gate_up, const mq_weight *w_down,
                                      const void *x_bf16, int64_t M, void *y_bf16,
                                      void *h_bf16, void *workspace, size_t ws_bytes,
                                      cudaStream_t stream) {
    if (!x_bf16 || !y_bf16 || !workspace) return MQ_ERR_INVALID_ARG;
    mq_status st = check_weight(w_gate_up);
    if (st == MQ_OK) st = check_weight(w_down);
    if (st != MQ_OK) return st;
    const int64_t K = w_gate_up->K, I = w_gate_up->N / 2;
    if (M < 1 || w_gate_up->N % 256 != 0 || w_down->K != I || !shape_fits(M, K) ||
        !shape_fits(M, I))
        return MQ_ERR_SHAPE;
    if (ws_bytes < mq_mlp_workspace_bytes(M, K, I)) return MQ_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(y_bf16) || (h_bf16 && !aligned16(h_bf16)) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    st = device_info(&d);
    if (st != MQ_OK) return st;
    uint8_t *base = static_cast<uint8_t *>(workspace);
    ActWs ax = carve_act(base, M, K);
    uint8_t *h_ws = base + ax.bytes;
    void *h = h_bf16 ? h_bf16 : h_ws;
    ActWs ah = carve_act(h_ws + align256(static_cast<size_t>(M) * I * 2), M, I);
    st = quantize_impl(d, x_bf16, M, K, K, ax.codes, ax.sf, ax.s_enc, nullptr, 0, ax.partials,
                       stream);
    if (st != MQ_OK) return st;
    int np = 0;
    st = gemm_impl(d, ax.codes, ax.sf, ax.s_enc, M, w_gate_up, h, I, true, ah.partials, &np,
                   stream);
    if (st != MQ_OK) return st;
    st = quantize_impl(d, h, M, I, I, ah.codes, ah.sf, ah.s_enc, ah.partials, np, nullptr, stream);
    if (st != MQ_OK) return st;
    return gemm_impl(d, ah.codes, ah.sf, ah.s_enc, M, w_down, y_bf16, w_down->N, false, nullptr,
                     nullptr, stream);
}

}  // extern "C"

// ---- fixed scratch for the allocation-free prefill entry point -------------
// One array per device, part of this library's device image: the driver
// places it when the library's device code is loaded, so a caller never
// allocates it.  Host code cannot use the symbol as a pointer; its device
// address is looked up once per device below.
static __device__ __align__(256) uint8_t g_mq_noalloc_scratch[MQ_NOALLOC_SCRATCH_BYTES];

namespace {

uint8_t *g_noalloc_ptr[kMaxDevices];
unsigned long long g_noalloc_ctx[kMaxDevices];  // context of each cached address
std::mutex g_noalloc_mu;

// The array's device address on the current device, looked up once per
// device context (again after a cudaDeviceReset, whose new context may place
// the library's device image elsewhere).
mq_status noalloc_scratch(uint8_t **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MQ_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    const unsigned long long ctx = current_context_id();
    if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_mq_noalloc_scratch) != cudaSuccess || !p)
            return MQ_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<uint8_t *>(p);
        g_noalloc_ctx[dev] = current_context_id();
    }
    *out = g_noalloc_ptr[dev];
    return MQ_OK;
}

}  // namespace

extern "C" {

mq_status mq_prefill_linear_nvfp4_noalloc(const mq_weight *w, const void *x_bf16, int64_t M,
                                          void *y_bf16, cudaStream_t stream) {
    if (!x_bf16 || !y_bf16) return MQ_ERR_INVALID_ARG;
    mq_status st = check_weight(w);
    if (st != MQ_OK) return st;
    if (M < 1 || !shape_fits(M, w->K)) return MQ_ERR_SHAPE;
    if (act_ws_bytes(M, w->K) > MQ_NOALLOC_SCRATCH_BYTES) return MQ_ERR_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(y_bf16)) return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    st = device_info(&d);
    if (st != MQ_OK) return st;
    uint8_t *scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != MQ_OK) return st;
    ActWs a = carve_act(scratch, M, w->K);
    st = quantize_impl(d, x_bf16, M, w->K, w->K, a.codes, a.sf, a.s_enc, nullptr, 0, a.partials,
                       stream);
    if (st != MQ_OK) return st;
    return gemm_impl(d, a.codes, a.sf, a.s_enc, M, w, y_bf16, w->N, false, nullptr, nullptr,
                     stream);
}

mq_status mq_decode_linear_nvfp4(const mq_weight *w, const void *x_bf16, int64_t M, void *y_bf16,
                                 void *workspace, size_t ws_bytes, cudaStream_t stream) {
    if (!x_bf16 || !y_bf16 || !workspace) return MQ_ERR_INVALID_ARG;
    mq_status st = check_weight(w);
    if (st != MQ_OK) return st;
    if (M < 1 || M > (1LL << 20) || !shape_fits(M, w->K)) return MQ_ERR_SHAPE;
    if (ws_bytes < act_ws_bytes(M, w->K)) return MQ_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(y_bf16) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    st = device_info(&d);
    if (st != MQ_OK) return st;
    // 1 to 4 tokens on a weight of up to 2^25 elements: the CUDA-core stream
    // (the tensor-core kernel's fixed per-CTA path costs more there); larger
    // weights stream faster through the tensor-core kernel below
    if (mq::decode_nvf4_gemv_fits(M, w->K) && w->N * w->K <= (int64_t(1) << 25))
        return cuda_status(mq::launch_decode_nvf4_gemv(w->codes, w->sf, w->s_enc, w->N, w->K, x_bf16,
                                                       M, y_bf16, d->num_sms, stream));
    const bool tc_fits = M <= mq::kDecodeTcTokens &&
                         mq::decode_tc_token_bytes(M, w->N, w->K, d->num_sms) <= mq::kDecodeTcTokenSmem;
    const size_t tok_bytes = static_cast<size_t>(M) * static_cast<size_t>(w->K) * 9u / 16u;
    // the tensor-core kernel (quantizes the tokens itself, one pass over the
    // weight) for up to 4 tokens and for 9 to 16; 5 to 8 tokens go to the
    // FP16-MMA kernel.  (On the 8B gate/up weight alone the tensor-core kernel
    // is faster at 5-8 tokens, 26.4 against 31.0 us at 5, but followed by the
    // down projection on the FP16-MMA kernel the pass took 62.7 us at 8
    // tokens against 54.0 us with both on the FP16-MMA kernel.)
    if (tc_fits && (M <= 4 || M > 8))
        return cuda_status(mq::launch_decode_nvf4_tc(w->tmap, w->sf, w->s_enc, w->N, w->K, x_bf16,
                                                     M, y_bf16, w->decode_scratch, d->err,
                                                     d->num_sms, stream));
    if (M <= 8 && tok_bytes <= mq::kDecodeNvf4TokenSmem)
        return cuda_status(mq::launch_decode_nvf4(nullptr, nullptr, nullptr, x_bf16, M, w->codes,
                                                  w->sf, w->s_enc, w->N, w->K, y_bf16,
                                                  w->decode_scratch, d->num_sms, stream));
    ActWs a = carve_act(static_cast<uint8_t *>(workspace), M, w->K);
    st = quantize_impl(d, x_bf16, M, w->K, w->K, a.codes, a.sf, a.s_enc, nullptr, 0, a.partials,
                       stream);
    if (st != MQ_OK) return st;
    return cuda_status(mq::launch_decode_nvf4(a.codes, a.sf, a.s_enc, nullptr, M, w->codes, w->sf,
                                              w->s_enc, w->N, w->K, y_bf16, w->decode_scratch,
                                              d->num_sms, stream));
}

mq_status mq_attention_prefill_bf16(const void *qkv_bf16, int64_t M, int64_t H, int64_t Hkv,
                                    int64_t D, void *k_cache, void *v_cache, int64_t S_max,
                                    void *o_bf16, float *o_amax_partials, int *n_partials,
                                    cudaStream_t stream) {
    if (!qkv_bf16 || !o_bf16 || !o_amax_partials || !n_partials) return MQ_ERR_INVALID_ARG;
    if ((k_cache == nullptr) != (v_cache == nullptr)) return MQ_ERR_INVALID_ARG;
    if (D != 128 || H < 1 || Hkv < 1 || H % Hkv != 0 || M < 1 || M > (1LL << 24) || H > 1024)
        return MQ_ERR_SHAPE;
    if (k_cache && (S_max < M || S_max > (1LL << 24))) return MQ_ERR_SHAPE;
    if (!aligned16(qkv_bf16) || !aligned16(o_bf16) || !aligned16(o_amax_partials) ||
        (k_cache && (!aligned16(k_cache) || !aligned16(v_cache))))
        return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    mq_status st = device_info(&d);
    if (st != MQ_OK) return st;
    const int grid = mq::attention_prefill_grid(M, H);
    int slots = 0;   // one partial per CTA when they fit, else atomic max into zeroed slots
    if (grid > MQ_AMAX_PARTIALS_MAX) {
        slots = MQ_AMAX_PARTIALS_MAX;
        if (cudaMemsetAsync(o_amax_partials, 0, sizeof(float) * MQ_AMAX_PARTIALS_MAX, stream) !=
            cudaSuccess)
            return MQ_ERR_CUDA;
    }
    *n_partials = slots ? slots : grid;
    return cuda_status(mq::launch_attention_prefill(qkv_bf16, M, H, Hkv, k_cache, v_cache, S_max,
                                                    o_bf16, o_amax_partials, slots, d->err, stream));
}

size_t mq_attention_decode_workspace_bytes(int64_t m, int64_t pos0, int64_t H, int64_t Hkv,
                                           int64_t D) {
    if (D != 128 || m < 1 || pos0 < 0 || H < 1 || Hkv < 1 || H % Hkv != 0) return 0;
    return mq::attention_decode_workspace_bytes(m, pos0, H, Hkv);
}

mq_status mq_attention_decode_bf16(const void *qkv_bf16, int64_t m, int64_t pos0, int64_t H,
                                   int64_t Hkv, int64_t D, void *k_cache, void *v_cache,
                                   int64_t S_max, void *o_bf16, void *workspace, size_t ws_bytes,
                                   cudaStream_t stream) {
    if (!qkv_bf16 || !k_cache || !v_cache || !o_bf16 || !workspace) return MQ_ERR_INVALID_ARG;
    if (D != 128 || H < 1 || Hkv < 1 || H % Hkv != 0 || m < 1 || pos0 < 0 ||
        (H / Hkv) * m > mq::attention_decode_max_rows() || pos0 + m > S_max || S_max > (1LL << 24))
        return MQ_ERR_SHAPE;
    if (ws_bytes < mq::attention_decode_workspace_bytes(m, pos0, H, Hkv)) return MQ_ERR_INVALID_ARG;
    if (!aligned16(qkv_bf16) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o_bf16) ||
        !aligned16(workspace))
        return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    mq_status st = device_info(&d);
    if (st != MQ_OK) return st;
    return cuda_status(mq::launch_attention_decode(qkv_bf16, m, pos0, H, Hkv, k_cache, v_cache,
                                                   S_max, o_bf16, workspace, stream));
}

mq_status mq_decode_linear_bf16(const mq_weight *w, const void *x_bf16, int64_t M, void *y_bf16,
                                cudaStream_t stream) {
    if (!x_bf16 || !y_bf16) return MQ_ERR_INVALID_ARG;
    mq_status st = check_weight(w);
    if (st != MQ_OK) return st;
    if (M < 1 || M > (1LL << 20)) return MQ_ERR_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(y_bf16)) return MQ_ERR_ALIGNMENT;
    DeviceInfo *d = nullptr;
    st = device_info(&d);
    if (st != MQ_OK) return st;
    return cuda_status(mq::launch_decode(x_bf16, M, w->bf16, w->N, w->K, y_bf16, w->decode_scratch,
                                         d->num_sms, stream));
}

}  // extern "C"
