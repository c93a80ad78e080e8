/*
 * mq_debug.h -- test-only entry points of libmq.  Not part of the public
 * interface (include/mq.h); they exist so that the test suite can drive
 * failure paths of the kernels without faulting the GPU.
 */
#ifndef MQ_DEBUG_H
#define MQ_DEBUG_H

#include "mq.h"

#ifdef __cplusplus
extern "C" {
#endif

/* The block-scaled GEMM of mq_gemm_nvfp4 (same arguments) launched with every
 * bounded wait limited to wait_limit_us (1000 .. 2000000) and with the first
 * K stage of the first tile never released to the producer.  The producers'
 * wait for that stage on the ring's second lap runs out, the kernel latches
 * the timeout bit, every role stops issuing, drains what it has issued and
 * the CTA pair exits; y is left undefined.  mq_check then reports
 * MQ_ERR_TIMEOUT once, and the device stays usable.  Needs K >= 2048 (more
 * K steps than ring stages); host-side errors as mq_gemm_nvfp4. */
mq_status mq_debug_gemm_withhold_release(const uint8_t *a_codes, const uint8_t *a_sf_swizzled,
                                         const float *a_s_enc_dev, int64_t M, const mq_weight *w,
                                         void *y_bf16, int64_t ldy, uint32_t wait_limit_us,
                                         cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MQ_DEBUG_H */
