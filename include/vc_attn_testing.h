/*
 * vc_attn_testing.h -- test hooks of libvcattn.so: primitive microkernels that
 * run exactly the device functions the production kernels use, so that their
 * rounding can be compared value by value with the CPU definition, and a check
 * of the bounded in-kernel wait. Same conventions as vc_attn.h (device pointers,
 * caller-owned buffers, asynchronous on `stream`, vc_status_t return).
 */
#ifndef VC_ATTN_TESTING_H
#define VC_ATTN_TESTING_H

#include "vc_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* codes[i] = E4M3 code of x[i] (round to nearest even, saturate to +-448), the
 * conversion used for the V residual and the Q/K codes. n >= 0. */
vc_status_t vc_attn_test_e4m3_round(const float* x, uint8_t* codes, int64_t n, void* stream);

/* codes[i] = E2M1 code (0..15, bit 3 = sign) of x[i] (round to nearest even,
 * saturate to +-6), the conversion used for the NVFP4 residual. */
vc_status_t vc_attn_test_e2m1_round(const float* x, uint8_t* codes, int64_t n, void* stream);

/* ExpCast probability code for score t[i], multiplier c[i] and integer frame
 * M[i] with bias B = bias_b (56 + 8 k_P): clip(rne(8 c t + B - 8 M), 0, 126).
 * hot = 0: the general device function (both clamps); hot = 1: the attention
 * kernel's hot-path form (lower clamp only), valid when M = ceil(fl32(c * max t))
 * over the scores of a row and |M| < 2^20. */
vc_status_t vc_attn_test_expcast(const float* t, const float* c, const float* M, int32_t bias_b,
                                 uint8_t* codes, int64_t n, int32_t hot, void* stream);

/* Launches one CTA that waits, with the same bounded wait the attention kernel
 * uses, on a barrier that nothing ever completes. After `limit_ns` nanoseconds
 * the kernel writes VC_ERR_TIMEOUT into *dev_status and returns; it never hangs. */
vc_status_t vc_attn_test_bounded_wait(int32_t* dev_status, uint64_t limit_ns, void* stream);

/* The fused E4M3-V attention of vc_attn_forward with one change, for
 * comparison: each probability is made the conventional way, 2^(c t - M + k_p)
 * on the special function unit (ex2.approx, flush-to-zero) and then converted
 * to E4M3 (round to nearest even, saturating), instead of ExpCast's single fma
 * on the score ("VC-Attention ...", Abstract: ExpCast replaces exactly this exp
 * and conversion). Frame, row sums, mean restore and layouts are those of
 * vc_attn_forward; the output differs from it by the approximation of 2^y.
 * Arguments and errors as vc_attn_forward. */
vc_status_t vc_attn_test_forward_exp2(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv, const vc_shape_t* shape,
                                      float softmax_scale, int32_t k_p, void* o, int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* VC_ATTN_TESTING_H */
