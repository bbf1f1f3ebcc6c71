/*
 * vc_attn.h -- C ABI of the VC-Attention forward hot path on one B200 (sm_100a).
 *
 * The method: "VC-Attention: Value Smoothing and Softmax Casting for Low-bit
 * Attention" (arXiv 2609.15810), Abstract -- V-Smooth reorders value tokens by
 * online clustering, quantises only the residual after subtracting each block's
 * mean and restores the mean from the online-softmax row sum; ExpCast-FP8 maps
 * log-domain scores to E4M3 probability codes with one fused multiply-add.
 * Per-(batch, head) k-means, 128-token blocks and the E4M3 / NVFP4 residual are
 * from "Nunchux AI lanza VC-Attention kernel ..." (news summary), second
 * paragraph. The input / output contract (FP16 or BF16 Q, K, V of shape
 * [S,H,128] or [B,S,H,128], BF16 O) and the prep / attention split are from
 * "Open VC Attention" (catalogue card), section "Описание".
 *
 * Conventions (every entry point):
 *  - Pointers named q, k, v, o and every field of vc_prepared_v_t / vc_qk_fp8_t
 *    are DEVICE pointers owned and allocated by the caller (except in
 *    vc_attn_run_host, whose q, k, v, o are host pointers); the library never
 *    allocates or frees device memory and keeps no pointer after a call returns.
 *  - Tensors are dense and row-major in the layouts stated per field. Q, K, V and
 *    O are [B, S, H, 128] (a [S, H, 128] tensor is B = 1). Device pointers must
 *    be 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). All work is
 *    enqueued asynchronously on it; no call synchronises the device.
 *  - Every call validates its arguments on the host before launching anything
 *    and returns a vc_status_t; on error nothing has been launched and
 *    vc_attn_last_error() gives a message (per calling thread). No call aborts,
 *    traps or prints.
 *  - Device-side failures (a bounded wait inside a kernel that ran out) are
 *    reported through the optional `dev_status` int (device memory, set by the
 *    caller to VC_OK before the call, read after the caller's own sync).
 *  - Sizes: S >= 1, H >= 1, B >= 1, D == 128, B*H*S_pad*128 < 2^31 elements per
 *    tensor, where nb = ceil(S/128) and S_pad = 128*nb; B*H <= 65535 (else
 *    VC_ERR_UNSUPPORTED: the kernels take one grid row per (b, h) slice).
 */
#ifndef VC_ATTN_H
#define VC_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VC_OK = 0,
  VC_ERR_INVALID_ARG = 1,   /* a shape, pointer, alignment or config is invalid   */
  VC_ERR_UNSUPPORTED = 2,   /* valid but not supported by the library or device  */
  VC_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required         */
  VC_ERR_CUDA = 4,          /* a CUDA runtime / driver call failed                */
  VC_ERR_TIMEOUT = 5        /* device side: a bounded wait in a kernel ran out    */
} vc_status_t;

typedef enum { VC_DTYPE_F16 = 0, VC_DTYPE_BF16 = 1 } vc_dtype_t;
typedef enum {
  VC_RESIDUAL_E4M3 = 0,              /* E4M3 codes, one scale per (b, h)                */
  VC_RESIDUAL_NVFP4 = 1,             /* E2M1 + E4M3 scale per 16 tokens + fp32 global   */
  VC_RESIDUAL_E4M3_PER_CHANNEL = 2,  /* E4M3 codes, one scale per (b, h, channel)       */
  VC_RESIDUAL_MXFP4 = 3              /* E2M1 + power-of-two scale per 32 tokens         */
} vc_residual_fmt_t;
typedef enum {
  VC_MODE_VSMOOTH = 0,      /* k-means + cluster sort + block means (the method)  */
  VC_MODE_MEANONLY = 1,     /* identity order, block means only (diagnostic)      */
  VC_MODE_NAIVE = 2         /* identity order, no block means: V itself at one scale
                               per (b, h), the unsmoothed baseline (diagnostic)    */
} vc_mode_t;

/* Problem shape. D must be 128. dtype is a vc_dtype_t for Q, K and V. */
typedef struct {
  int32_t B, S, H, D;
  int32_t dtype;
} vc_shape_t;

/* V-Smooth configuration. k in [1, 32] clusters, iters >= 1 assignment passes
 * (the last pass's assignment is final), seed for the k-means init. */
typedef struct {
  int32_t k;
  int32_t iters;
  uint64_t seed;
  int32_t residual_fmt;     /* vc_residual_fmt_t */
  int32_t mode;             /* vc_mode_t         */
} vc_vsmooth_cfg_t;

/* Output of vc_attn_prepare_v (caller-owned device buffers):
 *  perm     int32 [B,H,S]      original token index at each permuted position
 *  mu       fp32  [B,H,nb,128] mean of each 128-token block (permuted order)
 *  v_codes  E4M3, E4M3_PER_CHANNEL: uint8 [B,H,128,S_pad] residual codes, V^T
 *                  (token-contiguous)
 *           NVFP4, MXFP4: uint8 [B,H,128,S_pad/2] two E2M1 codes per byte, even
 *                  token in the low nibble (MXFP4: 32-byte aligned)
 *  v_scales NVFP4: uint8 [B,H,128,S_pad/16] E4M3 scale per 16 tokens
 *           MXFP4: uint8 [B,H,nb,128,4] biased exponent e + 127 of the scale 2^e
 *                  of channel d and tokens 128 j + 32 g .. 128 j + 32 g + 31 at
 *                  [b,h,j,d,g] (one 512-byte piece per 128-token block)
 *           otherwise unused (may be NULL)
 *  s_v      E4M3:  fp32 [B,H]     residual scale s_V
 *           E4M3_PER_CHANNEL: fp32 [B,H,128] residual scale of each channel
 *           NVFP4: fp32 [B,H]     global scale g
 *           MXFP4: fp32 [B,H]     written as 1 (the scales are in v_scales)
 * Padding columns (tokens >= S) of v_codes are written as 0 (MXFP4: exponent
 * byte 0 for groups that hold only padding). */
typedef struct {
  int32_t* perm;
  float* mu;
  uint8_t* v_codes;
  uint8_t* v_scales;
  float* s_v;
} vc_prepared_v_t;

/* Output of vc_attn_quant_qk (caller-owned device buffers):
 *  q_codes  uint8 [B,H,S_pad,128]  E4M3 codes of Q (original order)
 *  q_scales fp32  [B,H,nb]         one scale per 128-row block of Q
 *  k_codes  uint8 [B,H,S_pad,128]  E4M3 codes of K in permuted order
 *  k_scales fp32  [B,H,nb]         one scale per 128-row block of permuted K
 * Padding rows are written as 0. */
typedef struct {
  uint8_t* q_codes;
  float* q_scales;
  uint8_t* k_codes;
  float* k_scales;
} vc_qk_fp8_t;

/* Library version (major*10000 + minor*100 + patch). */
int32_t vc_attn_version(void);

/* Message for the last error returned on the calling thread ("" if none). */
const char* vc_attn_last_error(void);

/* Number of CUDA kernels this library has enqueued since it was loaded, over
 * all threads and devices (memset nodes not counted). Monotone; for measuring
 * how many launches a sequence of calls makes. */
uint64_t vc_attn_launch_count(void);

/* Bytes of workspace vc_attn_prepare_v needs for this shape and config
 * (0 if the arguments are invalid). */
size_t vc_attn_prepare_v_workspace_bytes(const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg);

/* V-Smooth prep ("VC-Attention ...", Abstract; "Nunchux AI lanza ...", 2nd
 * paragraph): per (b, h), seeded k-means over the value tokens (k clusters,
 * `iters` Lloyd assignment passes), a stable sort of the tokens by cluster id
 * (the permutation also applied to K by vc_attn_quant_qk), subtraction of each
 * 128-token block's mean, and quantisation of the residual (cfg->residual_fmt):
 *  - VC_RESIDUAL_E4M3: E4M3, one scale amax/448 per (b, h) ("Open VC Attention",
 *    "Описание": V scales per head);
 *  - VC_RESIDUAL_NVFP4: E2M1 + E4M3 scale per 16 tokens + fp32 global per (b, h)
 *    ("Nunchux AI lanza ...", 2nd paragraph);
 *  - VC_RESIDUAL_E4M3_PER_CHANNEL: E4M3 with one scale amax_d/448 per (b, h,
 *    channel d) (no passage: the per-head scale of the card, taken per channel);
 *    a channel whose amax is below 2^-100 gets scale 1 and codes 0;
 *  - VC_RESIDUAL_MXFP4: E2M1 codes of r * 2^-e with one power of two per
 *    channel and 32 consecutive permuted tokens, e the smallest integer >= -127
 *    with amax <= 6 * 2^e, so that nothing clips (no passage: the tensor cores'
 *    block-scaled FP4 operand, a neighbour of the NVFP4 residual).
 * cfg->mode VC_MODE_MEANONLY keeps the original order (perm = identity);
 * VC_MODE_NAIVE also writes all block means as 0, so V itself is quantised (the
 * baseline the method improves on; vc_attn_forward then adds no mean).
 *  v               device, [B,S,H,128] of shape->dtype
 *  out             fields as documented in vc_prepared_v_t (v_scales only NVFP4)
 *  workspace       device, >= vc_attn_prepare_v_workspace_bytes(), 256-B aligned;
 *                  contents on entry are ignored
 *  assign_history  optional device uint8 [iters,B,H,S]: the assignment of every
 *                  pass (for lock-step checking); NULL to skip
 * Errors: VC_ERR_INVALID_ARG (shape / cfg / pointers), VC_ERR_WORKSPACE,
 *         VC_ERR_CUDA (launch failure). */
vc_status_t vc_attn_prepare_v(const void* v, const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg,
                              const vc_prepared_v_t* out, void* workspace, size_t workspace_bytes,
                              uint8_t* assign_history, void* stream);

/* V-Smooth prep of a shard of heads of a larger problem: as vc_attn_prepare_v on
 * v = heads [h_base, h_base + shape->H) of a [B,S,H_total,128] problem, given as a
 * dense [B,S,shape->H,128] tensor. Every (b, h) slice of the method is independent
 * ("VC-Attention ...", Abstract: clustering, block means and the residual scale
 * are per value head; "Nunchux AI lanza ...", 2nd paragraph: k-means per batch and
 * head); the only link to the rest of the problem is the k-means init, whose seed
 * index is that of slice (b, h_base + h) of the whole problem, b*H_total + h_base + h.
 * So the outputs are, bit for bit, the heads [h_base, h_base + shape->H) of what
 * vc_attn_prepare_v gives for the whole problem: a problem can be split by heads over
 * several GPUs (or calls) with no exchange at all.
 *  h_base, H_total  0 <= h_base, h_base + shape->H <= H_total
 *  other arguments  as vc_attn_prepare_v (no assignment history)
 * Errors: as vc_attn_prepare_v, plus VC_ERR_INVALID_ARG for a head range outside
 * [0, H_total). */
vc_status_t vc_attn_prepare_v_shard(const void* v, const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg,
                                    int32_t h_base, int32_t H_total, const vc_prepared_v_t* out, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* Q/K FP8 quantisation ("Open VC Attention", "Описание": Q/K scales per block):
 * per (b, h, 128-row block) scale s = amax/448 and E4M3 codes of x*(448/amax);
 * K rows are gathered through `perm` (from vc_attn_prepare_v) first.
 *  q, k   device, [B,S,H,128] of shape->dtype
 *  perm   device int32 [B,H,S]
 * Errors: VC_ERR_INVALID_ARG, VC_ERR_CUDA. */
vc_status_t vc_attn_quant_qk(const void* q, const void* k, const vc_shape_t* shape,
                             const int32_t* perm, const vc_qk_fp8_t* out, void* stream);

/* Bytes of workspace vc_attn_prepare_v_repair needs for this shape and config
 * (0 if the arguments are invalid): that of vc_attn_prepare_v plus 4*B*H*S +
 * 8*B*H bytes (each part rounded up to 256). */
size_t vc_attn_prepare_v_repair_workspace_bytes(const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg);

/* V-Smooth prep with the V residual repair ("Open VC Attention", "Описание":
 * the repair re-adds the quantisation residual of the worst-rounded value
 * tokens, prepared with a budget such as 0.005), for the E4M3 residual. The
 * result is two E4M3 planes at the residual's scale s_V:
 *   plane 0 = the residual codes of vc_attn_prepare_v;
 *   plane 1 = for the m = min(S, ceil(budget * S)) kept tokens of each (b, h),
 *             E4M3 codes of each element's rounding error in code units,
 *             y - dec(code0) with y = fl32(fl32(v - mu) * fl32(448 / amax)) (the
 *             value that was rounded); 0 for the other and the padding tokens.
 * The kept tokens are the m largest by the error sum_d fl32(dlt_d^2), added in
 * fp32 from d = 0 to 127, ties to the lower permuted position.
 *  budget        share of the tokens of each (b, h) to repair, in [0, 1]
 *  out           as vc_attn_prepare_v, except that out->v_codes points to
 *                uint8 [2][B,H,128,S_pad] (plane 0, then plane 1)
 *  kept          optional device uint8 [B,H,S]: 1 for the kept permuted
 *                positions, else 0; NULL to skip
 *  workspace     device, >= vc_attn_prepare_v_repair_workspace_bytes(),
 *                256-B aligned
 * The planes feed vc_attn_forward_repair. Errors: as vc_attn_prepare_v, plus
 * VC_ERR_UNSUPPORTED for the NVFP4 residual and VC_ERR_INVALID_ARG for a budget
 * outside [0, 1]. */
vc_status_t vc_attn_prepare_v_repair(const void* v, const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg,
                                     double budget, const vc_prepared_v_t* out, uint8_t* kept,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* Attention over a repaired residual: as vc_attn_forward, with pv from
 * vc_attn_prepare_v_repair (pv->v_codes = the two planes). O = (s_V * P (plane 0
 * + plane 1) + sum_tiles rowsum(P_tile) mu_tile) / rowsum(P); the row sums come
 * from P alone, so the repaired tokens are counted once. Errors: as
 * vc_attn_forward. */
vc_status_t vc_attn_forward_repair(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv, const vc_shape_t* shape,
                                   float softmax_scale, int32_t k_p, void* o, int32_t* dev_status,
                                   void* stream);

/* Bytes of device workspace vc_attn_quant_qk_smoothk needs: B*H*128*12 (the
 * int64 token sums and the fp32 means; 0 for an invalid shape). */
size_t vc_attn_quant_qk_smoothk_workspace_bytes(const vc_shape_t* shape);

/* Q/K FP8 quantisation with K smoothing ("VC-Attention ...", Abstract: prior
 * work smooths queries and keys): as vc_attn_quant_qk, but K is first reduced by
 * its per-channel mean over the S tokens of each (b, h),
 *   kbar[d] = fl32((sum_t llrint(k[t][d] * 2^24) * 2^-24) / S)   (exact int64 sum,
 *             one double division)
 *   k'[t][d] = fl32(k[t][d] - kbar[d]),
 * and the per-block scales and E4M3 codes of K are those of k' (gathered through
 * perm). Every score of a query row moves by the same q . kbar, so softmax(Q K^T)
 * is unchanged, while keys with large channel offsets quantise with much finer
 * block scales. Q is quantised as by vc_attn_quant_qk. The outputs feed
 * vc_attn_forward / vc_attn_forward_nvfp4v unchanged.
 *  q, k, perm, out  as vc_attn_quant_qk
 *  workspace        device, >= vc_attn_quant_qk_smoothk_workspace_bytes(shape),
 *                   16-B aligned; contents on entry ignored, undefined after
 *  k_mean           optional device fp32 [B,H,128]: receives kbar; NULL to skip
 * The int64 sums wrap (as two's complement) only when |sum_t k[t][d]| reaches
 * 2^39, far beyond BF16 / FP16 activations of the supported sizes.
 * Errors: VC_ERR_INVALID_ARG, VC_ERR_WORKSPACE, VC_ERR_CUDA. */
vc_status_t vc_attn_quant_qk_smoothk(const void* q, const void* k, const vc_shape_t* shape,
                                     const int32_t* perm, const vc_qk_fp8_t* out, void* workspace,
                                     size_t workspace_bytes, float* k_mean, void* stream);

/* Residual energy of V-Smooth (diagnostic; "Nunchux AI lanza ...", 2nd
 * paragraph, reports the share of the sequence energy that the token ordering
 * removes, averaged over Wan2.2 heads): per (b, h)
 *   energy[b*H + h] = sum_{p < S} sum_d (v[b, perm[p], h, d] - mu[p / 128][d])^2
 * with the differences, squares and sums in fp64 (summation order unspecified,
 * so the last bits may vary between runs). With perm and mu from
 * vc_attn_prepare_v in VC_MODE_VSMOOTH this is the energy left for the residual
 * quantiser; in VC_MODE_MEANONLY, the same without the cluster sort; with
 * mu == NULL, the energy of V itself (VC_MODE_NAIVE).
 *  v       device, [B,S,H,128] of shape->dtype
 *  perm    device int32 [B,H,S] (permuted position -> token), or NULL for the
 *          identity order
 *  mu      device fp32 [B,H,nb,128] block means of the permuted order, or NULL
 *          for zero means
 *  energy  device fp64 [B,H], overwritten (zeroed on `stream`, then summed into)
 * Errors: VC_ERR_INVALID_ARG (shape, NULL v / energy, alignment), VC_ERR_CUDA. */
vc_status_t vc_attn_residual_energy(const void* v, const vc_shape_t* shape, const int32_t* perm,
                                    const float* mu, double* energy, void* stream);

/* Fused FP8 attention with ExpCast probabilities and the block-mean restore
 * ("VC-Attention ...", Abstract; "Hugging Face Introduces VC-Attention",
 * "Technical Breakthroughs and Core Innovations"), E4M3 V residual:
 *   t = Q_codes K_codes^T (FP8 tensor cores, fp32 accumulate)
 *   log2-domain score u = c t, c = (sQ sK) * fl32(softmax_scale * log2 e)
 *   P code = E4M3 bit pattern of 2^(u - M + k_p), M an integer running row frame
 *   O = (s_V * P V_codes + sum_tiles rowsum(P_tile) mu_tile) / rowsum(P)
 *  qk, pv        outputs of the two prep calls for the same shape
 *  softmax_scale usually 1/sqrt(128)
 *  k_p           probability bias exponent in [0, 8] (8 recommended)
 *  o             device bf16 [B,S,H,128], rows in original query order
 *  dev_status    optional device int32 (see conventions)
 * Non-causal, no mask. Errors: VC_ERR_INVALID_ARG, VC_ERR_UNSUPPORTED (device is
 * not sm_100), VC_ERR_CUDA. */
vc_status_t vc_attn_forward(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv, const vc_shape_t* shape,
                            float softmax_scale, int32_t k_p, void* o, int32_t* dev_status,
                            void* stream);

/* As vc_attn_forward, for a V residual prepared with
 * VC_RESIDUAL_E4M3_PER_CHANNEL (pv->s_v holds one scale per (b, h, channel)):
 * O = (s_V[d] * (P V_codes)[d] + sum_tiles rowsum(P_tile) mu_tile[d]) / rowsum(P)
 * for each output channel d (no passage: the per-head V scale of "Open VC
 * Attention", "Описание", taken per channel; the mean restore and the scores are
 * those of vc_attn_forward). Errors: as vc_attn_forward. */
vc_status_t vc_attn_forward_e4m3_per_channel(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv,
                                             const vc_shape_t* shape, float softmax_scale, int32_t k_p, void* o,
                                             int32_t* dev_status, void* stream);

/* As vc_attn_forward, for a V residual prepared with VC_RESIDUAL_MXFP4
 * (pv->v_codes packed E2M1 V^T, pv->v_scales the biased exponents): the P V
 * product runs on the block-scaled FP8 x FP4 tensor-core MMA, E4M3 probability
 * codes times E2M1 residual codes with the power of two 2^e of each channel and
 * 32 keys applied inside the product, so the residual is read at 4.25 bits per
 * value and no decoded copy is made (no passage: the block-scaled form of the
 * NVFP4 residual of "Nunchux AI lanza ...", 2nd paragraph).
 *   O = (P (e2m1 * 2^e) + sum_tiles rowsum(P_tile) mu_tile) / rowsum(P)
 * pv->v_codes must be 32-byte aligned. Errors: as vc_attn_forward. */
vc_status_t vc_attn_forward_mxfp4v(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv, const vc_shape_t* shape,
                                   float softmax_scale, int32_t k_p, void* o, int32_t* dev_status, void* stream);

/* Bytes of device workspace vc_attn_forward_nvfp4v needs: 2*B*H*128*S_pad
 * (S_pad = S rounded up to 128). 0 for an invalid shape. */
size_t vc_attn_forward_nvfp4v_workspace_bytes(const vc_shape_t* shape);

/* As vc_attn_forward, for a V residual prepared with VC_RESIDUAL_NVFP4 (pv->v_codes
 * packed E2M1, pv->v_scales E4M3 per 16 tokens, pv->s_v the global scale g;
 * "Hugging Face Introduces VC-Attention", "Technical Breakthroughs and Core
 * Innovations": NVFP4 storage of the smoothed V).
 * Each decoded value v = e2m1 * dec(scale16) / 8 is at most 6*448/8 = 336; the
 * call writes hi = E4M3(v) and lo = E4M3(v - hi) (round to nearest even) to
 * `workspace` (layout [2][B,H,128,S_pad] uint8), then runs the FP8 attention
 * over both planes with value scale 8*g. hi + lo equals v exactly for
 * v >= 1/16 and within 2^-10 below that (E4M3's subnormal step), i.e. an
 * absolute error of at most g/128 per element before the mean restore.
 *  workspace        device, >= vc_attn_forward_nvfp4v_workspace_bytes(shape),
 *                   16-B aligned; caller-owned, contents undefined afterwards;
 *                   must not be reused by other work until the call's stream
 *                   has passed it
 *  other arguments  as vc_attn_forward
 * Errors: as vc_attn_forward, plus VC_ERR_WORKSPACE (NULL or too small). */
vc_status_t vc_attn_forward_nvfp4v(const vc_qk_fp8_t* qk, const vc_prepared_v_t* pv,
                                   const vc_shape_t* shape, float softmax_scale, int32_t k_p,
                                   void* o, void* workspace, size_t workspace_bytes,
                                   int32_t* dev_status, void* stream);

/* Size of the fixed device scratch used by vc_attn_prepare_v_noalloc: 12 MiB. */
#define VC_ATTN_NOALLOC_SCRATCH_BYTES ((size_t)12 << 20)

/* V-Smooth prep exactly as vc_attn_prepare_v, but without a caller workspace:
 * the k-means and sort scratch lives in a fixed device array that this library
 * owns (VC_ATTN_NOALLOC_SCRATCH_BYTES per GPU, reserved on every GPU that loads
 * the library until the process exits). The paper has no counterpart; this is a
 * convenience for callers that cannot allocate device memory themselves, such as
 * a plugin that is handed only its input and output buffers by a host framework
 * with its own memory pool, or a latency-critical loop that must not call
 * cudaMalloc (which can synchronise the device). Inputs and outputs are still
 * caller-owned, as for vc_attn_prepare_v; nothing is allocated or freed.
 *  - Fits when vc_attn_prepare_v_workspace_bytes(shape, cfg) <=
 *    VC_ATTN_NOALLOC_SCRATCH_BYTES (about 10 MB for B=1, H=56, S=73397, k=16);
 *    larger problems return VC_ERR_WORKSPACE with a message naming both sizes
 *    (use vc_attn_prepare_v with a workspace for them).
 *  - The first call on a device looks up the array's device address there
 *    (one-time set-up per device, with that device current); make that first
 *    call before any stream capture.
 *  - Every call on a device shares the one array, and it keeps the last call's
 *    contents (each call clears what must start at zero). Calls whose work
 *    overlaps on the GPU (on different streams, or from different threads
 *    without ordering) race on it: serialise them on one stream.
 *  - The looked-up address is kept for the life of the process: calling
 *    cudaDeviceReset on a device after its first call here is not supported
 *    (the array would move, and the kept address would no longer be it).
 * Arguments, outputs and other errors are those of vc_attn_prepare_v. */
vc_status_t vc_attn_prepare_v_noalloc(const void* v, const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg,
                                      const vc_prepared_v_t* out, uint8_t* assign_history, void* stream);

/* Bytes of device workspace vc_attn_run_host needs for this shape, config and
 * head chunk (0 if the arguments are invalid): two slots, each with a chunk's
 * Q, K, V and O buffers (4 * S * head_chunk * 256 bytes) and its prep, code and
 * scratch buffers (about 3 * S * head_chunk * 128 bytes more). */
size_t vc_attn_run_host_workspace_bytes(const vc_shape_t* shape, const vc_vsmooth_cfg_t* cfg,
                                        int32_t head_chunk);

/* The whole path -- vc_attn_prepare_v, vc_attn_quant_qk and vc_attn_forward (or
 * the forward call of cfg->residual_fmt: vc_attn_forward_nvfp4v,
 * vc_attn_forward_e4m3_per_channel, vc_attn_forward_mxfp4v) -- for Q, K,
 * V and O in HOST memory, with the host<->device copies overlapped with the
 * compute. Every (b, h) slice of the method is independent ("VC-Attention ...",
 * Abstract: clustering, block means and the residual scale are per value head;
 * "Nunchux AI lanza ...", 2nd paragraph: k-means per batch and head), so the
 * call runs the problem in chunks of `head_chunk` heads of one batch entry: the
 * chunk's Q, K, V rows are copied to the device on one internal stream, its prep,
 * Q/K quantisation and attention run on `stream` (even chunks) or on a second
 * internal stream (odd chunks, so that one chunk's last wave of attention CTAs
 * shares the GPU with the next chunk's kernels), and its O rows are copied back
 * on a third internal stream, while the next chunks' inputs are already being
 * copied in. The first and the last chunk of the call take a single head, so
 * that the copies that cannot overlap any compute are short. The output is bit-identical to the three device calls on the whole
 * problem (each chunk's k-means is seeded by the slice's index in the whole
 * problem).
 *  q, k, v       HOST, [B,S,H,128] of shape->dtype. Page-locked memory
 *                (cudaHostAlloc / cudaHostRegister) lets the copies run
 *                asynchronously; with pageable memory the call still gives the
 *                same result, but the copies do not overlap the compute.
 *  o             HOST, bf16 [B,S,H,128]; valid once `stream` has passed the call
 *                (e.g. after cudaStreamSynchronize(stream))
 *  head_chunk    heads per chunk, >= 1 (values above H mean H); smaller chunks
 *                overlap more of the copies, larger ones keep more of the GPU
 *                busy per launch (4 for H = 56 on a B200 over PCIe 5)
 *  workspace     device, >= vc_attn_run_host_workspace_bytes(), 256-B aligned;
 *                must not be reused by other work until `stream` has passed the
 *                call
 *  other arguments as vc_attn_forward (cfg as vc_attn_prepare_v)
 * The host buffers must stay valid and unmodified until `stream` has passed the
 * call. The three internal streams of each device are created on the first
 * call there (not during stream capture) and live until the process exits; the
 * call enqueues its work and returns without waiting for it.
 * Errors: as vc_attn_prepare_v and vc_attn_forward, plus VC_ERR_INVALID_ARG for
 * head_chunk < 1 and VC_ERR_WORKSPACE. All arguments are checked before anything
 * is enqueued; a VC_ERR_CUDA from a failed launch or copy may leave earlier
 * chunks enqueued. */
vc_status_t vc_attn_run_host(const void* q, const void* k, const void* v, const vc_shape_t* shape,
                             const vc_vsmooth_cfg_t* cfg, float softmax_scale, int32_t k_p, void* o,
                             int32_t head_chunk, void* workspace, size_t workspace_bytes,
                             int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* VC_ATTN_H */
