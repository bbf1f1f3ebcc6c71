// vc_kernels.h -- internal launch interface between the C ABI (vc_api.cu) and
// the kernels (vc_prep.cu, vc_attn_fwd.cu). Not installed, not part of the ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>

#include "../../include/vc_attn.h"

namespace vc {

constexpr int kMaxClusters = 32;   // k-means clusters per (b, h)
constexpr int kChunk = 1024;       // tokens per k-means CTA (also the sort's chunk)

// Device buffers and sizes of one vc_attn_prepare_v call; the pointers are
// carved from the caller's workspace.
struct PrepPlan {
  int B, S, H, k, iters, fmt, mode;
  uint64_t seed;
  int seed_H, seed_b0, seed_h0;  // slice (b, h) of this plan is slice (seed_b0 + b, seed_h0 + h) of a
                                 // problem with seed_H heads (its k-means seed); H, 0, 0 unless the
                                 // problem is run in chunks or shards of heads
  int nb, S_pad, nchunks;
  float* cent;                 // [BH][k][128]
  unsigned long long* sums;    // [BH][k][128] int64 fixed-point
  int* counts;                 // [BH][k]
  uint8_t* assign;             // [BH][S] labels of the even passes
  uint8_t* assign2;            // [BH][S] labels of the odd passes
  int* hist;                   // [BH][nchunks][k]
  int* offs;                   // [BH][nchunks][k]
  unsigned int* amax;          // [BH] fp32 bits ([BH][128] for the per-channel scale)
  uint8_t* cops;               // [BH] centroid operand blocks of the tensor-core assignment
  int* work;                   // [iters] work counters of the tensor-core assignment passes
  bool tc_assign;              // BF16 V: k-means distances on the tensor cores through tm_v
  int num_sms;                 // streaming multiprocessors of the device (persistent grids)
  CUtensorMap tm_v;            // V as [B*S][H][128] bf16, 128 x 1 x 64 boxes, 128-byte swizzle
};

// Bytes of one (b, h) slice's centroid operand block of the tensor-core
// k-means assignment for k clusters (k <= 16: 16 rows, else 32).
constexpr size_t tc_cops_bytes(int k) { return k <= 16 ? 2 * 2 * 16 * 128 + 2 * 16 * 4 : 2 * 2 * 32 * 128 + 2 * 32 * 4; }

cudaError_t prep_configure();
// *nlaunch receives the number of kernels enqueued (memsets not counted).
cudaError_t launch_prepare_v(const void* v, int dtype, const PrepPlan& plan, const vc_prepared_v_t& out,
                             uint8_t* history, cudaStream_t st, int* nlaunch);
// ksum (optional, [B*H][128] int64, zeroed here): K smoothing by the token mean,
// written to k_mean ([B*H][128] fp32) when that is given. *nlaunch: kernels enqueued.
cudaError_t launch_quant_qk(const void* q, const void* k, int dtype, int B, int S, int H, const int32_t* perm,
                            const vc_qk_fp8_t& out, unsigned long long* ksum, float* k_mean, cudaStream_t st,
                            int* nlaunch);
// V residual repair on the two planes [2][B*H][128][S_pad] at `planes` (plane 0
// written by the E4M3 prep, plane 1 here); m tokens kept per slice (0: plane 1
// all zero); err [B*H][S] and thr [B*H] are scratch; kept (optional) [B*H][S].
cudaError_t launch_repair(const void* v, int dtype, int B, int S, int H, const int32_t* perm, const float* mu,
                          const unsigned int* amax_bits, uint8_t* planes, int m, float* err,
                          unsigned long long* thr, uint8_t* kept, cudaStream_t st, int* nlaunch);
// energy[B*H] (zeroed here) = sum of ||v[perm[p]] - mu[p/128]||^2 per slice; perm / mu may be NULL
cudaError_t launch_residual_energy(const void* v, int dtype, int B, int S, int H, const int32_t* perm,
                                   const float* mu, double* energy, cudaStream_t st);

// Attention forward.
struct AttnParams {
  int B, S, H, nb, S_pad;
  const float* q_scales;   // [BH][nb]
  const float* k_scales;   // [BH][nb]
  const float* mu;         // [BH][nb][128]
  const float* s_v;        // [BH] ([BH][128] for the per-channel scale)
  const uint8_t* v_scales; // NVFP4: [BH][128][S_pad/16]; MX-style: [BH][nb][128][4]
  float kappa;             // fl32(softmax_scale * log2 e)
  float v_mul;             // value scale = s_v * v_mul (1 for E4M3; 8 for the NVFP4 planes)
  int bias_b;              // 56 + 8 k_P
  void* o;                 // bf16 [B][S][H][128]
  int32_t* status;         // optional device status word
  uint64_t wait_ns;        // bound on every in-kernel wait
};

cudaError_t attn_configure();
// exp2 = true: the comparison kernel that makes the probabilities with ex2 +
// E4M3 conversion instead of ExpCast (test hook only)
cudaError_t launch_attn_e4m3(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const AttnParams& p, cudaStream_t st, bool exp2 = false);
// E4M3 residual with one scale per (b, h, channel) (p.s_v is [BH][128]).
cudaError_t launch_attn_channel(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const AttnParams& p, cudaStream_t st);
// MX-style FP4 residual: `tv_e2m1` maps the packed E2M1 codes as 16-byte smem
// containers (128 x 128 codes a box); p.v_scales holds the exponents [BH][nb][128][4].
cudaError_t launch_attn_mx(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv_e2m1,
                           const AttnParams& p, cudaStream_t st);
// NVFP4 residual: `tplanes` maps the two E4M3 planes written by launch_nvfp4_planes.
cudaError_t launch_attn_planes(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tplanes,
                               const AttnParams& p, cudaStream_t st);
// planes[pl][B*H][128][S_pad] (pl = 0 hi, 1 lo) with hi + lo = e2m1 * dec(scale16) / 8 exactly
// (down to the E4M3 subnormal grid); padding tokens 0.
cudaError_t launch_nvfp4_planes(const uint8_t* codes, const uint8_t* scales, int BH, int S_pad,
                                uint8_t* planes, cudaStream_t st);

}  // namespace vc
