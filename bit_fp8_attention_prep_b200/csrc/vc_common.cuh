// vc_common.cuh -- device helpers shared by the VC-Attention kernels (sm_100a).
//
// Number formats: OCP E4M3FN (residual, Q/K and probability codes) and E2M1
// (NVFP4 residual), as named by "Nunchux AI lanza VC-Attention kernel ..."
// (second paragraph) and "VC-Attention: Value Smoothing and Softmax Casting for
// Low-bit Attention", Abstract. Conversions use the hardware cvt instructions
// (round to nearest even, saturate to the largest finite value).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/vc_attn.h"

namespace vc {

constexpr int kD = 128;           // head dimension
constexpr int kBlock = 128;       // 128-token blocks (also the MMA tile)
constexpr int kGroup4 = 16;       // NVFP4: one E4M3 scale per 16 tokens
constexpr int kMxGroup = 32;      // MX-style FP4: one power-of-two scale per 32 tokens
constexpr float kE4M3Max = 448.0f;
constexpr float kE2M1Max = 6.0f;
constexpr float kTinyAmax = 7.888609052210118e-31f;  // 2^-100: below this a block is all zero
constexpr int kFixShift = 24;     // fixed-point sums of x * 2^24 (order-free)

// ---------------------------------------------------------------- conversions
// Two fp32 -> two E4M3 codes; `lo` lands in the low byte.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint8_t cvt_e4m3(float x) { return (uint8_t)(cvt_e4m3x2(x, 0.0f) & 0xFF); }

// Two fp32 -> two E2M1 codes in one byte; `lo` lands in the low nibble.
__device__ __forceinline__ uint8_t cvt_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return (uint8_t)r;
}

// E4M3 code -> fp32 value (exact). Subnormal codes are m * 2^-9.
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  const uint32_t mag = code & 0x7F;
  float v = mag >= 8 ? __uint_as_float((mag << 20) + 0x3C000000u) : (float)mag * 0.001953125f;
  return (code & 0x80) ? -v : v;
}

// E2M1 magnitude code (0..7) -> value {0, 0.5, 1, 1.5, 2, 3, 4, 6} (exact).
__device__ __forceinline__ float e2m1_value(uint32_t mag) {
  return mag < 4 ? 0.5f * (float)mag : (float)(2u << ((mag - 4) >> 1)) * ((mag & 1u) ? 1.5f : 1.0f);
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <> __device__ __forceinline__ float to_f32<__half>(__half x) { return __half2float(x); }

// Eight 16-bit values packed in a uint4 -> eight fp32.
template <typename T>
__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const T* h = reinterpret_cast<const T*>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = to_f32<T>(h[i]);
}

// Four 16-bit values packed in a uint2 -> four fp32.
template <typename T>
__device__ __forceinline__ void unpack4(const uint2& u, float* f) {
  const T* h = reinterpret_cast<const T*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) f[i] = to_f32<T>(h[i]);
}

// ---------------------------------------------------------------- ExpCast
// ExpCast-FP8 ("VC-Attention ...", Abstract; "Hugging Face Introduces
// VC-Attention", ExpCast-FP8 bullet): the E4M3 code of 2^(y + k_P) for the
// log2-domain score y = c*t - M is produced by ONE fma on a magic-biased fp32:
//   z = fma(t, 8c, MAGIC + B - 8M),  MAGIC = 1.5 * 2^23,  B = 56 + 8 k_P.
// In [2^23, 2^24) the fp32 spacing is 1, so the fma's single rounding is
// round-half-even to an integer of the exact value 8ct + B - 8M (B, 8M and MAGIC
// are even integers, so the shift does not move a tie), and the low byte of z's
// bit pattern is the code. Clamping z to [MAGIC, MAGIC + 126] clamps the code to
// [0, 126] (126 = 448, the largest finite E4M3).
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float expcast_bias(int32_t bias_b, float frame_m) {
  return (kMagic + (float)bias_b) - 8.0f * frame_m;  // exact for |frame_m| < 2^19
}

// General form (both clamps): used by the primitive test and by rows whose
// frame is outside the range where the upper clamp is provably inactive.
__device__ __forceinline__ uint32_t expcast_code(float t, float c8, float bias) {
  float z = __fmaf_rn(t, c8, bias);
  z = fminf(fmaxf(z, kMagic), kMagic + 126.0f);
  return __float_as_uint(z) & 0xFFu;
}

// Hot-path form: only the lower clamp. Valid when the frame M is the ceiling
// of fl32(c * max t) over the scores being cast and |M| < 2^20: then
// 8ct <= 8M + 8*ulp/2 <= 8M + 1/4 and the code is at most B <= 126.
__device__ __forceinline__ float expcast_z(float t, float c8, float bias) {
  return fmaxf(__fmaf_rn(t, c8, bias), kMagic);
}

// ---------------------------------------------------------------- packed fp32 math
// Two fp32 fused multiply-adds in one instruction (sm_100 f32x2), each rounded
// to nearest even exactly like __fmaf_rn.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t ra, rb, rc, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rc) : "f"(c.x), "f"(c.y));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}

// max of three fp32 values in one instruction (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ---------------------------------------------------------------- misc
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Device-side error report: first error wins.
__device__ __forceinline__ void report_status(int32_t* status, int32_t code) {
  if (status) atomicCAS(status, (int32_t)VC_OK, code);
}

}  // namespace vc
