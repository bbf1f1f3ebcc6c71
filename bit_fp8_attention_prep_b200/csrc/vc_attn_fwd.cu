// vc_attn_fwd.cu -- fused FP8 attention with ExpCast probabilities and the
// V-Smooth block-mean restore, for one B200 (sm_100a).
//
// Method: "VC-Attention: Value Smoothing and Softmax Casting for Low-bit
// Attention", Abstract, and "Hugging Face Introduces VC-Attention", section
// "Technical Breakthroughs and Core Innovations": low-bit tensor cores run QK^T
// and PV; between them ExpCast-FP8 turns log-domain scores into E4M3
// probability codes with one fused multiply-add; the value residual (V minus its
// 128-token block mean) goes through PV and the block means are restored from
// the block row sums of P ("restores that mean from the row sum the online
// softmax already maintains").
//
// One CTA = one 128-row query tile of one (b, h); it walks the (permuted) key
// blocks j = 0 .. nb-1:
//   warp 4 (TMA):     Q once; K_j, V^T_j and mu_j into ring buffers
//   warp 5 (MMA):     S_j = Q K_j^T   -> TMEM (two S buffers, 128 columns each)
//                     O  += P_{j-1} V_{j-1} -> TMEM (128 columns), issued after
//                     QK_j so that the tensor core works while warps 0-3 cast
//   warps 0-3:        row r = thread: tile max -> integer frame M (ceil of the
//                     log2-domain max, running) -> ExpCast codes -> P_j in shared
//                     memory (128-B swizzled K-major, the A operand of PV);
//                     rescale O / l / mean accumulator by 2^(M_old - M_new) when
//                     the frame moves; l += r_j, mean += r_j * mu_j (r_j = row
//                     sum of the cast P over block j); epilogue
//                     O = (s_V * O_acc + mean) / l -> BF16.
// All operands are E4M3; the MMA is tcgen05.mma kind::f8f6f4, M=128 N=128 K=32.
#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "vc_common.cuh"
#include "vc_kernels.h"
#include "vc_sm100.cuh"

namespace vc {
namespace {

constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t kTileBytes = 128 * 128;  // one 128 x 128 E4M3 tile
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;

struct __align__(1024) SmemE4M3 {
  uint8_t q[kTileBytes];
  uint8_t k[kKStages][kTileBytes];
  uint8_t v[kVStages][kTileBytes];
  uint8_t p[2][kTileBytes];
  float mu[kVStages][128];
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t o_final;
  uint64_t mma_drain;
  uint32_t tmem_base;
  int32_t abort_flag;
};

__device__ __forceinline__ float exp2_int(int n) {  // 2^n for integer n <= 0, exact (0 below 2^-126)
  return n < -126 ? 0.0f : __int_as_float((127 + n) << 23);
}

__device__ __forceinline__ bool wait_or_abort(SmemE4M3& s, uint64_t* bar, uint32_t parity, const AttnParams& P) {
  if (mbar_wait(bar, parity, P.wait_ns, P.status)) return true;
  s.abort_flag = 1;
  report_status(P.status, VC_ERR_TIMEOUT);
  return false;
}

__global__ void __launch_bounds__(kThreads, 1)
    vc_attn_fwd_e4m3_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  SmemE4M3& s = *reinterpret_cast<SmemE4M3*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, bh = blockIdx.y;
  const int nkv = P.nb;

  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.s_empty[i], 128);
      mbar_init(&s.p_full[i], 128);
      mbar_init(&s.p_empty[i], 1);
    }
    mbar_init(&s.o_final, 1);
    mbar_init(&s.mma_drain, 1);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const int rowq = bh * P.S_pad + qt * 128;
      mbar_arrive_expect_tx(&s.q_full, kTileBytes);
      tma_load_2d(s.q, &tmQ, &s.q_full, 0, rowq);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nkv && !*(volatile int32_t*)&s.abort_flag; ++j) {
        const int ks = j % kKStages;
        if (!wait_or_abort(s, &s.k_empty[ks], ((j / kKStages) & 1) ^ 1, P)) break;
        mbar_arrive_expect_tx(&s.k_full[ks], kTileBytes);
        tma_load_2d(s.k[ks], &tmK, &s.k_full[ks], 0, bh * P.S_pad + j * 128);
        k_issued = j + 1;
        const int vs = j % kVStages;
        if (!wait_or_abort(s, &s.v_empty[vs], ((j / kVStages) & 1) ^ 1, P)) break;
        mbar_arrive_expect_tx(&s.v_full[vs], kTileBytes + 512);
        tma_load_2d(s.v[vs], &tmV, &s.v_full[vs], j * 128, bh * 128);
        bulk_load(s.mu[vs], P.mu + ((size_t)bh * P.nb + j) * 128, 512, &s.v_full[vs]);
        v_issued = j + 1;
      }
      // Copies still in flight must land before the CTA exits (normally they all
      // have been consumed already and these waits return at once).
      const uint64_t drain_ns = 100000000ull;
      mbar_wait(&s.q_full, 0, drain_ns, nullptr);
      for (int j = max(0, k_issued - kKStages); j < k_issued; ++j)
        mbar_wait(&s.k_full[j % kKStages], (j / kKStages) & 1, drain_ns, nullptr);
      for (int j = max(0, v_issued - kVStages); j < v_issued; ++j)
        mbar_wait(&s.v_full[j % kVStages], (j / kVStages) & 1, drain_ns, nullptr);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f32acc(kFmtE4M3, kFmtE4M3, 128, 128);
      bool ok = wait_or_abort(s, &s.q_full, 0, P);
      const uint64_t qdesc = sdesc_k_sw128(smem_u32(s.q));
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          const int ks = j % kKStages, sb = j & 1;
          if (!(ok = wait_or_abort(s, &s.k_full[ks], (j / kKStages) & 1, P))) break;
          if (!(ok = wait_or_abort(s, &s.s_empty[sb], ((j >> 1) & 1) ^ 1, P))) break;
          tc_fence_after();
          const uint64_t kdesc = sdesc_k_sw128(smem_u32(s.k[ks]));
          const uint32_t dS = tmem + (sb ? kColS1 : kColS0);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) umma_f8f6f4_ss(dS, qdesc + 2 * kk, kdesc + 2 * kk, idesc, kk > 0);
          umma_commit(&s.s_full[sb]);
          umma_commit(&s.k_empty[ks]);
        }
        if (j >= 1) {
          const int jj = j - 1, pb = jj & 1;
          if (!(ok = wait_or_abort(s, &s.p_full[pb], (jj >> 1) & 1, P))) break;
          if (!(ok = wait_or_abort(s, &s.v_full[jj % kVStages], (jj / kVStages) & 1, P))) break;
          tc_fence_after();
          const uint64_t pdesc = sdesc_k_sw128(smem_u32(s.p[pb]));
          const uint64_t vdesc = sdesc_k_sw128(smem_u32(s.v[jj % kVStages]));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f8f6f4_ss(tmem + kColO, pdesc + 2 * kk, vdesc + 2 * kk, idesc, (jj > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&s.p_empty[pb]);
          umma_commit(&s.v_empty[jj % kVStages]);
          if (jj == nkv - 1) umma_commit(&s.o_final);
        }
      }
      // every MMA this thread issued has completed before TMEM is released
      umma_commit(&s.mma_drain);
      mbar_wait(&s.mma_drain, 0, 100000000ull, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int row = warp * 32 + lane;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float sQ = P.q_scales[(size_t)bh * P.nb + qt];
    float Mrun = 0.0f, l = 0.0f;
    float om[128];
#pragma unroll
    for (int d = 0; d < 128; ++d) om[d] = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1;
      const uint32_t sph = (j >> 1) & 1;
      if (!(ok = wait_or_abort(s, &s.s_full[sb], sph, P))) break;
      tc_fence_after();
      const uint32_t saddr = tmem + lane_base + (sb ? kColS1 : kColS0);
      const int valid = min(128, P.S - j * 128);
      // pass 1: tile max of the raw scores (c > 0, so max(c t) = c max(t))
      float tmax = -INFINITY;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t r[32];
        tmem_ld32(saddr + ch * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (ch * 32 + i < valid) tmax = fmaxf(tmax, __uint_as_float(r[i]));
      }
      const float c = __fmul_rn(__fmul_rn(sQ, P.k_scales[(size_t)bh * P.nb + j]), P.kappa);
      const float Mtile = ceilf(__fmul_rn(c, tmax));
      const float Mnew = j == 0 ? Mtile : fmaxf(Mrun, Mtile);
      const bool resc = j > 0 && Mnew > Mrun;
      const float alpha = resc ? exp2_int((int)(Mrun - Mnew)) : 1.0f;
      const float bias = expcast_bias(P.bias_b, Mnew);
      const float c8 = 8.0f * c;
      const bool hot = fabsf(Mnew) < 1048576.0f;
      // pass 2: codes -> P tile (swizzled), row sum of the cast P
      if (!(ok = wait_or_abort(s, &s.p_empty[sb], sph ^ 1, P))) break;
      uint8_t* prow = s.p[sb] + row * 128;
      float rsum = 0.0f;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t r[32];
        tmem_ld32(saddr + ch * 32, r);
        tmem_ld_wait();
        uint32_t w[8];
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          float z[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = ch * 32 + q4 * 4 + e;
            const float t = __uint_as_float(r[q4 * 4 + e]);
            float zz = hot ? expcast_z(t, c8, bias) : __uint_as_float(0x4B400000u + expcast_code(t, c8, bias));
            if (col >= valid) zz = kMagic;
            z[e] = zz;
            rsum += e4m3_to_f32(__float_as_uint(zz) & 0xFFu);
          }
          w[q4] = pack_codes4(z[0], z[1], z[2], z[3]);
        }
        const int c0 = (2 * ch) ^ (row & 7), c1 = (2 * ch + 1) ^ (row & 7);
        *reinterpret_cast<uint4*>(prow + c0 * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(prow + c1 * 16) = make_uint4(w[4], w[5], w[6], w[7]);
      }
      tc_fence_before();
      mbar_arrive(&s.s_empty[sb]);
      fence_proxy_async_smem();
      // rescale the TMEM accumulator when the frame moved (after PV_{j-1} is done)
      if (__any_sync(0xffffffffu, resc)) {
        const int jj = j - 1;
        if (!(ok = wait_or_abort(s, &s.p_empty[jj & 1], (jj >> 1) & 1, P))) break;
        tc_fence_after();
        const uint32_t oaddr = tmem + lane_base + kColO;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t r[32];
          tmem_ld32(oaddr + ch * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(oaddr + ch * 32, r);
        }
        tmem_st_wait();
      }
      // block-mean restore and row sum (same frame as O)
      if (!(ok = wait_or_abort(s, &s.v_full[j % kVStages], (j / kVStages) & 1, P))) break;
      const float4* mu4 = reinterpret_cast<const float4*>(s.mu[j % kVStages]);
      l = __fmaf_rn(l, alpha, rsum);
#pragma unroll
      for (int d4 = 0; d4 < 32; ++d4) {
        const float4 m = mu4[d4];
        om[4 * d4 + 0] = __fmaf_rn(rsum, m.x, om[4 * d4 + 0] * alpha);
        om[4 * d4 + 1] = __fmaf_rn(rsum, m.y, om[4 * d4 + 1] * alpha);
        om[4 * d4 + 2] = __fmaf_rn(rsum, m.z, om[4 * d4 + 2] * alpha);
        om[4 * d4 + 3] = __fmaf_rn(rsum, m.w, om[4 * d4 + 3] * alpha);
      }
      Mrun = Mnew;
      tc_fence_before();
      mbar_arrive(&s.p_full[sb]);
    }
    // epilogue: O = (s_V * O_acc + mean) / l, BF16, original query order
    ok = __all_sync(0xffffffffu, ok);
    if (ok) ok = __all_sync(0xffffffffu, wait_or_abort(s, &s.o_final, 0, P));
    if (ok) {
      tc_fence_after();
      const int q = qt * 128 + row;
      const float sV = P.s_v[bh];
      const float rl = 1.0f / l;
      const int b = bh / P.H, h = bh % P.H;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(P.o) + (((size_t)b * P.S + q) * P.H + h) * 128;
      const uint32_t oaddr = tmem + lane_base + kColO;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t r[32];
        tmem_ld32(oaddr + ch * 32, r);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int d = ch * 32 + 2 * i;
          const float a0 = __fmaf_rn(sV, __uint_as_float(r[2 * i]), om[d]) * rl;
          const float a1 = __fmaf_rn(sV, __uint_as_float(r[2 * i + 1]), om[d + 1]) * rl;
          __nv_bfloat162 b2 = __floats2bfloat162_rn(a0, a1);
          pk[i] = *reinterpret_cast<uint32_t*>(&b2);
        }
        if (q < P.S) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t attn_configure() {
  return cudaFuncSetAttribute(vc_attn_fwd_e4m3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)(sizeof(SmemE4M3) + 1024));
}

cudaError_t launch_attn_e4m3(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const AttnParams& p, cudaStream_t st) {
  const dim3 grid(p.nb, p.B * p.H);
  vc_attn_fwd_e4m3_kernel<<<grid, kThreads, sizeof(SmemE4M3) + 1024, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_nvfp4(const CUtensorMap&, const CUtensorMap&, const uint8_t*, const AttnParams&,
                              cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace vc
