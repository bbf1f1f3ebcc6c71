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
// One CTA = two 128-row query tiles (t = 0, 1) of one (b, h); both walk all key
// blocks j = 0 .. nb-1 (permuted order), sharing every K/V tile.
//   warps 0-7   softmax group of query tile 0: two threads per query row, warps
//               0-3 take score columns 0-63 and warps 4-7 columns 64-127 (a warp
//               reaches the 32 tensor-memory lanes of its rank mod 4); the halves
//               exchange their partial row maxima through shared memory
//   warps 8-15  softmax group of query tile 1
//   warp  16    TMA: both Q tiles once; K_j, V^T_j and mu_j into rings
//   warp  17    MMA issuer (one thread)
// Tensor memory (512 columns): S_t = [128t, 128t+128), O_t = [256+128t, ...).
// Per block j and tile t the tensor core runs, in this order per tile:
//   PV   O_t += P_t V_j                   P_t = ExpCast codes (smem), V_j = residual codes
//   ROW  S_t[:, 112:128) = P_t 1          exact row sums r of the cast P
//   QK   S_t  = Q_t K_{j+1}^T             kind::f8f6f4, M=128 K=128, as keys 0-111 (N=112)
//        and keys 112-127 (N=16); the second part waits until r has been read
//   MEAN after every 5 blocks:  O_t += R_t M    kind::f16 with bf16 operands:
//        R_t = the blocks' row sums, M = their block means / s_V, each split into
//        bf16 hi/lo parts (r_hi m_hi + r_hi m_lo + r_lo m_hi, three K slots a block);
//        both operands of a tile's mean MMA live in that tile's own 128-B-swizzled
//        smem tile (R in K chunks 0-1, M in chunks 2-3, alternating by batch), and
//        the softmax group writes it only while no MMA of its tile is in flight
// so O_t accumulates the whole output in residual-code units; the epilogue is
// O = s_V O_t / l. The softmax thread of row i keeps the integer running frame
// F (ceil of the largest log2-domain score so far); a block is cast in the frame
// current after it; when F moves, O_t, l and the not-yet-issued row sums are
// multiplied by the exact power of two 2^(F_old - F_new).
#include <cuda.h>
#include <cuda_bf16.h>
#include <stddef.h>
#include <stdint.h>

#include "vc_common.cuh"
#include "vc_kernels.h"
#include "vc_sm100.cuh"

namespace vc {
namespace {

// kPlanes = 1: the E4M3 residual; kPlanes = 2: the NVFP4 residual given as two
// exact E4M3 planes (hi + lo) by the pre-pass in vc_prep.cu, with PV run over both.
template <int kPlanes> struct Stages {
  static constexpr int K = 3;
  static constexpr int V = kPlanes == 1 ? 3 : 2;
};
constexpr uint32_t kTileBytes = 128 * 128;  // one 128 x 128 E4M3 tile (or 128 x 64 bf16)
constexpr int kThreads = 576;
constexpr int kTmaWarp = 16, kMmaWarp = 17;
constexpr uint32_t kTmemCols = 512;
constexpr int kMeanBlocks = 5;              // key blocks per mean MMA (3 K slots each: 15 of 16)
constexpr int kMeanChunks = 2;              // 16-slot K chunks per operand (R: 0-1, M: 2-3)
constexpr uint32_t kOneE4M3x4 = 0x38383838u;
constexpr uint32_t kRowCol = 112;            // score columns 112-127 also receive the row sums
constexpr uint64_t kKeyHiOff = (112 * 128) >> 4;  // descriptor offset of K rows 112.. (14 atoms)

template <int kPlanes>
struct __align__(1024) SmemAttn {
  static constexpr int kKStages = Stages<kPlanes>::K, kVStages = Stages<kPlanes>::V;
  uint8_t q[2][kTileBytes];
  uint8_t k[kKStages][kTileBytes];
  uint8_t v[kVStages][kPlanes][kTileBytes];
  uint8_t p[2][kTileBytes];
  uint8_t mop[2][kTileBytes];    // bf16 operands of the mean MMA, one tile per query tile
  uint8_t ones[2048];            // E4M3 1.0: B operand of the row-sum MMA (N=16, K=128)
  float mu[kVStages][128];
  float xmax[2][2][2][128];      // [block parity][query tile][column half][row] partial maxima
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages], mu_empty[kVStages];
  uint64_t s_full[2], p_full[2], o_done[2], r_free[2], fin_ready[2], o_final[2];
  uint64_t mma_drain;
  uint32_t tmem_base;
  int32_t abort_flag;
};

__device__ __forceinline__ float exp2_int(int n) {  // 2^n for integer n <= 0, exact (0 below 2^-126)
  return n < -126 ? 0.0f : __int_as_float((127 + n) << 23);
}

template <class Smem>
__device__ __forceinline__ bool wait_or_abort(Smem& s, uint64_t* bar, uint32_t parity, const AttnParams& P) {
  if (mbar_wait(bar, parity, P.wait_ns, P.status)) return true;
  s.abort_flag = 1;
  report_status(P.status, VC_ERR_TIMEOUT);
  return false;
}

// Byte offset of 16-bit element `slot` (K index 16*chunk + slot) of row `row` in
// a 128-B-swizzled K-major operand tile (rows of 128 B, 8-row atoms).
__device__ __forceinline__ uint32_t sw128_off16(int row, int chunk, int slot) {
  const int kb = chunk * 32 + slot * 2;  // byte within the unswizzled 128-B row
  return (uint32_t)(row * 128 + ((((kb >> 4) ^ (row & 7)) & 7) << 4) + (kb & 15));
}

__device__ __forceinline__ void st_bf16(uint8_t* base, uint32_t off, __nv_bfloat16 v) {
  *reinterpret_cast<__nv_bfloat16*>(base + off) = v;
}

// x = hi + lo with hi = bf16(x), lo = bf16(x - hi): 16 significant bits, fp32 range.
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(hi)));
}

template <int kPlanes>
__global__ void __launch_bounds__(kThreads, 1)
    vc_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnParams P) {
  using Smem = SmemAttn<kPlanes>;
  constexpr int kKStages = Smem::kKStages, kVStages = Smem::kVStages;
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y;
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
      mbar_init(&s.mu_empty[i], 256);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s.s_full[t], 1);
      mbar_init(&s.p_full[t], 256);
      mbar_init(&s.o_done[t], 1);
      mbar_init(&s.r_free[t], 256);
      mbar_init(&s.fin_ready[t], 256);
      mbar_init(&s.o_final[t], 1);
    }
    mbar_init(&s.mma_drain, 1);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  // mean-MMA operands start at zero (unused K slots stay zero); the row-sum B
  // operand is all E4M3 1.0 (every byte 0x38, so the swizzle does not matter)
  for (int i = threadIdx.x; i < (int)(2 * kTileBytes / 16); i += kThreads)
    *reinterpret_cast<uint4*>(&s.mop[0][0] + i * 16) = make_uint4(0u, 0u, 0u, 0u);
  for (int i = threadIdx.x; i < 2048 / 16; i += kThreads)
    *reinterpret_cast<uint4*>(s.ones + i * 16) = make_uint4(kOneE4M3x4, kOneE4M3x4, kOneE4M3x4, kOneE4M3x4);
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const int rowq = bh * P.S_pad + pair * 256;
      mbar_arrive_expect_tx(&s.q_full, 2 * kTileBytes);
      tma_load_2d(s.q[0], &tmQ, &s.q_full, 0, rowq);
      tma_load_2d(s.q[1], &tmQ, &s.q_full, 0, rowq + 128);  // past the head's last tile: unused rows
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nkv && !*(volatile int32_t*)&s.abort_flag; ++j) {
        const int ks = j % kKStages;
        if (!wait_or_abort(s, &s.k_empty[ks], ((j / kKStages) & 1) ^ 1, P)) break;
        mbar_arrive_expect_tx(&s.k_full[ks], kTileBytes);
        tma_load_2d(s.k[ks], &tmK, &s.k_full[ks], 0, bh * P.S_pad + j * 128);
        k_issued = j + 1;
        const int vs = j % kVStages;
        const uint32_t ph = ((j / kVStages) & 1) ^ 1;
        if (!wait_or_abort(s, &s.v_empty[vs], ph, P)) break;
        if (!wait_or_abort(s, &s.mu_empty[vs], ph, P)) break;
        mbar_arrive_expect_tx(&s.v_full[vs], kPlanes * kTileBytes + 512);
#pragma unroll
        for (int pl = 0; pl < kPlanes; ++pl)  // plane pl of head bh: rows (pl * BH + bh) * 128
          tma_load_2d(s.v[vs][pl], &tmV, &s.v_full[vs], j * 128, (pl * P.B * P.H + bh) * 128);
        bulk_load(s.mu[vs], P.mu + ((size_t)bh * P.nb + j) * 128, 512, &s.v_full[vs]);
        v_issued = j + 1;
      }
      // copies still in flight must land before the CTA exits
      const uint64_t drain_ns = 100000000ull;
      mbar_wait(&s.q_full, 0, drain_ns, nullptr);
      for (int j = max(0, k_issued - kKStages); j < k_issued; ++j)
        mbar_wait(&s.k_full[j % kKStages], (j / kKStages) & 1, drain_ns, nullptr);
      for (int j = max(0, v_issued - kVStages); j < v_issued; ++j)
        mbar_wait(&s.v_full[j % kVStages], (j / kVStages) & 1, drain_ns, nullptr);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_f32acc(kFmtE4M3, kFmtE4M3, 128, 128);
      constexpr uint32_t id_row = idesc_f32acc(kFmtE4M3, kFmtE4M3, 128, 16);     // also QK_hi
      constexpr uint32_t id_qk_lo = idesc_f32acc(kFmtE4M3, kFmtE4M3, 128, kRowCol);
      constexpr uint32_t id_mean = idesc_f32acc(kFmtBF16, kFmtBF16, 128, 128);
      const uint64_t dq[2] = {sdesc_k_sw128(smem_u32(s.q[0])), sdesc_k_sw128(smem_u32(s.q[1]))};
      const uint64_t dp[2] = {sdesc_k_sw128(smem_u32(s.p[0])), sdesc_k_sw128(smem_u32(s.p[1]))};
      const uint64_t dm[2] = {sdesc_k_sw128(smem_u32(s.mop[0])), sdesc_k_sw128(smem_u32(s.mop[1]))};
      const uint64_t dones = sdesc_k_sw128(smem_u32(s.ones));
      bool ok = wait_or_abort(s, &s.q_full, 0, P) && wait_or_abort(s, &s.k_full[0], 0, P);
      if (ok) {
        tc_fence_after();
        const uint64_t dk = sdesc_k_sw128(smem_u32(s.k[0]));
        for (int t = 0; t < 2; ++t) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) umma_f8f6f4_ss(tmem + 128 * t, dq[t] + 2 * kk, dk + 2 * kk, id_qk, kk > 0);
          umma_commit(&s.s_full[t]);
        }
        umma_commit(&s.k_empty[0]);
      }
      // Per block j, tile by tile: [mean batch], PV_t(j), ROW_t(j) as soon as P_t(j)
      // is ready, then at once the scores of keys 0-111 of block j+1 (QK_lo); the
      // last 16 keys (QK_hi) overwrite the row-sum columns 112-127, so they wait
      // until the softmax group has read its row sums, which overlaps QK_lo.
      for (int j = 0; ok && j < nkv; ++j) {
        const int vs = j % kVStages;
        const int ks = (j + 1) % kKStages;
        const uint64_t dk = sdesc_k_sw128(smem_u32(s.k[ks]));
        for (int t = 0; t < 2 && ok; ++t) {
          if (!(ok = wait_or_abort(s, &s.p_full[t], j & 1, P))) break;
          if (t == 0 && !(ok = wait_or_abort(s, &s.v_full[vs], (j / kVStages) & 1, P))) break;
          tc_fence_after();
          const uint32_t dO = tmem + 256 + 128 * t;
          if (j >= 1 && (j - 1) % kMeanBlocks == kMeanBlocks - 1) {
            const int ch = ((j - 1) / kMeanBlocks) % kMeanChunks;
            umma_f16_ss(dO, dm[t] + 2 * ch, dm[t] + 2 * (kMeanChunks + ch), id_mean, 1u);
          }
#pragma unroll
          for (int pl = 0; pl < kPlanes; ++pl) {  // O_t += P_t V_hi (+ P_t V_lo)
            const uint64_t dv = sdesc_k_sw128(smem_u32(s.v[vs][pl]));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f8f6f4_ss(dO, dp[t] + 2 * kk, dv + 2 * kk, id_qk, (j > 0 || pl > 0 || kk > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f8f6f4_ss(tmem + 128 * t + kRowCol, dp[t] + 2 * kk, dones + 2 * kk, id_row, kk > 0);
          umma_commit(&s.o_done[t]);
          if (t == 1) umma_commit(&s.v_empty[vs]);
          if (j + 1 < nkv) {
            if (t == 0 && !(ok = wait_or_abort(s, &s.k_full[ks], ((j + 1) / kKStages) & 1, P))) break;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f8f6f4_ss(tmem + 128 * t, dq[t] + 2 * kk, dk + 2 * kk, id_qk_lo, kk > 0);
            if (!(ok = wait_or_abort(s, &s.r_free[t], j & 1, P))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f8f6f4_ss(tmem + 128 * t + kRowCol, dq[t] + 2 * kk, dk + kKeyHiOff + 2 * kk, id_row, kk > 0);
            umma_commit(&s.s_full[t]);
            if (t == 1) umma_commit(&s.k_empty[ks]);
          }
        }
      }
      // the last (possibly partial) batch of block means, then the output is final
      for (int t = 0; t < 2 && ok; ++t) {
        if (!(ok = wait_or_abort(s, &s.fin_ready[t], 0, P))) break;
        tc_fence_after();
        const int ch = ((nkv - 1) / kMeanBlocks) % kMeanChunks;
        umma_f16_ss(tmem + 256 + 128 * t, dm[t] + 2 * ch, dm[t] + 2 * (kMeanChunks + ch), id_mean, 1u);
        umma_commit(&s.o_final[t]);
      }
      // every MMA this thread issued has completed before TMEM is released
      umma_commit(&s.mma_drain);
      mbar_wait(&s.mma_drain, 0, 100000000ull, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int t = warp >> 3;               // query tile
    const int hf = (warp >> 2) & 1;        // score / output column half
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + 128 * t;
    const uint32_t o_addr = tmem + lane_base + 256 + 128 * t + 64 * hf;
    const int qt = pair * 2 + t;
    const bool q_valid = qt < P.nb;
    const float sQ = q_valid ? P.q_scales[(size_t)bh * P.nb + qt] : 1.0f;
    const float sV = __fmul_rn(P.s_v[bh], P.v_mul);   // value scale of the residual codes
    const float inv_sV = __fdiv_rn(1.0f, sV);
    uint8_t* const mo = s.mop[t];
    uint8_t* const prow = s.p[t] + row * 128;
    float F = 0.0f, l = 0.0f;
    bool ok = true, range_ok = true, fail = false;
    const float* const ksc = P.k_scales + (size_t)bh * P.nb;
    float sK_next = ksc[0];
    for (int j = 0; j < nkv; ++j) {
      const float sK = sK_next;                      // this block's K scale, loaded one block ahead
      if (j + 1 < nkv) sK_next = ksc[j + 1];
      // A failed (timed-out) wait never breaks the loop on its own: the group
      // leaves together at the next row-max exchange, whose barrier ORs the
      // failures, so no thread is left waiting in that barrier.
      fail |= !wait_or_abort(s, &s.s_full[t], j & 1, P);
      tc_fence_after();
      uint32_t raw[2][32];
      tmem_ld32(s_addr + 64 * hf, raw[0]);
      tmem_ld32(s_addr + 64 * hf + 32, raw[1]);
      tmem_ld_wait();
      float sc[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) sc[i] = __uint_as_float(raw[i >> 5][i & 31]);
      const int valid = min(128, P.S - j * 128) - 64 * hf;   // valid columns of this half
      if (valid < 64) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i >= valid) sc[i] = -INFINITY;
      }
      // partial max of this half's raw scores, then the full row max
      float m0 = sc[0], m1 = sc[1];
#pragma unroll
      for (int i = 2; i < 62; i += 4) {
        m0 = fmax3(m0, sc[i + 0], sc[i + 1]);
        m1 = fmax3(m1, sc[i + 2], sc[i + 3]);
      }
      const float mp = fmax3(m0, m1, fmaxf(sc[62], sc[63]));
      s.xmax[j & 1][t][hf][row] = mp;
      if (named_bar_any(1 + t, 256, fail)) {
        ok = false;
        break;
      }
      const float tmax = fmaxf(mp, s.xmax[j & 1][t][hf ^ 1][row]);
      // c > 0, so max(c t) = c max(t)
      const float c = __fmul_rn(__fmul_rn(sQ, sK), P.kappa);
      const float Mtile = ceilf(__fmul_rn(c, tmax));
      const float Fn = j == 0 ? Mtile : fmaxf(F, Mtile);
      const bool resc = j > 0 && Fn > F;
      const float alpha = resc ? exp2_int((int)(F - Fn)) : 1.0f;
      const float bias = expcast_bias(P.bias_b, Fn);
      const float c8 = 8.0f * c;
      // The single-fma form below needs the frame's bias to be exact and the codes
      // to stay in the fp32 binade [2^23, 2^24): |F| < 2^19 (log2-domain scores
      // below 524288). Larger scores are reported, not computed.
      range_ok &= fabsf(Fn) < 524288.0f;
      // ExpCast: one fma per score on the magic-biased fp32; the low byte is the
      // code; the clamp at the magic value is code 0 (masked tail scores are -inf)
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t w[8];
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const int i = cc * 32 + q4 * 4;
          const float2 a = ffma2(make_float2(sc[i], sc[i + 1]), make_float2(c8, c8), make_float2(bias, bias));
          const float2 b = ffma2(make_float2(sc[i + 2], sc[i + 3]), make_float2(c8, c8), make_float2(bias, bias));
          w[q4] = pack_codes4(fmaxf(a.x, kMagic), fmaxf(a.y, kMagic), fmaxf(b.x, kMagic), fmaxf(b.y, kMagic));
        }
        const int k0 = 4 * hf + 2 * cc;
        *reinterpret_cast<uint4*>(prow + ((k0 ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(prow + (((k0 + 1) ^ (row & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
      }
      fence_proxy_async_smem();
      if (__any_sync(0xffffffffu, resc)) {
        // the frame moved: O_t (complete up to block j-1), l and the row sums not
        // yet handed to a mean MMA are rescaled by the exact 2^(F_old - F_new)
#pragma unroll 1
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t r[32];
          tmem_ld32(o_addr + 32 * cc, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(o_addr + 32 * cc, r);
          tmem_st_wait();  // the store reads r asynchronously: done before r is reused
        }
        if (resc && hf == 1) {
          const int jp = j - 1, ch = (jp / kMeanBlocks) % kMeanChunks;
          const int nslots = 3 * (jp % kMeanBlocks) + 3;
          for (int sl = 0; sl < nslots; ++sl) {
            __nv_bfloat16* e = reinterpret_cast<__nv_bfloat16*>(mo + sw128_off16(row, ch, sl));
            *e = __float2bfloat16_rn(__bfloat162float(*e) * alpha);
          }
          fence_proxy_async_smem();
        }
      }
      l *= alpha;
      F = Fn;
      tc_fence_before();
      mbar_arrive(&s.p_full[t]);
      // row sum of this block's cast P (tensor core), then the mean-MMA operands:
      // the upper half writes the row sums of its rows, the lower half the block
      // mean / s_V of channel `row`
      fail |= !wait_or_abort(s, &s.o_done[t], j & 1, P);
      tc_fence_after();
      const float r = __uint_as_float(tmem_ld1(s_addr + kRowCol));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&s.r_free[t]);
      l = __fadd_rn(l, r);
      const int g = j % kMeanBlocks, ch = (j / kMeanBlocks) % kMeanChunks;
      const bool last = j == nkv - 1;
      if (hf == 1) {
        __nv_bfloat16 rh, rl;
        split_bf16(r, rh, rl);
        st_bf16(mo, sw128_off16(row, ch, 3 * g + 0), rh);
        st_bf16(mo, sw128_off16(row, ch, 3 * g + 1), rh);
        st_bf16(mo, sw128_off16(row, ch, 3 * g + 2), rl);
        if (last)
          for (int sl = 3 * g + 3; sl < 16; ++sl) st_bf16(mo, sw128_off16(row, ch, sl), __float2bfloat16_rn(0.0f));
      } else {
        const int vs = j % kVStages;
        fail |= !wait_or_abort(s, &s.v_full[vs], (j / kVStages) & 1, P);
        const float m = __fmul_rn(s.mu[vs][row], inv_sV);
        mbar_arrive(&s.mu_empty[vs]);
        __nv_bfloat16 mh, ml;
        split_bf16(m, mh, ml);
        st_bf16(mo, sw128_off16(row, kMeanChunks + ch, 3 * g + 0), mh);
        st_bf16(mo, sw128_off16(row, kMeanChunks + ch, 3 * g + 1), ml);
        st_bf16(mo, sw128_off16(row, kMeanChunks + ch, 3 * g + 2), mh);
        if (last)
          for (int sl = 3 * g + 3; sl < 16; ++sl)
            st_bf16(mo, sw128_off16(row, kMeanChunks + ch, sl), __float2bfloat16_rn(0.0f));
      }
      if (g == kMeanBlocks - 1 || last) fence_proxy_async_smem();
    }
    if (!range_ok) report_status(P.status, VC_ERR_UNSUPPORTED);
    ok = __all_sync(0xffffffffu, ok && !fail);
    if (ok) {
      mbar_arrive(&s.fin_ready[t]);
      ok = __all_sync(0xffffffffu, wait_or_abort(s, &s.o_final[t], 0, P));
    }
    if (ok) {
      // epilogue: O = s_V O_t / l, BF16, original query order and layout; this
      // thread writes channels 64 hf .. 64 hf + 63 of its row
      tc_fence_after();
      const int q = qt * 128 + row;
      const float scale = __fdiv_rn(sV, l);
      const int b = bh / P.H, h = bh % P.H;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(P.o) + (((size_t)b * P.S + q) * P.H + h) * 128 + 64 * hf;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t r[32];
        tmem_ld32(o_addr + 32 * cc, r);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          __nv_bfloat162 b2 =
              __floats2bfloat162_rn(__uint_as_float(r[2 * i]) * scale, __uint_as_float(r[2 * i + 1]) * scale);
          pk[i] = *reinterpret_cast<uint32_t*>(&b2);
        }
        if (q_valid && q < P.S) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
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
  cudaError_t e = cudaFuncSetAttribute(vc_attn_fwd_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(sizeof(SmemAttn<1>) + 1024));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(vc_attn_fwd_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)(sizeof(SmemAttn<2>) + 1024));
}

cudaError_t launch_attn_e4m3(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const AttnParams& p, cudaStream_t st) {
  const dim3 grid((p.nb + 1) / 2, p.B * p.H);
  vc_attn_fwd_kernel<1><<<grid, kThreads, sizeof(SmemAttn<1>) + 1024, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_planes(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tplanes,
                               const AttnParams& p, cudaStream_t st) {
  const dim3 grid((p.nb + 1) / 2, p.B * p.H);
  vc_attn_fwd_kernel<2><<<grid, kThreads, sizeof(SmemAttn<2>) + 1024, st>>>(tq, tk, tplanes, p);
  return cudaGetLastError();
}

}  // namespace vc
