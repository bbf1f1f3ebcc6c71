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
//   warps 0-3   softmax of query tile 0: one thread per query row (warp w
//               reaches the 32 tensor-memory lanes 32w .. 32w+31)
//   warps 4-7   softmax of query tile 1
//   warp  8     TMA: both Q tiles once; K_j and V^T_j into rings; it also
//               writes the bf16 block-mean operand of the mean MMA
//   warp  9     issues the QK products of both tiles (one elected lane)
//   warps 10-11 issue the PV (and mean) products of tile 0 and tile 1
// The three issuing warps are independent streams into the tensor pipe, so an
// MMA whose inputs are ready never waits behind another stream's barrier.
// Tensor memory (512 columns):
//   O_0 [0, 144)    tile 0: output channels 0-127, then 16 row-sum columns
//   O_1 [144, 288)  tile 1: 16 row-sum columns, then output channels 0-127
//   S_0 [288, 416)  tile 0 scores
//   S_1 [320, 448)  tile 1 scores (shares 96 columns with S_0)
//   P_0 [448, 480), P_1 [480, 512)   E4M3 probability codes, 4 per column
// The QK products alternate between the tiles: each starts only after the
// other tile's softmax warps have loaded the scores in the shared columns
// (s_loaded). P has columns of its own, so the scores of block j+1 are computed
// while the softmax threads still cast block j.
// Per block j and tile t the tensor core runs
//   PV   O_t += P_t [V_j ; 1]     P_t (E4M3 codes) read from tensor memory,
//        V_j^T (residual codes) with 16 rows of E4M3 1.0 appended from shared
//        memory (N = 144): the extra columns accumulate the row sum l of the
//        cast P exactly as PV sees it
//   QK   S_t = Q_t K_{j+1}^T     kind::f8f6f4, M = N = K = 128
//   MEAN after every 5 blocks:  O_t += R_t M     kind::f16 with bf16 operands:
//        R_t = the blocks' row sums r_b (growth of l from block to block), M =
//        their block means / s_V, each split into bf16 hi/lo parts (r_hi m_hi +
//        r_hi m_lo + r_lo m_hi, three K slots a block). R_t sits in a 128-B-
//        swizzled smem tile of its own (K chunks 0-1, alternating by batch),
//        written by the softmax threads only between s_full and p_full, when
//        no MMA of their tile is in flight; M (shared by both tiles) in a
//        double-buffered unswizzled tile written by the TMA warp
// so O_t accumulates the whole output in residual-code units; the epilogue is
// O = s_V O_t / l (s_V per output channel for the per-channel residual scale).
// The MX-style FP4 residual (kVKind = kVMx) runs PV as the block-scaled
// kind::mxf8f6f4 product: V^T arrives as E2M1 codes (TMA widens each 16 packed
// codes into a 16-byte smem container), its power-of-two scale per channel and
// 32 tokens as UE8M0 bytes that the softmax threads of each tile copy into
// tensor memory (SFB_t) next to P_t, the probabilities' scale is a constant 2^0
// (SFA_t); the two score tiles then share all 128 of their columns, which frees
// the 32 columns the scale factors need. The softmax thread of row i keeps the integer running frame
// F (ceil of the largest log2-domain score so far); a block is cast in the frame
// current after it; when F moves, O_t (with its row-sum column) and the row sums
// not yet handed to a mean MMA (held in registers until their batch of 5 blocks
// is complete) are multiplied by the exact power 2^(F_old - F_new).
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
// kVKind: how the residual codes are scaled back to values.
constexpr int kVHead = 0;     // one scale s_V per (b, h)
constexpr int kVChannel = 1;  // one scale per (b, h, channel): applied per output channel
constexpr int kVMx = 2;       // MX-style FP4: a power of two per channel and 32 tokens, in the MMA
template <int kPlanes> struct Stages {
  static constexpr int K = 3;
  static constexpr int V = kPlanes == 1 ? 3 : 2;
};
constexpr uint32_t kTileBytes = 128 * 128;  // one 128 x 128 E4M3 tile (or 128 x 64 bf16)
constexpr uint32_t kOnesBytes = 16 * 128;   // 16 rows of E4M3 1.0 (K = 128 keys)
constexpr uint32_t kMopBytes = 128 * 16 * 2;  // M operand of one batch: 128 channels x 16 bf16
constexpr int kThreads = 384;
constexpr int kTmaWarp = 8, kQkWarp = 9, kPvWarp0 = 10;
constexpr uint32_t kTmemCols = 512;
constexpr int kMeanBlocks = 5;              // key blocks per mean MMA (3 K slots each: 15 of 16)
constexpr int kMeanChunks = 2;              // R: 16-slot K chunks 0 and 1, alternating by batch
constexpr uint32_t kOneE4M3x4 = 0x38383838u;
// E2M1 1.0 (code 2) in the 16-byte smem container of 16 FP4 codes: the low 8
// bytes hold the codes, two per byte, the high 8 bytes are padding
constexpr uint32_t kOneE2M1x8 = 0x22222222u, kE2M1Pad = 0u;
constexpr uint32_t kSfOne4 = 0x7F7F7F7Fu;   // four UE8M0 scale bytes of 2^0
constexpr uint32_t kSfBytes = 512;          // MX exponents of one V block: 128 channels x 4 groups
// transaction bytes of one 128 x 128 tile of E2M1 codes: the packed bytes read
// (64 per row), although each 16 codes land in a 16-byte shared-memory container
// whose upper 8 bytes the TMA leaves untouched (the MMA ignores them)
constexpr uint32_t kMxTileTx = kTileBytes / 2;
// tensor-memory columns (see the layout above)
__device__ __forceinline__ constexpr uint32_t col_o(int t) { return t ? 144u : 0u; }    // PV accumulator, N = 144
__device__ __forceinline__ constexpr uint32_t col_ch(int t) { return t ? 160u : 0u; }   // output channels 0-127
__device__ __forceinline__ constexpr uint32_t col_l(int t) { return t ? 144u : 128u; }  // first row-sum column
__device__ __forceinline__ constexpr uint32_t col_s(int t) { return t ? 320u : 288u; }  // scores
__device__ __forceinline__ constexpr uint32_t col_p(int t) { return t ? 480u : 448u; }  // P codes, 32 columns
// MX-style V: both score tiles in [320, 448); the scale factors of P (constant
// 2^0, 4 columns) and of V^T (5 of 8 columns) of each tile below them
__device__ __forceinline__ constexpr uint32_t col_s_mx() { return 320u; }
__device__ __forceinline__ constexpr uint32_t col_sfa(int t) { return t ? 292u : 288u; }
__device__ __forceinline__ constexpr uint32_t col_sfb(int t) { return t ? 304u : 296u; }

// One V ring stage: [16 rows of 1.0][plane 0: V^T tile][16 rows of 1.0][plane 1].
// Tile 0's PV reads plane 0 followed by the second band (ones last), tile 1's
// the first band followed by plane 0 (ones first), so that the row sums land
// at the ends of the two accumulators given above.
// The MX-style stage appends the block's 512 exponent bytes (kSf), padded to
// keep every stage 1024-byte aligned.
template <int kPlanes, bool kMx = false> struct VStage {
  static constexpr uint32_t kPlane0 = kOnesBytes;
  static constexpr uint32_t kOnes1 = kOnesBytes + kTileBytes;
  static constexpr uint32_t kPlane1 = 2 * kOnesBytes + kTileBytes;
  static constexpr uint32_t kSf = 2 * kOnesBytes + kPlanes * kTileBytes;
  static constexpr uint32_t kBytes = 2 * kOnesBytes + kPlanes * kTileBytes + (kMx ? 1024u : 0u);
};

template <int kPlanes, bool kMx = false>
struct __align__(1024) SmemAttn {
  static constexpr int kKStages = Stages<kPlanes>::K, kVStages = Stages<kPlanes>::V;
  uint8_t q[2][kTileBytes];
  uint8_t k[kKStages][kTileBytes];
  uint8_t v[kVStages][VStage<kPlanes, kMx>::kBytes];
  uint8_t rop[2][kTileBytes];    // R operand of the mean MMA, one 128-B-swizzled tile per query tile
  uint8_t mop[2][kMopBytes];     // M operand, unswizzled, one per batch parity
  uint64_t q_full;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t m_full[2], m_empty[2];
  uint64_t s_full[2], s_loaded[2], p_full[2], pv_done[2], fin_ready[2], o_final[2];
  uint64_t mma_drain[3];
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

// wait_or_abort for a whole warp: every lane returns the same answer.
template <class Smem>
__device__ __forceinline__ bool wait_warp(Smem& s, uint64_t* bar, uint32_t parity, const AttnParams& P) {
  return __all_sync(0xffffffffu, wait_or_abort(s, bar, parity, P));
}

// wait_warp for the TMA and MMA-issuing warps: they poll without asking to be
// suspended, so that an issuing warp sees its barrier complete at once (it is
// on the critical path between the two query tiles' score hand-overs). Bounded
// like every wait: the time limit and the CTA's abort flag are checked every 64
// polls.
template <class Smem>
__device__ __forceinline__ bool wait_spin_warp(Smem& s, uint64_t* bar, uint32_t parity, const AttnParams& P) {
  bool ok = mbar_try_wait(bar, parity);
  if (!ok) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
      if (mbar_try_wait(bar, parity)) {
        ok = true;
        break;
      }
      if ((it & 63u) == 0u &&
          (globaltimer_ns() - t0 > P.wait_ns || *reinterpret_cast<volatile int32_t*>(&s.abort_flag) != 0))
        break;
    }
    if (!ok) {
      s.abort_flag = 1;
      report_status(P.status, VC_ERR_TIMEOUT);
    }
  }
  return __all_sync(0xffffffffu, ok);
}

// x = hi + lo with hi = bf16(x), lo = bf16(x - hi): 16 significant bits, fp32 range.
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(hi)));
}

__device__ __forceinline__ uint32_t bf16_bits(__nv_bfloat16 x) {
  return (uint32_t)*reinterpret_cast<const uint16_t*>(&x);
}

// Writes one batch of row sums into chunk ch of row `row` of the R operand tile:
// r[i] for the batch's blocks i < n as the three K slots hi, hi, lo, the other
// slots 0. A chunk's 16 slots are two 16-byte pieces of the 128-B row.
__device__ __forceinline__ void put_r_batch(uint8_t* ro, int row, int ch, const float (&r)[kMeanBlocks], int n) {
  uint32_t h[16];
#pragma unroll
  for (int i = 0; i < kMeanBlocks; ++i) {
    __nv_bfloat16 hi, lo;
    split_bf16(i < n ? r[i] : 0.0f, hi, lo);
    h[3 * i] = h[3 * i + 1] = bf16_bits(hi);
    h[3 * i + 2] = bf16_bits(lo);
  }
  h[15] = 0u;
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = h[2 * i] | (h[2 * i + 1] << 16);
  uint8_t* base = ro + row * 128;
  const int x = row & 7;
  *reinterpret_cast<uint4*>(base + (((2 * ch) ^ x) & 7) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(base + (((2 * ch + 1) ^ x) & 7) * 16) = make_uint4(w[4], w[5], w[6], w[7]);
}

// M operand layout (unswizzled K-major, core matrices of 8 channels x 8 slots):
// channel c, slots 8h .. 8h+7 are the 16 bytes at (c/8)*256 + h*128 + (c%8)*16.
constexpr uint32_t kMopLbo = 128, kMopSbo = 256;


// Four magic-biased codes (low bytes of the fp32 patterns) into one word, a in
// the lowest byte. b*256 + a keeps a's and b's codes (< 256) in the low 16 bits
// (the magic's low 12 bits are zero, so nothing carries into them); the
// multiply-adds run on the fma pipe, one byte permute merges the halves.
__device__ __forceinline__ uint32_t pack4_imad(float a, float b, float c, float d) {
  const uint32_t lo = __float_as_uint(b) * 256u + __float_as_uint(a);
  const uint32_t hi = __float_as_uint(d) * 256u + __float_as_uint(c);
  return __byte_perm(lo, hi, 0x5410);
}

// kExp2 = true builds the comparison kernel: the same pipeline with the
// probabilities made the conventional way, 2^(c t - F + k_P) on the special
// function unit (ex2.approx) and then converted to E4M3 (round to nearest even,
// saturating), instead of ExpCast's single fma per score.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int kPlanes, bool kExp2 = false, int kVKind = kVHead>
__global__ void __launch_bounds__(kThreads, 1)
    vc_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnParams P) {
  constexpr bool kMx = kVKind == kVMx;
  static_assert(!kMx || kPlanes == 1, "the MX-style residual is one plane");
  using Smem = SmemAttn<kPlanes, kMx>;
  using VS = VStage<kPlanes, kMx>;
  constexpr int kKStages = Smem::kKStages, kVStages = Smem::kVStages;
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y;
  const int nkv = P.nb;
  const int nbatch = (nkv + kMeanBlocks - 1) / kMeanBlocks;

  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.v_empty[i], 2);   // PV_0(j) and PV_1(j) both read V_j
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s.m_full[t], 1);
      mbar_init(&s.m_empty[t], 2);   // both tiles' mean MMAs read it
      mbar_init(&s.s_full[t], 1);
      mbar_init(&s.s_loaded[t], 4);
      mbar_init(&s.p_full[t], 128);
      mbar_init(&s.pv_done[t], 1);
      mbar_init(&s.fin_ready[t], 128);
      mbar_init(&s.o_final[t], 1);
    }
    for (int i = 0; i < 3; ++i) mbar_init(&s.mma_drain[i], 1);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  // R operands start at zero (unused K slots stay zero); the two bands of every
  // V stage are all E4M3 1.0 (every byte 0x38, so the swizzle does not matter);
  // the TMA never writes them
  for (int i = threadIdx.x; i < (int)(2 * kTileBytes / 16); i += kThreads)
    *reinterpret_cast<uint4*>(&s.rop[0][0] + i * 16) = make_uint4(0u, 0u, 0u, 0u);
  for (int i = threadIdx.x; i < (int)(kVStages * 2 * kOnesBytes / 16); i += kThreads) {
    const int st = i / (2 * kOnesBytes / 16), r = i % (2 * kOnesBytes / 16);
    const uint32_t off = r < (int)(kOnesBytes / 16) ? r * 16 : VS::kOnes1 + (r - kOnesBytes / 16) * 16;
    *reinterpret_cast<uint4*>(&s.v[st][0] + off) =
        kMx ? make_uint4(kOneE2M1x8, kOneE2M1x8, kE2M1Pad, kE2M1Pad)   // a whole 16-byte container
            : make_uint4(kOneE4M3x4, kOneE4M3x4, kOneE4M3x4, kOneE4M3x4);
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  // value scale of the residual codes (per-channel scales are read where used;
  // the MX-style residual carries its scales inside the product: s_v is 1)
  const float sV = kVKind == kVChannel ? 1.0f : __fmul_rn(P.s_v[bh], P.v_mul);

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp runs the loop (its values stay warp-uniform); one elected
    // lane issues the copies. Every kMeanBlocks blocks the warp also writes the
    // M operand of one batch: lane l takes channels l, l+32, l+64, l+96.
    const bool leader = elect_one();
    float inv_sV[4];   // 1 / s_V of channels lane + 32 i
#pragma unroll
    for (int i = 0; i < 4; ++i)
      inv_sV[i] = __fdiv_rn(1.0f, kVKind == kVChannel ? P.s_v[(size_t)bh * 128 + lane + 32 * i] : sV);
    const float* const mu_bh = P.mu + (size_t)bh * P.nb * 128;
    float mnext[kMeanBlocks][4];  // block means of the next batch, loaded one batch ahead
    auto load_means = [&](int batch) {
#pragma unroll
      for (int g = 0; g < kMeanBlocks; ++g) {
        const int b = batch * kMeanBlocks + g;
#pragma unroll
        for (int i = 0; i < 4; ++i) mnext[g][i] = b < nkv ? __ldg(mu_bh + (size_t)b * 128 + lane + 32 * i) : 0.0f;
      }
    };
    load_means(0);
    if (leader) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const int rowq = bh * P.S_pad + pair * 256;
      mbar_arrive_expect_tx(&s.q_full, 2 * kTileBytes);
      tma_load_2d(s.q[0], &tmQ, &s.q_full, 0, rowq);
      tma_load_2d(s.q[1], &tmQ, &s.q_full, 0, rowq + 128);  // past the head's last tile: unused rows
    }
    int k_issued = 0, v_issued = 0;
    for (int j = 0; j < nkv && !*(volatile int32_t*)&s.abort_flag; ++j) {
      const int ks = j % kKStages;
      if (!wait_spin_warp(s, &s.k_empty[ks], ((j / kKStages) & 1) ^ 1, P)) break;
      if (leader) {
        mbar_arrive_expect_tx(&s.k_full[ks], kTileBytes);
        tma_load_2d(s.k[ks], &tmK, &s.k_full[ks], 0, bh * P.S_pad + j * 128);
      }
      k_issued = j + 1;
      const int vs = j % kVStages;
      if (!wait_spin_warp(s, &s.v_empty[vs], ((j / kVStages) & 1) ^ 1, P)) break;
      if (leader) {
        if (kMx) {
          // the E2M1 tile (x in codes: 64 bytes a block in HBM) and the block's exponents
          mbar_arrive_expect_tx(&s.v_full[vs], kMxTileTx + kSfBytes);
          tma_load_2d(&s.v[vs][0] + VS::kPlane0, &tmV, &s.v_full[vs], j * 128, bh * 128);
          bulk_load(&s.v[vs][0] + VS::kSf, P.v_scales + ((size_t)bh * P.nb + j) * kSfBytes, kSfBytes,
                    &s.v_full[vs]);
        } else {
          mbar_arrive_expect_tx(&s.v_full[vs], kPlanes * kTileBytes);
          // plane pl of head bh: rows (pl * BH + bh) * 128
          tma_load_2d(&s.v[vs][0] + VS::kPlane0, &tmV, &s.v_full[vs], j * 128, bh * 128);
          if (kPlanes == 2)
            tma_load_2d(&s.v[vs][0] + VS::kPlane1, &tmV, &s.v_full[vs], j * 128, (P.B * P.H + bh) * 128);
        }
      }
      v_issued = j + 1;
      if (j % kMeanBlocks == 0) {
        // M operand of batch n = j / kMeanBlocks: slots (hi, lo, hi) of mu_b / s_V
        // for its blocks, zero for blocks past the end and for slot 15
        const int n = j / kMeanBlocks, mb = n & 1;
        if (!wait_spin_warp(s, &s.m_empty[mb], ((n >> 1) & 1) ^ 1, P)) break;
        float cur[kMeanBlocks][4];
#pragma unroll
        for (int g = 0; g < kMeanBlocks; ++g)
#pragma unroll
          for (int i = 0; i < 4; ++i) cur[g][i] = mnext[g][i];
        if (n + 1 < nbatch) load_means(n + 1);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = lane + 32 * i;
          uint32_t h[8];  // 16 slots, two per word
          uint32_t sl[16];
#pragma unroll
          for (int g = 0; g < kMeanBlocks; ++g) {
            __nv_bfloat16 mh, ml;
            split_bf16(__fmul_rn(cur[g][i], inv_sV[i]), mh, ml);
            sl[3 * g + 0] = bf16_bits(mh);
            sl[3 * g + 1] = bf16_bits(ml);
            sl[3 * g + 2] = bf16_bits(mh);
          }
          sl[15] = 0u;
#pragma unroll
          for (int k2 = 0; k2 < 8; ++k2) h[k2] = sl[2 * k2] | (sl[2 * k2 + 1] << 16);
          uint8_t* dst = s.mop[mb] + (c >> 3) * kMopSbo + (c & 7) * 16;
          *reinterpret_cast<uint4*>(dst) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4*>(dst + kMopLbo) = make_uint4(h[4], h[5], h[6], h[7]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (leader) mbar_arrive(&s.m_full[mb]);
      }
    }
    // copies still in flight must land before the CTA exits
    const uint64_t drain_ns = 100000000ull;
    mbar_wait(&s.q_full, 0, drain_ns, nullptr);
    for (int j = max(0, k_issued - kKStages); j < k_issued; ++j)
      mbar_wait(&s.k_full[j % kKStages], (j / kKStages) & 1, drain_ns, nullptr);
    for (int j = max(0, v_issued - kVStages); j < v_issued; ++j)
      mbar_wait(&s.v_full[j % kVStages], (j / kVStages) & 1, drain_ns, nullptr);
  } else if (warp >= kQkWarp) {
    // ------------------------------------------------------------ MMA issuers
    // Each issuing warp runs its loop warp-wide so that descriptors and
    // addresses stay warp-uniform (uniform registers feed tcgen05.mma directly);
    // one elected lane issues the MMAs and the commits that track them.
    const bool leader = elect_one();
    auto commit = [&](uint64_t* bar) {
      if (leader) umma_commit(bar);
    };
    bool ok = true;
    if (warp == kQkWarp) {
      constexpr uint32_t id_qk = idesc_f32acc(kFmtE4M3, kFmtE4M3, 128, 128);
      const uint64_t dq[2] = {sdesc_k_sw128(smem_u32(s.q[0])), sdesc_k_sw128(smem_u32(s.q[1]))};
      auto qk = [&](int t, int ks) {  // S_t = Q_t K^T
        const uint64_t dk = sdesc_k_sw128(smem_u32(s.k[ks]));
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f8f6f4_ss(tmem + (kMx ? col_s_mx() : col_s(t)), dq[t] + 2 * kk, dk + 2 * kk, id_qk, kk > 0);
        }
      };
      // The QK products alternate between the tiles through the shared score
      // columns: S_1(j) once tile 0 has loaded S_0(j), S_0(j+1) once tile 1 has
      // loaded S_1(j).
      ok = wait_spin_warp(s, &s.q_full, 0, P);
      for (int j = 0; ok && j < nkv; ++j) {
        const int ks = j % kKStages;
        if (!(ok = wait_spin_warp(s, &s.k_full[ks], (j / kKStages) & 1, P))) break;
        if (j > 0 && !(ok = wait_spin_warp(s, &s.s_loaded[1], (j - 1) & 1, P))) break;
        tc_fence_after();
        qk(0, ks);
        commit(&s.s_full[0]);
        if (!(ok = wait_spin_warp(s, &s.s_loaded[0], j & 1, P))) break;
        tc_fence_after();
        qk(1, ks);
        commit(&s.s_full[1]);
        commit(&s.k_empty[ks]);
      }
      commit(&s.mma_drain[0]);
      mbar_wait(&s.mma_drain[0], 0, 100000000ull, nullptr);
    } else {
      const int t = warp - kPvWarp0;
      constexpr uint32_t id_pv = idesc_f32acc(kFmtE4M3, kFmtE4M3, 128, 144);
      constexpr uint32_t id_pv2 = idesc_f32acc(kFmtE4M3, kFmtE4M3, 128, 128);
      constexpr uint32_t id_mean = idesc_f32acc(kFmtBF16, kFmtBF16, 128, 128);
      const uint64_t dr = sdesc_k_sw128(smem_u32(s.rop[t]));
      // O_t += R_t M of one batch of blocks (both tiles read the same M tile)
      auto mean = [&](int batch) -> bool {
        const int mb = batch & 1;
        if (!wait_spin_warp(s, &s.m_full[mb], (batch >> 1) & 1, P)) return false;
        tc_fence_after();
        const uint64_t dmo = sdesc_k_noswz(smem_u32(s.mop[mb]), kMopLbo, kMopSbo);
        if (leader) umma_f16_ss(tmem + col_ch(t), dr + 2 * (batch % kMeanChunks), dmo, id_mean, 1u);
        commit(&s.m_empty[mb]);
        return true;
      };
      // Per block j: [mean batch], then O_t (+ row sums) += P_t(j) [V_j ; 1]
      // (tile 1: [1 ; V_j]) as soon as P_t(j) is in tensor memory.
      for (int j = 0; ok && j < nkv; ++j) {
        const int vs = j % kVStages;
        if (!(ok = wait_spin_warp(s, &s.p_full[t], j & 1, P))) break;
        if (!(ok = wait_spin_warp(s, &s.v_full[vs], (j / kVStages) & 1, P))) break;
        tc_fence_after();
        if (j >= kMeanBlocks && j % kMeanBlocks == 0 && !(ok = mean(j / kMeanBlocks - 1))) break;
        const uint32_t vb = smem_u32(&s.v[vs][0]);
        const uint64_t dv = sdesc_k_sw128(vb + (t == 0 ? VS::kPlane0 : 0u));
        if (leader) {
          if (kMx) {
            // K group kk of the block: scale byte kk of every SFB_t cell
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_mx_ts(tmem + col_o(t), tmem + col_p(t) + 8 * kk, dv + 2 * kk,
                         idesc_mx(kFmtE4M3, kFmtE2M1, 128, 144, 0, kk), tmem + col_sfa(t), tmem + col_sfb(t),
                         (j > 0 || kk > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f8f6f4_ts(tmem + col_o(t), tmem + col_p(t) + 8 * kk, dv + 2 * kk, id_pv,
                             (j > 0 || kk > 0) ? 1u : 0u);
          }
          if (kPlanes == 2) {
            const uint64_t dv2 = sdesc_k_sw128(vb + VS::kPlane1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f8f6f4_ts(tmem + col_ch(t), tmem + col_p(t) + 8 * kk, dv2 + 2 * kk, id_pv2, 1u);
          }
        }
        commit(&s.pv_done[t]);
        commit(&s.v_empty[vs]);
      }
      // the last (possibly partial) batch of block means, then the output is final
      if (ok) ok = wait_warp(s, &s.fin_ready[t], 0, P);
      if (ok) {
        tc_fence_after();
        ok = mean(nbatch - 1);
      }
      if (ok) commit(&s.o_final[t]);
      // every MMA this warp issued has completed before TMEM is released
      commit(&s.mma_drain[1 + t]);
      mbar_wait(&s.mma_drain[1 + t], 0, 100000000ull, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int t = warp >> 2;               // query tile
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + (kMx ? col_s_mx() : col_s(t));
    const uint32_t sfb_addr = tmem + lane_base + col_sfb(t);
    if (kMx) {
      // the probabilities' scale factors: 2^0 for every row and K group; written
      // once (each warp its own lane quarter), before the tile's first p_full
      tmem_st4(tmem + lane_base + col_sfa(t), kSfOne4, kSfOne4, kSfOne4, kSfOne4);
    }
    const uint32_t p_addr = tmem + lane_base + col_p(t);
    const uint32_t o_addr = tmem + lane_base + col_ch(t);
    const uint32_t l_addr = tmem + lane_base + col_l(t);
    const int qt = pair * 2 + t;
    const bool q_valid = qt < P.nb;
    const float sQ = q_valid ? P.q_scales[(size_t)bh * P.nb + qt] : 1.0f;
    uint8_t* const ro = s.rop[t];
    // F: running integer frame; Lp: row-sum column after the last block's own
    // rescale, so that the next read minus Lp is that block's row sum
    float F = 0.0f, Lp = 0.0f;
    // row sums of the current batch of blocks, in the current frame (written to
    // the R operand when the batch is complete)
    float rb[kMeanBlocks] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    bool ok = true, range_ok = true;
    const float* const ksc = P.k_scales + (size_t)bh * P.nb;
    float sK_next = ksc[0];
    for (int j = 0; j < nkv; ++j) {
      const float sK = sK_next;                      // this block's K scale, loaded one block ahead
      if (j + 1 < nkv) sK_next = ksc[j + 1];
      if (!(ok = wait_warp(s, &s.s_full[t], j & 1, P))) break;
      tc_fence_after();
      uint32_t sc[4][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(s_addr + 32 * cc, sc[cc]);
      tmem_ld_wait();
      // this warp's scores are in registers: the other tile's QK may now overwrite
      // the shared columns
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.s_loaded[t]);
      const int valid = min(128, P.S - j * 128);
      if (valid < 128) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i >= valid) sc[i >> 5][i & 31] = __float_as_uint(-INFINITY);
      }
#define SC(i) __uint_as_float(sc[(i) >> 5][(i) & 31])
      // row max of the raw scores (c > 0, so max(c t) = c max(t))
      float m0 = SC(0), m1 = SC(1), m2 = SC(2), m3 = SC(3);
#pragma unroll
      for (int i = 4; i < 124; i += 8) {
        m0 = fmax3(m0, SC(i + 0), SC(i + 1));
        m1 = fmax3(m1, SC(i + 2), SC(i + 3));
        m2 = fmax3(m2, SC(i + 4), SC(i + 5));
        m3 = fmax3(m3, SC(i + 6), SC(i + 7));
      }
      m0 = fmax3(m0, SC(124), SC(125));
      m1 = fmax3(m1, SC(126), SC(127));
      const float tmax = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
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
      uint32_t w[32];
      if (!kExp2) {
#pragma unroll
        for (int q4 = 0; q4 < 32; ++q4) {
          const int i = q4 * 4;
          const float2 a = ffma2(make_float2(SC(i), SC(i + 1)), make_float2(c8, c8), make_float2(bias, bias));
          const float2 b = ffma2(make_float2(SC(i + 2), SC(i + 3)), make_float2(c8, c8), make_float2(bias, bias));
          w[q4] = pack4_imad(fmaxf(a.x, kMagic), fmaxf(a.y, kMagic), fmaxf(b.x, kMagic), fmaxf(b.y, kMagic));
        }
      } else {
        const float off = (float)((P.bias_b - 56) / 8) - Fn;  // k_P - F
#pragma unroll
        for (int q4 = 0; q4 < 32; ++q4) {
          const int i = q4 * 4;
          const uint32_t lo = cvt_e4m3x2(ex2_approx(__fmaf_rn(SC(i), c, off)), ex2_approx(__fmaf_rn(SC(i + 1), c, off)));
          const uint32_t hi =
              cvt_e4m3x2(ex2_approx(__fmaf_rn(SC(i + 2), c, off)), ex2_approx(__fmaf_rn(SC(i + 3), c, off)));
          w[q4] = lo | (hi << 16);
        }
      }
#undef SC
      // MX-style V: the scale factors of V_j^T for this tile's B operand, one
      // cell per (lane, column c): the 4 group exponents of B row n = lane + 32 c,
      // which is channel n (tile 0: ones rows at n >= 128) or n - 16 (tile 1:
      // ones rows first); the ones rows and the unused cells take 2^0
      uint32_t sfr[8];
      if (kMx) {
        const int vs = j % kVStages;
        if (!(ok = wait_warp(s, &s.v_full[vs], (j / kVStages) & 1, P))) break;
        const uint32_t* sfw = reinterpret_cast<const uint32_t*>(&s.v[vs][0] + VS::kSf);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int ch = lane + 32 * c - (t ? 16 : 0);
          sfr[c] = (c < 5 && ch >= 0 && ch < 128) ? sfw[ch] : kSfOne4;
        }
      }
      // PV(j-1) has read P_t and added block j-1 to O_t: then the row-sum column
      // is read, O_t may be rescaled and P_t(j) written
      uint32_t lraw = 0u;
      if (j > 0) {
        if (!(ok = wait_warp(s, &s.pv_done[t], (j - 1) & 1, P))) break;
        tc_fence_after();
        lraw = tmem_ld1(l_addr);
        tmem_ld_wait();
      }
      tmem_st32(p_addr, w);
      if (kMx) tmem_st8(sfb_addr, sfr);
      const float Lc = __uint_as_float(lraw);
      if (__any_sync(0xffffffffu, resc)) {
        // the frame moved: O_t (complete up to block j-1) and its row-sum column
        // are rescaled by the exact 2^(F_old - F_new); so are the row sums of the
        // current batch not yet handed to a mean MMA
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t r[32];
          tmem_ld32(o_addr + 32 * cc, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(o_addr + 32 * cc, r);
          tmem_st_wait();  // the store reads r asynchronously: done before r is reused
        }
        tmem_st1(l_addr, __float_as_uint(Lc * alpha));
      }
      // R operand (no MMA of this tile is in flight between s_full and p_full):
      // the row sum of block j-1 is the column's growth since the last block,
      // carried into the new frame
      if (j > 0) {
        const int jp = j - 1, g = jp % kMeanBlocks;
        const float rj = __fsub_rn(Lc, Lp) * alpha;
#pragma unroll
        for (int i = 0; i < kMeanBlocks; ++i) rb[i] = i == g ? rj : rb[i] * alpha;  // exact: alpha = 2^-n
        // a batch is complete once the row sum of its last block is in: the mean
        // MMA that reads it is issued right after this block's p_full
        if (g == kMeanBlocks - 1) {
          put_r_batch(ro, row, (jp / kMeanBlocks) % kMeanChunks, rb, kMeanBlocks);
          fence_proxy_async_smem();
        }
      }
      Lp = Lc * alpha;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&s.p_full[t]);
      F = Fn;
    }
    if (!range_ok) report_status(P.status, VC_ERR_UNSUPPORTED);
    float l = 0.0f;
    // after the last PV: the total row sum, and the last block's share of it
    if (ok) ok = wait_warp(s, &s.pv_done[t], (nkv - 1) & 1, P);
    if (ok) {
      tc_fence_after();
      l = __uint_as_float(tmem_ld1(l_addr));
      tmem_ld_wait();
      const int jp = nkv - 1, g = jp % kMeanBlocks, ch = (jp / kMeanBlocks) % kMeanChunks;
      const float rl = __fsub_rn(l, Lp);
#pragma unroll
      for (int i = 0; i < kMeanBlocks; ++i)
        if (i == g) rb[i] = rl;
      put_r_batch(ro, row, ch, rb, g + 1);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&s.fin_ready[t]);
      ok = wait_warp(s, &s.o_final[t], 0, P);
    }
    if (ok) {
      // epilogue: O = s_V O_t / l, BF16, original query order and layout
      tc_fence_after();
      const int q = qt * 128 + row;
      const float scale = __fdiv_rn(sV, l);
      const int b = bh / P.H, h = bh % P.H;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(P.o) + (((size_t)b * P.S + q) * P.H + h) * 128;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        tmem_ld32(o_addr + 32 * cc, r);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float s0 = scale, s1 = scale;
          if (kVKind == kVChannel) {  // s_V of the two channels over l
            const float* sv = P.s_v + (size_t)bh * 128 + cc * 32 + 2 * i;
            s0 = __fdiv_rn(sv[0], l);
            s1 = __fdiv_rn(sv[1], l);
          }
          __nv_bfloat162 b2 =
              __floats2bfloat162_rn(__uint_as_float(r[2 * i]) * s0, __uint_as_float(r[2 * i + 1]) * s1);
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
  e = cudaFuncSetAttribute(vc_attn_fwd_kernel<1, false, kVChannel>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)(sizeof(SmemAttn<1>) + 1024));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(vc_attn_fwd_kernel<1, false, kVMx>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)(sizeof(SmemAttn<1, true>) + 1024));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(vc_attn_fwd_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)(sizeof(SmemAttn<1>) + 1024));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(vc_attn_fwd_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)(sizeof(SmemAttn<2>) + 1024));
}

cudaError_t launch_attn_e4m3(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const AttnParams& p, cudaStream_t st, bool exp2) {
  const dim3 grid((p.nb + 1) / 2, p.B * p.H);
  if (exp2)
    vc_attn_fwd_kernel<1, true><<<grid, kThreads, sizeof(SmemAttn<1>) + 1024, st>>>(tq, tk, tv, p);
  else
    vc_attn_fwd_kernel<1><<<grid, kThreads, sizeof(SmemAttn<1>) + 1024, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_channel(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const AttnParams& p, cudaStream_t st) {
  const dim3 grid((p.nb + 1) / 2, p.B * p.H);
  vc_attn_fwd_kernel<1, false, kVChannel><<<grid, kThreads, sizeof(SmemAttn<1>) + 1024, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_mx(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv_e2m1,
                           const AttnParams& p, cudaStream_t st) {
  const dim3 grid((p.nb + 1) / 2, p.B * p.H);
  vc_attn_fwd_kernel<1, false, kVMx><<<grid, kThreads, sizeof(SmemAttn<1, true>) + 1024, st>>>(tq, tk, tv_e2m1, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_planes(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tplanes,
                               const AttnParams& p, cudaStream_t st) {
  const dim3 grid((p.nb + 1) / 2, p.B * p.H);
  vc_attn_fwd_kernel<2><<<grid, kThreads, sizeof(SmemAttn<2>) + 1024, st>>>(tq, tk, tplanes, p);
  return cudaGetLastError();
}

}  // namespace vc
