// vc_prep.cu -- V-Smooth prep and Q/K FP8 quantisation kernels (sm_100a).
//
// V-Smooth ("VC-Attention: Value Smoothing and Softmax Casting for Low-bit
// Attention", Abstract; "Nunchux AI lanza VC-Attention kernel ...", second
// paragraph): per (batch, head), k-means over the value tokens, a stable sort of
// the tokens by cluster, the mean of every 128-token block of the sorted order,
// and E4M3 / NVFP4 codes of the residual. Q/K: one E4M3 scale per 128-row block
// ("Open VC Attention", "Описание": Q/K scales per block).
//
// Readings where the pages are silent: k-means init indices come from
// splitmix64 seeded by seed ^ (0x9E3779B97F4A7C15 * (b*H + h + 1)), redrawn
// while they repeat; assignment ties go to the lowest cluster index; centroid and
// block-mean sums are int64 sums of llrint(x * 2^24) (exact and order-free), then
// one double division, rounded to fp32; an empty cluster keeps its centroid; the
// last pass's assignment is final; the residual scale is one per (b, h); a block
// whose amax is below 2^-100 is all zero.
//
// Every kernel reads Q, K, V in the caller's [B, S, H, 128] layout (a token is a
// contiguous 256-byte row for one head; rows of one head are H*256 bytes apart).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

#include "vc_common.cuh"
#include "vc_kernels.h"
#include "vc_sm100.cuh"

namespace vc {

// --------------------------------------------------------------- k-means init
__device__ __forceinline__ uint64_t splitmix64_next(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ull;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

template <typename T>
__global__ void __launch_bounds__(128) kmeans_init_kernel(const T* __restrict__ v, int S, int H, int k,
                                                          uint64_t seed, int seed_H, int seed_b0, int seed_h0,
                                                          float* __restrict__ cent) {
  __shared__ int idx[kMaxClusters];
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  if (threadIdx.x == 0) {
    // the seed of slice (b, h) of this call is that of slice (seed_b0 + b, seed_h0 + h)
    // of the whole problem, which has seed_H heads
    const uint64_t g = (uint64_t)(seed_b0 + b) * (uint64_t)seed_H + (uint64_t)(seed_h0 + h);
    uint64_t st = seed ^ (0x9E3779B97F4A7C15ull * (g + 1));
    for (int i = 0; i < k; ++i) {
      int u;
      while (true) {
        u = (int)(splitmix64_next(st) % (uint64_t)S);
        bool dup = false;
        for (int j = 0; j < i; ++j) dup |= (idx[j] == u);
        if (!dup || i >= S) break;
      }
      idx[i] = u;
    }
  }
  __syncthreads();
  const int d = threadIdx.x;
  for (int i = 0; i < k; ++i) {
    const size_t off = (((size_t)b * S + idx[i]) * H + h) * kD + d;
    cent[((size_t)bh * k + i) * kD + d] = to_f32<T>(v[off]);
  }
}

// --------------------------------------------------------------- k-means assign
// One CTA (4 warps) = one chunk of kChunk tokens of one (b, h), in tiles of
// kTile tokens staged in shared memory with coalesced 16-byte loads.
//  - Assignment. Distances are translation-invariant, so with r the
//    coordinate-wise median of the centroids, x' = x - r and c' = c - r,
//    |x - c|^2 = |x'|^2 + g_c where g_c = |c'|^2 - 2 x'.c'. Thread (t, half)
//    takes tokens t and t + 64 of the tile and the centroids of its parity
//    (c = 2i + half): one packed f32x2 FMA per two dimensions, token and
//    centroid, against the direct form's subtract and FMA, with every centroid
//    value read from shared memory (all lanes of a warp read the same address)
//    feeding both tokens. Each half posts its nearest centroid per token; after
//    a barrier each half marks its centroids that the bound below cannot rule
//    out against the merged nearest, and the token's thread combines the two
//    (the proxies stay in registers, so 5 CTAs fit on an SM).
//    The proxies' rounding is bounded: g_c is within 199 u |c'|^2 + 68 u |x'|^2
//    of its exact value (u = 2^-24: 128-term FMA chains, the two translations,
//    one final FMA), and the direct fp32 form sum_d (x_d - c_d)^2 within
//    134 u (|x'|^2 + |c'|^2). A centroid c whose
//    g_c - 2^-15 |c'|^2 exceeds g_b + 2^-15 (|c'_b|^2 + |x'|^2) for the nearest
//    b is farther than b exactly and also by the direct form, so it cannot be
//    the answer. The rest (a near tie) are compared by the direct form, lowest
//    index on ties, which is the answer the direct form over all centroids
//    gives.
//  - The labels go to global memory (per pass, for the sums kernel below and
//    the final sort), and in the last pass a per-chunk cluster histogram.
constexpr int kTile = 128;

// Staged tile rows: 256 bytes, the 16-byte piece index XORed with the row's low
// three bits, so that eight lanes reading the same piece of eight consecutive
// rows hit distinct banks.
__device__ __forceinline__ int tile_off(int r, int piece) { return r * 256 + ((piece ^ (r & 7)) << 4); }
constexpr int kTileBytes = kTile * 256;

// 16 dimensions (16 ch .. 16 ch + 15) of staged row r, translated: x - r.
template <typename T>
__device__ __forceinline__ void load_translated(const uint8_t* tile, int r, int ch, const float* rneg,
                                                float2* x) {
  float f[16];
  unpack8<T>(*reinterpret_cast<const uint4*>(tile + tile_off(r, 2 * ch)), f);
  unpack8<T>(*reinterpret_cast<const uint4*>(tile + tile_off(r, 2 * ch + 1)), f + 8);
  const float4* rv = reinterpret_cast<const float4*>(rneg + ch * 16);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float4 q = rv[i];
    x[2 * i] = __fadd2_rn(make_float2(f[4 * i], f[4 * i + 1]), make_float2(q.x, q.y));
    x[2 * i + 1] = __fadd2_rn(make_float2(f[4 * i + 2], f[4 * i + 3]), make_float2(q.z, q.w));
  }
}

// Nearest centroid of staged row r among the centroids in the bit mask cand, by
// the direct form: squared fp32 distances sum_d (x_d - c_d)^2, even and odd
// dimensions in the two halves of a packed f32x2 accumulator, 16 dimensions at
// a time, the halves added last; the lowest index wins ties. cg: the centroids
// of this (b, h), fp32 [k][128].
template <typename T>
__device__ __noinline__ int nearest_direct(const uint8_t* tile, int r, const float* __restrict__ cg, uint32_t cand) {
  int best = -1;
  float best_d = 0.0f;
#pragma unroll 1
  for (; cand != 0u; cand &= cand - 1u) {
    const int c = __ffs(cand) - 1;
    float2 dist = make_float2(0.f, 0.f);
#pragma unroll 1
    for (int ch = 0; ch < 8; ++ch) {
      float f[16];
      unpack8<T>(*reinterpret_cast<const uint4*>(tile + tile_off(r, 2 * ch)), f);
      unpack8<T>(*reinterpret_cast<const uint4*>(tile + tile_off(r, 2 * ch + 1)), f + 8);
      const float4* cc = reinterpret_cast<const float4*>(cg + c * kD + ch * 16);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 p = __ldg(cc + i);
        const float2 d0 = __fadd2_rn(make_float2(f[4 * i], f[4 * i + 1]), make_float2(-p.x, -p.y));
        const float2 d1 = __fadd2_rn(make_float2(f[4 * i + 2], f[4 * i + 3]), make_float2(-p.z, -p.w));
        dist = __ffma2_rn(d0, d0, dist);
        dist = __ffma2_rn(d1, d1, dist);
      }
    }
    const float dd = dist.x + dist.y;
    if (best < 0 || dd < best_d) {
      best_d = dd;
      best = c;
    }
  }
  return best;
}

template <typename T, int KC>
__global__ void __launch_bounds__(kTile, 5) kmeans_assign_kernel(const T* __restrict__ v, int S, int H, int k,
                                                              const float* __restrict__ cent,
                                                              uint8_t* __restrict__ assign, int* __restrict__ hist,
                                                              uint8_t* __restrict__ history) {
  constexpr int kHalfC = KC / 2;
  static_assert(KC % 2 == 0, "cluster capacity must keep the staged tile 16-byte aligned");
  extern __shared__ __align__(16) uint8_t smem[];
  float* cpr = reinterpret_cast<float*>(smem);                                         // [KC][128]: c - r
  float* rneg = cpr + (size_t)KC * kD;                                                 // [128]: -r
  float* ncs = rneg + kD;                                                              // [KC]: |c - r|^2
  float* kns = ncs + KC;                                                               // [KC]: 2^-15 |c - r|^2
  float* pg = kns + KC;                                                                // [2][kTile]: each half's nearest g
  float* xs = pg + 2 * kTile;                                                          // [kTile]: |x'|^2
  uint32_t* pn = reinterpret_cast<uint32_t*>(xs + kTile);                              // [2][kTile]: near-tie bits
  int8_t* pi = reinterpret_cast<int8_t*>(pn + 2 * kTile);                              // [2][kTile]: nearest c
  uint8_t* tile = reinterpret_cast<uint8_t*>(pi + 2 * kTile);                          // staged rows
  int* scount = reinterpret_cast<int*>(tile + kTileBytes);                     // [KC]

  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int chunk = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t row_stride = (size_t)H * kD;  // elements between consecutive tokens of one head
  const T* vbase = v + ((size_t)b * S * H + h) * kD;
  const float* cg = cent + (size_t)bh * k * kD;

  {  // translation r = coordinate-wise lower median of the centroids; c' = c - r
    const int d = tid;
    float cv[KC];
#pragma unroll
    for (int c = 0; c < KC; ++c) cv[c] = c < k ? cg[c * kD + d] : 0.0f;
    const int m = (k - 1) / 2;
    float r = cv[0];
#pragma unroll
    for (int i = 0; i < KC; ++i) {
      int lt = 0, le = 0;
#pragma unroll
      for (int j = 0; j < KC; ++j) {
        lt += (j < k && cv[j] < cv[i]);
        le += (j < k && cv[j] <= cv[i]);
      }
      if (i < k && lt <= m && m < le) r = cv[i];
    }
    rneg[d] = -r;
#pragma unroll
    for (int c = 0; c < KC; ++c)
      if (c < k) cpr[c * kD + d] = __fsub_rn(cv[c], r);
  }
  if (tid < KC) scount[tid] = 0;
  __syncthreads();
  for (int c = warp; c < k; c += 4) {  // |c'|^2
    float q = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float x = cpr[c * kD + lane + 32 * j];
      q = fmaf(x, x, q);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    if (lane == 0) {
      ncs[c] = q;
      kns[c] = q * 0x1p-15f;
    }
  }
  __syncthreads();

  const int t = tid & 63, half = tid >> 6;
  const int s_chunk0 = chunk * kChunk;
  const int s_chunk1 = min(S, s_chunk0 + kChunk);
  for (int s0 = s_chunk0; s0 < s_chunk1; s0 += kTile) {
    const int ntok = min(kTile, s_chunk1 - s0);
    __syncthreads();
    // stage the tile: 16 x 16-byte pieces per token, a warp covers two tokens
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
      const int idx = i * kTile + tid, r = idx >> 4, c = idx & 15;
      if (r < ntok) {
        const uint4 val = *reinterpret_cast<const uint4*>(vbase + (size_t)(s0 + r) * row_stride + c * 8);
        *reinterpret_cast<uint4*>(tile + tile_off(r, c)) = val;
      }
    }
    __syncthreads();
    // proxies g_c of tokens t and t + 64 (rows past ntok hold stale data; unused)
    float2 ga[kHalfC], gb[kHalfC];
#pragma unroll
    for (int i = 0; i < kHalfC; ++i) ga[i] = gb[i] = make_float2(0.f, 0.f);
    float2 xx = make_float2(0.f, 0.f);  // |x'|^2 of token tid = t + 64 half
#pragma unroll 1
    for (int ch = 0; ch < 8; ++ch) {
      float2 xa[8], xb[8];
      load_translated<T>(tile, t, ch, rneg, xa);
      load_translated<T>(tile, t + 64, ch, rneg, xb);
      if (half == 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) xx = __ffma2_rn(xa[i], xa[i], xx);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) xx = __ffma2_rn(xb[i], xb[i], xx);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int i = 0; i < kHalfC; ++i) {
          const int c = 2 * i + half;
          if (c < k) {
            const float4 p = *reinterpret_cast<const float4*>(cpr + c * kD + ch * 16 + 4 * q);
            const float2 p01 = make_float2(p.x, p.y), p23 = make_float2(p.z, p.w);
            ga[i] = __ffma2_rn(xa[2 * q], p01, ga[i]);
            gb[i] = __ffma2_rn(xb[2 * q], p01, gb[i]);
            ga[i] = __ffma2_rn(xa[2 * q + 1], p23, ga[i]);
            gb[i] = __ffma2_rn(xb[2 * q + 1], p23, gb[i]);
          }
        }
      }
    }
    // this half's proxies of both tokens, and its nearest centroid of each
    float g[2][kHalfC];
#pragma unroll
    for (int tok = 0; tok < 2; ++tok) {
      int ib = -1;  // the lowest index wins ties within the half
      float gmin = __int_as_float(0x7f800000);
#pragma unroll
      for (int i = 0; i < kHalfC; ++i) {
        const int c = 2 * i + half;
        const float2 dot = tok ? gb[i] : ga[i];
        g[tok][i] = c < k ? fmaf(-2.0f, dot.x + dot.y, ncs[c]) : __int_as_float(0x7f800000);
        if (c < k && (ib < 0 || g[tok][i] < gmin)) {
          gmin = g[tok][i];
          ib = c;
        }
      }
      pg[half * kTile + t + 64 * tok] = gmin;
      pi[half * kTile + t + 64 * tok] = (int8_t)ib;
    }
    xs[tid] = xx.x + xx.y;  // token tid = t + 64 half is this thread's own
    __syncthreads();
    // nearest of the two halves (lowest index on equal g), then this half's
    // centroids that the rounding bound cannot rule out (a near tie)
    auto merged = [&](int tk, float& g_best) -> int {
      const float a1 = pg[tk], c1 = pg[kTile + tk];
      const int ai = pi[tk], ci = pi[kTile + tk];
      const bool first = ci < 0 || a1 < c1 || (a1 == c1 && ai < ci) || !(c1 == c1);
      g_best = first ? a1 : c1;
      return first ? ai : ci;
    };
#pragma unroll
    for (int tok = 0; tok < 2; ++tok) {
      const int tk = t + 64 * tok;
      float g_best;
      const int bc = merged(tk, g_best);
      const float lim = g_best + (kns[bc] + xs[tk] * 0x1p-15f);
      uint32_t near = 0;
#pragma unroll
      for (int i = 0; i < kHalfC; ++i) {
        const int c = 2 * i + half;
        if (c < k && c != bc && !(g[tok][i] - kns[c] > lim)) near |= 1u << c;
      }
      pn[half * kTile + tk] = near;
    }
    __syncthreads();
    const bool valid = tid < ntok;
    int best = 0;
    if (valid) {
      float g_best;
      best = merged(tid, g_best);
      const uint32_t near = pn[tid] | pn[kTile + tid];
      if (near != 0u) best = nearest_direct<T>(tile, tid, cg, near | (1u << best));
      assign[(size_t)bh * S + s0 + tid] = (uint8_t)best;
      if (history) history[(size_t)bh * S + s0 + tid] = (uint8_t)best;
      if (hist != nullptr) atomicAdd(&scount[best], 1);
    }
  }
  __syncthreads();
  if (hist != nullptr && tid < k) hist[((size_t)bh * gridDim.x + chunk) * k + tid] = scount[tid];
}

template <int KC>
constexpr size_t assign_smem() {
  return (size_t)KC * kD * 4 + kD * 4 + 2 * KC * 4 + kTile * (2 * 4 + 4 + 2 * 4 + 2) + kTileBytes + KC * 4;
}

// --------------------------------------------------------------- k-means assign on the tensor cores
// The assignment for BF16 V, in two kernels.
// (1) kmeans_cops_kernel, before each pass: per (b, h) the centroid operand block
//     of the pass: the hi and mid bf16 parts of every centroid as the MMA's B
//     operand (two halves of 64 dimensions, rows 0..KC-1 hi, KC..2KC-1 mid, in
//     the 128-byte-swizzled layout a 1024-byte-aligned copy reproduces), then
//     |c|^2 (fp64 sum rounded once) and |c| for the KC centroids.
// (2) kmeans_assign_tc_kernel: one persistent CTA (10 warps) per SM takes work
//     items (b, h, chunk of kChunk tokens) from a global counter, so that CTAs
//     whose tokens need the fallback below more often do not hold back the rest,
//     and streams their 128-token tiles through a ring of stages:
//  - warp 8 takes the items, writes each tile's descriptor next to its stage
//    and loads the tile with TMA (two 128-byte-swizzled boxes of 64 dimensions)
//    with the slice's centroid operand block (one bulk copy);
//  - warp 9 issues the tile's dot products on the tensor cores into one of four
//    tensor-memory stages of 2 KC fp32 columns;
//  - warps 0-3 (even tiles) and 4-7 (odd tiles) take one token per thread:
//    proxies, argmin, fallback, label, and in the last pass the cluster
//    histogram of each chunk (zeroed by the launcher; one global atomic per
//    cluster present in a warp's 32 tokens).
// Dots. A centroid c (fp32) is hi + mid + r with hi = bf16(c), mid = bf16(c - hi)
// and |r_d| <= 2^-18 |c_d|, so x . c = x . hi + x . mid within 2^-18 |x| |c| (x
// bf16; sum_d |x_d c_d| <= |x| |c|). One kind::f16 MMA chain (M = 128 tokens,
// N = 2 KC, K = 128 dimensions: eight instructions a tile) gives both dots of
// every centroid in fp32; their sum is the dot.
// Decision. g_c = |c|^2 - 2 x . c ranks the centroids as |x - c|^2 = |x|^2 + g_c
// does. The tensor core's accumulation order and rounding are not specified;
// measured on a B200 over mixture, outlier and wide-exponent inputs, the error
// of its fp32 dot products stayed below 2^-20 of sum_d |x_d hi_d|. Each dot is
// allowed 2^-15 |x| |c| (the dropped part 2^-18, the accumulation 2^-17: eight
// times the largest error measured, the final add far less) and |c|^2 with the
// final fma 2^-19 |c|^2: with e_c = 2^-19 |c|^2 + 2^-14 |x| |c|, a centroid whose
// g_c - e_c exceeds g_b + e_b, b the smallest proxy, is farther than b. Any other
// centroid is a candidate. b and its candidates are then compared by the squared
// distance sum_d (x_d - c_d)^2 in fp32 (all terms positive: the rounding of the
// differences, squares and 128-term sum, in any order, stays within 2^-16 of the
// distance itself; the whole warp makes one such token's distances, four
// dimensions a lane), and those still within that bound of the nearest once more
// in fp64 by the token's own thread (differences exact, squares rounded at
// 2^-53), the lowest index winning ties: the exact argmin but for ties below fp64
// rounding.
constexpr int kTcWarps = 10, kTcThreads = kTcWarps * 32;
constexpr int kTcTmaWarp = 8, kTcMmaWarp = 9;
constexpr int kTcDStages = 4;                  // tensor-memory dot stages (two per token-warp group)
constexpr uint32_t kTcStageCols = 64;          // tensor-memory columns per dot stage (N = 2 KC <= 64)
constexpr uint32_t kTcTileBytes = kTile * 256; // 128 tokens x 128 bf16 (two 16 KB boxes)

// Bytes of one slice's centroid operand block: [2 halves][2 KC rows][128 B], then
// |c|^2 [KC] and |c| [KC] (fp32).
template <int KC> __host__ __device__ constexpr uint32_t cops_bytes() { return 2 * 2 * KC * 128 + 2 * KC * 4; }
template <int KC> __host__ __device__ constexpr int tc_stages() { return KC == 32 ? 4 : 5; }   // tile ring depth (shared memory)

// Byte offset of dimension-half piece j (16 bytes, 8 dims) of row r in a
// 128-byte-swizzled block of rows: rows of 128 B, the piece index XORed with r mod 8.
__device__ __forceinline__ uint32_t sw128_off(int r, int j) { return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4)); }

template <int KC>
__global__ void __launch_bounds__(128) kmeans_cops_kernel(int k, const float* __restrict__ cent,
                                                          uint8_t* __restrict__ cops) {
  __shared__ double wq[4][KC];
  const int bh = blockIdx.x, d = threadIdx.x, lane = d & 31, warp = d >> 5;
  uint8_t* blk = cops + (size_t)bh * cops_bytes<KC>();
  const float* cg = cent + (size_t)bh * k * kD;
#pragma unroll 4
  for (int c = 0; c < KC; ++c) {
    const float x = c < k ? cg[c * kD + d] : 0.0f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    const __nv_bfloat16 mid = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(hi)));
    uint8_t* half = blk + (d >> 6) * (2 * KC * 128);
    *reinterpret_cast<__nv_bfloat16*>(half + sw128_off(c, (d & 63) >> 3) + (d & 7) * 2) = hi;
    *reinterpret_cast<__nv_bfloat16*>(half + sw128_off(KC + c, (d & 63) >> 3) + (d & 7) * 2) = mid;
    double q = (double)x * (double)x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    if (lane == 0) wq[warp][c] = q;
  }
  __syncthreads();
  if (d < KC) {
    const double q = (wq[0][d] + wq[1][d]) + (wq[2][d] + wq[3][d]);
    float* nrm = reinterpret_cast<float*>(blk + 2 * 2 * KC * 128);
    nrm[d] = __double2float_rn(q);
    nrm[KC + d] = __double2float_rn(sqrt(q));
  }
}

struct TcTile {
  int bh, chunk, t, end;   // slice, chunk, tile of the chunk; end = 1 marks the end of the stream
};

template <int KC>
struct __align__(1024) SmemAssignTc {
  static constexpr int kStages = tc_stages<KC>();
  uint8_t a[kStages][2][kTile * 128];      // [stage][64-dimension half] 128-B-swizzled rows of 64 bf16
  uint8_t cop[kStages][cops_bytes<KC>() + 1024 - cops_bytes<KC>() % 1024];  // the tile's centroid operand block
  TcTile desc[kStages];
  uint64_t a_full[kStages], a_empty[kStages], d_full[kTcDStages], d_empty[kTcDStages], drain;
  uint32_t tmem_base;
  int32_t abort_flag;                      // a wait ran out: every role skips the remaining tiles
};

// Bounded wait on an mbarrier phase (1 s), for a whole warp; false (and the CTA's
// abort flag set) when the time ran out or another role already gave up. The
// waiting thread is suspended in the barrier unit (up to 20 us at a time), so
// idle warps leave the issue slots to the working ones.
template <class Smem>
__device__ __forceinline__ bool tc_wait(Smem& s, uint64_t* bar, uint32_t parity) {
  bool ok = mbar_try_wait(bar, parity);
  if (!ok) {
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      if (mbar_try_wait_sleep(bar, parity, 20000u)) {
        ok = true;
        break;
      }
      if (globaltimer_ns() - t0 > 1000000000ull || *reinterpret_cast<volatile int32_t*>(&s.abort_flag) != 0) break;
    }
    if (!ok) s.abort_flag = 1;
  }
  return __all_sync(0xffffffffu, ok);
}

template <int KC>
__global__ void __launch_bounds__(kTcThreads, 1) kmeans_assign_tc_kernel(const __grid_constant__ CUtensorMap tmV,
                                                                       int S, int H, int k, int nchunks, int BH,
                                                                       const float* __restrict__ cent,
                                                                       const uint8_t* __restrict__ cops,
                                                                       int* __restrict__ work,
                                                                       uint8_t* __restrict__ assign,
                                                                       int* __restrict__ hist,
                                                                       uint8_t* __restrict__ history) {
  static_assert(KC == 16 || KC == 32, "N of the dot MMA");
  using Smem = SmemAssignTc<KC>;
  constexpr int NS = Smem::kStages;
  constexpr uint32_t kCopBytes = cops_bytes<KC>();
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total = BH * nchunks;
  constexpr uint32_t idesc = idesc_f32acc(kFmtBF16, kFmtBF16, 128, 2 * KC);

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&s.a_full[i], 1);
      mbar_init(&s.a_empty[i], 1 + 4);   // the MMA's commit and the four warps of the tile's group
    }
    for (int i = 0; i < kTcDStages; ++i) {
      mbar_init(&s.d_full[i], 1);
      mbar_init(&s.d_empty[i], 4);
    }
    mbar_init(&s.drain, 1);
    s.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, kTcDStages * kTcStageCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const bool leader = elect_one();   // the issuing lane of the TMA and MMA warps
  int ntiles = 0;                    // tiles this CTA streamed (the TMA warp's count)

  if (warp == kTcTmaWarp) {
    // ------------------------------------------------ work items, TMA producer
    // tile g goes to stage g % NS; after the last item, two end tiles (one for
    // each token-warp group) close the stream
    int g = 0, ends = 0;
    int item = 0, ntile_item = 0, ti = 0;
    bool have = false;
    while (ends < 2) {
      if (*reinterpret_cast<volatile int32_t*>(&s.abort_flag)) break;
      if (ends == 0 && (!have || ti == ntile_item)) {
        int it = 0;
        if (leader) it = atomicAdd(work, 1);
        item = __shfl_sync(0xffffffffu, it, __ffs(__ballot_sync(0xffffffffu, leader)) - 1);
        have = item < total;
        if (have) {
          const int chunk = item % nchunks;
          ntile_item = (min(kChunk, S - chunk * kChunk) + kTile - 1) / kTile;
          ti = 0;
        }
      }
      const int st = g % NS;
      if (g >= NS && !tc_wait(s, &s.a_empty[st], ((g / NS) & 1) ^ 1)) break;
      if (leader) {
        TcTile d;
        if (have) {
          d.bh = item / nchunks;
          d.chunk = item % nchunks;
          d.t = ti;
          d.end = 0;
          s.desc[st] = d;
          if (g == 0) prefetch_tmap(&tmV);
          const int b = d.bh / H, h = d.bh % H;
          const int z = b * S + d.chunk * kChunk + ti * kTile;   // rows past the tensor read as zeros
          mbar_arrive_expect_tx(&s.a_full[st], kTcTileBytes + kCopBytes);
          tma_load_3d(s.a[st][0], &tmV, &s.a_full[st], 0, h, z);
          tma_load_3d(s.a[st][1], &tmV, &s.a_full[st], 64, h, z);
          bulk_load(s.cop[st], cops + (size_t)d.bh * kCopBytes, kCopBytes, &s.a_full[st]);
        } else {
          d.bh = d.chunk = d.t = 0;
          d.end = 1;
          s.desc[st] = d;
          mbar_arrive(&s.a_full[st]);
        }
      }
      __syncwarp();
      if (have) {
        ++ti;
        ++ntiles;
      } else {
        ++ends;
      }
      ++g;
    }
    // copies still in flight land before the CTA exits
    for (int i = max(0, g - NS); i < g; ++i) mbar_wait(&s.a_full[i % NS], (i / NS) & 1, 100000000ull, nullptr);
  } else if (warp == kTcMmaWarp) {
    // ------------------------------------------------ dot products
    for (int g = 0;; ++g) {
      const int st = g % NS, ds = g % kTcDStages;
      if (!tc_wait(s, &s.a_full[st], (g / NS) & 1)) break;
      if (s.desc[st].end) break;
      if (g >= kTcDStages && !tc_wait(s, &s.d_empty[ds], ((g / kTcDStages) & 1) ^ 1)) break;
      tc_fence_after();
      if (leader) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint64_t da = sdesc_k_sw128(smem_u32(s.a[st][half]));
          const uint64_t db = sdesc_k_sw128(smem_u32(s.cop[st] + half * (2 * KC * 128)));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16_ss(tmem + ds * kTcStageCols, da + 2 * kk, db + 2 * kk, idesc, (half | kk) != 0);
        }
        umma_commit(&s.d_full[ds]);
        umma_commit(&s.a_empty[st]);
      }
      __syncwarp();
    }
    if (leader) umma_commit(&s.drain);
    __syncwarp();
    mbar_wait(&s.drain, 0, 100000000ull, nullptr);
  } else {
    // ------------------------------------------------ one token per thread
    // group grp = warp / 4 takes the tiles g with g % 2 == grp
    const int grp = warp >> 2;
    const int r = tid & 127;                             // row of the tile, tensor-memory lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
#pragma unroll 1
    for (int g = grp;; g += 2) {
      const int st = g % NS, ds = g % kTcDStages;
      if (!tc_wait(s, &s.a_full[st], (g / NS) & 1)) break;
      const TcTile d = s.desc[st];
      if (d.end) break;
      if (!tc_wait(s, &s.d_full[ds], (g / kTcDStages) & 1)) break;
      tc_fence_after();
      uint32_t dr[32], dm[32];   // x . hi and x . mid of each centroid
      tmem_ld32(tmem + lane_base + ds * kTcStageCols, dr);
      tmem_ld32(tmem + lane_base + ds * kTcStageCols + KC, dm);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.d_empty[ds]);
      const int bh = d.bh, chunk = d.chunk;
      const int p = d.t * kTile + r;                       // token of the chunk
      const int ntok = min(kChunk, S - chunk * kChunk);
      const float* const nrm = reinterpret_cast<const float*>(s.cop[st] + 2 * 2 * KC * 128);  // |c|^2, |c|
      const float* const cg = cent + (size_t)bh * k * kD;
      const uint8_t* const arow0 = s.a[st][0];
      const uint8_t* const arow1 = s.a[st][1];
      auto piece = [&](int j, float* f) {                // dims 8j .. 8j+7 of row r
        const uint8_t* base = j < 8 ? arow0 : arow1;
        unpack8<__nv_bfloat16>(*reinterpret_cast<const uint4*>(base + sw128_off(r, j & 7)), f);
      };
      float2 xx2 = make_float2(0.f, 0.f);
#pragma unroll 4
      for (int j = 0; j < 16; ++j) {
        float f[8];
        piece(j, f);
#pragma unroll
        for (int e = 0; e < 8; e += 2) xx2 = __ffma2_rn(make_float2(f[e], f[e + 1]), make_float2(f[e], f[e + 1]), xx2);
      }
      const float xabs = sqrtf(xx2.x + xx2.y);
      int best = 0;
      float gb = 0.0f;
      float gv[KC];
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        gv[c] = fmaf(-2.0f, __uint_as_float(dr[c]) + __uint_as_float(dm[c]), nrm[c]);
        if (c < k && (c == 0 || gv[c] < gb)) {
          gb = gv[c];
          best = c;
        }
      }
      const float xs = 0x1p-14f * xabs;
      const float lim = gb + fmaf(0x1p-19f, nrm[best], xs * nrm[KC + best]);
      uint32_t cand = 0u;
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        const float e = fmaf(0x1p-19f, nrm[c], xs * nrm[KC + c]);
        if (c < k && c != best && !(gv[c] - e > lim)) cand |= 1u << c;
      }
      // Near ties: the best proxy and its candidates by their direct squared
      // distances. The fp32 distances of a token are made by the whole warp (four
      // dimensions a lane, the partial sums added by shuffles), one such token
      // after another, so that a lane's near tie does not hold the other 31 lanes
      // for its serial 128-term sums. The fp32 values only set aside the centroids
      // clearly farther than the nearest (any order of adding the positive terms
      // stays within 2^-16 of the distance); those still within that bound are
      // compared in fp64 by the token's own thread, dimension after dimension, the
      // lowest index winning ties.
      const uint32_t cm_own = cand != 0u ? (cand | (1u << best)) : 0u;
      uint32_t close_own = 0u;
      int bmin_own = best;
      {
        const int jx = lane >> 1;                          // piece of the lane's four dimensions
        const uint8_t* const xbase = (jx < 8 ? arow0 : arow1) + (lane & 1) * 8;
#pragma unroll 1
        for (uint32_t todo = __ballot_sync(0xffffffffu, cand != 0u); todo != 0u; todo &= todo - 1u) {
          const int src = __ffs(todo) - 1;
          const uint32_t cm = __shfl_sync(0xffffffffu, cm_own, src);
          float xf[4];
          unpack4<__nv_bfloat16>(*reinterpret_cast<const uint2*>(xbase + sw128_off((warp & 3) * 32 + src, jx & 7)), xf);
          float dd[KC];
          float dmin = __int_as_float(0x7f800000);
          int bmin = -1;
#pragma unroll 1
          for (uint32_t m = cm; m != 0u; m &= m - 1u) {
            const int c = __ffs(m) - 1;
            const float4 cc = __ldg(reinterpret_cast<const float4*>(cg + c * kD + 4 * lane));
            const float d0 = xf[0] - cc.x, d1 = xf[1] - cc.y, d2 = xf[2] - cc.z, d3 = xf[3] - cc.w;
            float part = (d0 * d0 + d1 * d1) + (d2 * d2 + d3 * d3);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
#pragma unroll
            for (int q = 0; q < KC; ++q)
              if (q == c) dd[q] = part;
            if (bmin < 0 || part < dmin) {
              dmin = part;
              bmin = c;
            }
          }
          uint32_t close = 0u;   // within the fp32 bound of the nearest
#pragma unroll
          for (int q = 0; q < KC; ++q)
            if (((cm >> q) & 1u) && q != bmin && !(dd[q] - 0x1p-16f * dd[q] > dmin + 0x1p-16f * dmin))
              close |= 1u << q;
          if (lane == src) {
            bmin_own = bmin;
            close_own = close;
          }
        }
      }
      if (cand != 0u) {
        best = bmin_own;
        if (close_own != 0u) {
          uint32_t close = close_own | (1u << bmin_own);
          double bd = 0.0;
          best = -1;
#pragma unroll 1
          for (; close != 0u; close &= close - 1u) {
            const int c = __ffs(close) - 1;
            double dist = 0.0;
#pragma unroll 1
            for (int j = 0; j < 16; ++j) {
              float f[8];
              piece(j, f);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const double df = (double)f[e] - (double)__ldg(cg + c * kD + 8 * j + e);
                dist = fma(df, df, dist);
              }
            }
            if (best < 0 || dist < bd) {
              bd = dist;
              best = c;
            }
          }
        }
      }
      const bool valid = p < ntok;
      if (valid) {
        const size_t o = (size_t)bh * S + (size_t)chunk * kChunk + p;
        assign[o] = (uint8_t)best;
        if (history) history[o] = (uint8_t)best;
      }
      if (hist != nullptr) {
        // the warp's tokens of each cluster, added once by the lowest such lane
        const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
        const uint32_t same = __match_any_sync(0xffffffffu, valid ? best : -1) & vmask;
        if (valid && (same & ((1u << lane) - 1u)) == 0u)
          atomicAdd(&hist[((size_t)bh * nchunks + chunk) * k + best], __popc(same));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.a_empty[st]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcDStages * kTcStageCols);
  }
  (void)ntiles;
}

template <int KC>
constexpr size_t assign_tc_smem() {
  return sizeof(SmemAssignTc<KC>) + 1024;
}

// --------------------------------------------------------------- k-means sums
// sums[c] and counts[c] are running totals over the whole (b, h): the int64 sum
// of llrint(x * 2^24) over the tokens of cluster c, and their number. One CTA
// (4 warps) = one chunk of kChunk tokens, in tiles of 128. The first pass adds
// every token to its cluster; a later ("delta") pass compares each token's
// cluster with the previous pass's and, for the tokens that moved, adds x to the
// new cluster and subtracts it from the old one (exact integer arithmetic, so the
// totals equal a fresh sum). The tile's entries go into cluster order, + before -
// within a cluster (a counting sort: match_any ranks within each warp, offsets
// across warps and the two signs), as words holding the token, the cluster and
// the sign. Each warp walks a contiguous quarter of the sorted entries, eight
// entries in flight, lane l owning dimensions 4l .. 4l+3 of each entry's row (one
// coalesced 256-byte read per warp load); it keeps int64 running sums and adds
// them to the CTA's accumulators (shared-memory atomics: a segment can span two
// warps) where a (cluster, sign) segment ends. A tile without entries reads
// nothing; no global atomics until the chunk's totals go to global memory.
template <typename T, int KC>
__global__ void __launch_bounds__(kTile) kmeans_sums_kernel(const T* __restrict__ v, int S, int H, int k, bool delta,
                                                            const uint8_t* __restrict__ lab_new,
                                                            const uint8_t* __restrict__ lab_old,
                                                            unsigned long long* __restrict__ sums,
                                                            int* __restrict__ counts) {
  __shared__ long long acc[KC * kD];
  __shared__ __align__(16) uint32_t sent[2 * kTile];
  __shared__ int scount[KC];
  __shared__ int woff[8 * KC + 1];  // [sign][warp][cluster], then the number of entries
  const int bh = blockIdx.y, b = bh / H, h = bh % H, chunk = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t row_stride = (size_t)H * kD;
  const T* vbase4 = v + ((size_t)b * S * H + h) * kD + 4 * lane;
  for (int i = tid; i < KC * kD; i += kTile) acc[i] = 0;
  if (tid < KC) scount[tid] = 0;
  const int s_chunk0 = chunk * kChunk, s_chunk1 = min(S, s_chunk0 + kChunk);
  for (int s0 = s_chunk0; s0 < s_chunk1; s0 += kTile) {
    const bool valid = tid < s_chunk1 - s0;
    const int cn = valid ? lab_new[(size_t)bh * S + s0 + tid] : 0;
    const int co = valid && delta ? lab_old[(size_t)bh * S + s0 + tid] : cn;
    const bool add = valid && (!delta || co != cn), sub = valid && delta && co != cn;
    __syncthreads();  // the previous tile's walk is done with sent and woff
    for (int i = tid; i < 8 * KC; i += kTile) woff[i] = 0;
    if (add) atomicAdd(&scount[cn], 1);
    if (sub) atomicAdd(&scount[co], -1);
    const unsigned pa = __match_any_sync(0xffffffffu, add ? cn : 0xFF);
    const unsigned ps = __match_any_sync(0xffffffffu, sub ? co : 0xFF);
    const int ra = __popc(pa & ((1u << lane) - 1u)), rs = __popc(ps & ((1u << lane) - 1u));
    __syncthreads();
    if (add && ra == 0) woff[(0 * 4 + warp) * KC + cn] = __popc(pa);
    if (sub && rs == 0) woff[(1 * 4 + warp) * KC + co] = __popc(ps);
    __syncthreads();
    if (tid < 32) {
      int w[8], tot = 0;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        w[g] = tid < KC ? woff[g * KC + tid] : 0;
        tot += w[g];
      }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t2 = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += t2;
      }
      if (tid < KC) {
        int base = incl - tot;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          woff[g * KC + tid] = base;
          base += w[g];
        }
      }
      if (tid == 31) woff[8 * KC] = incl;
    }
    __syncthreads();
    if (add) sent[woff[(0 * 4 + warp) * KC + cn] + ra] = (uint32_t)tid | ((uint32_t)cn << 16);
    if (sub) sent[woff[(1 * 4 + warp) * KC + co] + rs] = (uint32_t)tid | ((uint32_t)co << 16) | 0x80000000u;
    __syncthreads();
    const int nent = woff[8 * KC];
    if (nent == 0) continue;
    // warp w walks entries [w n / 4, (w + 1) n / 4); lane l owns dimensions
    // 4l .. 4l+3 of each entry's row (one coalesced 256-byte read per warp load)
    const int e_lo = (warp * nent) >> 2, e_hi = ((warp + 1) * nent) >> 2;
    if (e_lo == e_hi) continue;
    const T* trow = vbase4 + (size_t)s0 * row_stride;
    auto flush = [&](uint32_t key, const long long* run) {  // key = e >> 16: cluster, sign in bit 15
      unsigned long long* a = reinterpret_cast<unsigned long long*>(acc + (key & 0xFFu) * kD + 4 * lane);
#pragma unroll
      for (int q = 0; q < 4; ++q) atomicAdd(a + q, (unsigned long long)((key & 0x8000u) ? -run[q] : run[q]));
    };
    long long run[4] = {0, 0, 0, 0};
    uint32_t cur = sent[e_lo] >> 16;
    int pos = e_lo;
    for (; pos + 8 <= e_hi; pos += 8) {
      uint32_t e[8];
      uint2 x[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) e[j] = sent[pos + j];
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = *reinterpret_cast<const uint2*>(trow + (size_t)(e[j] & 0xFFu) * row_stride);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t key = e[j] >> 16;
        if (key != cur) {
          flush(cur, run);
          run[0] = run[1] = run[2] = run[3] = 0;
          cur = key;
        }
        float f[4];
        unpack4<T>(x[j], f);
#pragma unroll
        for (int q = 0; q < 4; ++q) run[q] += __float2ll_rn(f[q] * 16777216.0f);  // x * 2^24, exact
      }
    }
    for (; pos < e_hi; ++pos) {
      const uint32_t e = sent[pos], key = e >> 16;
      if (key != cur) {
        flush(cur, run);
        run[0] = run[1] = run[2] = run[3] = 0;
        cur = key;
      }
      float f[4];
      unpack4<T>(*reinterpret_cast<const uint2*>(trow + (size_t)(e & 0xFFu) * row_stride), f);
#pragma unroll
      for (int q = 0; q < 4; ++q) run[q] += __float2ll_rn(f[q] * 16777216.0f);
    }
    flush(cur, run);
  }
  __syncthreads();
  for (int i = tid; i < k * kD; i += kTile)
    if (acc[i] != 0) atomicAdd(&sums[(size_t)bh * k * kD + i], (unsigned long long)acc[i]);
  if (tid < k && scount[tid] != 0) atomicAdd(&counts[(size_t)bh * k + tid], scount[tid]);
}

template <typename T, int KC>
// Returns the number of kernels it enqueued.
static int launch_kmeans_pass(dim3 grid, cudaStream_t st, const T* v, const PrepPlan& pl, int it, bool last,
                              uint8_t* hist_t) {
  uint8_t* lab = it & 1 ? pl.assign2 : pl.assign;
  bool done = false;
  int n = 0;
  if constexpr (std::is_same<T, __nv_bfloat16>::value && KC >= 16) {
    if (pl.tc_assign) {
      // the pass's centroid operands, then one persistent CTA per SM over all
      // (b, h, chunk) items, taken from the pass's work counter
      const int items = pl.nchunks * pl.B * pl.H;
      const int ctas = std::max(1, std::min(items, pl.num_sms));
      if (last) cudaMemsetAsync(pl.hist, 0, sizeof(int) * (size_t)items * pl.k, st);  // summed by atomics
      kmeans_cops_kernel<KC><<<pl.B * pl.H, 128, 0, st>>>(pl.k, pl.cent, pl.cops);
      kmeans_assign_tc_kernel<KC><<<ctas, kTcThreads, assign_tc_smem<KC>(), st>>>(
          pl.tm_v, pl.S, pl.H, pl.k, pl.nchunks, pl.B * pl.H, pl.cent, pl.cops, pl.work + it, lab,
          last ? pl.hist : nullptr, hist_t);
      done = true;
      n += 2;
    }
  }
  if (!done) {
    kmeans_assign_kernel<T, KC><<<grid, kTile, assign_smem<KC>(), st>>>(v, pl.S, pl.H, pl.k, pl.cent, lab,
                                                                         last ? pl.hist : nullptr, hist_t);
    ++n;
  }
  if (!last) {
    kmeans_sums_kernel<T, KC><<<grid, kTile, 0, st>>>(v, pl.S, pl.H, pl.k, it > 0, lab, it & 1 ? pl.assign : pl.assign2,
                                                      pl.sums, pl.counts);
    ++n;
  }
  return n;
}

template <typename T>
static int launch_kmeans_pass_k(dim3 grid, cudaStream_t st, const T* v, const PrepPlan& pl, int it, bool last,
                                uint8_t* hist_t) {
  if (pl.k <= 8 && !(std::is_same<T, __nv_bfloat16>::value && pl.tc_assign))
    return launch_kmeans_pass<T, 8>(grid, st, v, pl, it, last, hist_t);
  if (pl.k <= 16) return launch_kmeans_pass<T, 16>(grid, st, v, pl, it, last, hist_t);
  return launch_kmeans_pass<T, 32>(grid, st, v, pl, it, last, hist_t);
}

// --------------------------------------------------------------- centroid update
// c = (double) sum * 2^-24 / count, rounded to fp32; an empty cluster keeps its
// centroid. sums and counts stay as running totals for the next delta pass.
__global__ void __launch_bounds__(128) kmeans_update_kernel(int k, float* __restrict__ cent,
                                                            unsigned long long* __restrict__ sums,
                                                            int* __restrict__ counts) {
  const int bh = blockIdx.x, d = threadIdx.x;
  for (int c = 0; c < k; ++c) {
    const int n = counts[(size_t)bh * k + c];
    const size_t i = ((size_t)bh * k + c) * kD + d;
    if (n > 0) {
      const double s = (double)(long long)sums[i] * 5.9604644775390625e-08;  // * 2^-24, exact
      cent[i] = __double2float_rn(__ddiv_rn(s, (double)n));
    }
  }
}

// --------------------------------------------------------------- stable cluster sort
// offs[bh][chunk][c] = (tokens of clusters < c) + (tokens of cluster c in earlier chunks)
__global__ void __launch_bounds__(32) perm_offsets_kernel(int k, int nchunks, const int* __restrict__ hist,
                                                          int* __restrict__ offs) {
  const int bh = blockIdx.x, c = threadIdx.x;
  int total = 0;
  if (c < k)
    for (int ch = 0; ch < nchunks; ++ch) total += hist[((size_t)bh * nchunks + ch) * k + c];
  // exclusive scan of the cluster totals across the warp
  int incl = total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (c >= o) incl += t;
  }
  int run = incl - total;
  if (c < k)
    for (int ch = 0; ch < nchunks; ++ch) {
      const size_t i = ((size_t)bh * nchunks + ch) * k + c;
      const int n = hist[i];
      offs[i] = run;
      run += n;
    }
}

// One CTA = one chunk of kChunk tokens; each warp ranks its 32 tokens with
// match_any, warps are ordered by an exclusive scan of their per-cluster counts.
__global__ void __launch_bounds__(kChunk) perm_scatter_kernel(int S, int k, const uint8_t* __restrict__ assign,
                                                              const int* __restrict__ offs,
                                                              int32_t* __restrict__ perm) {
  __shared__ int wcount[kChunk / 32][kMaxClusters];
  const int bh = blockIdx.y, chunk = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < (kChunk / 32) * kMaxClusters; i += kChunk) (&wcount[0][0])[i] = 0;
  __syncthreads();
  const int s = chunk * kChunk + tid;
  const bool valid = s < S;
  const int a = valid ? assign[(size_t)bh * S + s] : 0xFF;
  const unsigned peers = __match_any_sync(0xffffffffu, a);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (valid && rank == 0) wcount[warp][a] = __popc(peers);
  __syncthreads();
  if (tid < k) {
    int run = 0;
    for (int w = 0; w < kChunk / 32; ++w) {
      const int n = wcount[w][tid];
      wcount[w][tid] = run;
      run += n;
    }
  }
  __syncthreads();
  if (valid) {
    const int pos = offs[((size_t)bh * gridDim.x + chunk) * k + a] + wcount[warp][a] + rank;
    perm[(size_t)bh * S + pos] = s;
  }
}

__global__ void identity_perm_kernel(int S, int32_t* __restrict__ perm) {
  for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < S; s += gridDim.x * blockDim.x)
    perm[(size_t)blockIdx.y * S + s] = s;
}

// --------------------------------------------------------------- block mean + residual amax
// One CTA (4 warps) = one 128-token block of permuted positions, loaded as in
// quant_qk_kernel: warp w takes rows 32w .. 32w+31, two rows per load (lanes 0-15
// row 2i, lanes 16-31 row 2i+1, 16 bytes each), eight loads in flight at a time;
// lane l owns dimensions 8(l%16) .. 8(l%16)+7. The amax pass reads the rows
// again (from L1 / L2). Means use the int64 fixed-point sum (naive mode: all
// means are 0 and the first pass is skipped); the residual amax is merged into
// amax[bh] with an integer atomicMax on the (non-negative) fp32 bits; with
// kPerCh, one amax per channel, amax[bh * 128 + d].
template <typename T, bool kPerCh = false>
__global__ void __launch_bounds__(128) block_stats_kernel(const T* __restrict__ v, int S, int H,
                                                          const int32_t* __restrict__ perm, bool naive,
                                                          float* __restrict__ mu,
                                                          unsigned int* __restrict__ amax) {
  __shared__ long long wsum[8][kD];
  __shared__ float smu[kD];
  __shared__ float wmax[4];
  const int bh = blockIdx.y, b = bh / H, h = bh % H, blk = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int half = lane >> 4, c = lane & 15;
  const int p0 = blk * kBlock, cnt = min(kBlock, S - p0);
  const size_t row_stride = (size_t)H * kD;
  const T* vbase = v + ((size_t)b * S * H + h) * kD + c * 8;
  const int32_t* pbase = perm + (size_t)bh * S + p0;

  // rows warp*32 + i0*2 + 2i + half, i < 8 (rows past cnt read as 0)
  auto load8 = [&](int i0, uint4* x) {
    int src[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = warp * 32 + 2 * (i0 + i) + half;
      src[i] = r < cnt ? pbase[r] : -1;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      x[i] = src[i] >= 0 ? *reinterpret_cast<const uint4*>(vbase + (size_t)src[i] * row_stride)
                         : make_uint4(0u, 0u, 0u, 0u);
  };
  long long acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 1
  for (int i0 = 0; i0 < (naive ? 0 : 16); i0 += 8) {
    uint4 x[8];
    load8(i0, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float f[8];
      unpack8<T>(x[i], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __float2ll_rn(f[e] * 16777216.0f);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) wsum[warp * 2 + half][c * 8 + e] = acc[e];
  __syncthreads();
  {
    const int d = tid;
    long long s = 0;
#pragma unroll
    for (int g = 0; g < 8; ++g) s += wsum[g][d];
    const float m = naive ? 0.0f : __double2float_rn(__ddiv_rn((double)s * 5.9604644775390625e-08, (double)cnt));
    smu[d] = m;
    mu[((size_t)bh * gridDim.x + blk) * kD + d] = m;
  }
  __syncthreads();
  float m8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m8[e] = smu[c * 8 + e];
  float mx8[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};  // per channel of this lane
#pragma unroll 1
  for (int i0 = 0; i0 < 16; i0 += 8) {
    uint4 x[8];
    load8(i0, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (warp * 32 + 2 * (i0 + i) + half >= cnt) continue;
      float f[8];
      unpack8<T>(x[i], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], fabsf(__fsub_rn(f[e], m8[e])));
    }
  }
  if (!kPerCh) {
    float mx = mx8[0];
#pragma unroll
    for (int e = 1; e < 8; ++e) mx = fmaxf(mx, mx8[e]);
    mx = warp_max(mx);
    if (lane == 0) wmax[warp] = mx;
    __syncthreads();
    if (tid == 0) {
      const float m = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
      atomicMax(&amax[bh], __float_as_uint(m));
    }
  } else {
    // lanes c and c + 16 hold the same channels; then the four warps
    __shared__ float cmax[4][kD];
#pragma unroll
    for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(mx8[e], __shfl_xor_sync(0xffffffffu, mx8[e], 16));
    if (half == 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) cmax[warp][c * 8 + e] = mx8[e];
    }
    __syncthreads();
    const float m = fmaxf(fmaxf(cmax[0][tid], cmax[1][tid]), fmaxf(cmax[2][tid], cmax[3][tid]));
    atomicMax(&amax[(size_t)bh * kD + tid], __float_as_uint(m));
  }
}

// --------------------------------------------------------------- residual E4M3
// One CTA (8 warps) = one 128-token block of permuted positions. Loads as in
// quant_qk_kernel (two gathered 256-byte rows per warp instruction); each lane
// keeps the same 8 channels, so it subtracts 8 block means held in registers.
// The codes go to a shared tile [token][channel] (136-byte rows: the two half
// warps' 8-byte stores fall on disjoint banks) and leave transposed, as V^T rows
// of 128 tokens per channel (the K-major B operand of the PV product): a lane
// reads a 4 x 4 block of codes (4 channels of 4 consecutive tokens, one word per
// token), transposes it with byte permutes and stores 4 words, one per channel.
// A warp reads 8 channel groups of 4 token quads, which fall on 32 distinct banks.
constexpr int kResStride = 136;

// With kPerCh the scale is one per channel (amax_bits[bh * 128 + d], s_v
// [bh][128]): a channel whose amax is below 2^-100 gets scale 1 and codes 0.
template <typename T, bool kPerCh = false>
__global__ void __launch_bounds__(256) residual_e4m3_kernel(const T* __restrict__ v, int S, int H, int S_pad,
                                                            const int32_t* __restrict__ perm,
                                                            const float* __restrict__ mu,
                                                            const unsigned int* __restrict__ amax_bits,
                                                            uint8_t* __restrict__ vt, float* __restrict__ s_v) {
  __shared__ __align__(16) uint8_t ct[kBlock * kResStride];
  const int bh = blockIdx.y, b = bh / H, h = bh % H, blk = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4, c = lane & 15;
  float inv8[8];   // 448 / amax of each of this lane's 8 channels (0 for an all-zero one)
  bool zero = false;
  if (!kPerCh) {
    const float amax = __uint_as_float(amax_bits[bh]);
    zero = !(amax >= kTinyAmax);
    const float inv = zero ? 0.0f : __fdiv_rn(kE4M3Max, amax);
#pragma unroll
    for (int e = 0; e < 8; ++e) inv8[e] = inv;
    if (blk == 0 && threadIdx.x == 0) s_v[bh] = zero ? 1.0f : __fdiv_rn(amax, kE4M3Max);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float a = __uint_as_float(amax_bits[(size_t)bh * kD + c * 8 + e]);
      inv8[e] = a >= kTinyAmax ? __fdiv_rn(kE4M3Max, a) : 0.0f;
    }
    if (blk == 0 && threadIdx.x < kD) {
      const float a = __uint_as_float(amax_bits[(size_t)bh * kD + threadIdx.x]);
      s_v[(size_t)bh * kD + threadIdx.x] = a >= kTinyAmax ? __fdiv_rn(a, kE4M3Max) : 1.0f;
    }
  }
  float m8[8];
  {
    const float4* mp = reinterpret_cast<const float4*>(mu + ((size_t)bh * gridDim.x + blk) * kD + c * 8);
    const float4 m0 = mp[0], m1 = mp[1];
    m8[0] = m0.x; m8[1] = m0.y; m8[2] = m0.z; m8[3] = m0.w;
    m8[4] = m1.x; m8[5] = m1.y; m8[6] = m1.z; m8[7] = m1.w;
  }
  // the 8 row indices, then the 8 row loads, all in flight before the first use
  int src[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int p = blk * kBlock + warp * 16 + 2 * i + half;
    src[i] = p < S && !zero ? perm[(size_t)bh * S + p] : -1;
  }
  uint4 xs[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    xs[i] = src[i] >= 0 ? *reinterpret_cast<const uint4*>(v + (((size_t)b * S + src[i]) * H + h) * kD + c * 8)
                        : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = warp * 16 + 2 * i + half;
    uint2 w = make_uint2(0u, 0u);
    if (src[i] >= 0) {
      float f[8];
      unpack8<T>(xs[i], f);
      float rr[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)  // an all-zero channel codes to +0 (no -0 from a negative tiny residual)
        rr[e] = inv8[e] != 0.0f ? __fmul_rn(__fsub_rn(f[e], m8[e]), inv8[e]) : 0.0f;
      w.x = (uint32_t)cvt_e4m3x2(rr[0], rr[1]) | ((uint32_t)cvt_e4m3x2(rr[2], rr[3]) << 16);
      w.y = (uint32_t)cvt_e4m3x2(rr[4], rr[5]) | ((uint32_t)cvt_e4m3x2(rr[6], rr[7]) << 16);
    }
    *reinterpret_cast<uint2*>(ct + r * kResStride + c * 8) = w;
  }
  __syncthreads();
  uint8_t* const out = vt + (size_t)bh * kD * S_pad + (size_t)blk * kBlock;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    // a 4 x 4 block of codes: channels 4cg .. 4cg+3 of tokens 4tq .. 4tq+3
    const int combo = warp * 4 + it;
    const int cg = 8 * (combo & 3) + (lane & 7), tq = 4 * (combo >> 2) + (lane >> 3);
    const uint8_t* src = ct + (4 * tq) * kResStride + 4 * cg;
    const uint32_t r0 = *reinterpret_cast<const uint32_t*>(src);                   // token 4tq, 4 channels
    const uint32_t r1 = *reinterpret_cast<const uint32_t*>(src + kResStride);
    const uint32_t r2 = *reinterpret_cast<const uint32_t*>(src + 2 * kResStride);
    const uint32_t r3 = *reinterpret_cast<const uint32_t*>(src + 3 * kResStride);
    const uint32_t lo01 = __byte_perm(r0, r1, 0x5140), hi01 = __byte_perm(r0, r1, 0x7362);
    const uint32_t lo23 = __byte_perm(r2, r3, 0x5140), hi23 = __byte_perm(r2, r3, 0x7362);
    uint8_t* dst = out + (size_t)(4 * cg) * S_pad + 4 * tq;                          // 4 tokens of a channel
    *reinterpret_cast<uint32_t*>(dst) = __byte_perm(lo01, lo23, 0x5410);
    *reinterpret_cast<uint32_t*>(dst + S_pad) = __byte_perm(lo01, lo23, 0x7632);
    *reinterpret_cast<uint32_t*>(dst + 2 * (size_t)S_pad) = __byte_perm(hi01, hi23, 0x5410);
    *reinterpret_cast<uint32_t*>(dst + 3 * (size_t)S_pad) = __byte_perm(hi01, hi23, 0x7632);
  }
}

// --------------------------------------------------------------- residual NVFP4
// Global scale g = amax / (448 * 6) per (b, h); per channel and group of 16
// consecutive permuted tokens an E4M3 scale s = E4M3(fl32(fl32(gmax/6)/g)), and
// E2M1 codes of r / fl32(dec(s) * g) (0 where dec(s) == 0). One CTA (8 warps) =
// one 128-token block, loaded as in residual_e4m3_kernel: warp w holds rows
// 16w .. 16w+15, which is exactly group w of the block, so a group's amax per
// channel is a lane's max over its rows merged with the other half warp's. The
// codes leave through a shared tile and 4 x 4 byte transposes as in
// residual_mxfp4_kernel; the scales through a shared [channel][group] tile.
template <typename T>
__global__ void __launch_bounds__(256) residual_nvfp4_kernel(const T* __restrict__ v, int S, int H, int S_pad,
                                                             const int32_t* __restrict__ perm,
                                                             const float* __restrict__ mu,
                                                             const unsigned int* __restrict__ amax_bits,
                                                             uint8_t* __restrict__ codes,
                                                             uint8_t* __restrict__ scales, float* __restrict__ gsc) {
  __shared__ __align__(16) uint8_t ct[kBlock * kResStride];
  __shared__ __align__(8) uint8_t ssc[kD][8];   // [channel][group] scale codes of the block
  const int bh = blockIdx.y, b = bh / H, h = bh % H, blk = blockIdx.x, nb = gridDim.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4, c = lane & 15;
  const float amax = __uint_as_float(amax_bits[bh]);
  const bool zero = !(amax >= kTinyAmax);
  const float g = zero ? 1.0f : __fdiv_rn(amax, kE4M3Max * kE2M1Max);
  if (blk == 0 && threadIdx.x == 0) gsc[bh] = g;
  float m8[8];
  {
    const float4* mp = reinterpret_cast<const float4*>(mu + ((size_t)bh * nb + blk) * kD + c * 8);
    const float4 m0 = mp[0], m1 = mp[1];
    m8[0] = m0.x; m8[1] = m0.y; m8[2] = m0.z; m8[3] = m0.w;
    m8[4] = m1.x; m8[5] = m1.y; m8[6] = m1.z; m8[7] = m1.w;
  }
  int src[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int p = blk * kBlock + warp * 16 + 2 * i + half;
    src[i] = p < S && !zero ? perm[(size_t)bh * S + p] : -1;
  }
  uint4 xs[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    xs[i] = src[i] >= 0 ? *reinterpret_cast<const uint4*>(v + (((size_t)b * S + src[i]) * H + h) * kD + c * 8)
                        : make_uint4(0u, 0u, 0u, 0u);
  float rr[8][8], mx[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mx[e] = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float f[8];
    unpack8<T>(xs[i], f);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      rr[i][e] = src[i] >= 0 ? __fsub_rn(f[e], m8[e]) : 0.0f;
      mx[e] = fmaxf(mx[e], fabsf(rr[i][e]));
    }
  }
  float den[8];
  uint32_t scw0 = 0u, scw1 = 0u;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float gmax = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 16));   // group `warp`, channel c*8+e
    const uint32_t sc = zero ? 0u : cvt_e4m3(__fdiv_rn(__fdiv_rn(gmax, kE2M1Max), g));
    den[e] = sc != 0u ? __fmul_rn(e4m3_to_f32(sc), g) : 0.0f;
    if (e < 4) scw0 |= sc << (8 * e); else scw1 |= sc << (8 * (e - 4));
  }
  if (half == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) ssc[c * 8 + e][warp] = (uint8_t)(((e < 4 ? scw0 : scw1) >> (8 * (e & 3))) & 0xFFu);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = warp * 16 + 2 * i + half;
    uint32_t w0 = 0u, w1 = 0u;   // one code per byte, channels c*8 .. c*8+7
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (den[e] != 0.0f) w0 |= (uint32_t)(cvt_e2m1x2(__fdiv_rn(rr[i][e], den[e]), 0.0f) & 0xFu) << (8 * e);
      if (den[4 + e] != 0.0f)
        w1 |= (uint32_t)(cvt_e2m1x2(__fdiv_rn(rr[i][4 + e], den[4 + e]), 0.0f) & 0xFu) << (8 * e);
    }
    *reinterpret_cast<uint2*>(ct + r * kResStride + c * 8) = make_uint2(w0, w1);
  }
  __syncthreads();
  if (threadIdx.x < kD) {
    const int d = threadIdx.x;
    *reinterpret_cast<uint2*>(scales + ((size_t)bh * kD + d) * (S_pad / kGroup4) + (size_t)blk * (kBlock / kGroup4)) =
        *reinterpret_cast<const uint2*>(ssc[d]);
  }
  uint8_t* const out = codes + (size_t)bh * kD * (S_pad / 2) + (size_t)blk * (kBlock / 2);
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int combo = warp * 4 + it;
    const int cg = 8 * (combo & 3) + (lane & 7), tq = 4 * (combo >> 2) + (lane >> 3);
    const uint8_t* sp = ct + (4 * tq) * kResStride + 4 * cg;
    const uint32_t r0 = *reinterpret_cast<const uint32_t*>(sp);
    const uint32_t r1 = *reinterpret_cast<const uint32_t*>(sp + kResStride);
    const uint32_t r2 = *reinterpret_cast<const uint32_t*>(sp + 2 * kResStride);
    const uint32_t r3 = *reinterpret_cast<const uint32_t*>(sp + 3 * kResStride);
    const uint32_t lo01 = __byte_perm(r0, r1, 0x5140), hi01 = __byte_perm(r0, r1, 0x7362);
    const uint32_t lo23 = __byte_perm(r2, r3, 0x5140), hi23 = __byte_perm(r2, r3, 0x7362);
    const uint32_t ch4[4] = {__byte_perm(lo01, lo23, 0x5410), __byte_perm(lo01, lo23, 0x7632),
                             __byte_perm(hi01, hi23, 0x5410), __byte_perm(hi01, hi23, 0x7632)};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t w = ch4[q];
      const uint32_t packed = (w & 0xFu) | ((w >> 4) & 0xF0u) | (((w >> 16) & 0xFu) << 8) | ((w >> 12) & 0xF000u);
      *reinterpret_cast<uint16_t*>(out + (size_t)(4 * cg + q) * (S_pad / 2) + 2 * tq) = (uint16_t)packed;
    }
  }
}

// --------------------------------------------------------------- residual MX-style FP4
// Per channel and group of 32 consecutive permuted tokens, the power of two
// X = 2^e with e the smallest integer for which the group's amax <= 6 * 2^e (so
// no value clips), e >= -127; E2M1 codes of r * 2^-e (exact scaling, then one
// round to nearest even). From the fp32 bits of the amax, amax = f * 2^E with f
// in [1, 2): 6 * 2^(E-2) = 1.5 * 2^E covers it iff f <= 1.5, else 6 * 2^(E-1);
// an amax below 2^-126 (zero or subnormal) gives the clamp value -127.
// Outputs: packed codes as the NVFP4 residual ([BH][128][S_pad/2], even token in
// the low nibble) and the biased exponents e + 127 as [BH][nb][128][4] bytes
// (block, channel, group of the block), so that a block's exponents are one
// 512-byte piece with one word per channel.
__device__ __forceinline__ int mx_exponent(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int be = (int)(bits >> 23);
  if (be == 0) return -127;
  const int E = be - 127;
  return max(-127, (bits & 0x7FFFFFu) <= 0x400000u ? E - 2 : E - 1);
}

// One CTA (8 warps) = one 128-token block of permuted positions, loaded as in
// residual_e4m3_kernel (warp w: rows 16w .. 16w+15, two rows per load; lane l
// owns channels 8(l%16) .. 8(l%16)+7). A group of 32 tokens is warps 2g and 2g+1:
// each lane takes the amax of its channels over its rows, the two half warps and
// then the two warps of the group merge theirs through shared memory. The codes go
// to a shared tile [token][channel] (one code per byte) and leave transposed as
// in residual_e4m3_kernel (4 x 4 byte blocks and byte permutes), then packed two
// tokens a byte.
template <typename T>
__global__ void __launch_bounds__(256) residual_mxfp4_kernel(const T* __restrict__ v, int S, int H, int S_pad,
                                                             const int32_t* __restrict__ perm,
                                                             const float* __restrict__ mu,
                                                             uint8_t* __restrict__ codes,
                                                             uint32_t* __restrict__ exps, float* __restrict__ s_v) {
  __shared__ __align__(16) uint8_t ct[kBlock * kResStride];
  __shared__ float wmx[8][kD];   // per warp: the amax of each channel over its 16 rows
  const int bh = blockIdx.y, b = bh / H, h = bh % H, blk = blockIdx.x, nb = gridDim.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4, c = lane & 15;
  if (blk == 0 && threadIdx.x == 0) s_v[bh] = 1.0f;   // no per-head scale
  float m8[8];
  {
    const float4* mp = reinterpret_cast<const float4*>(mu + ((size_t)bh * nb + blk) * kD + c * 8);
    const float4 m0 = mp[0], m1 = mp[1];
    m8[0] = m0.x; m8[1] = m0.y; m8[2] = m0.z; m8[3] = m0.w;
    m8[4] = m1.x; m8[5] = m1.y; m8[6] = m1.z; m8[7] = m1.w;
  }
  int src[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int p = blk * kBlock + warp * 16 + 2 * i + half;
    src[i] = p < S ? perm[(size_t)bh * S + p] : -1;
  }
  uint4 xs[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    xs[i] = src[i] >= 0 ? *reinterpret_cast<const uint4*>(v + (((size_t)b * S + src[i]) * H + h) * kD + c * 8)
                        : make_uint4(0u, 0u, 0u, 0u);
  // residuals (padding rows 0) and their per-channel amax over this lane's rows
  float rr[8][8], mx[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mx[e] = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float f[8];
    unpack8<T>(xs[i], f);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      rr[i][e] = src[i] >= 0 ? __fsub_rn(f[e], m8[e]) : 0.0f;
      mx[e] = fmaxf(mx[e], fabsf(rr[i][e]));
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 16));
  if (half == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) wmx[warp][c * 8 + e] = mx[e];
  }
  __syncthreads();
  // this group's exponents (group g = warp / 2) and the codes of this lane's values
  const int g = warp >> 1;
  float sc[8];
  uint32_t ew = 0u;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int ex = mx_exponent(fmaxf(wmx[2 * g][c * 8 + e], wmx[2 * g + 1][c * 8 + e]));
    sc[e] = __uint_as_float((uint32_t)(127 - ex) << 23);   // 2^-ex, normal for ex in [-127, 126]
    (void)ew;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = warp * 16 + 2 * i + half;
    uint32_t w0 = 0u, w1 = 0u;   // one code per byte, channels c*8 .. c*8+7
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      w0 |= (uint32_t)(cvt_e2m1x2(__fmul_rn(rr[i][e], sc[e]), 0.0f) & 0xFu) << (8 * e);
      w1 |= (uint32_t)(cvt_e2m1x2(__fmul_rn(rr[i][4 + e], sc[4 + e]), 0.0f) & 0xFu) << (8 * e);
    }
    *reinterpret_cast<uint2*>(ct + r * kResStride + c * 8) = make_uint2(w0, w1);
  }
  // the block's exponent bytes: channel d, groups 0..3 in one word
  if (threadIdx.x < kD) {
    const int d = threadIdx.x;
    uint32_t w = 0u;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      w |= (uint32_t)(mx_exponent(fmaxf(wmx[2 * q][d], wmx[2 * q + 1][d])) + 127) << (8 * q);
    exps[((size_t)bh * nb + blk) * kD + d] = w;
  }
  __syncthreads();
  uint8_t* const out = codes + (size_t)bh * kD * (S_pad / 2) + (size_t)blk * (kBlock / 2);
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    // a 4 x 4 block of codes: channels 4cg .. 4cg+3 of tokens 4tq .. 4tq+3
    const int combo = warp * 4 + it;
    const int cg = 8 * (combo & 3) + (lane & 7), tq = 4 * (combo >> 2) + (lane >> 3);
    const uint8_t* sp = ct + (4 * tq) * kResStride + 4 * cg;
    const uint32_t r0 = *reinterpret_cast<const uint32_t*>(sp);
    const uint32_t r1 = *reinterpret_cast<const uint32_t*>(sp + kResStride);
    const uint32_t r2 = *reinterpret_cast<const uint32_t*>(sp + 2 * kResStride);
    const uint32_t r3 = *reinterpret_cast<const uint32_t*>(sp + 3 * kResStride);
    const uint32_t lo01 = __byte_perm(r0, r1, 0x5140), hi01 = __byte_perm(r0, r1, 0x7362);
    const uint32_t lo23 = __byte_perm(r2, r3, 0x5140), hi23 = __byte_perm(r2, r3, 0x7362);
    // channel 4cg + q: its 4 tokens' codes, one per byte, then two per byte
    const uint32_t ch4[4] = {__byte_perm(lo01, lo23, 0x5410), __byte_perm(lo01, lo23, 0x7632),
                             __byte_perm(hi01, hi23, 0x5410), __byte_perm(hi01, hi23, 0x7632)};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t w = ch4[q];
      const uint32_t packed = (w & 0xFu) | ((w >> 4) & 0xF0u) | (((w >> 16) & 0xFu) << 8) | ((w >> 12) & 0xF000u);
      *reinterpret_cast<uint16_t*>(out + (size_t)(4 * cg + q) * (S_pad / 2) + 2 * tq) = (uint16_t)packed;
    }
  }
}

// --------------------------------------------------------------- token sums (K smoothing)
// sums[bh][d] += sum over tokens of llrint(x * 2^24), the exact, order-free
// int64 fixed-point sum (two's complement in the unsigned atomics). One CTA
// (4 warps) = kSumRows tokens of one (b, h); row group g = 2 warp + half takes
// rows g, g + 8, ...: each warp load reads two whole 256-byte rows, eight loads
// in flight; lane l owns dimensions 8 (l % 16) .. 8 (l % 16) + 7.
constexpr int kSumRows = 1024;

template <typename T>
__global__ void __launch_bounds__(128) token_sums_kernel(const T* __restrict__ x, int S, int H,
                                                         unsigned long long* __restrict__ sums) {
  __shared__ long long part[8][kD];
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, half = lane >> 4, c = lane & 15;
  const int g = warp * 2 + half;
  const int p0 = blockIdx.x * kSumRows, cnt = min(kSumRows, S - p0);
  const size_t rs = (size_t)H * kD;
  const T* base = x + (((size_t)b * S + p0) * H + h) * kD + c * 8;
  long long acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 1
  for (int r0 = g; r0 < cnt; r0 += 64) {
    uint4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int r = r0 + 8 * j;
      v[j] = r < cnt ? *reinterpret_cast<const uint4*>(base + (size_t)r * rs) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float f[8];
      unpack8<T>(v[j], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __float2ll_rn(f[e] * 16777216.0f);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[g][c * 8 + e] = acc[e];
  __syncthreads();
  const int d = threadIdx.x;
  long long t = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) t += part[i][d];
  atomicAdd(&sums[(size_t)bh * kD + d], (unsigned long long)t);
}

// kbar[bh][d] = fl32((sum * 2^-24) / S) from the token sums, once per (b, h) and
// channel (one fp64 division each); also into k_mean when that is given.
__global__ void __launch_bounds__(128) kbar_kernel(const unsigned long long* __restrict__ sums, int S,
                                                   float* __restrict__ kbar, float* __restrict__ k_mean) {
  const size_t i = (size_t)blockIdx.x * kD + threadIdx.x;
  const long long sum = (long long)sums[i];
  const float m = __double2float_rn(__ddiv_rn((double)sum * 5.9604644775390625e-08, (double)S));
  kbar[i] = m;
  if (k_mean != nullptr) k_mean[i] = m;
}

// --------------------------------------------------------------- Q/K quantisation
// One CTA (8 warps) = one 128-row block of Q (original order) or K (gathered by
// perm). Warp w takes rows 16w .. 16w+15, two rows per load: lanes 0-15 read row
// 2i and lanes 16-31 row 2i+1, 16 bytes each, so every load instruction reads two
// whole 256-byte rows. The values stay in registers while the block amax is
// reduced (warp shuffles, then shared memory); each lane then writes the 8 E4M3
// codes of its 8 values (rows of 128 codes, contiguous per half warp).
// With kbar (K smoothing: the per-channel token mean of K made by kbar_kernel),
// the K CTAs first subtract kbar from every valid row (an fp32 subtraction;
// padding rows stay 0) (a separate instantiation, so that the plain one keeps its
// register count and occupancy).
template <typename T, bool kSmooth>
__global__ void __launch_bounds__(256, 3) quant_qk_kernel(const T* __restrict__ q, const T* __restrict__ k, int S,
                                                       int H, int S_pad, const int32_t* __restrict__ perm,
                                                       const float* __restrict__ kbar,
                                                       uint8_t* __restrict__ qc, float* __restrict__ qs,
                                                       uint8_t* __restrict__ kc, float* __restrict__ ks) {
  __shared__ float wmax[8];
  const int bh = blockIdx.y, b = bh / H, h = bh % H, blk = blockIdx.x;
  const bool is_k = blockIdx.z == 1;
  const bool smooth = kSmooth && is_k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4, c = lane & 15;  // row parity and 16-byte piece of the row
  const T* const src = is_k ? k : q;
  // the 8 row indices, then the 8 row loads, all in flight before the first use
  int row[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int p = blk * kBlock + warp * 16 + 2 * i + half;
    row[i] = p < S ? (is_k ? perm[(size_t)bh * S + p] : p) : -1;
  }
  uint4 x[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    x[i] = row[i] >= 0 ? *reinterpret_cast<const uint4*>(src + (((size_t)b * S + row[i]) * H + h) * kD + c * 8)
                       : make_uint4(0u, 0u, 0u, 0u);
  float kb[8];
  if (smooth) {
    const float4* m4 = reinterpret_cast<const float4*>(kbar + (size_t)bh * kD + c * 8);
    const float4 m0 = __ldg(m4), m1 = __ldg(m4 + 1);
    kb[0] = m0.x, kb[1] = m0.y, kb[2] = m0.z, kb[3] = m0.w;
    kb[4] = m1.x, kb[5] = m1.y, kb[6] = m1.z, kb[7] = m1.w;
  }
  // the values of row i (K smoothed when asked; rows past S are 0)
  auto values = [&](int i, float* f) {
    unpack8<T>(x[i], f);
    if (smooth && row[i] >= 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = __fsub_rn(f[e], kb[e]);
    }
  };
  float mx = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float f[8];
    values(i, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(f[e]));
  }
  mx = warp_max(mx);
  if (lane == 0) wmax[warp] = mx;
  __syncthreads();
  float amax = wmax[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, wmax[w]);
  const bool zero = !(amax >= kTinyAmax);
  const float inv = zero ? 0.0f : __fdiv_rn(kE4M3Max, amax);
  const int nbk = gridDim.x;
  if (threadIdx.x == 0) (is_k ? ks : qs)[(size_t)bh * nbk + blk] = zero ? 1.0f : __fdiv_rn(amax, kE4M3Max);
  uint8_t* const out = (is_k ? kc : qc) + ((size_t)bh * S_pad + (size_t)blk * kBlock) * kD;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = warp * 16 + 2 * i + half;
    uint2 w = make_uint2(0u, 0u);
    if (!zero) {  // rows past S hold zeros, which code to 0
      float f[8];
      values(i, f);
      w.x = (uint32_t)cvt_e4m3x2(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv)) |
            ((uint32_t)cvt_e4m3x2(__fmul_rn(f[2], inv), __fmul_rn(f[3], inv)) << 16);
      w.y = (uint32_t)cvt_e4m3x2(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv)) |
            ((uint32_t)cvt_e4m3x2(__fmul_rn(f[6], inv), __fmul_rn(f[7], inv)) << 16);
    }
    *reinterpret_cast<uint2*>(out + (size_t)r * kD + c * 8) = w;
  }
}

// --------------------------------------------------------------- NVFP4 -> two E4M3 planes
// The attention kernel multiplies E4M3 probabilities with E4M3 operands only.
// An NVFP4 residual value e2m1 * dec(s16) (times the global g) has at most 6
// significant bits, so v = e2m1 * dec(s16) / 8 (at most 336) splits exactly into
// hi = E4M3(v) and lo = E4M3(v - hi); the product P (hi + lo) is then P v exactly
// wherever lo lies on the E4M3 grid (|v| >= 2^-4, i.e. down to 1/5376 of the
// head's largest value; below that lo rounds to the 2^-9 subnormal grid).
// One CTA = one 128-token block of one (b, h); thread d owns channel d.
__global__ void __launch_bounds__(128) nvfp4_planes_kernel(const uint8_t* __restrict__ codes,
                                                           const uint8_t* __restrict__ scales, int S_pad,
                                                           size_t plane_stride, uint8_t* __restrict__ planes) {
  const int bh = blockIdx.y, blk = blockIdx.x, d = threadIdx.x;
  const size_t row = (size_t)bh * kD + d;
  const uint8_t* crow = codes + row * (S_pad / 2) + (size_t)blk * (kBlock / 2);
  const uint2 sc2 = *reinterpret_cast<const uint2*>(scales + row * (S_pad / kGroup4) + (size_t)blk * (kBlock / kGroup4));
  uint8_t* hi = planes + row * S_pad + (size_t)blk * kBlock;
  uint8_t* lo = hi + plane_stride;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {  // 32 tokens (16 code bytes) at a time
    const uint4 cw = *reinterpret_cast<const uint4*>(crow + c * 16);
    const uint8_t* cb = reinterpret_cast<const uint8_t*>(&cw);
    // the two scale bytes of these 32 tokens (scale byte 2c and 2c+1 of the block)
    const uint32_t sw = ((c < 2) ? sc2.x : sc2.y) >> (16 * (c & 1));
    const float sc_lo = e4m3_to_f32(sw & 0xFFu), sc_hi = e4m3_to_f32((sw >> 8) & 0xFFu);
    uint32_t wh[8], wl[8];
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      float v[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const uint32_t nib = (cb[(i + e) >> 1] >> (4 * ((i + e) & 1))) & 0xFu;
        const float mag = e2m1_value(nib & 7u);
        v[e] = __fmul_rn(__fmul_rn((nib & 8u) ? -mag : mag, (i + e) < kGroup4 ? sc_lo : sc_hi), 0.125f);
      }
      const uint16_t h2 = cvt_e4m3x2(v[0], v[1]);
      const uint16_t l2 = cvt_e4m3x2(__fsub_rn(v[0], e4m3_to_f32(h2 & 0xFF)), __fsub_rn(v[1], e4m3_to_f32(h2 >> 8)));
      const int k = i >> 1;  // byte pair index 0..15
      if ((k & 1) == 0) {
        wh[k >> 1] = h2;
        wl[k >> 1] = l2;
      } else {
        wh[k >> 1] |= (uint32_t)h2 << 16;
        wl[k >> 1] |= (uint32_t)l2 << 16;
      }
    }
    uint4* oh = reinterpret_cast<uint4*>(hi + c * 32);
    uint4* ol = reinterpret_cast<uint4*>(lo + c * 32);
    oh[0] = make_uint4(wh[0], wh[1], wh[2], wh[3]);
    oh[1] = make_uint4(wh[4], wh[5], wh[6], wh[7]);
    ol[0] = make_uint4(wl[0], wl[1], wl[2], wl[3]);
    ol[1] = make_uint4(wl[4], wl[5], wl[6], wl[7]);
  }
}

cudaError_t launch_nvfp4_planes(const uint8_t* codes, const uint8_t* scales, int BH, int S_pad, uint8_t* planes,
                                cudaStream_t st) {
  const dim3 grid(S_pad / kBlock, BH);
  nvfp4_planes_kernel<<<grid, 128, 0, st>>>(codes, scales, S_pad, (size_t)BH * kD * S_pad, planes);
  return cudaGetLastError();
}

// --------------------------------------------------------------- residual energy (diagnostic)
// E[bh] = sum over permuted positions p < S of ||v[perm[p]] - mu[p / 128]||^2:
// the energy the residual quantiser sees. One CTA (4 warps) = one 128-token
// block, rows gathered as in block_stats_kernel (two 256-byte rows per warp
// load, eight loads in flight). Each lane forms its differences, squares and
// sums in fp64 (a 16-bit input minus an fp32 mean is exact there unless the two
// lie some 28 binades apart, and rounded once otherwise); the CTA's sum goes to
// energy[bh] (zeroed by the launcher) with one double atomicAdd, so only the
// summation order varies from run to run.
// perm == NULL reads the identity order, mu == NULL zero means.
template <typename T>
__global__ void __launch_bounds__(128) residual_energy_kernel(const T* __restrict__ v, int S, int H,
                                                              const int32_t* __restrict__ perm,
                                                              const float* __restrict__ mu,
                                                              double* __restrict__ energy) {
  __shared__ double wsum[4];
  const int bh = blockIdx.y, b = bh / H, h = bh % H, blk = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int half = lane >> 4, c = lane & 15;
  const int p0 = blk * kBlock, cnt = min(kBlock, S - p0);
  const size_t row_stride = (size_t)H * kD;
  const T* vbase = v + ((size_t)b * S * H + h) * kD + c * 8;
  double m8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e)
    m8[e] = mu ? (double)mu[((size_t)bh * gridDim.x + blk) * kD + c * 8 + e] : 0.0;
  double acc = 0.0;
#pragma unroll 1
  for (int i0 = 0; i0 < 16; i0 += 8) {
    int src[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = warp * 32 + 2 * (i0 + i) + half;
      src[i] = r < cnt ? (perm ? perm[(size_t)bh * S + p0 + r] : p0 + r) : -1;
    }
    uint4 x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      x[i] = src[i] >= 0 ? *reinterpret_cast<const uint4*>(vbase + (size_t)src[i] * row_stride)
                         : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (src[i] < 0) continue;
      float f[8];
      unpack8<T>(x[i], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const double d = (double)f[e] - m8[e];
        acc = fma(d, d, acc);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) wsum[warp] = acc;
  __syncthreads();
  if (tid == 0) atomicAdd(&energy[bh], (wsum[0] + wsum[1]) + (wsum[2] + wsum[3]));
}

// --------------------------------------------------------------- V residual repair
// "Open VC Attention", "Описание": the repair re-adds the quantisation residual
// of the worst-rounded value tokens (budget e.g. 0.005). Two E4M3 planes at the
// residual's scale s_V: plane 0 holds the residual codes (residual_e4m3_kernel),
// plane 1, for the kept tokens, the E4M3 codes of each element's rounding error
// in code units, dlt = y - dec(code) with y = fl32(fl32(x - mu) * fl32(448/amax))
// the value that was rounded (exact in fp32), and 0 elsewhere; the two-plane
// attention kernel then adds P (plane 0 + plane 1) at scale s_V.
// A token's error is sum_d fl32(dlt_d^2), added in fp32 from d = 0 to 127; the
// kept tokens are the m largest by the key (error, then lower position).

// y - dec(code) of channel d of one token: the rounding error in code units.
__device__ __forceinline__ float repair_dlt(float x, float m, float inv, uint32_t code) {
  return __fsub_rn(__fmul_rn(__fsub_rn(x, m), inv), e4m3_to_f32(code));
}

// 64-bit ranking key: larger error first, then lower position (errors are >= 0,
// so their bit patterns order like their values).
__device__ __forceinline__ unsigned long long repair_key(float err, int p) {
  return ((unsigned long long)__float_as_uint(err) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)p);
}

// The tile of one 128-token block of permuted positions in shared memory: rows
// gathered through perm with coalesced 16-byte loads (two rows per warp
// instruction, every load of a thread issued before the first store), at
// tile_off(r, piece). Rows past S are left unwritten.
template <typename T>
__device__ __forceinline__ void stage_perm_tile(uint8_t* tile, const T* __restrict__ v, int S, int H, int b, int h,
                                                const int32_t* __restrict__ prow, int ntok) {
  const int tid = threadIdx.x;
  uint4 x[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int idx = i * kTile + tid, r = idx >> 4, c = idx & 15;
    if (r < ntok) x[i] = *reinterpret_cast<const uint4*>(v + (((size_t)b * S + prow[r]) * H + h) * kD + c * 8);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int idx = i * kTile + tid, r = idx >> 4, c = idx & 15;
    if (r < ntok) *reinterpret_cast<uint4*>(tile + tile_off(r, c)) = x[i];
  }
}

// err[bh][p] for every permuted position p < S. One CTA = one 128-token block:
// the block's rows are staged in shared memory, then each thread takes one token,
// recomputes its codes exactly as the residual kernel does (so plane 0 need not
// be read) and sums the squared rounding errors channel by channel in order.
template <typename T>
__global__ void __launch_bounds__(128) repair_err_kernel(const T* __restrict__ v, int S, int H, int S_pad,
                                                         const int32_t* __restrict__ perm,
                                                         const float* __restrict__ mu,
                                                         const unsigned int* __restrict__ amax_bits,
                                                         float* __restrict__ err) {
  __shared__ float smu[kD];
  extern __shared__ __align__(16) uint8_t tile[];
  const int bh = blockIdx.y, b = bh / H, h = bh % H, blk = blockIdx.x, t = threadIdx.x;
  const int p0 = blk * kBlock, ntok = min(kBlock, S - p0);
  smu[t] = mu[((size_t)bh * gridDim.x + blk) * kD + t];
  const float amax = __uint_as_float(amax_bits[bh]);
  const bool zero = !(amax >= kTinyAmax);
  if (!zero) stage_perm_tile<T>(tile, v, S, H, b, h, perm + (size_t)bh * S + p0, ntok);
  __syncthreads();
  if (t >= ntok) return;
  float e = 0.0f;
  if (!zero) {
    const float inv = __fdiv_rn(kE4M3Max, amax);
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
      float f[8];
      unpack8<T>(*reinterpret_cast<const uint4*>(tile + tile_off(t, c)), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float y = __fmul_rn(__fsub_rn(f[i], smu[c * 8 + i]), inv);
        const float dl = __fsub_rn(y, e4m3_to_f32(cvt_e4m3(y)));
        e = __fadd_rn(e, __fmul_rn(dl, dl));
      }
    }
  }
  err[(size_t)bh * S + p0 + t] = e;
}

// thr[bh] = the key of the m-th largest token (1 <= m <= S): a radix select over
// the 64-bit keys, 8 bits per pass from the top, one CTA per (b, h). Each pass
// counts the candidates (keys matching the digits chosen so far) per next digit
// in shared memory and keeps the digit where the count from the top reaches the
// remaining rank; keys are distinct, so exactly m keys are >= thr.
__global__ void __launch_bounds__(256) repair_select_kernel(const float* __restrict__ err, int S, int m,
                                                            unsigned long long* __restrict__ thr) {
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ int s_left;
  const int bh = blockIdx.x, t = threadIdx.x;
  const float* e = err + (size_t)bh * S;
  unsigned long long prefix = 0ull, mask = 0ull;
  int left = m;
#pragma unroll 1
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    hist[t] = 0u;
    __syncthreads();
    for (int p = t; p < S; p += 256) {
      const unsigned long long k = repair_key(e[p], p);
      if ((k & mask) == prefix) atomicAdd(&hist[(uint32_t)(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (t == 0) {
      int above = 0, digit = 0;
      for (int d = 255; d >= 0; --d) {
        const int c = (int)hist[d];
        if (above + c >= left) {
          digit = d;
          break;
        }
        above += c;
      }
      s_left = left - above;
      s_prefix = prefix | ((unsigned long long)digit << shift);
    }
    __syncthreads();
    prefix = s_prefix;
    left = s_left;
    mask |= 0xFFull << shift;
    __syncthreads();
  }
  if (t == 0) thr[bh] = prefix;
}

// Plane 1 (and the optional kept flags): one CTA = one 128-token block of
// permuted positions, its rows staged in shared memory when any is kept; one
// thread per token, which recomputes its codes as the residual kernel does; channel
// by channel the 128 threads write 128 consecutive bytes of the V^T plane. Tokens
// not kept, padding tokens and slices whose residual is all zero get 0.
template <typename T>
__global__ void __launch_bounds__(128) repair_plane_kernel(const T* __restrict__ v, int S, int H, int S_pad,
                                                           const int32_t* __restrict__ perm,
                                                           const float* __restrict__ mu,
                                                           const unsigned int* __restrict__ amax_bits,
                                                           const float* __restrict__ err,
                                                           const unsigned long long* __restrict__ thr, bool any,
                                                           uint8_t* __restrict__ plane1, uint8_t* __restrict__ kept) {
  __shared__ float smu[kD];
  __shared__ int nkeep;
  extern __shared__ __align__(16) uint8_t tile[];
  const int bh = blockIdx.y, b = bh / H, h = bh % H, blk = blockIdx.x, t = threadIdx.x;
  const int p0 = blk * kBlock, ntok = min(kBlock, S - p0), p = p0 + t;
  smu[t] = mu[((size_t)bh * gridDim.x + blk) * kD + t];
  if (t == 0) nkeep = 0;
  __syncthreads();
  const float amax = __uint_as_float(amax_bits[bh]);
  const bool zero = !(amax >= kTinyAmax);
  const bool keep = any && p < S && repair_key(err[(size_t)bh * S + p], p) >= thr[bh];
  if (kept != nullptr && p < S) kept[(size_t)bh * S + p] = keep ? 1 : 0;
  if (keep && !zero) atomicAdd(&nkeep, 1);
  __syncthreads();
  const bool stage = nkeep > 0;   // uniform: the block has a kept token
  if (stage) stage_perm_tile<T>(tile, v, S, H, b, h, perm + (size_t)bh * S + p0, ntok);
  __syncthreads();
  uint8_t* out = plane1 + (size_t)bh * kD * S_pad + p;
  if (!keep || zero) {
#pragma unroll 4
    for (int d = 0; d < kD; ++d) out[(size_t)d * S_pad] = 0;
    return;
  }
  const float inv = __fdiv_rn(kE4M3Max, amax);
#pragma unroll 4
  for (int c = 0; c < 16; ++c) {
    float f[8];
    unpack8<T>(*reinterpret_cast<const uint4*>(tile + tile_off(t, c)), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float y = __fmul_rn(__fsub_rn(f[i], smu[c * 8 + i]), inv);
      out[(size_t)(c * 8 + i) * S_pad] = cvt_e4m3(__fsub_rn(y, e4m3_to_f32(cvt_e4m3(y))));
    }
  }
}

// --------------------------------------------------------------- launchers
template <typename T>
static cudaError_t launch_prepare_v_t(const T* v, const PrepPlan& pl, const vc_prepared_v_t& out,
                                      uint8_t* history, cudaStream_t st, int* nlaunch) {
  const int S = pl.S, H = pl.H, BH = pl.B * pl.H, k = pl.k;
  cudaError_t e;
  int n = 0;
  const size_t namax = (size_t)BH * (pl.fmt == VC_RESIDUAL_E4M3_PER_CHANNEL ? kD : 1);  // per (b, h) or channel
  if ((e = cudaMemsetAsync(pl.amax, 0, sizeof(unsigned) * namax, st)) != cudaSuccess) return e;
  if (pl.mode == VC_MODE_VSMOOTH) {
    if ((e = cudaMemsetAsync(pl.sums, 0, sizeof(unsigned long long) * BH * k * kD, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(pl.counts, 0, sizeof(int) * BH * k, st)) != cudaSuccess) return e;
    if (pl.tc_assign && (e = cudaMemsetAsync(pl.work, 0, sizeof(int) * pl.iters, st)) != cudaSuccess) return e;
    kmeans_init_kernel<T><<<BH, 128, 0, st>>>(v, S, H, k, pl.seed, pl.seed_H, pl.seed_b0, pl.seed_h0, pl.cent);
    ++n;
    const dim3 grid(pl.nchunks, BH);
    // pass it writes its labels to assign (even) or assign2 (odd); the sums of
    // every pass but the last feed the centroid update
    for (int it = 0; it < pl.iters; ++it) {
      uint8_t* hist_t = history ? history + (size_t)it * BH * S : nullptr;
      const bool last = it + 1 == pl.iters;
      n += launch_kmeans_pass_k<T>(grid, st, v, pl, it, last, hist_t);
      if (!last) {
        kmeans_update_kernel<<<BH, 128, 0, st>>>(k, pl.cent, pl.sums, pl.counts);
        ++n;
      }
    }
    perm_offsets_kernel<<<BH, 32, 0, st>>>(k, pl.nchunks, pl.hist, pl.offs);
    perm_scatter_kernel<<<grid, kChunk, 0, st>>>(S, k, (pl.iters - 1) & 1 ? pl.assign2 : pl.assign, pl.offs,
                                                 out.perm);
    n += 2;
  } else {
    identity_perm_kernel<<<dim3(std::max(1, std::min(1024, (S + 255) / 256)), BH), 256, 0, st>>>(S, out.perm);
    ++n;
  }
  const dim3 gb(pl.nb, BH);
  const bool naive = pl.mode == VC_MODE_NAIVE;
  if (pl.fmt == VC_RESIDUAL_E4M3_PER_CHANNEL)
    block_stats_kernel<T, true><<<gb, 128, 0, st>>>(v, S, H, out.perm, naive, out.mu, pl.amax);
  else
    block_stats_kernel<T><<<gb, 128, 0, st>>>(v, S, H, out.perm, naive, out.mu, pl.amax);
  if (pl.fmt == VC_RESIDUAL_E4M3) {
    residual_e4m3_kernel<T><<<gb, 256, 0, st>>>(v, S, H, pl.S_pad, out.perm, out.mu, pl.amax, out.v_codes,
                                                out.s_v);
  } else if (pl.fmt == VC_RESIDUAL_E4M3_PER_CHANNEL) {
    residual_e4m3_kernel<T, true><<<gb, 256, 0, st>>>(v, S, H, pl.S_pad, out.perm, out.mu, pl.amax,
                                                      out.v_codes, out.s_v);
  } else if (pl.fmt == VC_RESIDUAL_MXFP4) {
    residual_mxfp4_kernel<T><<<gb, 256, 0, st>>>(v, S, H, pl.S_pad, out.perm, out.mu, out.v_codes,
                                                 reinterpret_cast<uint32_t*>(out.v_scales), out.s_v);
  } else {
    residual_nvfp4_kernel<T><<<gb, 256, 0, st>>>(v, S, H, pl.S_pad, out.perm, out.mu, pl.amax, out.v_codes,
                                                 out.v_scales, out.s_v);
  }
  *nlaunch = n + 2;
  return cudaGetLastError();
}

cudaError_t launch_prepare_v(const void* v, int dtype, const PrepPlan& pl, const vc_prepared_v_t& out,
                             uint8_t* history, cudaStream_t st, int* nlaunch) {
  if (dtype == VC_DTYPE_BF16)
    return launch_prepare_v_t(static_cast<const __nv_bfloat16*>(v), pl, out, history, st, nlaunch);
  return launch_prepare_v_t(static_cast<const __half*>(v), pl, out, history, st, nlaunch);
}

cudaError_t launch_quant_qk(const void* q, const void* k, int dtype, int B, int S, int H, const int32_t* perm,
                            const vc_qk_fp8_t& out, unsigned long long* ksum, float* k_mean, cudaStream_t st,
                            int* nlaunch) {
  const int nb = (S + kBlock - 1) / kBlock;
  const dim3 grid(nb, B * H, 2);
  const bool bf = dtype == VC_DTYPE_BF16;
  int n = 1;
  // K smoothing: the token sums, then the means (fp32, right after the sums in
  // the same workspace)
  float* const kbar = ksum != nullptr ? reinterpret_cast<float*>(ksum + (size_t)B * H * kD) : nullptr;
  if (ksum != nullptr) {
    cudaError_t e;
    if ((e = cudaMemsetAsync(ksum, 0, sizeof(unsigned long long) * B * H * kD, st)) != cudaSuccess) return e;
    const dim3 gs((S + kSumRows - 1) / kSumRows, B * H);
    if (bf)
      token_sums_kernel<__nv_bfloat16><<<gs, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(k), S, H, ksum);
    else
      token_sums_kernel<__half><<<gs, 128, 0, st>>>(static_cast<const __half*>(k), S, H, ksum);
    kbar_kernel<<<B * H, kD, 0, st>>>(ksum, S, kbar, k_mean);
    n += 2;
  }
  auto qk = bf ? (ksum ? quant_qk_kernel<__nv_bfloat16, true> : quant_qk_kernel<__nv_bfloat16, false>)
              : nullptr;
  auto qh = bf ? nullptr : (ksum ? quant_qk_kernel<__half, true> : quant_qk_kernel<__half, false>);
  if (bf)
    qk<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), S, H,
                             nb * kBlock, perm, kbar, out.q_codes, out.q_scales, out.k_codes, out.k_scales);
  else
    qh<<<grid, 256, 0, st>>>(static_cast<const __half*>(q), static_cast<const __half*>(k), S, H, nb * kBlock, perm,
                             kbar, out.q_codes, out.q_scales, out.k_codes, out.k_scales);
  *nlaunch = n;
  return cudaGetLastError();
}

cudaError_t launch_residual_energy(const void* v, int dtype, int B, int S, int H, const int32_t* perm,
                                   const float* mu, double* energy, cudaStream_t st) {
  cudaError_t e;
  if ((e = cudaMemsetAsync(energy, 0, sizeof(double) * B * H, st)) != cudaSuccess) return e;
  const dim3 grid((S + kBlock - 1) / kBlock, B * H);
  if (dtype == VC_DTYPE_BF16)
    residual_energy_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(v), S, H, perm,
                                                                mu, energy);
  else
    residual_energy_kernel<__half><<<grid, 128, 0, st>>>(static_cast<const __half*>(v), S, H, perm, mu, energy);
  return cudaGetLastError();
}

cudaError_t launch_repair(const void* v, int dtype, int B, int S, int H, const int32_t* perm, const float* mu,
                          const unsigned int* amax_bits, uint8_t* planes, int m, float* err,
                          unsigned long long* thr, uint8_t* kept, cudaStream_t st, int* nlaunch) {
  const int nb = (S + kBlock - 1) / kBlock, S_pad = nb * kBlock, BH = B * H;
  const dim3 grid(nb, BH);
  uint8_t* plane1 = planes + (size_t)BH * kD * S_pad;
  const bool bf = dtype == VC_DTYPE_BF16;
  int n = 0;
  if (m > 0) {
    if (bf)
      repair_err_kernel<__nv_bfloat16><<<grid, 128, kTileBytes, st>>>(static_cast<const __nv_bfloat16*>(v), S, H,
                                                                      S_pad, perm, mu, amax_bits, err);
    else
      repair_err_kernel<__half><<<grid, 128, kTileBytes, st>>>(static_cast<const __half*>(v), S, H, S_pad, perm, mu,
                                                               amax_bits, err);
    repair_select_kernel<<<BH, 256, 0, st>>>(err, S, m, thr);
    n += 2;
  }
  if (bf)
    repair_plane_kernel<__nv_bfloat16><<<grid, 128, kTileBytes, st>>>(static_cast<const __nv_bfloat16*>(v), S, H,
                                                                      S_pad, perm, mu, amax_bits, err, thr, m > 0,
                                                                      plane1, kept);
  else
    repair_plane_kernel<__half><<<grid, 128, kTileBytes, st>>>(static_cast<const __half*>(v), S, H, S_pad, perm, mu,
                                                               amax_bits, err, thr, m > 0, plane1, kept);
  *nlaunch = n + 1;
  return cudaGetLastError();
}

cudaError_t prep_configure() {
  cudaError_t e;
  const struct {
    const void* f;
    size_t bytes;
  } assign_fns[] = {
      {(const void*)kmeans_assign_kernel<__nv_bfloat16, 8>, assign_smem<8>()},
      {(const void*)kmeans_assign_kernel<__nv_bfloat16, 16>, assign_smem<16>()},
      {(const void*)kmeans_assign_kernel<__nv_bfloat16, 32>, assign_smem<32>()},
      {(const void*)kmeans_assign_kernel<__half, 8>, assign_smem<8>()},
      {(const void*)kmeans_assign_kernel<__half, 16>, assign_smem<16>()},
      {(const void*)kmeans_assign_kernel<__half, 32>, assign_smem<32>()},
  };
  for (const auto& a : assign_fns)
    if ((e = cudaFuncSetAttribute(a.f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)a.bytes)) != cudaSuccess)
      return e;
  static_assert(assign_tc_smem<16>() <= 227 * 1024 && assign_tc_smem<32>() <= 227 * 1024, "shared memory per CTA");
  if ((e = cudaFuncSetAttribute(kmeans_assign_tc_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)assign_tc_smem<16>())) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(kmeans_assign_tc_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)assign_tc_smem<32>())) != cudaSuccess)
    return e;
  return cudaSuccess;
}

}  // namespace vc
