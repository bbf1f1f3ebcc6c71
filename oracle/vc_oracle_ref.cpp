// vc_oracle_ref.cpp -- the VC-Attention forward path written out plainly in C++.
//
// TEST INFRASTRUCTURE ONLY, like the numpy oracle beside it: a second, independent
// CPU statement of the same definitions (readings R1-R14 of the oracle package),
// which the tests hold bit for bit against the numpy oracle. Only tests/, the
// smoke test and the benchmark's CPU baseline may load it; it shares no code with
// the CUDA library. Plain loops, one (batch, head) slice at a time, in the order
// each step is defined; no blocking, fusion or reordering.
//
// Sources (web pages describing the method):
//   "VC-Attention: Value Smoothing and Softmax Casting for Low-bit Attention",
//     Abstract: V-Smooth (clustering, block means, residual quantisation) and
//     ExpCast-FP8 (log-domain scores to E4M3 codes with one fused multiply-add,
//     the mean restored from the online softmax's row sum).
//   "Hugging Face Introduces VC-Attention", section "Technical Breakthroughs and
//     Core Innovations": the same two steps.
//   "Nunchux AI lanza VC-Attention kernel", second paragraph: k-means per batch
//     and head, 128-token block means, E4M3 or NVFP4 residual.
//   "Open VC Attention", section "Описание": Q/K scales per block, V per head.
//
// Build: g++ -O2 -ffp-contract=off -shared -fPIC (no fused multiply-add: every
// fp32 operation is rounded on its own, as the definitions state).
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <vector>

namespace {

const int kBlock = 128;              // 128-token blocks
const double kE4M3Max = 448.0;
const double kE2M1Max = 6.0;
const double kLog2e = 1.4426950408889634;   // nearest double to log2(e)
const float kTinyAmax = 7.888609052210118e-31f;  // 2^-100 (R10)
const int kFixShift = 24;            // fixed-point sums of x * 2^24 (R2, R4)
const uint64_t kGolden = 0x9E3779B97F4A7C15ull;

int num_blocks(int S) { return (S + kBlock - 1) / kBlock; }

// E4M3FN value of a code (0..255): sign, 4 exponent bits (bias 7), 3 mantissa
// bits; exponent field 0 is subnormal (m 2^-9); S.1111.111 is NaN.
double e4m3_value(int code) {
  const double sign = (code & 0x80) ? -1.0 : 1.0;
  const int e = (code >> 3) & 0xF, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) return sign * m * ldexp(1.0, -9);
  return sign * (1.0 + m / 8.0) * ldexp(1.0, e - 7);
}

// fp32 -> E4M3 code: round the magnitude to 3 mantissa bits in its binade (the
// binade floored at the normal minimum 2^-6), ties to even, saturate at 448; the
// code of the rounded magnitude is found by walking the increasing codes 0..126.
uint8_t e4m3_code(float x) {
  if (isnan(x)) return (uint8_t)(signbit(x) ? 0xFF : 0x7F);
  const double a = fabs((double)x);
  double mag;
  if (a == 0.0) {
    mag = 0.0;
  } else if (isinf(a)) {
    mag = kE4M3Max;
  } else {
    int E;
    frexp(a, &E);                        // a = f 2^E, f in [0.5, 1)
    int e = E - 1;
    if (e < -6) e = -6;
    const double quantum = ldexp(1.0, e - 3);
    mag = nearbyint(a / quantum) * quantum;   // the default rounding: ties to even
    if (mag > kE4M3Max) mag = kE4M3Max;
  }
  int code = 0;
  while (code < 126 && e4m3_value(code) < mag) ++code;
  return (uint8_t)(signbit(x) ? (code | 0x80) : code);
}

const double kE2M1Values[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

// fp32 -> E2M1 code (bit 3 the sign): 1 mantissa bit, exponent bias 1 (smallest
// binade [1, 2), below it steps of 0.5), ties to even, saturate at 6.
uint8_t e2m1_code(float x) {
  const double a = fabs((double)x);
  double mag;
  if (isnan(x) || isinf(a)) {
    mag = kE2M1Max;
  } else if (a == 0.0) {
    mag = 0.0;
  } else {
    int E;
    frexp(a, &E);
    int e = E - 1;
    if (e < 0) e = 0;
    const double quantum = ldexp(1.0, e - 1);
    mag = nearbyint(a / quantum) * quantum;
    if (mag > kE2M1Max) mag = kE2M1Max;
  }
  int code = 0;
  while (code < 7 && kE2M1Values[code] < mag) ++code;
  return (uint8_t)(signbit(x) ? (code | 8) : code);
}

// splitmix64 (Steele, Lea and Flood, OOPSLA 2014)
struct SplitMix {
  uint64_t state;
  uint64_t next() {
    state += kGolden;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
};

int64_t fix(float x) { return llrint((double)x * ldexp(1.0, kFixShift)); }   // ties to even

}  // namespace

extern "C" {

int orc_version(void) { return 1; }

void orc_e4m3_round(const float* x, long n, uint8_t* out) {
  for (long i = 0; i < n; ++i) out[i] = e4m3_code(x[i]);
}

void orc_e2m1_round(const float* x, long n, uint8_t* out) {
  for (long i = 0; i < n; ++i) out[i] = e2m1_code(x[i]);
}

// R1: k token indices of slice bh, drawn with splitmix64 from
// seed ^ (golden * (bh + 1)); a draw that repeats an earlier index is drawn again
// unless every index is already taken.
void orc_kmeans_init(int S, int k, uint64_t seed, long bh, int* idx) {
  SplitMix rng{seed ^ (kGolden * (uint64_t)(bh + 1))};
  int n = 0;
  std::vector<char> taken(S, 0);
  int distinct = 0;
  while (n < k) {
    const int u = (int)(rng.next() % (uint64_t)S);
    if (taken[u] && distinct < S) continue;
    if (!taken[u]) {
      taken[u] = 1;
      ++distinct;
    }
    idx[n++] = u;
  }
}

// R2: Lloyd passes over X (S x D, fp32). Each pass assigns every token to the
// centroid at the smallest fp64 squared distance (first index on ties); between
// passes a centroid becomes its members' mean (int64 sum of x 2^24, one fp64
// division, rounded to fp32; an empty cluster keeps its centroid). history[t*S+j]
// is pass t's label of token j; cent holds the centroids of the last pass.
void orc_kmeans_lloyd(const float* X, int S, int D, int k, int iters, uint64_t seed, long bh, int* assign,
                      float* cent, int* history) {
  std::vector<int> idx(k);
  orc_kmeans_init(S, k, seed, bh, idx.data());
  for (int c = 0; c < k; ++c)
    for (int d = 0; d < D; ++d) cent[c * D + d] = X[(size_t)idx[c] * D + d];
  std::vector<int64_t> sums((size_t)k * D);
  std::vector<int64_t> count(k);
  for (int t = 0; t < iters; ++t) {
    for (int j = 0; j < S; ++j) {
      int best = 0;
      double bd = 0.0;
      for (int c = 0; c < k; ++c) {
        double dist = 0.0;
        for (int d = 0; d < D; ++d) {
          const double df = (double)X[(size_t)j * D + d] - (double)cent[c * D + d];
          dist += df * df;
        }
        if (c == 0 || dist < bd) {
          bd = dist;
          best = c;
        }
      }
      assign[j] = best;
      history[(size_t)t * S + j] = best;
    }
    if (t == iters - 1) break;
    memset(sums.data(), 0, sums.size() * sizeof(int64_t));
    memset(count.data(), 0, count.size() * sizeof(int64_t));
    for (int j = 0; j < S; ++j) {
      ++count[assign[j]];
      for (int d = 0; d < D; ++d) sums[(size_t)assign[j] * D + d] += fix(X[(size_t)j * D + d]);
    }
    for (int c = 0; c < k; ++c) {
      if (count[c] == 0) continue;
      for (int d = 0; d < D; ++d)
        cent[c * D + d] = (float)(((double)sums[(size_t)c * D + d] * ldexp(1.0, -kFixShift)) / (double)count[c]);
    }
  }
}

// R3: stable order of the tokens by cluster: perm[p] is the original index of the
// token at permuted position p (a counting sort, ties in original order).
void orc_cluster_perm(const int* assign, int S, int k, int* perm) {
  std::vector<int> start(k + 1, 0);
  for (int j = 0; j < S; ++j) ++start[assign[j] + 1];
  for (int c = 0; c < k; ++c) start[c + 1] += start[c];
  for (int j = 0; j < S; ++j) perm[start[assign[j]]++] = j;
}

// R4: mean of each 128-token block in permuted order over its valid tokens.
void orc_block_means(const float* X, int S, int D, const int* perm, float* mu) {
  const int nb = num_blocks(S);
  for (int b = 0; b < nb; ++b) {
    const int p0 = b * kBlock, p1 = p0 + kBlock < S ? p0 + kBlock : S;
    for (int d = 0; d < D; ++d) {
      int64_t s = 0;
      for (int p = p0; p < p1; ++p) s += fix(X[(size_t)perm[p] * D + d]);
      mu[b * D + d] = (float)(((double)s * ldexp(1.0, -kFixShift)) / (double)(p1 - p0));
    }
  }
}

// The residual of permuted token p, channel d: fl32(x - mu_block).
static float residual(const float* X, int D, const int* perm, const float* mu, int p, int d) {
  return X[(size_t)perm[p] * D + d] - mu[(p / kBlock) * D + d];
}

// R5: E4M3 residual with one scale per slice. vt is V^T (D x S_pad) with zero
// padding; s_v = fl32(amax / 448), codes E4M3(fl32(r * fl32(448 / amax))).
void orc_residual_e4m3(const float* X, int S, int D, const int* perm, const float* mu, uint8_t* vt, float* s_v,
                       float* amax_out) {
  const int Sp = num_blocks(S) * kBlock;
  memset(vt, 0, (size_t)D * Sp);
  float amax = 0.0f;
  for (int p = 0; p < S; ++p)
    for (int d = 0; d < D; ++d) {
      const float a = fabsf(residual(X, D, perm, mu, p, d));
      if (a > amax) amax = a;
    }
  *amax_out = amax;
  if (!(amax >= kTinyAmax)) {
    *s_v = 1.0f;
    return;
  }
  const float inv = (float)kE4M3Max / amax;
  *s_v = amax / (float)kE4M3Max;
  for (int p = 0; p < S; ++p)
    for (int d = 0; d < D; ++d) vt[(size_t)d * Sp + p] = e4m3_code(residual(X, D, perm, mu, p, d) * inv);
}

// R6: NVFP4 residual. g = fl32(amax / 2688); per channel and group of 16
// permuted tokens an E4M3 scale E4M3(fl32(fl32(gmax / 6) / g)); codes
// E2M1(fl32(r / fl32(dec(scale) g))), 0 where the scale decodes to 0; packed
// two per byte, the even token in the low nibble.
void orc_residual_nvfp4(const float* X, int S, int D, const int* perm, const float* mu, uint8_t* packed,
                        uint8_t* scales, float* g_out, float* amax_out) {
  const int Sp = num_blocks(S) * kBlock, ng = Sp / 16;
  memset(packed, 0, (size_t)D * Sp / 2);
  memset(scales, 0, (size_t)D * ng);
  float amax = 0.0f;
  for (int p = 0; p < S; ++p)
    for (int d = 0; d < D; ++d) {
      const float a = fabsf(residual(X, D, perm, mu, p, d));
      if (a > amax) amax = a;
    }
  *amax_out = amax;
  if (!(amax >= kTinyAmax)) {
    *g_out = 1.0f;
    return;
  }
  const float g = amax / (float)(kE4M3Max * kE2M1Max);
  *g_out = g;
  for (int d = 0; d < D; ++d)
    for (int q = 0; q < ng; ++q) {
      float gmax = 0.0f;
      for (int i = 0; i < 16; ++i) {
        const int p = q * 16 + i;
        if (p < S) {
          const float a = fabsf(residual(X, D, perm, mu, p, d));
          if (a > gmax) gmax = a;
        }
      }
      const uint8_t sc = e4m3_code((gmax / (float)kE2M1Max) / g);
      scales[(size_t)d * ng + q] = sc;
      const float sdec = (float)e4m3_value(sc);
      const float den = sdec * g;
      for (int i = 0; i < 16; ++i) {
        const int p = q * 16 + i;
        const float r = p < S ? residual(X, D, perm, mu, p, d) : 0.0f;
        const uint8_t code = sdec == 0.0f ? 0 : e2m1_code(r / den);
        packed[(size_t)d * (Sp / 2) + p / 2] |= (uint8_t)((p & 1) ? code << 4 : code);
      }
    }
}

// R14: E4M3 residual with one scale per channel: s_v[d] = fl32(amax_d / 448), codes
// E4M3(fl32(r fl32(448 / amax_d))); a channel below 2^-100 keeps scale 1, codes 0.
void orc_residual_e4m3_per_channel(const float* X, int S, int D, const int* perm, const float* mu, uint8_t* vt,
                                   float* s_v, float* amax) {
  const int Sp = num_blocks(S) * kBlock;
  memset(vt, 0, (size_t)D * Sp);
  for (int d = 0; d < D; ++d) {
    float a = 0.0f;
    for (int p = 0; p < S; ++p) {
      const float v = fabsf(residual(X, D, perm, mu, p, d));
      if (v > a) a = v;
    }
    amax[d] = a;
    s_v[d] = 1.0f;
    if (!(a >= kTinyAmax)) continue;
    const float inv = (float)kE4M3Max / a;
    s_v[d] = a / (float)kE4M3Max;
    for (int p = 0; p < S; ++p) vt[(size_t)d * Sp + p] = e4m3_code(residual(X, D, perm, mu, p, d) * inv);
  }
}

// R13: the exponent of an MX group: the smallest integer e with amax <= 6 2^e,
// clamped to [-127, 127]; -127 for an all-zero group.
int orc_mx_exponent(double amax) {
  if (!(amax > 0.0)) return -127;
  int e = -127;
  while (e < 127 && kE2M1Max * ldexp(1.0, e) < amax) ++e;
  return e;
}

// R13: MX-style FP4 residual: per channel and group of 32 permuted tokens the
// exponent e of the group's amax, codes E2M1(fl32(r / 2^e)) (exact division by a
// power of two); codes (D x S_pad) one per byte, exponents (D x S_pad/32) as e + 127.
void orc_residual_mxfp4(const float* X, int S, int D, const int* perm, const float* mu, uint8_t* codes,
                        uint8_t* e8) {
  const int Sp = num_blocks(S) * kBlock, ng = Sp / 32;
  memset(codes, 0, (size_t)D * Sp);
  for (int d = 0; d < D; ++d)
    for (int q = 0; q < ng; ++q) {
      double gmax = 0.0;
      for (int i = 0; i < 32; ++i) {
        const int p = q * 32 + i;
        if (p < S) {
          const double a = fabs((double)residual(X, D, perm, mu, p, d));
          if (a > gmax) gmax = a;
        }
      }
      const int e = orc_mx_exponent(gmax);
      e8[(size_t)d * ng + q] = (uint8_t)(e + 127);
      for (int i = 0; i < 32; ++i) {
        const int p = q * 32 + i;
        const double r = p < S ? (double)residual(X, D, perm, mu, p, d) : 0.0;
        codes[(size_t)d * Sp + p] = e2m1_code((float)(r / ldexp(1.0, e)));
      }
    }
}

// R12: the repair planes of an E4M3 residual. Plane 0 is the residual's codes
// (R5); for the ceil(budget S) tokens with the largest error, plane 1 holds the
// E4M3 codes of each element's rounding error in code units, dlt = fl32(y -
// dec(code)) with y = fl32(r fl32(448 / amax)); a token's error is the fp32 sum
// of fl32(dlt^2) over the channels from d = 0; ties go to the lower position.
// pos receives the kept positions in ascending order; returns their number.
int orc_residual_repair_planes(const float* X, int S, int D, const int* perm, const float* mu, double budget,
                               uint8_t* vt, uint8_t* lo, float* s_v, int* pos) {
  const int Sp = num_blocks(S) * kBlock;
  float amax = 0.0f;
  orc_residual_e4m3(X, S, D, perm, mu, vt, s_v, &amax);
  memset(lo, 0, (size_t)D * Sp);
  double mm = ceil(budget * (double)S);
  const int m = mm < (double)S ? (int)mm : S;
  std::vector<float> err(S, 0.0f);
  std::vector<float> dlt((size_t)S * D, 0.0f);
  if (amax >= kTinyAmax) {
    const float inv = (float)kE4M3Max / amax;
    for (int p = 0; p < S; ++p) {
      float e = 0.0f;
      for (int d = 0; d < D; ++d) {
        const float y = residual(X, D, perm, mu, p, d) * inv;
        const float dl = y - (float)e4m3_value(vt[(size_t)d * Sp + p]);
        dlt[(size_t)p * D + d] = dl;
        e = e + dl * dl;
      }
      err[p] = e;
    }
  }
  std::vector<int> order(S);
  for (int p = 0; p < S; ++p) order[p] = p;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return err[a] > err[b]; });
  std::sort(order.begin(), order.begin() + m);
  for (int i = 0; i < m; ++i) {
    const int p = order[i];
    pos[i] = p;
    for (int d = 0; d < D; ++d) lo[(size_t)d * Sp + p] = e4m3_code(dlt[(size_t)p * D + d]);
  }
  return m;
}

// Residual energy of one slice: sum over permuted positions p of
// ||x[perm[p]] - mu[p / 128]||^2 in fp64.
double orc_residual_energy(const float* X, int S, int D, const int* perm, const float* mu) {
  double e = 0.0;
  for (int p = 0; p < S; ++p)
    for (int d = 0; d < D; ++d) {
      const double r = (double)X[(size_t)perm[p] * D + d] - (double)mu[(p / kBlock) * D + d];
      e += r * r;
    }
  return e;
}

// Decoded E4M3 residual (S x D, fp64, permuted order): s_v dec(code).
void orc_vres_from_e4m3(const uint8_t* vt, int S_pad, int S, int D, float s_v, double* vres) {
  for (int p = 0; p < S; ++p)
    for (int d = 0; d < D; ++d) vres[(size_t)p * D + d] = (double)s_v * e4m3_value(vt[(size_t)d * S_pad + p]);
}

// R7: per 128-token block scale fl32(amax / 448) and codes E4M3(fl32(x fl32(448 /
// amax))), rows taken in `order` (K: the permutation) or as given (Q: NULL);
// codes (S_pad x D) with zero padding; a block below 2^-100 keeps scale 1, codes 0.
void orc_quant_blocks_e4m3(const float* X, int S, int D, const int* order, uint8_t* codes, float* scales) {
  const int nb = num_blocks(S);
  memset(codes, 0, (size_t)nb * kBlock * D);
  for (int b = 0; b < nb; ++b) {
    const int p0 = b * kBlock, p1 = p0 + kBlock < S ? p0 + kBlock : S;
    float amax = 0.0f;
    for (int p = p0; p < p1; ++p)
      for (int d = 0; d < D; ++d) {
        const float a = fabsf(X[(size_t)(order ? order[p] : p) * D + d]);
        if (a > amax) amax = a;
      }
    scales[b] = 1.0f;
    if (!(amax >= kTinyAmax)) continue;
    const float inv = (float)kE4M3Max / amax;
    scales[b] = amax / (float)kE4M3Max;
    for (int p = p0; p < p1; ++p)
      for (int d = 0; d < D; ++d) codes[(size_t)p * D + d] = e4m3_code(X[(size_t)(order ? order[p] : p) * D + d] * inv);
  }
}

// R11: the per-channel token mean of one slice (int64 sum of llrint(x 2^24), one
// fp64 division, rounded to fp32) and K - kbar in fp32 (xs: S x D, written).
void orc_smooth_k(const float* K, int S, int D, float* kbar, float* xs) {
  for (int d = 0; d < D; ++d) {
    int64_t s = 0;
    for (int j = 0; j < S; ++j) s += fix(K[(size_t)j * D + d]);
    kbar[d] = (float)(((double)s * ldexp(1.0, -kFixShift)) / (double)S);
  }
  for (int j = 0; j < S; ++j)
    for (int d = 0; d < D; ++d) xs[(size_t)j * D + d] = K[(size_t)j * D + d] - kbar[d];
}

// R8: kappa = fl32(softmax_scale log2 e).
float orc_softmax_kappa(float softmax_scale) { return (float)((double)softmax_scale * kLog2e); }

// VC-Attention output of query rows `rows` of one slice (R8, R9): scores
// t = fl32(sum_d dec(q) dec(k)) (the fp64 sum is exact: products of 4-bit
// significands), multipliers c = fl32(fl32(sQ sK) kappa); blocks of 128 keys in
// permuted order, each cast in the running integer frame F = max(F, ceil(max_j
// fl32(c t))) as code = clip(56 + 8 k_P - 8F + rne(8 c t), 0, 126) (8 c t exact
// in fp64); P = dec(code) 2^(F_block - F_final); O = (sum_j P_j v~_j + sum_b r_b
// mu_b) / l with r_b the block row sums and l their total. Outputs O (nrows x D),
// the codes (nrows x S) and l, all in fp64.
void orc_vc_attention_rows(const uint8_t* q_codes, const float* q_scales, const uint8_t* k_codes,
                           const float* k_scales, const double* vres, const float* mu, int S, int D, const int* rows,
                           int nrows, float softmax_scale, int k_p, double* O, uint8_t* codes, double* l_out) {
  const int nb = num_blocks(S);
  const float kappa = orc_softmax_kappa(softmax_scale);
  const double bias = 56.0 + 8.0 * k_p;
  std::vector<float> t(S), c(S);
  std::vector<double> frame(nb), P(S), r(nb);
  for (int ri = 0; ri < nrows; ++ri) {
    const int i = rows[ri];
    const float sq = q_scales[i / kBlock];
    for (int j = 0; j < S; ++j) {
      double acc = 0.0;
      for (int d = 0; d < D; ++d)
        acc += e4m3_value(q_codes[(size_t)i * D + d]) * e4m3_value(k_codes[(size_t)j * D + d]);
      t[j] = (float)acc;
      c[j] = (sq * k_scales[j / kBlock]) * kappa;
    }
    double F = 0.0;
    for (int b = 0; b < nb; ++b) {
      const int j0 = b * kBlock, j1 = j0 + kBlock < S ? j0 + kBlock : S;
      float umax = c[j0] * t[j0];
      for (int j = j0 + 1; j < j1; ++j) {
        const float u = c[j] * t[j];
        if (u > umax) umax = u;
      }
      const double Fb = ceil((double)umax);
      F = (b == 0 || Fb > F) ? Fb : F;
      frame[b] = F;
      for (int j = j0; j < j1; ++j) {
        double code = (bias - 8.0 * F) + nearbyint(8.0 * (double)c[j] * (double)t[j]);
        if (code < 0.0) code = 0.0;
        if (code > 126.0) code = 126.0;
        codes[(size_t)ri * S + j] = (uint8_t)code;
      }
    }
    double l = 0.0;
    for (int b = 0; b < nb; ++b) {
      const int j0 = b * kBlock, j1 = j0 + kBlock < S ? j0 + kBlock : S;
      const double scale = ldexp(1.0, (int)(frame[b] - F));
      r[b] = 0.0;
      for (int j = j0; j < j1; ++j) {
        P[j] = e4m3_value(codes[(size_t)ri * S + j]) * scale;
        r[b] += P[j];
      }
      l += r[b];
    }
    for (int d = 0; d < D; ++d) {
      double o = 0.0;
      for (int j = 0; j < S; ++j) o += P[j] * vres[(size_t)j * D + d];
      for (int b = 0; b < nb; ++b) o += r[b] * (double)mu[b * D + d];
      O[(size_t)ri * D + d] = o / l;
    }
    l_out[ri] = l;
  }
}

// softmax(Q K^T scale) V in fp64 from the unquantised inputs, for query rows `rows`
// (the scale in fp64 as given).
void orc_exact_attention_rows(const float* Q, const float* K, const float* V, int S, int D, const int* rows,
                              int nrows, double softmax_scale, double* O) {
  std::vector<double> s(S);
  for (int ri = 0; ri < nrows; ++ri) {
    const int i = rows[ri];
    double smax = -INFINITY;
    for (int j = 0; j < S; ++j) {
      double acc = 0.0;
      for (int d = 0; d < D; ++d) acc += (double)Q[(size_t)i * D + d] * (double)K[(size_t)j * D + d];
      s[j] = acc * softmax_scale;
      if (s[j] > smax) smax = s[j];
    }
    double l = 0.0;
    for (int j = 0; j < S; ++j) {
      s[j] = exp(s[j] - smax);
      l += s[j];
    }
    for (int d = 0; d < D; ++d) {
      double o = 0.0;
      for (int j = 0; j < S; ++j) o += s[j] * (double)V[(size_t)j * D + d];
      O[(size_t)ri * D + d] = o / l;
    }
  }
}

}  // extern "C"
