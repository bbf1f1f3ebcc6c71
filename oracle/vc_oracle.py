"""VC-Attention forward path written out plainly on the CPU (numpy, fp64).

TEST INFRASTRUCTURE ONLY. This module is the oracle the CUDA path is checked
against. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
``cpu_baseline`` / ``--impl reference`` legs may import it. It shares no code with
the CUDA library and imports nothing from it. It is slow on purpose: every step is
the plain definition, one (batch, head) slice at a time, with no blocking, fusion
or reordering beyond what the step itself states.

Sources (web pages describing the method) cited below as:
  [ABS] "VC-Attention: Value Smoothing and Softmax Casting for Low-bit Attention"
        (arXiv 2609.15810), Abstract.
  [HF]  "Hugging Face Introduces VC-Attention: Breakthrough Optimization for
        Low-bit Attention Mechanisms", section "Technical Breakthroughs and Core
        Innovations" (V-Smooth and ExpCast-FP8 bullets).
  [OVC] "Open VC Attention" (catalogue card), section "Описание" (description):
        FP16/BF16 [S,H,128] / [B,S,H,128] in, BF16 out; Q/K scales per block,
        V scales per head.
  [NUN] "Nunchux AI lanza VC-Attention kernel para acelerar generacion de video"
        (news summary), second paragraph: k-means per (batch, head), 128-token
        block means, E4M3 or NVFP4 residual.

Readings taken where the pages are silent (R-numbers are used in comments):
  R1  k-means init: k distinct token indices drawn per (b, h) with splitmix64
      seeded by ``seed ^ (0x9E3779B97F4A7C15 * (b*H + h + 1))``; u = next() mod S,
      redrawn while it repeats (duplicates allowed only once all S are taken).
  R2  Lloyd: ``iters`` assignment passes; distance = sum_d (x_d - c_d)^2 in fp64;
      ties go to the lowest cluster index; between passes the centroid is
      (float)(((double) sum_j llrint(x_j * 2^24)) * 2^-24 / n); an empty cluster
      keeps its centroid; the last pass's assignment is final.
  R3  Permutation: stable sort of token indices by final cluster id, ascending;
      K is permuted with V; Q is not.
  R4  Block means over the valid (<= 128) permuted tokens of each block, with the
      same int64 fixed-point sum as R2.
  R5  Residual scale per (b, h) (Open-VC's "V per head"); E4M3 is OCP E4M3FN,
      round-to-nearest-even, saturating to +-448.
  R6  NVFP4 residual: fp32 global g = amax / 2688 per (b, h); one E4M3 scale per
      16 consecutive permuted tokens of one channel; E2M1 codes, RNE, saturating.
  R7  Q/K: one scale per 128-token block (Q in original order, K in permuted
      order); softmax scale enters the score multiplier, not the codes.
  R8  ExpCast: log2-domain score u = c_j * t_ij with c_j = fl32(fl32(sQ*sK) *
      kappa), kappa = fl32(softmax_scale * log2 e); the online softmax visits the
      128-key blocks in permuted order and keeps an integer running frame per row,
      F_i(b) = max(F_i(b-1), ceil(max_{j in block b} fl32(u_ij))), F_i(0) from
      block 0 alone; the keys of block b are cast in the frame current after
      block b: code = clip(B - 8 F_i(b) + rne(8 c_j t_ij), 0, 126),
      B = 56 + 8 k_P (k_P = 8 by default: P is carried scaled by 2^8); when the
      frame moves, what was accumulated so far is multiplied by the exact power
      of two 2^(F_old - F_new), so key j carries dec(code_ij) 2^(F_i(b) - F_i(nb-1)).
      ([ABS]: the mean is restored from the row sum "the online softmax already
      maintains" -- the cast happens inside that online pass.) Where the frame
      never moves this is the single-frame cast with M_i = ceil(max_j fl32(u_ij)).
  R9  Row sum and block restore use the cast P (the E4M3 values the PV product
      uses); O = (sum_j P_ij v~_j + sum_b r_ib mu_b) / l_i, then BF16 RNE.
  R10 A block (or head) whose amax is below 2^-100 is treated as all zero:
      scale 1, codes 0.
  R11 Optional K smoothing ([ABS]: prior work smooths queries and keys; the
      pages give no form): K minus its per-channel mean over all tokens of the
      (b, h) slice, the mean an int64 fixed-point sum as in R4, the difference
      taken in fp32, before the per-block quantisation of R7. Every score of a
      query row moves by the same q.kbar, so the softmax is unchanged. Q is not
      smoothed (its mean would shift each key's score differently).
  R12 Optional V residual repair ([OVC]: re-adds the quantisation residual of
      the worst-rounded value tokens, with a budget such as 0.005): for an E4M3
      residual, the ceil(budget * S) tokens of the slice whose decoded value
      s_V dec(code) is farthest from the residual r it codes (squared L2 over
      the channels, fp64; ties to the lower permuted position) get their error
      r - s_V dec(code) back, stored in fp32. The probabilities are untouched:
      only those tokens' values in the P V product change.
  R13 MX-style FP4 residual (not described by the pages; the block-scaled FP4
      operand form of the B200 tensor cores, a neighbour of the NVFP4 residual):
      E2M1 codes with one power-of-two scale per 32 consecutive permuted tokens
      of one channel, X = 2^e with e the smallest integer for which the group's
      amax <= 6 * 2^e (so nothing clips; the OCP MX rule 2^(floor(log2 amax) - 2)
      can clip a group's largest values by up to a quarter), e clamped to
      [-127, 127] (an 8-bit biased exponent), codes E2M1(r / X) with RNE; an
      all-zero group has e = -127 and codes 0. No per-head scale.
  R14 Optional per-channel residual scale (an accuracy knob beside [OVC]'s
      per-head V scale): s_V[d] = amax_d / 448 over the slice's
      residual in channel d, codes E4M3(r * fl32(448 / amax_d)); a channel with
      amax_d below 2^-100 gets scale 1 and codes 0 (R10).
"""
import math

import numpy as np

D_HEAD = 128
BLOCK = 128                 # [NUN]: 128-token blocks (also the MMA tile)
NVFP4_GROUP = 16            # R6: one E4M3 scale per 16 elements
E4M3_MAX = 448.0
E2M1_MAX = 6.0
LOG2E = 1.4426950408889634  # nearest double to log2(e)
TINY_AMAX = 2.0 ** -100     # R10
FIX_SHIFT = 24              # R2/R4: fixed-point sums of x * 2^24
MASK64 = (1 << 64) - 1
GOLDEN64 = 0x9E3779B97F4A7C15
K_P_DEFAULT = 8

__all__ = [
    "D_HEAD", "BLOCK", "NVFP4_GROUP", "E4M3_MAX", "LOG2E", "K_P_DEFAULT",
    "e4m3_table", "e4m3_round", "e2m1_table", "e2m1_round", "bf16_round",
    "SplitMix64", "kmeans_init_indices", "kmeans_lloyd", "centroid_update",
    "cluster_permutation", "block_means", "residual_e4m3", "residual_nvfp4",
    "vres_from_e4m3", "vres_from_nvfp4", "quant_blocks_e4m3", "softmax_kappa",
    "expcast_codes", "expcast_bias", "expcast_online_probs", "vc_attention_rows", "vc_attention_exact_prob",
    "exact_attention_rows", "naive_v_e4m3", "prepare_v_head", "quant_qk_head",
    "padded_len", "num_blocks", "residual_energy", "token_mean", "smooth_k", "residual_repair",
    "residual_repair_planes", "mx_exponent", "residual_mxfp4", "vres_from_mxfp4", "residual_e4m3_per_channel",
    "vres_from_e4m3_per_channel",
]


def num_blocks(S):
    return (S + BLOCK - 1) // BLOCK


def padded_len(S):
    return num_blocks(S) * BLOCK


# ----------------------------------------------------------------- formats
def e4m3_table():
    """float64 value of every E4M3 code 0..255 (NaN at 0x7F and 0xFF).

    OCP FP8 E4M3FN: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent
    field 0 is subnormal (m * 2^-9); no infinities; S.1111.111 is NaN. [NUN] and
    [ABS] name E4M3 for both the residual and the probability codes.
    """
    vals = np.empty(256, np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 15 and m == 7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * m * 2.0 ** -9
        else:
            vals[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_E4M3 = e4m3_table()
_E4M3_POS = _E4M3[:127]     # codes 0..126: strictly increasing 0 .. 448


def e4m3_round(x):
    """fp32 -> E4M3 code, round to nearest even, saturate to +-448 (R5).

    The sign bit is copied (so -0 and negative values that round to zero give
    0x80); NaN gives 0x7F with the sign bit of the input.
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    with np.errstate(all="ignore"):
        _, E = np.frexp(a)                       # a = f * 2^E, f in [0.5, 1)
        e = np.maximum(E - 1, -6)                # binade, floored at the normal minimum
        quantum = np.ldexp(1.0, e - 3)           # 3 mantissa bits
        q = np.rint(a / quantum)                 # ties to even
        mag = np.minimum(q * quantum, E4M3_MAX)  # satfinite (inf -> 448 too)
    mag = np.where(np.isnan(a), 0.0, mag)
    code = np.searchsorted(_E4M3_POS, mag).astype(np.uint16)
    assert np.all(_E4M3_POS[np.minimum(code, 126)] == mag), "E4M3 encode off-grid"
    code = np.where(np.isnan(x), 0x7F, code)
    code = np.where(np.signbit(x), code | 0x80, code)
    return code.astype(np.uint8)


E2M1_VALUES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def e2m1_table():
    """float64 value of the 16 E2M1 codes (bit 3 is the sign) [NUN: NVFP4]."""
    vals = np.array(E2M1_VALUES + tuple(-v for v in E2M1_VALUES), np.float64)
    vals[8] = -0.0
    return vals


def e2m1_round(x):
    """fp32 -> E2M1 code (0..15), round to nearest even, saturate to +-6 (R6)."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    with np.errstate(all="ignore"):
        _, E = np.frexp(a)
        e = np.maximum(E - 1, 0)                 # exponent bias 1: smallest binade [1, 2)
        quantum = np.ldexp(1.0, e - 1)           # 1 mantissa bit
        q = np.rint(a / quantum)
        mag = np.minimum(q * quantum, E2M1_MAX)
    mag = np.where(np.isnan(a), E2M1_MAX, mag)
    code = np.searchsorted(np.array(E2M1_VALUES), mag).astype(np.uint8)
    code = np.where(np.signbit(x), code | 0x8, code)
    return code.astype(np.uint8)


def bf16_round(x):
    """float64 -> nearest bfloat16 (ties to even), returned as float64 values."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)   # fp64 -> fp32 RNE
    b = f.view(np.uint32).astype(np.uint64)
    # RNE on the low 16 bits of the fp32 pattern (fp32 -> bf16 is the top half)
    lsb = (b >> 16) & 1
    b = (b + 0x7FFF + lsb) & 0xFFFF0000
    out = b.astype(np.uint32).view(np.float32).astype(np.float64)
    return np.where(np.isnan(f), np.nan, out)


# ------------------------------------------------------------ k-means (A2)
class SplitMix64:
    """splitmix64 (Steele, Lea & Flood, OOPSLA 2014), used only for R1."""

    def __init__(self, state):
        self.state = state & MASK64

    def next(self):
        self.state = (self.state + GOLDEN64) & MASK64
        z = self.state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        return z ^ (z >> 31)


def kmeans_init_indices(S, k, seed, bh):
    """R1: k token indices for slice bh = b*H + h ([NUN]: k-means per batch and head)."""
    rng = SplitMix64((seed ^ ((GOLDEN64 * (bh + 1)) & MASK64)) & MASK64)
    chosen = []
    while len(chosen) < k:
        u = rng.next() % S
        if u in chosen and len(set(chosen)) < S:
            continue
        chosen.append(u)
    return chosen


def _sq_distances(X64, C64, chunk=8192):
    """fp64 sum_d (x_d - c_d)^2 for every token and centroid (R2)."""
    S = X64.shape[0]
    out = np.empty((S, C64.shape[0]), np.float64)
    for s0 in range(0, S, chunk):
        diff = X64[s0:s0 + chunk, None, :] - C64[None, :, :]
        out[s0:s0 + chunk] = np.einsum("skd,skd->sk", diff, diff)
    return out


def centroid_update(Xfix, a, C_old, k):
    """R2 update: fixed-point member sums, one fp64 division, rounded to fp32."""
    C = C_old.copy()
    for c in range(k):
        members = a == c
        n = int(members.sum())
        if n == 0:
            continue                                   # empty cluster keeps its centroid
        s = Xfix[members].sum(axis=0)                  # exact int64
        assert np.all(np.abs(s) < 2 ** 53)
        C[c] = ((s.astype(np.float64) * 2.0 ** -FIX_SHIFT) / n).astype(np.float32)
    return C


def kmeans_lloyd(X, k, iters, seed, bh, adopt=None, near_tie_rel=1e-6):
    """Online k-means over one slice's value tokens ([ABS] "lightweight online
    clustering"; [NUN] k-means per batch and head), per R1/R2.

    X: (S, D) float32 values (the BF16/FP16 inputs, exactly).
    adopt: optional list of per-pass assignments from another implementation.
      Where it disagrees with this oracle and the oracle's relative distance gap
      (d_other - d_best) / d_best is below ``near_tie_rel``, the other choice is
      adopted and counted as a near tie; any other disagreement is counted as a
      mismatch and the oracle keeps its own choice.
    Returns (final assignment, final centroids, per-pass assignments, stats).
    """
    X = np.asarray(X, np.float32)
    S = X.shape[0]
    X64 = X.astype(np.float64)
    Xfix = np.rint(X64 * 2.0 ** FIX_SHIFT).astype(np.int64)
    C = X[kmeans_init_indices(S, k, seed, bh)].astype(np.float32)
    history = []
    stats = {"near_ties": 0, "mismatches": 0}
    a = None
    for t in range(iters):
        dist = _sq_distances(X64, C.astype(np.float64))
        a = np.argmin(dist, axis=1).astype(np.int64)   # first minimum = lowest index
        if adopt is not None:
            g = np.asarray(adopt[t]).astype(np.int64)
            for j in np.nonzero(g != a)[0]:
                d_best = dist[j, a[j]]
                d_other = dist[j, g[j]] if 0 <= g[j] < k else np.inf
                gap = (d_other - d_best) / d_best if d_best > 0 else (0.0 if d_other == 0 else np.inf)
                if gap < near_tie_rel:
                    a[j] = g[j]
                    stats["near_ties"] += 1
                else:
                    stats["mismatches"] += 1
        history.append(a.copy())
        if t < iters - 1:
            C = centroid_update(Xfix, a, C, k)
    return a, C, history, stats


def cluster_permutation(a):
    """R3: perm[p] = original index of the token at permuted position p
    ([ABS]/[HF]: V-Smooth reorders value tokens so a block quantises well)."""
    return np.argsort(np.asarray(a), kind="stable").astype(np.int32)


def block_means(X, perm):
    """R4: mean of each 128-token block in permuted order ([NUN]: subtract the
    mean of each 128-token block), int64 fixed-point sum, fp32 result."""
    X = np.asarray(X, np.float32)
    S = len(perm)
    Xfix = np.rint(X.astype(np.float64) * 2.0 ** FIX_SHIFT).astype(np.int64)
    mu = np.zeros((num_blocks(S), X.shape[1]), np.float32)
    for b in range(num_blocks(S)):
        rows = perm[b * BLOCK: min(b * BLOCK + BLOCK, S)]
        s = Xfix[rows].sum(axis=0)
        mu[b] = ((s.astype(np.float64) * 2.0 ** -FIX_SHIFT) / len(rows)).astype(np.float32)
    return mu


def _residual_f32(X, perm, mu):
    X = np.asarray(X, np.float32)
    S = len(perm)
    return X[perm] - mu[np.arange(S) // BLOCK]          # fp32 subtraction


def residual_e4m3(X, perm, mu):
    """R5: quantise only the residual x - mu_block ([ABS], [HF], [NUN]) to E4M3
    with one scale per (b, h) ([OVC]: V scales per head).

    Returns (V^T codes (D, S_pad) uint8 with zero padding, s_V, amax).
    """
    r = _residual_f32(X, perm, mu)
    S, D = r.shape
    amax = np.float32(np.max(np.abs(r))) if S else np.float32(0)
    vt = np.zeros((D, padded_len(S)), np.uint8)
    if not amax >= TINY_AMAX:
        return vt, np.float32(1.0), amax
    inv = np.float32(E4M3_MAX) / amax
    s_v = amax / np.float32(E4M3_MAX)
    vt[:, :S] = e4m3_round(r * inv).T
    return vt, np.float32(s_v), amax


def residual_e4m3_per_channel(X, perm, mu):
    """R14: the E4M3 residual with one scale per channel. Returns (V^T codes
    (D, S_pad) uint8 with zero padding, s_V (D,) fp32, amax (D,) fp32)."""
    r = _residual_f32(X, perm, mu)
    S, D = r.shape
    amax = np.max(np.abs(r), axis=0).astype(np.float32) if S else np.zeros(D, np.float32)
    vt = np.zeros((D, padded_len(S)), np.uint8)
    s_v = np.ones(D, np.float32)
    for d in range(D):
        if not amax[d] >= TINY_AMAX:
            continue
        inv = np.float32(E4M3_MAX) / amax[d]
        s_v[d] = amax[d] / np.float32(E4M3_MAX)
        vt[d, :S] = e4m3_round(r[:, d] * inv)
    return vt, s_v, amax


def vres_from_e4m3_per_channel(vt, s_v, S):
    """Decoded per-channel residual (S, D) float64: s_V[d] * dec(code)."""
    return (np.asarray(s_v, np.float64)[:, None] * _E4M3[vt[:, :S]]).T


def residual_nvfp4(X, perm, mu):
    """R6: NVFP4 residual ([NUN]: "o 4 bits (NVFP4)").

    Returns (packed codes (D, S_pad/2) uint8 -- token 2i in the low nibble --,
    E4M3 group scales (D, S_pad/16) uint8, global scale g, amax).
    """
    r = _residual_f32(X, perm, mu)
    S, D = r.shape
    Sp = padded_len(S)
    amax = np.float32(np.max(np.abs(r))) if S else np.float32(0)
    packed = np.zeros((D, Sp // 2), np.uint8)
    scales = np.zeros((D, Sp // NVFP4_GROUP), np.uint8)
    if not amax >= TINY_AMAX:
        return packed, scales, np.float32(1.0), amax
    g = amax / np.float32(E4M3_MAX * E2M1_MAX)
    rt = np.zeros((D, Sp), np.float32)
    rt[:, :S] = r.T
    grp = rt.reshape(D, Sp // NVFP4_GROUP, NVFP4_GROUP)
    gmax = np.max(np.abs(grp), axis=2)                                    # (D, groups)
    scales[:] = e4m3_round((gmax / np.float32(E2M1_MAX)) / g)
    sdec = _E4M3[scales].astype(np.float32)
    den = sdec * g                                                        # fp32
    with np.errstate(all="ignore"):
        q = grp / den[:, :, None]                                         # fp32 division
    codes = np.where(sdec[:, :, None] == 0, 0, e2m1_round(q)).astype(np.uint8)
    codes = codes.reshape(D, Sp)
    packed[:] = codes[:, 0::2] | (codes[:, 1::2] << 4)
    return packed, scales, np.float32(g), amax


def vres_from_e4m3(vt, s_v, S):
    """Decoded residual values (S, D) float64: s_V * dec(code)."""
    return float(s_v) * _E4M3[vt[:, :S]].T


def residual_repair(X, perm, mu, vt, s_v, budget):
    """R12: the repair of an E4M3 residual. Returns (positions, corrections,
    repaired values): the permuted positions of the kept tokens (ascending),
    their fp32 corrections (m, D), and the decoded residual (S, D, fp64) with the
    corrections added at those positions."""
    r = _residual_f32(X, perm, mu).astype(np.float64)
    S = r.shape[0]
    vres = vres_from_e4m3(vt, s_v, S)
    err = np.sum((r - vres) ** 2, axis=1)
    m = min(S, int(math.ceil(budget * S)))
    order = np.lexsort((np.arange(S), -err))     # largest error first, then lower position
    pos = np.sort(order[:m])
    delta = (r[pos] - vres[pos]).astype(np.float32)
    rep = vres.copy()
    rep[pos] += delta.astype(np.float64)
    return pos, delta, rep


MX_GROUP = 32


def mx_exponent(amax):
    """R13: smallest integer e with amax <= 6 * 2^e, clamped to [-127, 127]
    (-127 for amax == 0). Exact: 6 * 2^e is exact in fp64."""
    a = float(amax)
    if not a > 0:
        return -127
    e = int(math.ceil(math.log2(a / E2M1_MAX)))
    while e > -127 and E2M1_MAX * 2.0 ** (e - 1) >= a:
        e -= 1
    while E2M1_MAX * 2.0 ** e < a:
        e += 1
    return max(-127, min(127, e))


def residual_mxfp4(X, perm, mu):
    """R13: MX-style FP4 residual. Returns (codes (D, S_pad) uint8, one E2M1 code
    per element, unpacked; biased exponents (D, S_pad/32) uint8 = e + 127)."""
    r = _residual_f32(X, perm, mu)
    S, D = r.shape
    Sp = padded_len(S)
    rt = np.zeros((D, Sp), np.float64)
    rt[:, :S] = r.T
    grp = rt.reshape(D, Sp // MX_GROUP, MX_GROUP)
    gmax = np.max(np.abs(grp), axis=2)
    e = np.vectorize(mx_exponent, otypes=[np.int64])(gmax)
    scaled = grp / np.ldexp(1.0, e)[:, :, None]              # exact: a power of two
    codes = e2m1_round(scaled.astype(np.float32)).reshape(D, Sp)
    return codes.astype(np.uint8), (e + 127).astype(np.uint8)


def vres_from_mxfp4(codes, e8, S):
    """Decoded MX-style residual (S, D) float64: e2m1(code) * 2^(e8 - 127)."""
    x = np.ldexp(1.0, np.repeat(e8.astype(np.int64) - 127, MX_GROUP, axis=1))
    return (e2m1_table()[codes] * x)[:, :S].T


def residual_repair_planes(X, perm, mu, budget):
    """R12 in the form of two E4M3 planes at the residual's scale s_V: plane 0
    holds the residual codes of R5; plane 1, for the kept tokens, the E4M3 codes
    of each element's rounding error in code units, dlt = y - dec(code) with
    y = fl32(r * fl32(448 / amax)) the value that was rounded (dlt is exact in
    fp32), and 0 elsewhere. A token's error is sum_d fl32(dlt_d^2), added in fp32
    channel by channel from d = 0 (a fixed order, so that any implementation
    that follows it ranks the tokens identically); the ceil(budget * S) largest
    are kept, ties to the lower permuted position.

    Returns (positions ascending, plane 0 (D, S_pad), plane 1 (D, S_pad), s_V,
    repaired values (S, D) fp64 = s_V (dec(plane 0) + dec(plane 1)))."""
    r = _residual_f32(X, perm, mu)
    S, D = r.shape
    vt, s_v, amax = residual_e4m3(X, perm, mu)
    lo = np.zeros_like(vt)
    m = min(S, int(math.ceil(budget * S)))
    if amax >= TINY_AMAX:
        inv = np.float32(E4M3_MAX) / amax
        y = r * inv                                                  # fp32, as R5 codes it
        dlt = (y - _E4M3[vt[:, :S]].T.astype(np.float32)).astype(np.float32)
        sq = dlt * dlt
        err = np.zeros(S, np.float32)
        for d in range(D):
            err = err + sq[:, d]
    else:
        dlt = np.zeros((S, D), np.float32)
        err = np.zeros(S, np.float32)
    order = np.lexsort((np.arange(S), -err.astype(np.float64)))
    pos = np.sort(order[:m])
    lo[:, pos] = e4m3_round(dlt[pos]).T
    rep = float(s_v) * (_E4M3[vt[:, :S]] + _E4M3[lo[:, :S]]).T
    return pos, vt, lo, s_v, rep


def vres_from_nvfp4(packed, scales, g, S):
    """Decoded NVFP4 residual values (S, D) float64: e2m1 * dec(scale) * g."""
    D = packed.shape[0]
    codes = np.empty((D, packed.shape[1] * 2), np.uint8)
    codes[:, 0::2] = packed & 0xF
    codes[:, 1::2] = packed >> 4
    vals = e2m1_table()[codes] * np.repeat(_E4M3[scales], NVFP4_GROUP, axis=1) * float(g)
    return vals[:, :S].T


def residual_energy(X, perm, mu):
    """Energy left for the residual quantiser: sum over permuted positions p of
    ||x[perm[p]] - mu[p // 128]||^2, in fp64 ([NUN]: the share of this energy that
    the token ordering removes is the method's reported diagnostic; the ratio is
    taken between the cluster order and the original order, both with block means).
    """
    r = np.asarray(X, np.float64)[perm] - np.asarray(mu, np.float64)[np.arange(len(perm)) // BLOCK]
    return float(np.sum(r * r))


# ------------------------------------------------------------ Q/K (A11)
def quant_blocks_e4m3(X, order=None):
    """R7: per 128-token block scale and E4M3 codes ([OVC]: Q/K scales per block).

    X: (S, D) float32; ``order`` (the permutation) reorders rows first (for K).
    Returns (codes (S_pad, D) uint8 with zero padding, scales (nb,) float32).
    """
    X = np.asarray(X, np.float32)
    if order is not None:
        X = X[order]
    S, D = X.shape
    codes = np.zeros((padded_len(S), D), np.uint8)
    scales = np.ones(num_blocks(S), np.float32)
    for b in range(num_blocks(S)):
        blk = X[b * BLOCK: min(b * BLOCK + BLOCK, S)]
        amax = np.float32(np.max(np.abs(blk)))
        if not amax >= TINY_AMAX:
            continue
        inv = np.float32(E4M3_MAX) / amax
        scales[b] = amax / np.float32(E4M3_MAX)
        codes[b * BLOCK: b * BLOCK + blk.shape[0]] = e4m3_round(blk * inv)
    return codes, scales


# ------------------------------------------------------------ ExpCast (A8)
def softmax_kappa(softmax_scale):
    """kappa = fl32(softmax_scale * log2 e): scores enter the log2 domain (R8)."""
    return np.float32(float(np.float32(softmax_scale)) * LOG2E)


def expcast_bias(k_p=K_P_DEFAULT):
    """B = 56 + 8 k_P: code of 2^k_P (E4M3 exponent bias 7 times 8 mantissa steps)."""
    return 56 + 8 * k_p


def expcast_codes(t, c, M, bias):
    """ExpCast-FP8 ([ABS]/[HF]: log-domain scores straight to E4M3 probability
    codes with one fused multiply-add), per R8.

    code = clip(bias - 8 M + rne(8 c t), 0, 126). 8 c t is exact in fp64 (a
    product of two fp32 values times 8); bias - 8M is an even integer, so adding
    it after the round-half-even step equals rounding the full sum.
    """
    v = 8.0 * np.asarray(c, np.float32).astype(np.float64) * np.asarray(t, np.float32).astype(np.float64)
    code = (bias - 8.0 * np.asarray(M, np.float64)) + np.rint(v)
    return np.clip(code, 0, 126).astype(np.uint8)


def _combine(P, vres, mu, S):
    """R9: O = (P v~ + sum_b r_b mu_b) / l with r_b the block row sums of P."""
    nb = num_blocks(S)
    starts = np.arange(nb) * BLOCK
    R = np.add.reduceat(P, starts, axis=1)            # per-block row sums (A7)
    l = P.sum(axis=1)
    return (P @ vres + R @ np.asarray(mu, np.float64)) / l[:, None], l


def expcast_online_probs(t, c, S, k_p=K_P_DEFAULT):
    """R8: probabilities of one or more query rows, cast block by block in the
    online running frame and expressed in the final frame.

    t, c: (rows, S) fp32 scores and multipliers. Returns (P float64, codes
    uint8, frames (rows, nb) float64 = F_i(b), final frame F_i(nb-1)).
    """
    t = np.asarray(t, np.float32)
    c = np.asarray(c, np.float32)
    u = c * t                                                        # fl32(c t)
    nb = num_blocks(S)
    bias = expcast_bias(k_p)
    codes = np.zeros(t.shape, np.uint8)
    frames = np.zeros((t.shape[0], nb), np.float64)
    F = None
    for b in range(nb):
        cols = slice(b * BLOCK, min(b * BLOCK + BLOCK, S))
        Fb = np.ceil(u[:, cols].max(axis=1).astype(np.float64))    # this block's frame
        F = Fb if F is None else np.maximum(F, Fb)                   # running frame
        frames[:, b] = F
        codes[:, cols] = expcast_codes(t[:, cols], c[:, cols], F[:, None], bias)
    shift = np.repeat(frames - F[:, None], BLOCK, axis=1)[:, :S]     # F(b) - F(final) <= 0
    P = _E4M3[codes] * np.exp2(shift)                                # exact powers of two
    return P, codes, frames, F


def vc_attention_rows(q_codes, q_scales, k_codes, k_scales, vres, mu, S, rows,
                      softmax_scale, k_p=K_P_DEFAULT, return_codes=False):
    """VC-Attention output for query rows ``rows`` of one (b, h) slice, in fp64.

    q_codes/k_codes: (S_pad, D) E4M3 codes (K in permuted order); q_scales/
    k_scales: per-block fp32 scales; vres: (S, D) decoded residual values in
    permuted order; mu: (nb, D) block means. Scores t = sum_d dec(q) dec(k) are
    exact in fp64 (products of 4-bit significands) and then rounded to fp32.
    Probabilities follow R8 (online integer frame per 128-key block), the
    combination R9.
    """
    rows = np.asarray(rows)
    Kd = _E4M3[k_codes[:S]]
    Qd = _E4M3[q_codes[rows]]
    t = (Qd @ Kd.T).astype(np.float32)
    kappa = softmax_kappa(softmax_scale)
    sq = np.asarray(q_scales, np.float32)[rows // BLOCK]
    sk = np.asarray(k_scales, np.float32)[np.arange(S) // BLOCK]
    c = (sq[:, None] * sk[None, :]) * kappa                         # fp32, fp32
    P, codes, frames, M = expcast_online_probs(t, c, S, k_p)
    O, l = _combine(P, vres, mu, S)
    if return_codes:
        return O, codes, M, l
    return O


def vc_attention_exact_prob(Q, K_perm, vres, mu, rows, softmax_scale):
    """The same combination with exact probabilities and unquantised inputs:
    P = 2^(u - max u), u = q.k * scale * log2 e, all fp64. With vres = V_perm - mu
    this must reproduce exact attention (V-Smooth is lossless before rounding)."""
    Q = np.asarray(Q, np.float64)[np.asarray(rows)]
    u = (Q @ np.asarray(K_perm, np.float64).T) * (float(softmax_scale) * LOG2E)
    P = np.exp2(u - u.max(axis=1, keepdims=True))
    O, _ = _combine(P, np.asarray(vres, np.float64), mu, K_perm.shape[0])
    return O


def exact_attention_rows(Q, K, V, rows, softmax_scale):
    """softmax(Q K^T * scale) V in fp64 from the original inputs (no permutation,
    no quantisation): the accuracy reference for the whole method."""
    Q = np.asarray(Q, np.float64)[np.asarray(rows)]
    s = (Q @ np.asarray(K, np.float64).T) * float(softmax_scale)
    P = np.exp(s - s.max(axis=1, keepdims=True))
    return (P @ np.asarray(V, np.float64)) / P.sum(axis=1, keepdims=True)


def naive_v_e4m3(V):
    """Baseline without V-Smooth: V itself per-(b, h) E4M3 in original order.
    Returns (decoded values (S, D) float64, s_V)."""
    V = np.asarray(V, np.float32)
    amax = np.float32(np.max(np.abs(V)))
    if not amax >= TINY_AMAX:
        return np.zeros(V.shape, np.float64), np.float32(1.0)
    inv = np.float32(E4M3_MAX) / amax
    s_v = amax / np.float32(E4M3_MAX)
    return float(s_v) * _E4M3[e4m3_round(V * inv)], np.float32(s_v)


# ------------------------------------------------------------ per-slice pipeline
def prepare_v_head(V, k, iters, seed, bh, fmt="e4m3", adopt=None, mode="vsmooth"):
    """V-Smooth prep for one (b, h) slice: k-means -> permutation -> block means
    -> residual quantisation ([ABS], [HF], [NUN]).

    mode "vsmooth" is the method; "meanonly" skips the clustering (identity
    permutation) and keeps the block means, for the residual-energy comparison;
    "naive" is the baseline the method improves on ([ABS]: low-bit V without
    smoothing): identity order and no block means, so V itself is quantised with
    the per-(b, h) scale.
    """
    V = np.asarray(V, np.float32)
    S = V.shape[0]
    out = {}
    if mode == "vsmooth":
        a, C, hist, stats = kmeans_lloyd(V, k, iters, seed, bh, adopt=adopt)
        out.update(assign=a, centroids=C, history=hist, stats=stats)
        perm = cluster_permutation(a)
    elif mode in ("meanonly", "naive"):
        perm = np.arange(S, dtype=np.int32)
    else:
        raise ValueError(mode)
    mu = block_means(V, perm) if mode != "naive" else np.zeros((num_blocks(S), V.shape[1]), np.float32)
    out.update(perm=perm, mu=mu)
    if fmt == "e4m3":
        vt, s_v, amax = residual_e4m3(V, perm, mu)
        out.update(v_codes=vt, s_v=s_v, amax=amax, vres=vres_from_e4m3(vt, s_v, S))
    elif fmt == "e4m3c":
        vt, s_v, amax = residual_e4m3_per_channel(V, perm, mu)
        out.update(v_codes=vt, s_v=s_v, amax=amax, vres=vres_from_e4m3_per_channel(vt, s_v, S))
    elif fmt == "mxfp4":
        codes, e8 = residual_mxfp4(V, perm, mu)
        out.update(v_codes=codes, v_scales=e8, vres=vres_from_mxfp4(codes, e8, S))
    elif fmt == "nvfp4":
        packed, scales, g, amax = residual_nvfp4(V, perm, mu)
        out.update(v_codes=packed, v_scales=scales, g=g, amax=amax,
                   vres=vres_from_nvfp4(packed, scales, g, S))
    else:
        raise ValueError(fmt)
    return out


def token_mean(X):
    """R11: per-channel mean over all tokens of one slice, int64 fixed-point sum
    of x * 2^24, one fp64 division, rounded to fp32."""
    X = np.asarray(X, np.float32)
    s = np.rint(X.astype(np.float64) * 2.0 ** FIX_SHIFT).astype(np.int64).sum(axis=0)
    return ((s.astype(np.float64) * 2.0 ** -FIX_SHIFT) / X.shape[0]).astype(np.float32)


def smooth_k(K):
    """R11: K minus its token mean (fp32 subtraction); returns (K - kbar, kbar)."""
    K = np.asarray(K, np.float32)
    kbar = token_mean(K)
    return K - kbar, kbar


def quant_qk_head(Q, K, perm, smooth=False):
    """Q/K per-block E4M3 quantisation for one slice; K gathered by ``perm``
    (after the R11 smoothing when ``smooth``)."""
    qc, qs = quant_blocks_e4m3(Q)
    if smooth:
        K = smooth_k(K)[0]
    kc, ks = quant_blocks_e4m3(K, order=perm)
    return qc, qs, kc, ks


def _check():  # pragma: no cover - import-time sanity of the constants
    assert math.isclose(LOG2E, 1.0 / math.log(2.0), rel_tol=1e-15)


_check()
