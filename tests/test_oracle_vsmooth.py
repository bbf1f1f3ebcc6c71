"""Pins for the oracle's V-Smooth prep and Q/K quantisation (CPU only).

Brute force with exact rational arithmetic on tiny inputs, a published
splitmix64 output, and the closed-form properties of each step.
"""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from bit_fp8_attention_prep_b200 import synth


def _bf16_values(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).float().numpy()
    # keep every value on the 2^-24 fixed-point grid (|x| >= 2^-17 or 0) so that
    # the fixed-point sums are the exact sums
    x[np.abs(x) < 2.0 ** -16] = 0.0
    return x


def test_splitmix64_published_outputs():
    # First two outputs of the splitmix64 reference implementation from state 0.
    r = O.SplitMix64(0)
    assert r.next() == 0xE220A8397B1DCDAF
    assert r.next() == 0x6E789E6AA1B965F4


def test_init_indices_distinct_in_range_and_seeded():
    for S, k in [(256, 4), (4096, 16), (73397, 16), (5, 5)]:
        idx = O.kmeans_init_indices(S, k, 0, 3)
        assert len(idx) == k and len(set(idx)) == k and all(0 <= i < S for i in idx)
    assert O.kmeans_init_indices(4096, 16, 0, 0) != O.kmeans_init_indices(4096, 16, 0, 1)
    assert O.kmeans_init_indices(4096, 16, 0, 0) != O.kmeans_init_indices(4096, 16, 1, 0)
    assert O.kmeans_init_indices(4096, 16, 7, 2) == O.kmeans_init_indices(4096, 16, 7, 2)
    # fewer tokens than clusters: all tokens taken once, then repeats are allowed
    idx = O.kmeans_init_indices(3, 8, 0, 0)
    assert len(idx) == 8 and set(idx) == {0, 1, 2}


def _exact_lloyd(X, k, iters, seed, bh):
    """Lloyd's algorithm in exact rational arithmetic (brute force)."""
    S, D = X.shape
    C = [[Fraction(float(v)) for v in X[i]] for i in O.kmeans_init_indices(S, k, seed, bh)]
    Xf = [[Fraction(float(v)) for v in row] for row in X]
    hist = []
    for t in range(iters):
        a = []
        for j in range(S):
            d = [sum((Xf[j][e] - C[c][e]) ** 2 for e in range(D)) for c in range(k)]
            a.append(min(range(k), key=lambda c: (d[c], c)))
        hist.append(a)
        if t < iters - 1:
            for c in range(k):
                mem = [j for j in range(S) if a[j] == c]
                if mem:
                    C[c] = [Fraction(float(np.float32(float(sum(Xf[j][e] for j in mem) / len(mem)))))
                            for e in range(D)]
    return hist, C


@pytest.mark.parametrize("S,D,k,iters,seed", [(40, 3, 4, 3, 0), (64, 8, 5, 4, 1), (33, 128, 3, 3, 2)])
def test_lloyd_matches_exact_brute_force(S, D, k, iters, seed):
    # tight clusters so that Lloyd moves tokens between passes
    X = _bf16_values((S, D), seed)
    X[: S // 2] += 3.0
    X = torch.from_numpy(X).to(torch.bfloat16).float().numpy()
    a, C, hist, stats = O.kmeans_lloyd(X, k, iters, seed, bh=5)
    ehist, eC = _exact_lloyd(X, k, iters, seed, bh=5)
    for t in range(iters):
        assert list(hist[t]) == ehist[t]
    assert stats == {"near_ties": 0, "mismatches": 0}


def test_lloyd_centroid_is_rounded_exact_mean():
    X = _bf16_values((300, 128), 4)
    a = np.arange(300) % 7
    Xfix = np.rint(X.astype(np.float64) * 2.0 ** 24).astype(np.int64)
    C = O.centroid_update(Xfix, a, np.zeros((8, 128), np.float32), 8)
    for c in range(7):
        mem = X[a == c]
        for e in (0, 17, 127):
            exact = sum(Fraction(float(v)) for v in mem[:, e]) / len(mem)
            assert C[c, e] == np.float32(float(exact))
    assert np.all(C[7] == 0)          # empty cluster keeps its centroid


def test_lloyd_recovers_planted_clusters():
    # Plant 16 generator centres far apart (pairwise distance >= 8) with noise of
    # norm < 1, and give the token at the i-th seeded init index generator i, so
    # that every generator holds one init pick. Lloyd must then label every token
    # with its own generator's pick after the first pass and keep that labelling,
    # and the centroids must be the generators' exact member means (fp32-rounded).
    S, k, D, seed, bh = 3000, 16, 128, 5, 2
    init = O.kmeans_init_indices(S, k, seed, bh)
    rng = np.random.default_rng(11)
    centres = np.zeros((k, D))
    for i in range(k):
        centres[i, 8 * i: 8 * i + 8] = 4.0 * (1 + (i % 3))     # disjoint supports: |c_i - c_j| >= 8
    gen = rng.integers(0, k, S)
    gen[np.asarray(init)] = np.arange(k)
    noise = rng.standard_normal((S, D))
    noise *= (0.9 * rng.random(S) / np.linalg.norm(noise, axis=1))[:, None]
    X = (centres[gen] + noise).astype(np.float32)
    X = torch.from_numpy(X).to(torch.bfloat16).float().numpy()
    X[np.abs(X) < 2.0 ** -16] = 0.0                   # on the fixed-point grid: exact sums
    a, C, hist, stats = O.kmeans_lloyd(X, k, 4, seed, bh)
    for h in hist:
        assert np.array_equal(h, gen)
    for i in range(k):
        mem = X[gen == i]
        for e in (0, 8 * i, 8 * i + 7, 127):
            exact = sum(Fraction(float(v)) for v in mem[:, e]) / len(mem)
            assert C[i, e] == np.float32(float(exact))


def test_lloyd_objective_does_not_increase():
    # Lloyd's two steps each lower sum_j |x_j - c_a(j)|^2 (exact means; here the
    # means are rounded to fp32, so allow a relative 1e-6 per pass).
    cfg, Q, K, V = synth.make_workload("mid", B=1, H=1, S=2048)
    X = V[0, :, 0].float().numpy()
    a, C, hist, stats = O.kmeans_lloyd(X, 16, 6, 0, 0)
    X64 = X.astype(np.float64)
    Cs = [X[O.kmeans_init_indices(2048, 16, 0, 0)].astype(np.float64)]
    Xfix = np.rint(X64 * 2.0 ** 24).astype(np.int64)
    for h in hist[:-1]:
        Cs.append(O.centroid_update(Xfix, h, Cs[-1].astype(np.float32), 16).astype(np.float64))
    J = [np.sum((X64 - Cs[t][h]) ** 2) for t, h in enumerate(hist)]
    for j0, j1 in zip(J, J[1:]):
        assert j1 <= j0 * (1 + 1e-6)
    assert J[-1] < J[0]
    # the final centroids are the ones the last pass assigned against
    assert np.array_equal(Cs[-1].astype(np.float32), C)


def test_permutation_is_stable_sort():
    rng = np.random.default_rng(5)
    for S, k in [(1, 1), (257, 4), (1000, 16)]:
        a = rng.integers(0, k, S)
        perm = O.cluster_permutation(a)
        assert list(perm) == sorted(range(S), key=lambda j: (a[j], j))


def test_block_means_exact_and_tail():
    X = _bf16_values((300, 128), 6, scale=3.0)
    perm = np.random.default_rng(6).permutation(300).astype(np.int32)
    mu = O.block_means(X, perm)
    assert mu.shape == (3, 128)
    for b, (lo, hi) in enumerate([(0, 128), (128, 256), (256, 300)]):
        rows = X[perm[lo:hi]]
        for e in (0, 64, 127):
            exact = sum(Fraction(float(v)) for v in rows[:, e]) / (hi - lo)
            assert mu[b, e] == np.float32(float(exact))


def _nearest_code_brute(v, tab, ncodes):
    d = np.abs(tab[:ncodes] - v)
    best = np.flatnonzero(d == d.min())
    return best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]


def test_residual_e4m3_codes_are_nearest_and_amax_maps_to_max():
    X = _bf16_values((300, 128), 7, scale=2.0)
    perm = np.random.default_rng(7).permutation(300).astype(np.int32)
    mu = O.block_means(X, perm)
    vt, s_v, amax = O.residual_e4m3(X, perm, mu)
    assert vt.shape == (128, 384) and np.all(vt[:, 300:] == 0)
    r = X[perm] - mu[np.arange(300) // 128]
    assert amax == np.max(np.abs(r))
    assert s_v == amax / np.float32(448)
    tab = O.e4m3_table()
    inv = np.float32(448) / amax
    jmax, emax = np.unravel_index(np.argmax(np.abs(r)), r.shape)
    assert vt[emax, jmax] & 0x7F == 0x7E
    rng = np.random.default_rng(8)
    for _ in range(300):
        j, e = rng.integers(0, 300), rng.integers(0, 128)
        v = float(np.float32(r[j, e] * inv))
        want = _nearest_code_brute(abs(v), tab, 127) | (0x80 if math.copysign(1, v) < 0 else 0)
        assert vt[e, j] == want


def test_residual_nvfp4_brute_force_and_fp16_exactness():
    X = _bf16_values((200, 128), 9, scale=2.0)
    perm = np.arange(200, dtype=np.int32)[::-1].copy()
    mu = O.block_means(X, perm)
    packed, scales, g, amax = O.residual_nvfp4(X, perm, mu)
    assert packed.shape == (128, 128) and scales.shape == (128, 16)
    r = X[perm] - mu[np.arange(200) // 128]
    assert g == amax / np.float32(2688)
    t4, t8 = O.e2m1_table(), O.e4m3_table()
    codes = np.empty((128, 256), np.uint8)
    codes[:, 0::2], codes[:, 1::2] = packed & 15, packed >> 4
    rng = np.random.default_rng(10)
    for _ in range(200):
        e, grp = rng.integers(0, 128), rng.integers(0, 200 // 16)
        vals = np.zeros(16, np.float32)
        n = min(16, 200 - 16 * grp)
        vals[:n] = r[16 * grp:16 * grp + n, e]
        target = float(np.float32(np.float32(np.max(np.abs(vals)) / np.float32(6)) / g))
        assert scales[e, grp] == _nearest_code_brute(target, t8, 127)
        den = np.float32(np.float32(t8[scales[e, grp]]) * g)
        for i in range(16):
            q = float(np.float32(vals[i] / den))
            want = _nearest_code_brute(min(abs(q), 6.0), t4, 8) | (8 if math.copysign(1, q) < 0 else 0)
            assert codes[e, 16 * grp + i] == want
    # every e2m1 x (positive) E4M3 product is exact in fp16, so the PV operand can
    # be dequantised exactly
    prods = np.outer(t4[:8], t8[:127])
    assert np.array_equal(prods.astype(np.float16).astype(np.float64), prods)


def test_quant_blocks_scales_codes_and_zero_block():
    X = _bf16_values((300, 128), 11)
    X[128:256] = 0.0
    perm = np.random.default_rng(11).permutation(300).astype(np.int32)
    codes, scales = O.quant_blocks_e4m3(X, order=perm)
    Xp = X[perm]
    assert codes.shape == (384, 128) and np.all(codes[300:] == 0)
    tab = O.e4m3_table()
    for b, (lo, hi) in enumerate([(0, 128), (128, 256), (256, 300)]):
        amax = np.max(np.abs(Xp[lo:hi]))
        if amax == 0:
            assert scales[b] == 1.0 and np.all(codes[lo:hi] == 0)
            continue
        assert scales[b] == amax / np.float32(448)
        deq = tab[codes[lo:hi]] * float(scales[b])
        # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 (normals), plus the
        # subnormal half-step
        assert np.all(np.abs(deq - Xp[lo:hi]) <= 2.0 ** -4 * np.abs(Xp[lo:hi]) + 2.0 ** -10 * scales[b] + 1e-30)


def test_naive_mode_is_v_itself_with_one_scale_per_head():
    # the baseline without smoothing: identity order, no means, and the decoded
    # residual equals the direct per-head E4M3 quantisation of V (a separate
    # routine), which is within half an E4M3 step of every value
    g = torch.Generator().manual_seed(11)
    V = (torch.randn(300, 128, generator=g) * 3 + 5).to(torch.bfloat16).float().numpy()
    out = O.prepare_v_head(V, 16, 4, 0, 0, mode="naive")
    assert np.array_equal(out["perm"], np.arange(300))
    assert not out["mu"].any()
    direct, s_v = O.naive_v_e4m3(V)
    assert out["s_v"] == s_v == np.float32(np.abs(V).max() / 448)
    assert np.array_equal(out["vres"], direct)
    # E4M3: half a mantissa step (|v| / 16) for normals, half the 2^-9 step below
    assert np.all(np.abs(direct - V) <= np.abs(V) / 16 + float(s_v) * 2.0 ** -10)
    # with a common offset in V, the block means of V-Smooth shrink the range to code
    vs = O.prepare_v_head(V, 16, 4, 0, 0)
    assert vs["s_v"] < out["s_v"]


def test_residual_energy_block_variance_parallel_axis_and_zero_means():
    # With the exact fp64 mean of every block of the permuted order, the energy
    # is sum_b n_b * sum_d var_bd (numpy's population variance per block, the
    # ragged 44-token tail included). Any other means add sum_b n_b |mu_b - m_b|^2
    # (the parallel-axis identity), which pins the block that each permuted
    # position is charged to; zero means give the squared Frobenius norm of V.
    S = 300
    rng = np.random.default_rng(5)
    X = _bf16_values((S, 128), 21, 2.0) + np.float32(3.0)
    perm = rng.permutation(S).astype(np.int32)
    Xp = X.astype(np.float64)[perm]
    blocks = [Xp[i:i + 128] for i in range(0, S, 128)]
    assert [len(b) for b in blocks] == [128, 128, 44]
    m = np.stack([b.mean(axis=0) for b in blocks])
    var_sum = sum(len(b) * np.var(b, axis=0).sum() for b in blocks)
    assert O.residual_energy(X, perm, m) == pytest.approx(var_sum, rel=1e-12)
    mu = rng.normal(size=m.shape).astype(np.float32)
    shift = sum(len(b) * np.sum((mu[i].astype(np.float64) - m[i]) ** 2) for i, b in enumerate(blocks))
    assert O.residual_energy(X, perm, mu) == pytest.approx(var_sum + shift, rel=1e-12)
    zero = np.zeros_like(mu)
    frob = np.linalg.norm(X.astype(np.float64)) ** 2
    assert O.residual_energy(X, perm, zero) == pytest.approx(frob, rel=1e-12)
    assert O.residual_energy(X, np.arange(S, dtype=np.int32), zero) == pytest.approx(frob, rel=1e-12)


def test_residual_energy_depends_on_blocks_not_order_within_them():
    S = 300
    rng = np.random.default_rng(6)
    X = _bf16_values((S, 128), 22, 1.0)
    perm = rng.permutation(S).astype(np.int32)
    mu = O.block_means(X, perm)
    e = O.residual_energy(X, perm, mu)
    # shuffling positions inside each block changes nothing ...
    p2 = perm.copy()
    for lo in range(0, S, 128):
        p2[lo:lo + 128] = rng.permutation(p2[lo:lo + 128])
    assert O.residual_energy(X, p2, mu) == pytest.approx(e, rel=1e-12)
    # ... moving a token to another block does
    p3 = perm.copy()
    p3[[0, 200]] = p3[[200, 0]]
    assert O.residual_energy(X, p3, mu) != pytest.approx(e, rel=1e-9)


def test_cluster_sort_leaves_only_within_cluster_energy():
    # Four groups of 128 tokens each, interleaved in the original order. Sorted
    # by group, every block is one group, so with the block means of the sorted
    # order the energy is the within-group scatter sum_c n_c sum_d var_cd; in
    # the original order each block mixes the groups and keeps their spread.
    rng = np.random.default_rng(7)
    centers = rng.normal(size=(4, 128)) * 4.0
    lab = rng.permutation(np.repeat(np.arange(4), 128))
    X = (centers[lab] + rng.normal(size=(512, 128))).astype(np.float32)
    X = torch.from_numpy(X).to(torch.bfloat16).float().numpy()
    perm = O.cluster_permutation(lab)
    within = sum(128 * np.var(X[lab == c].astype(np.float64), axis=0).sum() for c in range(4))
    e_sorted = O.residual_energy(X, perm, O.block_means(X, perm))
    assert e_sorted == pytest.approx(within, rel=1e-6)
    ident = np.arange(512, dtype=np.int32)
    e_orig = O.residual_energy(X, ident, O.block_means(X, ident))
    assert e_orig > 5 * e_sorted


def test_token_mean_is_the_rounded_exact_mean():
    # on the 2^-24 grid the fixed-point sum is exact, so the mean is the exact sum
    # divided once in fp64 and rounded to fp32: numpy's own fp64 mean, rounded
    X = _bf16_values((1000, 128), 31, 3.0) + np.float32(2.5)
    assert np.array_equal(O.token_mean(X), X.astype(np.float64).mean(axis=0).astype(np.float32))
    assert np.array_equal(O.token_mean(np.full((7, 128), -1.25, np.float32)), np.full(128, -1.25, np.float32))


def test_k_smoothing_keeps_the_softmax_and_tightens_the_k_codes():
    # Subtracting one vector from every key moves all scores of a query row by the
    # same amount, so exact attention is unchanged. With a per-channel offset in K
    # the smoothed block scales are several times smaller, the decoded smoothed K
    # is within half an E4M3 step of K - kbar, and the VC-Attention output moves
    # closer to exact attention.
    rng = np.random.default_rng(9)
    S = 300
    bf = lambda a: torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()
    Q = bf(rng.normal(size=(S, 128)))
    K = bf(rng.normal(size=(S, 128)) + rng.normal(size=128) * 6.0)
    V = bf(rng.normal(size=(S, 128)))
    Ks, kbar = O.smooth_k(K)
    assert np.array_equal(Ks, K - kbar)
    assert np.abs(O.token_mean(Ks)).max() < 1e-5
    rows = np.arange(0, S, 7)
    scale = 1.0 / math.sqrt(128)
    ref = O.exact_attention_rows(Q, K, V, rows, scale)
    exact_diff = K.astype(np.float64) - kbar.astype(np.float64)
    assert np.allclose(O.exact_attention_rows(Q, exact_diff, V, rows, scale), ref, rtol=1e-12, atol=1e-14)
    # the fp32 difference is rounded (to 2^-21 of |K| here): scores move by ~1e-6 at most
    assert np.allclose(O.exact_attention_rows(Q, Ks, V, rows, scale), ref, rtol=0, atol=1e-7)
    prep = O.prepare_v_head(V, 16, 4, 0, 0)
    err = {}
    for smooth in (False, True):
        qc, qs, kc, ks = O.quant_qk_head(Q, K, prep["perm"], smooth=smooth)
        if smooth:
            assert np.all(ks < ks_plain / 3)
            dec = O.e4m3_table()[kc[:S]] * np.repeat(ks, 128)[:S, None]
            Kp = Ks[prep["perm"]]
            step = np.repeat(ks, 128)[:S, None] * 2.0 ** -10
            assert np.all(np.abs(dec - Kp) <= np.abs(Kp) / 16 + step)
        else:
            ks_plain = ks
        o = O.vc_attention_rows(qc, qs, kc, ks, prep["vres"], prep["mu"], S, rows, scale)
        o = o[0] if isinstance(o, tuple) else o
        err[smooth] = np.linalg.norm(o - ref) / np.linalg.norm(ref)
    assert err[True] < 0.7 * err[False], err


def _repair_case(S, seed, k=4):
    g = torch.Generator().manual_seed(seed)
    V = torch.randn(S, 128, generator=g) * 2
    V[::17] *= 20                                  # a few outlier tokens
    X = V.to(torch.bfloat16).float().numpy()
    return X, O.prepare_v_head(X, k, 2, 0, 0)


def test_residual_repair_ends_and_exactness():
    X, prep = _repair_case(300, 41)
    args = (X, prep["perm"], prep["mu"], prep["v_codes"], prep["s_v"])
    pos, delta, rep = O.residual_repair(*args, 0.0)
    assert len(pos) == 0 and np.array_equal(rep, prep["vres"])
    # budget 1: every token gets its value back, up to the fp32 rounding of its correction
    r = (X[prep["perm"]] - prep["mu"][np.arange(300) // 128]).astype(np.float64)
    pos, delta, rep = O.residual_repair(*args, 1.0)
    assert np.array_equal(pos, np.arange(300))
    assert np.all(np.abs(rep - r) <= 2.0 ** -24 * np.abs(r - prep["vres"]))
    # the budget is a share of the slice's tokens, rounded up
    assert [len(O.residual_repair(*args, b)[0]) for b in (0.005, 0.01, 0.1)] == [2, 3, 30]


def test_residual_repair_keeps_the_worst_tokens_by_brute_force():
    # 12 tokens, two pairs of them identical (exact ties of the error). For m of
    # 3, 9 and 11 every m-subset is tried: the kept one removes the most squared
    # error (exactly rounded sums), and among equal errors the lower permuted
    # positions are kept (the pairs straddle the cut at m = 9 and m = 11)
    g = torch.Generator().manual_seed(43)
    V = torch.randn(12, 128, generator=g) * 3
    V[7] = V[2]
    V[9] = V[4]
    X = V.to(torch.bfloat16).float().numpy()
    prep = O.prepare_v_head(X, 1, 1, 0, 0, mode="meanonly")     # identity order, one block
    args = (X, prep["perm"], prep["mu"], prep["v_codes"], prep["s_v"])
    vres = prep["vres"]
    r = [[float(X[j, d]) - float(prep["mu"][0, d]) for d in range(128)] for j in range(12)]
    err = [math.fsum((r[j][d] - vres[j, d]) ** 2 for d in range(128)) for j in range(12)]
    assert err[2] == err[7] and err[4] == err[9]
    for m in (3, 9, 11):
        pos = O.residual_repair(*args, m / 12)[0].tolist()
        best = max(itertools.combinations(range(12), m),
                   key=lambda c: (math.fsum(err[j] for j in c), [-j for j in c]))
        assert pos == list(best), (m, pos, best)
    assert 2 in O.residual_repair(*args, 9 / 12)[0] and 7 not in O.residual_repair(*args, 9 / 12)[0]
    assert 4 in O.residual_repair(*args, 11 / 12)[0] and 9 not in O.residual_repair(*args, 11 / 12)[0]


def test_residual_repair_lowers_the_value_error_and_the_output_error():
    X, prep = _repair_case(300, 47)
    args = (X, prep["perm"], prep["mu"], prep["v_codes"], prep["s_v"])
    r = (X[prep["perm"]] - prep["mu"][np.arange(300) // 128]).astype(np.float64)
    left = []
    for b in (0.0, 0.01, 0.05, 0.2):
        pos, delta, rep = O.residual_repair(*args, b)
        left.append(float(np.sum((rep - r) ** 2)))
    assert left[0] > left[1] > left[2] > left[3]
    g = torch.Generator().manual_seed(48)
    Q = torch.randn(300, 128, generator=g).to(torch.bfloat16).float().numpy()
    K = torch.randn(300, 128, generator=g).to(torch.bfloat16).float().numpy()
    qc, qs, kc, ks = O.quant_qk_head(Q, K, prep["perm"])
    rows = np.arange(0, 300, 5)
    scale = 1.0 / math.sqrt(128)
    ref = O.exact_attention_rows(Q, K, X, rows, scale)
    e = {}
    for b in (0.0, 0.05):
        rep = O.residual_repair(*args, b)[2]
        o = O.vc_attention_rows(qc, qs, kc, ks, rep, prep["mu"], 300, rows, scale)
        e[b] = np.linalg.norm(o - ref) / np.linalg.norm(ref)
    assert e[0.05] < e[0.0], e


def test_residual_e4m3_per_channel_scales_codes_and_error():
    # every channel's largest residual maps to the largest code; every code is the
    # nearest (brute force) to r * 448 / amax_d; a zero channel gets scale 1 and
    # codes 0; each channel's decoded error stays within its own half-step bound
    X = _bf16_values((300, 128), 17, scale=1.0)
    X[:, 9] = 0
    perm = np.random.default_rng(18).permutation(300).astype(np.int32)
    mu = O.block_means(X, perm)
    vt, s_v, amax = O.residual_e4m3_per_channel(X, perm, mu)
    r = X[perm] - mu[np.arange(300) // 128]
    assert np.array_equal(amax, np.max(np.abs(r), axis=0))
    assert s_v[9] == 1.0 and not vt[9].any() and not vt[:, 300:].any()
    tab = O.e4m3_table()
    for d in (0, 20, 127):
        assert s_v[d] == amax[d] / np.float32(448)
        j = int(np.argmax(np.abs(r[:, d])))
        assert vt[d, j] & 0x7F == 0x7E
        inv = np.float32(448) / amax[d]
        for jj in range(0, 300, 7):
            v = float(np.float32(r[jj, d] * inv))
            want = _nearest_code_brute(abs(v), tab, 127) | (0x80 if math.copysign(1, v) < 0 else 0)
            assert vt[d, jj] == want
    dec = O.vres_from_e4m3_per_channel(vt, s_v, 300)
    assert np.all(np.abs(dec - r) <= np.abs(r) / 16 + s_v[None, :] * 2.0 ** -10)


@pytest.mark.parametrize("wide,gain", [(30.0, False), (3e4, True)])
def test_per_channel_scale_helps_only_below_the_e4m3_normal_range(wide, gain):
    # E4M3 keeps its relative precision over a 2^15 range below its maximum, so a
    # head scale set by channels 30x wider costs the narrow channels nothing; only
    # channels pushed into the subnormal codes (here 3e4x narrower) gain from
    # their own scale
    X = _bf16_values((300, 128), 19, scale=1.0)
    X[:, :8] *= wide
    X = torch.from_numpy(X).to(torch.bfloat16).float().numpy()
    perm = np.arange(300, dtype=np.int32)
    mu = O.block_means(X, perm)
    r = X[perm] - mu[np.arange(300) // 128]
    vt, s_v, _ = O.residual_e4m3_per_channel(X, perm, mu)
    dec = O.vres_from_e4m3_per_channel(vt, s_v, 300)
    vh, sh, _ = O.residual_e4m3(X, perm, mu)
    head = O.vres_from_e4m3(vh, sh, 300)
    e_ch = np.sum((dec - r)[:, 8:] ** 2)
    e_head = np.sum((head - r)[:, 8:] ** 2)
    if gain:
        assert e_ch < 0.1 * e_head
    else:
        assert 0.8 * e_head < e_ch < 1.25 * e_head


def test_residual_repair_planes_selection_codes_and_agreement():
    # Plane 0 is the residual code plane; the kept tokens are the largest by the
    # fp32 channel-ordered error (recomputed here with scalar fp32 arithmetic);
    # plane 1 holds the nearest E4M3 code of each kept element's error in code
    # units and 0 elsewhere; on continuous data the kept set is the exact form's
    # (fp64) one, and the repaired values sit within 2^-4 of the exact form's
    # correction (plus E4M3's subnormal floor) of the residual.
    X, prep = _repair_case(300, 51)
    perm, mu = prep["perm"], prep["mu"]
    pos, p0, p1, s_v, rep = O.residual_repair_planes(X, perm, mu, 0.05)
    vt, s_ref, amax = O.residual_e4m3(X, perm, mu)
    assert np.array_equal(p0, vt) and s_v == s_ref and len(pos) == 15
    r = X[perm] - mu[np.arange(300) // 128]
    inv = np.float32(448) / amax
    tab = O.e4m3_table()
    err = []
    for j in range(300):
        acc = np.float32(0)
        for d in range(128):
            dl = np.float32(np.float32(r[j, d] * inv) - np.float32(tab[vt[d, j]]))
            acc = np.float32(acc + np.float32(dl * dl))
        err.append(float(acc))
    want = sorted(sorted(range(300), key=lambda j: (-err[j], j))[:15])
    assert pos.tolist() == want
    keep = np.zeros(300, bool)
    keep[pos] = True
    assert not p1[:, :300][:, ~keep].any() and not p1[:, 300:].any()
    for j in pos[:4]:
        for d in range(0, 128, 9):
            dl = float(np.float32(np.float32(r[j, d] * inv) - np.float32(tab[vt[d, j]])))
            want_c = _nearest_code_brute(abs(dl), tab, 127) | (0x80 if math.copysign(1, dl) < 0 else 0)
            assert p1[d, j] == want_c or (dl == 0 and p1[d, j] & 0x7F == 0)
    epos, delta, _ = O.residual_repair(X, perm, mu, vt, s_v, 0.05)
    assert np.array_equal(epos, pos)
    r64 = r.astype(np.float64)
    assert np.all(np.abs(rep[pos] - r64[pos]) <= np.abs(delta) / 16 + float(s_v) * 2.0 ** -10)
    assert np.sum((rep - r64) ** 2) < np.sum((prep["vres"] - r64) ** 2)


def test_residual_repair_planes_ties_and_zero_head():
    # identical tokens tie exactly and the lower position is kept; an all-zero
    # slice repairs nothing
    g = torch.Generator().manual_seed(52)
    V = torch.randn(12, 128, generator=g) * 3
    V[7] = V[2]
    V[9] = V[4]
    X = V.to(torch.bfloat16).float().numpy()
    perm = np.arange(12, dtype=np.int32)
    mu = np.zeros((1, 128), np.float32)
    for m in range(1, 12):
        pos = O.residual_repair_planes(X, perm, mu, m / 12)[0].tolist()
        assert not (7 in pos and 2 not in pos) and not (9 in pos and 4 not in pos)
    Z = np.zeros((40, 128), np.float32)
    pos, p0, p1, s_v, rep = O.residual_repair_planes(Z, np.arange(40, dtype=np.int32), np.zeros((1, 128), np.float32), 0.5)
    assert s_v == 1.0 and not p0.any() and not p1.any() and not rep.any()
