"""Pins for the oracle's attention outputs (CPU only).

- exact attention against torch's scaled_dot_product_attention in fp64;
- invariance of exact attention under a joint K/V permutation;
- V-Smooth recovery: with exact probabilities and unquantised inputs, the
  block-mean split (residual through PV, mean through the block row sums)
  reproduces exact attention;
- the ExpCast VC-attention output against a brute-force loop with exact sums;
- kappa against softmax_scale * log2(e) at 60 digits.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from bit_fp8_attention_prep_b200 import synth

SCALE = 1.0 / math.sqrt(128)


def _head(name="tiny", b=0, h=0, **kw):
    cfg, Q, K, V = synth.make_workload(name, **kw)
    f = lambda X: X[b, :, h].float().numpy()
    return cfg, f(Q), f(K), f(V)


def test_exact_attention_matches_torch_sdpa():
    _, Q, K, V = _head("tiny", S=200)
    rows = np.arange(200)
    ours = O.exact_attention_rows(Q, K, V, rows, SCALE)
    t = lambda X: torch.from_numpy(X.astype(np.float64))[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V), scale=SCALE)[0, 0].numpy()
    assert np.max(np.abs(ours - ref)) < 1e-12


def test_exact_attention_joint_permutation_invariance():
    _, Q, K, V = _head("tiny")
    perm = np.random.default_rng(0).permutation(256)
    rows = np.arange(0, 256, 7)
    a = O.exact_attention_rows(Q, K, V, rows, SCALE)
    b = O.exact_attention_rows(Q, K[perm], V[perm], rows, SCALE)
    assert np.linalg.norm(a - b) <= 1e-12 * np.linalg.norm(a)


def test_vsmooth_mean_split_recovers_exact_attention():
    cfg, Q, K, V = _head("mid", S=700, B=1, H=1)          # ragged: 5 full blocks + 60
    prep = O.prepare_v_head(V, 16, 4, 0, 0)
    perm, mu = prep["perm"], prep["mu"]
    vres = V[perm].astype(np.float64) - mu[np.arange(700) // 128].astype(np.float64)
    rows = np.arange(0, 700, 11)
    got = O.vc_attention_exact_prob(Q, K[perm], vres, mu, rows, SCALE)
    ref = O.exact_attention_rows(Q, K, V, rows, SCALE)
    assert np.linalg.norm(got - ref) <= 1e-12 * np.linalg.norm(ref)
    # a wrong block index in the restore is caught: shift the means by one block
    bad = O.vc_attention_exact_prob(Q, K[perm], vres, np.roll(mu, 1, axis=0), rows, SCALE)
    assert np.linalg.norm(bad - ref) > 1e-3 * np.linalg.norm(ref)


def _brute_vc_row(i, qc, qs, kc, ks, vres, mu, S, scale, k_p):
    """One output row by loops: exact sums, exact round-half-even, the online
    softmax visiting the 128-key blocks in order with an integer running frame
    (a key of block b is cast in the frame reached after block b and carried
    into the final frame by the exact power of two)."""
    tab = O.e4m3_table()
    kappa = np.float32(float(np.float32(scale)) * O.LOG2E)
    B = 56 + 8 * k_p
    nb = (S + 127) // 128
    ts, cs, us = [], [], []
    for j in range(S):
        t = math.fsum(tab[qc[i, d]] * tab[kc[j, d]] for d in range(128))
        t32 = np.float32(t)
        c = np.float32(np.float32(qs[i // 128] * ks[j // 128]) * kappa)
        ts.append(t32)
        cs.append(c)
        us.append(float(np.float32(float(c) * float(t32))))
    frame_of_block = []
    F = None
    for b in range(nb):
        Fb = math.ceil(max(us[b * 128:min(b * 128 + 128, S)]))
        F = Fb if F is None else max(F, Fb)
        frame_of_block.append(F)
    P = []
    for j, (t32, c) in enumerate(zip(ts, cs)):
        Fj = frame_of_block[j // 128]
        v = Fraction(B) - 8 * Fj + 8 * Fraction(float(c)) * Fraction(float(t32))
        P.append(tab[min(max(round(v), 0), 126)] * 2.0 ** (Fj - F))
    l = math.fsum(P)
    out = []
    for d in range(128):
        pv = math.fsum(P[j] * vres[j, d] for j in range(S))
        restore = math.fsum(math.fsum(P[j] for j in range(b * 128, min(b * 128 + 128, S))) * float(mu[b, d])
                            for b in range(nb))
        out.append((pv + restore) / l)
    return np.array(out)


def test_vc_attention_matches_brute_force_loops():
    # 300 keys = three blocks (the last ragged), so the running frame can move
    cfg, Q, K, V = _head("mid", S=300, B=1, H=1)
    prep = O.prepare_v_head(V, 16, 4, 0, 0)
    qc, qs, kc, ks = O.quant_qk_head(Q, K, prep["perm"])
    rows = np.array([0, 77, 131, 299])
    moved = 0
    for k_p in (0, 8):
        got, codes, M, l = O.vc_attention_rows(qc, qs, kc, ks, prep["vres"], prep["mu"], 300, rows, SCALE,
                                               k_p=k_p, return_codes=True)
        for n, i in enumerate(rows):
            want = _brute_vc_row(i, qc, qs, kc, ks, prep["vres"], prep["mu"], 300, SCALE, k_p)
            assert np.max(np.abs(got[n] - want)) <= 1e-12 * (1 + np.max(np.abs(want)))
    t = O.e4m3_table()
    kd, qd = t[kc[:300]], t[qc[rows]]
    u = ((qs[rows // 128][:, None] * ks[np.arange(300) // 128][None, :]) * O.softmax_kappa(SCALE)) * (qd @ kd.T).astype(np.float32)
    first = np.ceil(u[:, :128].max(axis=1).astype(np.float64))
    assert np.any(first < M), "the test rows must include one whose frame moves"


def test_vc_attention_close_to_exact_and_better_than_naive_v():
    # Statistic, not a pin: on the outlier-bearing tiny workload V-Smooth should
    # beat per-head FP8 V with the same Q/K codes and ExpCast.
    cfg, Q, K, V = _head("tiny", h=1)
    S = 256
    prep = O.prepare_v_head(V, 4, 3, 0, 1)
    qc, qs, kc, ks = O.quant_qk_head(Q, K, prep["perm"])
    rows = np.arange(S)
    vc = O.vc_attention_rows(qc, qs, kc, ks, prep["vres"], prep["mu"], S, rows, SCALE)
    ref = O.exact_attention_rows(Q, K, V, rows, SCALE)
    qc0, qs0, kc0, ks0 = O.quant_qk_head(Q, K, np.arange(S))
    vnaive, _ = O.naive_v_e4m3(V)
    naive = O.vc_attention_rows(qc0, qs0, kc0, ks0, vnaive, np.zeros((2, 128), np.float32), S, rows, SCALE)
    e_vc = np.linalg.norm(vc - ref) / np.linalg.norm(ref)
    e_naive = np.linalg.norm(naive - ref) / np.linalg.norm(ref)
    assert e_vc < 0.1
    assert e_vc < e_naive


def _scores(name="mid", S=1000, h=1):
    cfg, Q, K, V = _head(name, S=S, B=1, H=2, h=h)
    prep = O.prepare_v_head(V, 16, 4, 0, h)
    qc, qs, kc, ks = O.quant_qk_head(Q, K, prep["perm"])
    tab = O.e4m3_table()
    t = (tab[qc[:S]] @ tab[kc[:S]].T).astype(np.float32)
    c = (qs[np.arange(S) // 128][:, None] * ks[np.arange(S) // 128][None, :]) * O.softmax_kappa(SCALE)
    return t, c.astype(np.float32), S


def test_online_cast_equals_single_frame_cast_on_normal_codes():
    # Codes in integer frames differ by exactly 8 per unit of frame, so casting a
    # block in an earlier (lower) frame and scaling by 2^(F_old - F_new) gives the
    # same value as casting it in the final frame wherever the final-frame code is
    # a normal E4M3 number (>= 8); only final-frame subnormals and zeros differ, and
    # there the online value is the finer one.
    t, c, S = _scores()
    P, codes, frames, F = O.expcast_online_probs(t, c, S, 8)
    single = O.expcast_codes(t, c, F[:, None], O.expcast_bias(8))
    tab = O.e4m3_table()
    normal = single >= 8
    assert np.array_equal(P[normal], tab[single[normal]])
    assert np.any(frames[:, :1] < F[:, None]), "some frame must move on this workload"
    moved = ~normal & (P != tab[single])
    assert moved.any()
    exact = np.exp2((c.astype(np.float64) * t.astype(np.float64)) - F[:, None] + 8)
    err_online = np.abs(P[moved] - exact[moved])
    err_single = np.abs(tab[single[moved]] - exact[moved])
    # each online value keeps its own frame's resolution, while below code 8 the
    # final-frame cast only bounds the absolute error by the smallest normal
    # value 2^(k_P - 14) (times 2^(1/16) for the code rounding)
    assert err_online.sum() < 0.5 * err_single.sum()
    assert np.all(err_single <= 2.0 ** -6 * 2 ** (1 / 16))


def test_online_probs_within_piecewise_linear_bound():
    # Each key's carried probability against 2^(u - F_final + k_P): inside the
    # E4M3 piecewise-linear bound [2^(-1/16), 1.5/sqrt(2) 2^(1/16)] wherever its
    # own-frame code is normal; the frame never drops below the row max.
    t, c, S = _scores(h=0)
    P, codes, frames, F = O.expcast_online_probs(t, c, S, 8)
    u = (c * t).astype(np.float64)
    assert np.all(u.max(axis=1) <= F)
    own_normal = codes >= 8
    exact = np.exp2(c.astype(np.float64) * t.astype(np.float64) - F[:, None] + 8)
    ratio = P[own_normal] / exact[own_normal]
    assert ratio.min() >= 2 ** (-1 / 16) - 1e-12
    assert ratio.max() <= 1.5 / math.sqrt(2) * 2 ** (1 / 16) + 1e-12
    # the largest probability of every row sits in the top binade below 2^k_P
    assert np.all(P.max(axis=1) <= 2.0 ** 8) and np.all(P.max(axis=1) >= 2.0 ** 7 * 2 ** (-1 / 16))


def test_softmax_kappa_is_scale_times_log2e():
    # exp(s x) = 2^(kappa x) with kappa = s log2(e), rounded once to fp32: the
    # oracle's fp64 product then fp32 rounding lands within half an fp32 ulp
    # (plus 2^-53 relative) of the exact value computed at 60 digits.
    from decimal import Decimal, getcontext
    getcontext().prec = 60
    log2e = 1 / Decimal(2).ln()
    for s in (1 / math.sqrt(128), 1 / math.sqrt(64), 1.0, 0.125, 0.3):
        s32 = Decimal(float(np.float32(s)))
        k = O.softmax_kappa(s)
        assert k.dtype == np.float32
        ulp = Decimal(float(np.spacing(k)))
        assert abs(Decimal(float(k)) - s32 * log2e) <= ulp * Decimal("0.5000001")
        x = 7.0
        assert 2.0 ** (float(k) * x) == pytest.approx(math.exp(float(np.float32(s)) * x), rel=1e-6)
