"""Pins for the oracle's attention outputs (CPU only).

- exact attention against torch's scaled_dot_product_attention in fp64;
- invariance of exact attention under a joint K/V permutation;
- V-Smooth recovery: with exact probabilities and unquantised inputs, the
  block-mean split (residual through PV, mean through the block row sums)
  reproduces exact attention;
- the ExpCast VC-attention output against a brute-force loop with exact sums.
"""
import math
from fractions import Fraction

import numpy as np
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
    """One output row by loops: exact sums, exact round-half-even."""
    tab = O.e4m3_table()
    kappa = np.float32(float(np.float32(scale)) * O.LOG2E)
    B = 56 + 8 * k_p
    ts, cs, us = [], [], []
    for j in range(S):
        t = math.fsum(tab[qc[i, d]] * tab[kc[j, d]] for d in range(128))
        t32 = np.float32(t)
        c = np.float32(np.float32(qs[i // 128] * ks[j // 128]) * kappa)
        ts.append(t32)
        cs.append(c)
        us.append(float(np.float32(float(c) * float(t32))))
    M = math.ceil(max(us))
    P = []
    for t32, c in zip(ts, cs):
        v = Fraction(B) - 8 * M + 8 * Fraction(float(c)) * Fraction(float(t32))
        P.append(tab[min(max(round(v), 0), 126)])
    l = math.fsum(P)
    out = []
    for d in range(128):
        pv = math.fsum(P[j] * vres[j, d] for j in range(S))
        restore = math.fsum(math.fsum(P[j] for j in range(b * 128, min(b * 128 + 128, S))) * float(mu[b, d])
                            for b in range((S + 127) // 128))
        out.append((pv + restore) / l)
    return np.array(out)


def test_vc_attention_matches_brute_force_loops():
    cfg, Q, K, V = _head("mid", S=150, B=1, H=1)
    prep = O.prepare_v_head(V, 16, 4, 0, 0)
    qc, qs, kc, ks = O.quant_qk_head(Q, K, prep["perm"])
    rows = np.array([0, 77, 131, 149])
    for k_p in (0, 8):
        got = O.vc_attention_rows(qc, qs, kc, ks, prep["vres"], prep["mu"], 150, rows, SCALE, k_p=k_p)
        for n, i in enumerate(rows):
            want = _brute_vc_row(i, qc, qs, kc, ks, prep["vres"], prep["mu"], 150, SCALE, k_p)
            assert np.max(np.abs(got[n] - want)) <= 1e-12 * (1 + np.max(np.abs(want)))


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
