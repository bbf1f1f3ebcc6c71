"""Pins for the oracle's number formats and the ExpCast mapping (CPU only).

Each check ties the oracle to something other than itself: the OCP FP8 /
NVFP4 format definitions (closed-form values), torch's own fp8 / bf16 casts
(library routines), exact rational arithmetic, and the closed-form error bound
of a piecewise-linear 2^y.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O


# ------------------------------------------------------------------ E4M3
def test_e4m3_table_closed_forms():
    t = O.e4m3_table()
    # OCP FP8 E4M3FN: max normal 448 = 1.75 * 2^8, min subnormal 2^-9,
    # min normal 2^-6, 1.0 at exponent field 7, NaN only at S.1111.111.
    assert t[0x7E] == 448.0
    assert t[0x01] == 2.0 ** -9
    assert t[0x07] == 7 * 2.0 ** -9
    assert t[0x08] == 2.0 ** -6
    assert t[0x38] == 1.0
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.isnan(t).sum() == 2
    assert t[0x80] == 0.0 and math.copysign(1.0, t[0x80]) == -1.0
    pos = t[:127]
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(t[128:255], -pos)


def test_e4m3_round_matches_torch_cast():
    # torch's CPU float8_e4m3fn cast is round-to-nearest-even; compare on a dense
    # sweep of fp32 bit patterns inside the finite range, and on every midpoint.
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2 ** 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x) & (np.abs(x) <= 448.0)]
    t = O.e4m3_table()
    pos = t[:127]
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1000)])
    ours = O.e4m3_round(x)
    ref = torch.from_numpy(x.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_round_roundtrip_ties_and_saturation():
    t = O.e4m3_table()
    finite = [c for c in range(256) if not np.isnan(t[c])]
    assert np.array_equal(O.e4m3_round(t[finite].astype(np.float32)), np.array(finite, np.uint8))
    # ties go to the even mantissa
    pos = t[:127]
    for c in range(126):
        mid = np.float32((pos[c] + pos[c + 1]) / 2)
        want = c if c % 2 == 0 else c + 1
        assert O.e4m3_round(np.array([mid]))[0] == want
    big = np.array([448.0, 460.0, 464.0, 1e6, np.inf, -np.inf], np.float32)
    assert list(O.e4m3_round(big)) == [0x7E] * 4 + [0x7E, 0xFE]


# ------------------------------------------------------------------ E2M1
def test_e2m1_table_and_round_brute_force():
    t = O.e2m1_table()
    assert list(t[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # NVFP4 E2M1 values
    assert np.array_equal(t[8:], -t[:8])
    xs = np.linspace(-8, 8, 64001).astype(np.float32)
    got = O.e2m1_round(xs)
    vals = t[:8]
    for x, g in zip(xs, got):
        a = min(abs(float(x)), 6.0)
        d = np.abs(vals - a)
        best = np.flatnonzero(d == d.min())
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        if math.copysign(1.0, float(x)) < 0:
            want |= 8
        assert g == want, (x, g, want)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(200_000) * np.exp(rng.uniform(-20, 20, 200_000))
    ref = torch.from_numpy(x).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_round(x), ref)


# ------------------------------------------------------------------ ExpCast
@pytest.mark.parametrize("k_p", [0, 8])
def test_expcast_exact_at_integer_y(k_p):
    # c = 1, t = y integer, frame M = 0  =>  code = B + 8y, and the decoded E4M3
    # value must be exactly 2^(y + k_P) wherever the code is a normal number.
    B = O.expcast_bias(k_p)
    t = O.e4m3_table()
    for y in range(-30, 1):
        code = int(O.expcast_codes(np.float32(y), np.float32(1.0), 0.0, B))
        if code >= 8:
            assert code == B + 8 * y
            assert t[code] == math.ldexp(1.0, y + k_p)
        else:
            assert code == max(0, B + 8 * y)


def test_expcast_matches_exact_rational_rounding():
    # Independent exact computation with Fractions: code = clip(rne(B - 8M + 8ct)).
    rng = np.random.default_rng(3)
    for k_p in (0, 8):
        B = O.expcast_bias(k_p)
        tt = (rng.standard_normal(4000) * 40).astype(np.float32)
        cc = np.exp(rng.uniform(-6, 1, 4000)).astype(np.float32)
        MM = np.ceil((cc * tt).max())
        # add exact ties: 8 c t = n + 1/2
        cc = np.concatenate([cc, np.full(64, 1.0, np.float32)])
        tt = np.concatenate([tt, (np.arange(64) - 40 + 0.5).astype(np.float32) / 8])
        got = O.expcast_codes(tt, cc, MM, B)
        for t_, c_, g in zip(tt, cc, got):
            v = Fraction(B) - 8 * Fraction(float(MM)) + 8 * Fraction(float(c_)) * Fraction(float(t_))
            want = min(max(round(v), 0), 126)      # Python rounds Fractions half to even
            assert g == want


@pytest.mark.parametrize("k_p", [0, 8])
def test_expcast_monotone_over_code_range(k_p):
    B = O.expcast_bias(k_p)
    t = np.sort(np.linspace(-40, 1, 200001).astype(np.float32))
    codes = O.expcast_codes(t, np.float32(1.0), 1.0, B)
    assert np.all(np.diff(codes.astype(int)) >= 0)
    assert codes[0] == 0 and codes[-1] == B
    assert set(range(0, B + 1)) <= set(codes.tolist())


@pytest.mark.parametrize("k_p", [0, 8])
def test_expcast_piecewise_linear_error_bound(k_p):
    # E4M3 decoding of code n = 8e + m is 2^(e-7)(1 + m/8): a piecewise-linear 2^y.
    # Against 2^(y+k_P) the ratio lies in [2^(-1/16), (1.5/sqrt 2) 2^(1/16)]:
    # (1+f)/2^f <= 1.5/sqrt(2) on the grid f = m/8 (max at m = 4) and the code
    # rounding moves the exponent by at most 1/16.
    B = O.expcast_bias(k_p)
    tab = O.e4m3_table()
    y = np.linspace(-B / 8.0 - 0.5, 0.0, 300001).astype(np.float32)
    codes = O.expcast_codes(y, np.float32(1.0), 0.0, B)
    normal = codes >= 8
    ratio = tab[codes[normal]] / np.exp2(y[normal].astype(np.float64) + k_p)
    lo, hi = 2 ** (-1 / 16), 1.5 / math.sqrt(2) * 2 ** (1 / 16)
    assert ratio.min() >= lo - 1e-12 and ratio.max() <= hi + 1e-12
    assert ratio.max() > 1.09            # the bound is nearly reached
    sub = (codes < 8) & (codes > 0)
    assert sub.sum() > 0
    err = np.abs(tab[codes[sub]] - np.exp2(y[sub].astype(np.float64) + k_p))
    # subnormal codes (below the smallest normal 2^-6) sit on a linear 2^-9 grid:
    # the absolute error there stays below 2^-7.
    assert err.max() <= 2.0 ** -7


def test_mx_exponent_is_the_smallest_non_clipping_power_of_two():
    # brute force over every 8-bit exponent, at the boundaries 6 * 2^k, their
    # fp64 neighbours, and random values
    rng = np.random.default_rng(12)
    vals = [0.0, 6.0 * 2.0 ** -127, 6.0 * 2.0 ** -130, 1e-30, 3e38]
    for k in (-20, -3, 0, 1, 7):
        b = 6.0 * 2.0 ** k
        vals += [b, np.nextafter(b, 0.0), np.nextafter(b, np.inf)]
    vals += list(np.abs(rng.normal(size=50)) * 10.0 ** rng.integers(-6, 6, size=50))
    for a in vals:
        want = min([k for k in range(-127, 128) if a <= 6.0 * 2.0 ** k])
        assert O.mx_exponent(a) == want, (a, O.mx_exponent(a), want)


def test_residual_mxfp4_nearest_codes_no_clipping_and_minimal_scale():
    g = torch.Generator().manual_seed(13)
    S = 300                                   # 9 full groups of 32 and a ragged one per channel
    X = (torch.randn(S, 128, generator=g) * 2).to(torch.bfloat16).float().numpy()
    X[::29] *= 40
    X[:, 5] = 0                               # an all-zero channel
    perm = np.random.default_rng(14).permutation(S).astype(np.int32)
    mu = O.block_means(X, perm)
    codes, e8 = O.residual_mxfp4(X, perm, mu)
    Sp = O.padded_len(S)
    assert codes.shape == (128, Sp) and e8.shape == (128, Sp // 32)
    assert not codes[:, S:].any()
    r = (X[perm] - mu[np.arange(S) // 128]).astype(np.float64)       # the residual, fp32 values
    grid = np.array(O.e2m1_table(), np.float64)
    dec = O.vres_from_mxfp4(codes, e8, S)
    for d in (0, 5, 77):
        for gi in range(Sp // 32):
            seg = r[gi * 32: min(gi * 32 + 32, S), d]
            if seg.size == 0:
                continue
            x = 2.0 ** (int(e8[d, gi]) - 127)
            amax = np.abs(seg).max()
            assert amax <= 6 * x                                      # nothing clips
            assert amax == 0 and e8[d, gi] == 0 or amax > 3 * x       # a smaller power of two would clip
            cand = np.abs(grid[None, :] * x - seg[:, None])           # every grid point
            got = np.abs(dec[gi * 32: gi * 32 + seg.size, d] - seg)
            assert np.all(got <= cand.min(axis=1))                    # nearest point of the scaled grid
    assert not dec[:, 5].any()


def test_residual_mxfp4_exact_on_the_scaled_grid():
    # a group whose values are E2M1 values times one power of two decodes exactly
    rng = np.random.default_rng(15)
    grid = np.array(O.e2m1_table(), np.float32)
    X = (grid[rng.integers(0, 16, size=(64, 128))] * np.float32(2.0 ** -9)).astype(np.float32)
    X[0, :] = np.float32(6 * 2.0 ** -9)       # every group reaches the top of the grid
    X[32, :] = np.float32(-6 * 2.0 ** -9)
    perm = np.arange(64, dtype=np.int32)
    codes, e8 = O.residual_mxfp4(X, perm, np.zeros((1, 128), np.float32))
    assert (e8[:, :2] == 127 - 9).all() and (e8[:, 2:] == 0).all()     # the padding groups are all zero
    assert np.array_equal(O.vres_from_mxfp4(codes, e8, 64), X.astype(np.float64))
