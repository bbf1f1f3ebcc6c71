"""GPU: the device functions the kernels use for E4M3 / E2M1 rounding and for
ExpCast produce exactly the oracle's codes, and the bounded in-kernel wait ends
with a status instead of hanging."""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def va():
    from bit_fp8_attention_prep_b200 import build, vc_attn
    build.build()
    vc_attn.load()
    return vc_attn


def _structured_floats():
    """Every sign and exponent x the top 12 mantissa bits x low-bit patterns
    around the rounding points (exact ties included); no NaNs."""
    se = np.arange(512, dtype=np.uint64) << np.uint64(23)
    hi = np.arange(4096, dtype=np.uint64) << np.uint64(11)
    lo = np.array([0, 1, 0x3FF, 0x400, 0x401, 0x7FF], dtype=np.uint64)
    bits = (se[:, None, None] | hi[None, :, None] | lo[None, None, :]).reshape(-1).astype(np.uint32)
    x = bits.view(np.float32)
    return x[~np.isnan(x)]


def test_e4m3_cvt_matches_oracle(va):
    x = _structured_floats()
    got = va.test_e4m3_round(torch.from_numpy(x).cuda()).cpu().numpy()
    want = O.e4m3_round(x)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, [(float(x[i]), int(got[i]), int(want[i])) for i in bad[:10]]


def test_e2m1_cvt_matches_oracle(va):
    x = _structured_floats()
    got = va.test_e2m1_round(torch.from_numpy(x).cuda()).cpu().numpy()
    want = O.e2m1_round(x)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, [(float(x[i]), int(got[i]), int(want[i])) for i in bad[:10]]


@pytest.mark.parametrize("k_p", [0, 8])
def test_expcast_general_matches_oracle(va, k_p):
    rng = np.random.default_rng(k_p)
    n = 2_000_000
    t = (rng.standard_normal(n) * np.exp(rng.uniform(-3, 8, n))).astype(np.float32)
    c = np.exp(rng.uniform(-12, 2, n)).astype(np.float32)
    M = np.rint(rng.standard_normal(n) * 50).astype(np.float32)
    # exact ties: c = 1/8, t = integer + 1/2 puts 8ct - 8M + B on .5
    t[:4096] = (np.arange(4096) - 2048 + 0.5).astype(np.float32)
    c[:4096] = 1.0
    M[:4096] = 0.0
    B = O.expcast_bias(k_p)
    got = va.test_expcast(*(torch.from_numpy(a).cuda() for a in (t, c, M)), B, hot=False).cpu().numpy()
    want = O.expcast_codes(t, c, M, B)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, [(float(t[i]), float(c[i]), float(M[i]), int(got[i]), int(want[i])) for i in bad[:10]]


def test_expcast_hot_path_matches_oracle_on_rows(va):
    # Rows of scores with the frame M = ceil(fl32(c * max t)), as in the kernel.
    rng = np.random.default_rng(7)
    rows, cols = 2048, 512
    t = (rng.standard_normal((rows, cols)) * np.exp(rng.uniform(0, 9, (rows, 1)))).astype(np.float32)
    c = np.exp(rng.uniform(-12, 0, (rows, 1))).astype(np.float32) * np.ones((1, cols), np.float32)
    M = np.ceil((c * t.max(axis=1, keepdims=True)).astype(np.float64)).astype(np.float32) * np.ones((1, cols), np.float32)
    assert np.all(np.abs(M) < 2 ** 20)
    got = va.test_expcast(*(torch.from_numpy(a.reshape(-1).copy()).cuda() for a in (t, c, M)), 120, hot=True)
    want = O.expcast_codes(t, c, M, 120).reshape(-1)
    assert np.array_equal(got.cpu().numpy(), want)


def test_bounded_wait_returns_timeout(va):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    va.test_bounded_wait(status, 50_000_000)      # 50 ms on a barrier nothing completes
    end.record()
    torch.cuda.synchronize()
    assert int(status.item()) == va.VC_ERR_TIMEOUT
    assert 40.0 <= start.elapsed_time(end) < 5000.0
    # the context is still usable afterwards
    assert float(torch.ones(4, device="cuda").sum().item()) == 4.0


# ---------------------------------------------------------------- all 2^32 inputs
# On the non-negative fp32 bit patterns 0 .. 0x7F800000 (+0 to +inf, in order of
# value), round-to-nearest-even with saturation is a non-decreasing step function
# of the pattern with at most 127 (E4M3) or 7 (E2M1) steps. The kernel's output on
# every such pattern is checked to be non-decreasing, and its steps (positions and
# codes) to be the oracle's, found by bisection over the oracle (whose rounding of
# a value to a power-of-two grid is exact, hence monotone). Together these fix the
# kernel's output on all of them. Negative patterns must give the positive one's
# code with the sign bit set, NaN patterns the oracle's NaN code; both are checked
# on every pattern.
_POS_END = 0x7F800000          # +inf
_CHUNK = 1 << 28


def _oracle_code(fn, p):
    return int(fn(np.array([p], dtype=np.uint32).view(np.float32))[0])


def _oracle_steps(fn):
    """[(p, code)]: p = 0 and every pattern whose code differs from p - 1's."""
    steps = [(0, _oracle_code(fn, 0))]
    cur = 0
    while True:
        c = steps[-1][1]
        if _oracle_code(fn, _POS_END) == c:
            return steps
        lo, hi = cur, _POS_END          # fn(lo) == c, fn(hi) != c
        while hi - lo > 1:
            mid = (lo + hi) // 2
            if _oracle_code(fn, mid) == c:
                lo = mid
            else:
                hi = mid
        steps.append((hi, _oracle_code(fn, hi)))
        cur = hi


def _gpu_codes(va_fn, p0, n):
    bits = torch.arange(p0, p0 + n, dtype=torch.int64, device="cuda")
    bits = torch.where(bits >= 1 << 31, bits - (1 << 32), bits).to(torch.int32)
    return va_fn(bits.view(torch.float32)).to(torch.int32)


def _exhaustive(va_fn, oracle_fn, sign_bit):
    steps, prev = [], None
    for p0 in range(0, _POS_END + 1, _CHUNK):
        n = min(_CHUNK, _POS_END + 1 - p0)
        got = _gpu_codes(va_fn, p0, n)
        neg = _gpu_codes(va_fn, p0 + (1 << 31), n)
        assert torch.equal(neg, got | sign_bit), f"negative patterns of chunk {p0:#x}"
        if prev is not None:
            got = torch.cat([prev.view(1), got])
        assert bool((got[1:] >= got[:-1]).all()), f"not monotone in chunk {p0:#x}"
        idx = torch.nonzero(got[1:] != got[:-1]).flatten() + 1
        base = p0 - (1 if prev is not None else 0)
        if prev is None:
            steps.append((0, int(got[0])))
        steps += [(base + int(i), int(got[i])) for i in idx.cpu()]
        prev = got[-1]
    assert steps == _oracle_steps(oracle_fn)
    # NaN has no defined sign in the conversion: the oracle's NaN code and the same
    # code with the sign bit flipped are both accepted (for E4M3 the two NaN
    # encodings; E2M1 has none and both sides saturate the magnitude to 6)
    nan_code = _oracle_code(oracle_fn, 0x7FC00000)
    assert _oracle_code(oracle_fn, 0xFFC00000) == nan_code | sign_bit
    for lo, hi in ((_POS_END + 1, 1 << 31), ((1 << 31) + _POS_END + 1, 1 << 32)):
        for p0 in range(lo, hi, _CHUNK):
            got = _gpu_codes(va_fn, p0, min(_CHUNK, hi - p0))
            assert bool(((got | sign_bit) == (nan_code | sign_bit)).all()), f"NaN patterns from {p0:#x}"


def test_e4m3_cvt_all_fp32_inputs(va):
    _exhaustive(va.test_e4m3_round, O.e4m3_round, 0x80)
    assert O.e4m3_round(np.array([np.nan], np.float32))[0] == 0x7F    # an E4M3 NaN code


def test_e2m1_cvt_all_fp32_inputs(va):
    _exhaustive(va.test_e2m1_round, O.e2m1_round, 0x8)
    assert O.e2m1_round(np.array([np.nan], np.float32))[0] == 0x7     # saturated to 6
