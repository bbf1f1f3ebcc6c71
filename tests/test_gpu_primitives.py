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
