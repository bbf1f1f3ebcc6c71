"""GPU: the two further residual formats, each bit-exact in the prep and
within the parity bars in the output.

- E4M3 with one scale per (b, h, channel): codes and scales against the oracle's
  residual_e4m3_per_channel, O against the oracle's VC-Attention on those values.
- MX-style FP4 (E2M1 with a power of two per channel and 32 tokens): codes and
  exponents against residual_mxfp4, O through the block-scaled FP8 x FP4 tensor-core
  product against the oracle's VC-Attention on the decoded MX values."""
import numpy as np
import pytest
import torch

import oracle as O
from parity_helpers import (SCALE, assert_o_close, assert_prep_bit_exact, gpu_pipeline, head, make, oracle_head,
                            oracle_rows, rel_l2)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def va():
    from bit_fp8_attention_prep_b200 import build, vc_attn
    build.build()
    vc_attn.load()
    return vc_attn


def _check(va, cfg, Q, K, V, fmt, rows=None, k_p=8, elementwise=True):
    g = gpu_pipeline(va, Q, K, V, cfg["k"], cfg["iters"], fmt=fmt, k_p=k_p)
    assert g["status"] == 0
    S = cfg["S"]
    rows = np.arange(S) if rows is None else rows
    worst = 0.0
    for b in range(cfg["B"]):
        for h in range(cfg["H"]):
            ref = oracle_head(g, Q, K, V, b, h, cfg["k"], cfg["iters"], fmt=fmt)
            assert_prep_bit_exact(g, ref, b, h, fmt=fmt)
            want = oracle_rows(ref, S, rows, k_p=k_p)
            if elementwise:
                r, _ = assert_o_close(g["o"][b, rows, h], want)
            else:
                r = rel_l2(g["o"][b, rows, h], O.bf16_round(want))
                assert r <= 2e-3, r
            worst = max(worst, r)
    return g, worst


@pytest.mark.parametrize("fmt", ["e4m3c", "mxfp4"])
@pytest.mark.parametrize("name,kw", [("tiny", {}), ("mid", dict(B=1, H=2, S=1000)), ("mid", dict(B=2, H=1, S=129)),
                                     ("mid", dict(B=1, H=1, S=5)), ("mid", dict(B=1, H=2, S=641))])
def test_format_prep_and_output(va, fmt, name, kw):
    # full and ragged tiles (1000 = 7 blocks + 104; 129 = one block + 1 token)
    cfg, Q, K, V = make(name, **kw)
    _check(va, cfg, Q, K, V, fmt)


@pytest.mark.parametrize("fmt", ["e4m3c", "mxfp4"])
def test_format_kp0_fp16_and_zero_channels(va, fmt):
    cfg, Q, K, V = make("mid", B=1, H=2, S=640)
    V[:, :, 0, 5] = 0.0          # one all-zero channel: its residual is the block mean's error only
    V[:, :, 1, :] = 0.0          # an all-zero head
    _check(va, cfg, Q, K, V, fmt, k_p=0)
    _check(va, cfg, Q.half(), K.half(), V.half(), fmt)


def test_mx_group_scales_span_the_exponent_range(va):
    # channels scaled from 2^-32 to 2^19: the exponents stay exact and no group
    # clips (prep bit-exact). The output is held to the rel-L2 bar only: with
    # values up to 2^24 in one channel, one probability code that the two sides
    # cast differently (an fp32 score on a rounding boundary, which the element
    # bar allows elsewhere) moves that channel's output by more than one BF16 step
    cfg, Q, K, V = make("mid", B=1, H=1, S=512)
    ch = torch.arange(128, dtype=torch.float64)
    V = (V.double() * torch.pow(2.0, (ch - 80) / 2.5)).to(torch.bfloat16)
    g, _ = _check(va, cfg, Q, K, V, "mxfp4", elementwise=False)
    e8 = g["v_scales"][0, 0]
    assert e8.min() < 100 and e8.max() > 140


def test_mid_size_sampled_rows(va):
    cfg, Q, K, V = make("mid", B=1, H=2, S=4096)
    rows = np.sort(np.random.default_rng(1).choice(4096, 80, replace=False))
    rows[0], rows[-1] = 0, 4095
    for fmt in ("e4m3c", "mxfp4"):
        _check(va, cfg, Q, K, V, fmt, rows=rows)


def test_per_channel_scale_gains_on_narrow_channels(va):
    # a head whose channels span 3e4 in range: the per-channel scale keeps the
    # narrow channels out of E4M3's subnormal codes (the oracle's finding); both
    # paths run on the GPU against exact fp64 attention on the same rows
    cfg, Q, K, V = make("mid", B=1, H=1, S=2048)
    w = torch.ones(128, dtype=torch.float64)
    w[64:] = 3.0e-5
    V = (V.double() * w).to(torch.bfloat16)
    rows = np.arange(0, 2048, 16)
    ex = O.exact_attention_rows(head(Q, 0, 0), head(K, 0, 0), head(V, 0, 0), rows, SCALE)
    err = {}
    for fmt in ("e4m3", "e4m3c"):
        g = gpu_pipeline(va, Q, K, V, 16, 4, fmt=fmt, history=False)
        o = g["o"][0, rows, 0]
        err[fmt] = rel_l2(o[:, 64:], ex[:, 64:])
    assert err["e4m3c"] < 0.5 * err["e4m3"], err
