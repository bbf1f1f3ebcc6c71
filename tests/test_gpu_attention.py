"""GPU: the fused ExpCast attention matches the oracle's VC-attention output
within the acceptance bars (rel-L2 <= 2e-3, max-abs <= 1e-2), across full and
ragged tiles, both probability biases, FP16 input and the NVFP4 residual."""
import math

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


def _check_all_heads(va, cfg, Q, K, V, rows=None, k_p=8, fmt="e4m3"):
    g = gpu_pipeline(va, Q, K, V, cfg["k"], cfg["iters"], k_p=k_p, fmt=fmt)
    assert g["status"] == 0
    S = cfg["S"]
    rows = np.arange(S) if rows is None else rows
    worst = 0.0
    for b in range(cfg["B"]):
        for h in range(cfg["H"]):
            ref = oracle_head(g, Q, K, V, b, h, cfg["k"], cfg["iters"], fmt=fmt)
            o_ref = oracle_rows(ref, S, rows, k_p=k_p)
            r, _ = assert_o_close(g["o"][b, rows, h], o_ref)
            worst = max(worst, r)
    return g, worst


def test_attention_tiny_all_rows(va):
    cfg, Q, K, V = make("tiny")
    _check_all_heads(va, cfg, Q, K, V)


# 1 and 5: a single partial block; 128: one full block (the pair's second tile is
# past the end); 257: an odd block count with a one-token tail; 641: one mean
# batch in the loop and a one-block batch after it
@pytest.mark.parametrize("S", [1, 5, 128, 129, 257, 641, 700, 1000])
def test_attention_ragged(va, S):
    cfg, Q, K, V = make("mid", B=1, H=2, S=S)
    _check_all_heads(va, cfg, Q, K, V)


def test_attention_kp0_and_fp16(va):
    cfg, Q, K, V = make("mid", B=1, H=2, S=640)
    _check_all_heads(va, cfg, Q, K, V, k_p=0)
    _check_all_heads(va, cfg, Q.half(), K.half(), V.half())


def test_attention_mid_sampled_rows(va):
    cfg, Q, K, V = make("mid")
    rows = np.sort(np.random.default_rng(0).choice(cfg["S"], 96, replace=False))
    rows[0], rows[-1] = 0, cfg["S"] - 1
    _check_all_heads(va, cfg, Q, K, V, rows=rows)


def test_attention_nvfp4_tiny_all_rows(va):
    cfg, Q, K, V = make("tiny")
    _check_all_heads(va, cfg, Q, K, V, fmt="nvfp4")


@pytest.mark.parametrize("S", [1, 129, 257, 700, 1000])
def test_attention_nvfp4_ragged(va, S):
    cfg, Q, K, V = make("mid", B=1, H=2, S=S)
    _check_all_heads(va, cfg, Q, K, V, fmt="nvfp4")


def test_attention_nvfp4_mid_sampled_rows_kp0(va):
    cfg, Q, K, V = make("mid")
    rows = np.sort(np.random.default_rng(1).choice(cfg["S"], 64, replace=False))
    rows[0], rows[-1] = 0, cfg["S"] - 1
    _check_all_heads(va, cfg, Q, K, V, rows=rows, fmt="nvfp4")
    _check_all_heads(va, cfg, Q, K, V, rows=rows, fmt="nvfp4", k_p=0)


def test_attention_nvfp4_plan_matches_one_shot_calls(va):
    # The preallocated Plan (caller-owned plane workspace) gives the same bits as
    # the one-shot calls (workspace allocated per call).
    cfg, Q, K, V = make("mid", B=1, H=2, S=777)
    q, k, v = Q.cuda(), K.cuda(), V.cuda()
    plan = va.Plan(1, 777, 2, k=cfg["k"], iters=cfg["iters"], fmt="nvfp4")
    o_plan = plan.run(q, k, v).clone()
    pv = va.prepare_v(v, k=cfg["k"], iters=cfg["iters"], fmt="nvfp4")
    o_one = va.forward(va.quant_qk(q, k, pv["perm"]), pv, va.shape_of(q), SCALE, 8)
    torch.cuda.synchronize()
    assert int(plan.status.item()) == 0
    assert torch.equal(o_plan.view(torch.int16), o_one.view(torch.int16))


def test_attention_accuracy_vs_exact_and_naive(va):
    # V-Smooth against the unsmoothed baseline, both on the GPU (VC_MODE_NAIVE:
    # V itself at one E4M3 scale per head) with the same Q/K codes and ExpCast,
    # measured against exact fp64 attention. The values sit on 16 well separated
    # centres (N(0, 6^2) per channel, spread 0.2), so each token is mostly its
    # cluster's offset, which the block means of the sorted order carry exactly;
    # the queries are scaled by 0.3 so that the probabilities' own FP8 error
    # (equal in both runs) does not hide the value error. The oracle predicts a
    # factor of about 2 on these inputs.
    cfg, Q, K, V = make("mid", B=1, H=2, S=2048)
    g = torch.Generator().manual_seed(5)
    for h in range(2):
        cent = torch.randn(16, 128, generator=g) * 6.0
        lab = torch.randint(0, 16, (2048,), generator=g)
        V[0, :, h] = (cent[lab] + 0.2 * torch.randn(2048, 128, generator=g)).to(torch.bfloat16)
    Q = (Q.float() * 0.3).to(torch.bfloat16)
    rows = np.arange(0, 2048, 8)
    err = {}
    for mode in ("vsmooth", "naive"):
        gp = gpu_pipeline(va, Q, K, V, 16, 4, mode=mode, history=False)
        assert gp["status"] == 0
        num = den = 0.0
        for h in range(2):
            exact = O.exact_attention_rows(head(Q, 0, h), head(K, 0, h), head(V, 0, h), rows, SCALE)
            num += float(((gp["o"][0, rows, h] - exact) ** 2).sum())
            den += float((exact ** 2).sum())
        err[mode] = math.sqrt(num / den)
    print(f"rel-L2 vs exact fp64: V-Smooth {err['vsmooth']:.5f}, naive V {err['naive']:.5f}")
    assert err["vsmooth"] < 0.02 and err["vsmooth"] < 0.7 * err["naive"], err


def test_attention_exp2_comparison_kernel(va):
    # The comparison kernel (2^y on the special function unit, then an E4M3
    # conversion, in place of ExpCast) runs the same pipeline: close to exact
    # attention and to the ExpCast output, not equal to it.
    cfg, Q, K, V = make("mid", B=1, H=2, S=700)
    q, k, v = Q.cuda(), K.cuda(), V.cuda()
    pv = va.prepare_v(v, k=cfg["k"], iters=cfg["iters"])
    qk = va.quant_qk(q, k, pv["perm"])
    sh = va.shape_of(q)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o_cast = va.forward(qk, pv, sh, SCALE, 8).float().cpu().numpy()
    o_exp2 = va.test_forward_exp2(qk, pv, sh, SCALE, 8, status=status).float().cpu().numpy()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = np.arange(0, 700, 7)
    for h in range(2):
        exact = O.exact_attention_rows(head(Q, 0, h), head(K, 0, h), head(V, 0, h), rows, SCALE)
        e_exp2 = rel_l2(o_exp2[0, rows, h], exact)
        e_cast = rel_l2(o_cast[0, rows, h], exact)
        print(f"head {h}: rel-L2 vs exact: ExpCast {e_cast:.4f}, exp2 + E4M3 {e_exp2:.4f}")
        assert e_exp2 < 0.05 and rel_l2(o_exp2[0, rows, h], o_cast[0, rows, h]) < 0.05


def test_forward_with_smoothed_keys(va):
    # K smoothing end to end: prep bit-exact with the oracle, O within the parity
    # bar of the oracle's VC-Attention on the same smoothed codes, and closer to
    # exact fp64 attention than without smoothing
    from test_gpu_prep import _offset_keys
    cfg, Q, K, V = make("mid", B=1, H=2, S=1000)
    K = _offset_keys(K, 3)
    rows = np.arange(0, 1000, 9)
    errs = {}
    for smooth in (False, True):
        g = gpu_pipeline(va, Q, K, V, 16, 4, smooth_k=smooth)
        assert g["status"] == 0
        num = den = 0.0
        for h in range(2):
            ref = oracle_head(g, Q, K, V, 0, h, 16, 4, smooth_k=smooth)
            assert_prep_bit_exact(g, ref, 0, h)
            if smooth:
                assert_o_close(g["o"][0, rows, h], oracle_rows(ref, 1000, rows))
            ex = O.exact_attention_rows(head(Q, 0, h), head(K, 0, h), head(V, 0, h), rows, SCALE)
            num += float(((g["o"][0, rows, h] - ex) ** 2).sum())
            den += float((ex ** 2).sum())
        errs[smooth] = math.sqrt(num / den)
    assert errs[True] < 0.8 * errs[False], errs


def test_plan_and_attention_with_smoothed_keys_match_the_calls(va):
    # the preallocated plan and the one-call helper give the same bytes as the
    # separate calls with K smoothing
    from test_gpu_prep import _offset_keys
    cfg, Q, K, V = make("mid", B=1, H=2, S=700)
    K = _offset_keys(K, 8)
    q, k, v = Q.cuda(), K.cuda(), V.cuda()
    pv = va.prepare_v(v)
    qk = va.quant_qk(q, k, pv["perm"], smooth_k=True)
    o_calls = va.forward(qk, pv, va.shape_of(q))
    plan = va.Plan(1, 700, 2, smooth_k=True)
    o_plan = plan.run(q, k, v).clone()
    o_one = va.attention(q, k, v, smooth_k=True)
    torch.cuda.synchronize()
    assert torch.equal(o_plan, o_calls) and torch.equal(o_one, o_calls)
    assert torch.equal(plan.k_mean, qk["k_mean"]) and torch.equal(plan.k_codes, qk["k_codes"])
