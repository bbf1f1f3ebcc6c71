"""GPU: V-Smooth prep and Q/K quantisation are bit-exact with the oracle
(k-means assignments compared pass by pass; near ties counted, no mismatch)."""
import numpy as np
import pytest
import torch

import oracle as O
from parity_helpers import assert_prep_bit_exact, gpu_pipeline, make, oracle_head

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def va():
    from bit_fp8_attention_prep_b200 import build, vc_attn
    build.build()
    vc_attn.load()
    return vc_attn


@pytest.mark.parametrize("name,kw", [
    ("tiny", {}),
    ("mid", dict(B=2, H=2, S=1000)),          # ragged: 7 full blocks + 104
    ("mid", dict(B=1, H=3, S=2500)),          # several k-means chunks, ragged chunk
])
def test_prep_bit_exact(va, name, kw):
    cfg, Q, K, V = make(name, **kw)
    g = gpu_pipeline(va, Q, K, V, cfg["k"], cfg["iters"])
    assert g["status"] == 0
    ties = 0
    for b in range(cfg["B"]):
        for h in range(cfg["H"]):
            ref = oracle_head(g, Q, K, V, b, h, cfg["k"], cfg["iters"])
            assert_prep_bit_exact(g, ref, b, h)
            ties += ref["stats"]["near_ties"]
    print(f"near ties adopted: {ties}")


def test_prep_nvfp4_bit_exact(va):
    cfg, Q, K, V = make("mid", B=1, H=2, S=777)
    g = gpu_pipeline(va, Q, K, V, 16, 4, fmt="nvfp4", attend=False)
    for h in range(2):
        ref = oracle_head(g, Q, K, V, 0, h, 16, 4, fmt="nvfp4")
        assert_prep_bit_exact(g, ref, 0, h, fmt="nvfp4")


@pytest.mark.parametrize("S,k", [(1, 4), (5, 16), (129, 16), (130, 1)])
def test_prep_edge_sizes(va, S, k):
    # fewer tokens than clusters, a single token, one token past a block, k = 1
    cfg, Q, K, V = make("mid", B=1, H=2, S=S)
    g = gpu_pipeline(va, Q, K, V, k, 3)
    for h in range(2):
        ref = oracle_head(g, Q, K, V, 0, h, k, 3)
        assert_prep_bit_exact(g, ref, 0, h)


def test_prep_zero_head_and_fp16(va):
    cfg, Q, K, V = make("mid", B=1, H=2, S=300)
    V[:, :, 1] = 0                       # an all-zero head: amax 0 -> s_V = 1, codes 0
    Q[:, 128:256, 0] = 0                 # an all-zero Q block -> scale 1, codes 0
    for dt in (torch.bfloat16, torch.float16):
        Qd, Kd, Vd = Q.to(dt), K.to(dt), V.to(dt)
        g = gpu_pipeline(va, Qd, Kd, Vd, 16, 4)
        for h in range(2):
            ref = oracle_head(g, Qd, Kd, Vd, 0, h, 16, 4)
            assert_prep_bit_exact(g, ref, 0, h)
        assert g["s_v"][0, 1] == 1.0 and not g["v_codes"][0, 1].any()
        assert g["q_scales"][0, 0, 1] == 1.0


def test_meanonly_mode(va):
    cfg, Q, K, V = make("mid", B=1, H=2, S=400)
    v = V.cuda()
    pv = va.prepare_v(v, mode="meanonly")
    torch.cuda.synchronize()
    for h in range(2):
        ref = O.prepare_v_head(V[0, :, h].float().numpy(), 16, 4, 0, h, mode="meanonly")
        assert np.array_equal(pv["perm"][0, h].cpu().numpy(), ref["perm"])
        assert np.array_equal(pv["mu"][0, h].cpu().numpy().view(np.uint32), ref["mu"].view(np.uint32))
        assert np.array_equal(pv["v_codes"][0, h].cpu().numpy(), ref["v_codes"])


def test_prep_exact_ties(va):
    # Values from three integer vectors and the midpoints of their pairs (all exact
    # in bf16): the initial centroids repeat and many tokens are exactly as far
    # from two centroids, so most assignments are decided by the direct-form
    # fallback and the lowest-index rule.
    g0 = torch.Generator().manual_seed(5)
    base = torch.randint(-4, 5, (3, 128), generator=g0).float()
    pool = torch.cat([base, 0.5 * (base[[0, 0, 1]] + base[[1, 2, 2]])])
    S, H = 700, 2
    V = pool[torch.randint(0, 6, (1, S, H), generator=g0)].to(torch.bfloat16)
    Q = torch.randn(1, S, H, 128, generator=g0).to(torch.bfloat16)
    K = torch.randn(1, S, H, 128, generator=g0).to(torch.bfloat16)
    g = gpu_pipeline(va, Q, K, V, 8, 3)
    for h in range(H):
        ref = oracle_head(g, Q, K, V, 0, h, 8, 3)
        assert ref["stats"]["near_ties"] == 0, ref["stats"]   # exact ties: both sides take the lowest index
        assert_prep_bit_exact(g, ref, 0, h)


@pytest.mark.parametrize("fmt", ["e4m3", "nvfp4"])
def test_naive_mode(va, fmt):
    # no reordering and no block means: the codes are V's own, one scale per head
    cfg, Q, K, V = make("mid", B=1, H=2, S=400)
    g = gpu_pipeline(va, Q, K, V, 16, 4, fmt=fmt, history=False, attend=False, mode="naive")
    for h in range(2):
        ref = O.prepare_v_head(V[0, :, h].float().numpy(), 16, 4, 0, h, fmt=fmt, mode="naive")
        assert np.array_equal(g["perm"][0, h], ref["perm"])
        assert not g["mu"][0, h].any()
        assert np.array_equal(g["v_codes"][0, h], ref["v_codes"])
        if fmt == "e4m3":
            assert g["s_v"][0, h] == ref["s_v"]
        else:
            assert np.array_equal(g["v_scales"][0, h], ref["v_scales"]) and g["s_v"][0, h] == ref["g"]


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_residual_energy(va, dt):
    # fp64 residual energy per slice: in the V-Smooth order with its block means,
    # in the original order with its block means (perm given, and perm NULL), and
    # of V itself (mu NULL), each against the oracle's own permutation and means
    cfg, Q, K, V = make("mid", B=2, H=3, S=1000)      # 7 full blocks + 104
    V = V.to(dt)
    B, S, H = 2, 1000, 3
    v = V.cuda()
    pv = va.prepare_v(v, history=True)
    pm = va.prepare_v(v, mode="meanonly")
    e_vs = va.residual_energy(v, pv["perm"], pv["mu"]).cpu().numpy()
    e_mo = va.residual_energy(v, pm["perm"], pm["mu"]).cpu().numpy()
    e_id = va.residual_energy(v, None, pm["mu"]).cpu().numpy()
    e_v = va.residual_energy(v).cpu().numpy()
    hist = pv["history"].cpu().numpy()
    ident = np.arange(S, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            X = V[b, :, h].float().numpy()
            ref = O.prepare_v_head(X, 16, 4, 0, b * H + h, adopt=[hist[t, b, h] for t in range(4)])
            assert ref["stats"]["mismatches"] == 0, ref["stats"]
            mo = O.prepare_v_head(X, 16, 4, 0, b * H + h, mode="meanonly")
            # fp64 sums of 128 000 non-negative terms in two orders: a few ulps apart
            assert e_vs[b, h] == pytest.approx(O.residual_energy(X, ref["perm"], ref["mu"]), rel=1e-12)
            assert e_mo[b, h] == pytest.approx(O.residual_energy(X, ident, mo["mu"]), rel=1e-12)
            assert e_id[b, h] == pytest.approx(e_mo[b, h], rel=1e-12)
            assert e_v[b, h] == pytest.approx(O.residual_energy(X, ident, np.zeros((8, 128))), rel=1e-12)
            assert e_vs[b, h] <= e_mo[b, h] <= e_v[b, h]


def test_residual_energy_edges(va):
    # one token (its own block mean: energy 0) and an all-zero head
    V = torch.zeros(1, 1, 2, 128, dtype=torch.bfloat16)
    V[0, 0, 0] = torch.arange(128) / 16
    v = V.cuda()
    pv = va.prepare_v(v, k=4, iters=2)
    e = va.residual_energy(v, pv["perm"], pv["mu"]).cpu().numpy()
    e_v = va.residual_energy(v).cpu().numpy()
    assert e[0, 0] == 0.0 and e[0, 1] == 0.0
    assert e_v[0, 0] == float(np.sum((np.arange(128) / 16.0) ** 2)) and e_v[0, 1] == 0.0


def _offset_keys(K, seed, size=6.0):
    # a per-(head, channel) offset on every key, as in the keys of DiT attention
    g = torch.Generator().manual_seed(seed)
    off = torch.randn(K.shape[2], K.shape[3], generator=g) * size
    return (K.float() + off).to(K.dtype)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_quant_qk_smoothk_bit_exact(va, dt):
    # K smoothing through a random permutation: codes, scales and the token mean
    # are bit-exact with the oracle's; Q is untouched
    cfg, Q, K, V = make("mid", B=2, H=3, S=1000)
    Q, K = Q.to(dt), _offset_keys(K, 3).to(dt)
    B, S, H = 2, 1000, 3
    rng = np.random.default_rng(4)
    perm = np.stack([np.stack([rng.permutation(S) for _ in range(H)]) for _ in range(B)]).astype(np.int32)
    out = va.quant_qk(Q.cuda(), K.cuda(), torch.from_numpy(perm).cuda(), smooth_k=True)
    plain = va.quant_qk(Q.cuda(), K.cuda(), torch.from_numpy(perm).cuda())
    torch.cuda.synchronize()
    g = {n: t.cpu().numpy() for n, t in out.items() if n != "workspace"}
    for b in range(B):
        for h in range(H):
            Kh = K[b, :, h].float().numpy()
            qc, qs, kc, ks = O.quant_qk_head(Q[b, :, h].float().numpy(), Kh, perm[b, h], smooth=True)
            assert np.array_equal(g["k_mean"][b, h].view(np.uint32), O.token_mean(Kh).view(np.uint32))
            assert np.array_equal(g["k_codes"][b, h], kc)
            assert np.array_equal(g["k_scales"][b, h].view(np.uint32), ks.view(np.uint32))
            assert np.array_equal(g["q_codes"][b, h], qc)
            assert np.array_equal(g["q_scales"][b, h].view(np.uint32), qs.view(np.uint32))
    assert np.array_equal(g["q_codes"], plain["q_codes"].cpu().numpy())
    # the offsets dominate the plain block amax; the smoothed one is the spread alone
    ratio = g["k_scales"] / plain["k_scales"].cpu().numpy()
    assert (ratio < 1).all() and ratio.mean() < 0.7, (ratio.min(), ratio.mean(), ratio.max())


@pytest.mark.parametrize("S", [1, 129])
def test_quant_qk_smoothk_edges(va, S):
    # one token (K - kbar = 0: scale 1, codes 0) and one token past a block
    cfg, Q, K, V = make("mid", B=1, H=2, S=S)
    K = _offset_keys(K, 5)
    perm = torch.arange(S, dtype=torch.int32).repeat(1, 2, 1).contiguous()
    out = va.quant_qk(Q.cuda(), K.cuda(), perm.cuda(), smooth_k=True)
    torch.cuda.synchronize()
    for h in range(2):
        Kh = K[0, :, h].float().numpy()
        qc, qs, kc, ks = O.quant_qk_head(Q[0, :, h].float().numpy(), Kh, np.arange(S), smooth=True)
        assert np.array_equal(out["k_codes"][0, h].cpu().numpy(), kc)
        assert np.array_equal(out["k_scales"][0, h].cpu().numpy().view(np.uint32), ks.view(np.uint32))
    if S == 1:
        assert not out["k_codes"].any() and (out["k_scales"] == 1).all()
