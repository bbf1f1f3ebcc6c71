"""CPU: the C++ statement of the oracle (oracle/vc_oracle_ref.cpp) against the
numpy oracle, step by step, on seeded inputs of the method's shapes: integer,
byte and index outputs bit for bit, fp32 results bit for bit, fp64 combinations
within 1e-12 (the two sum in different orders). Two independent statements of
the same readings agreeing is what these tests pin; each statement is pinned to
the pages and the mathematics by the other test_oracle_* files."""
import math

import numpy as np
import pytest

import oracle as O
from oracle import ref_cpp as C
from bit_fp8_attention_prep_b200 import synth

SCALE = 1.0 / math.sqrt(128)


@pytest.fixture(scope="module", autouse=True)
def lib():
    C.build()
    return C.load()


def torch_free_bf16(x):
    """Round fp32 values to bf16 (ties to even) with integer arithmetic."""
    b = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def _slice(name, b=0, h=0, **kw):
    cfg, Q, K, V = synth.make_workload(name, **kw)
    f = lambda X: X[b, :, h].float().numpy()
    return cfg, f(Q), f(K), f(V)


def test_e4m3_every_bf16_pattern_and_specials():
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    x = bits.view(np.float32)
    assert np.array_equal(C.e4m3_round(x), O.e4m3_round(x))
    # midpoints between neighbouring codes (ties), their fp32 neighbours, specials
    vals = O.e4m3_table()[:127]
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    sp = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, -np.nan, 448.0, 464.0, 480.0, 1e30, 2.0 ** -10, 2.0 ** -11,
                   1.5 * 2.0 ** -10, 3 * 2.0 ** -11, 1e-45], np.float32)
    x = np.concatenate([near, -near, sp, np.random.default_rng(0).standard_normal(20000).astype(np.float32) * 100])
    assert np.array_equal(C.e4m3_round(x), O.e4m3_round(x))


def test_e2m1_every_bf16_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    x = bits.view(np.float32)
    assert np.array_equal(C.e2m1_round(x), O.e2m1_round(x))


@pytest.mark.parametrize("S,k,seed,bh", [(256, 4, 0, 0), (4096, 16, 0, 5), (73397, 16, 3, 55), (5, 16, 0, 1),
                                         (1, 4, 7, 2)])
def test_kmeans_init(S, k, seed, bh):
    assert C.kmeans_init_indices(S, k, seed, bh) == O.kmeans_init_indices(S, k, seed, bh)


@pytest.mark.parametrize("name,kw,h", [("tiny", {}, 1), ("mid", dict(B=1, H=2, S=1000), 1),
                                       ("mid", dict(B=1, H=1, S=129), 0)])
def test_prep_steps_bit_exact(name, kw, h):
    cfg, Q, K, V = _slice(name, h=h, **kw)
    k, iters, bh = cfg["k"], cfg["iters"], h
    a_c, C_c, hist_c = C.kmeans_lloyd(V, k, iters, 0, bh)
    a_o, C_o, hist_o, stats = O.kmeans_lloyd(V, k, iters, 0, bh)
    for hc, ho in zip(hist_c, hist_o):
        assert np.array_equal(hc, ho)
    assert np.array_equal(C_c.view(np.uint32), C_o.view(np.uint32))
    perm = C.cluster_permutation(a_c, k)
    assert np.array_equal(perm, O.cluster_permutation(a_o))
    mu = C.block_means(V, perm)
    assert np.array_equal(mu.view(np.uint32), O.block_means(V, perm).view(np.uint32))
    vt_c, sv_c, am_c = C.residual_e4m3(V, perm, mu)
    vt_o, sv_o, am_o = O.residual_e4m3(V, perm, mu)
    assert np.array_equal(vt_c, vt_o) and sv_c == sv_o and am_c == am_o
    assert np.array_equal(C.vres_from_e4m3(vt_c, sv_c, len(perm)), O.vres_from_e4m3(vt_o, sv_o, len(perm)))
    pk_c, sc_c, g_c, _ = C.residual_nvfp4(V, perm, mu)
    pk_o, sc_o, g_o, _ = O.residual_nvfp4(V, perm, mu)
    assert np.array_equal(pk_c, pk_o) and np.array_equal(sc_c, sc_o) and g_c == g_o
    vt_c, sv_c, am_c = C.residual_e4m3_per_channel(V, perm, mu)
    vt_o, sv_o, am_o = O.residual_e4m3_per_channel(V, perm, mu)
    assert np.array_equal(vt_c, vt_o) and np.array_equal(sv_c.view(np.uint32), sv_o.view(np.uint32))
    cd_c, e8_c = C.residual_mxfp4(V, perm, mu)
    cd_o, e8_o = O.residual_mxfp4(V, perm, mu)
    assert np.array_equal(cd_c, cd_o) and np.array_equal(e8_c, e8_o)
    for X, order in ((Q, None), (K, perm)):
        cc, scc = C.quant_blocks_e4m3(X, order)
        co, sco = O.quant_blocks_e4m3(X, order)
        assert np.array_equal(cc, co) and np.array_equal(scc.view(np.uint32), sco.view(np.uint32))


@pytest.mark.parametrize("budget", [0.0, 0.005, 0.05, 1.0])
def test_repair_planes_and_energy(budget):
    cfg, Q, K, V = _slice("mid", B=1, H=1, S=1000)
    ref = O.prepare_v_head(V, cfg["k"], cfg["iters"], 0, 0)
    perm, mu = ref["perm"], ref["mu"]
    pos_c, vt_c, lo_c, sv_c = C.residual_repair_planes(V, perm, mu, budget)
    pos_o, vt_o, lo_o, sv_o, _ = O.residual_repair_planes(V, perm, mu, budget)
    assert np.array_equal(pos_c, pos_o) and np.array_equal(vt_c, vt_o) and np.array_equal(lo_c, lo_o)
    assert sv_c == sv_o
    e_c, e_o = C.residual_energy(V, perm, mu), O.residual_energy(V, perm, mu)
    assert abs(e_c - e_o) <= 1e-12 * e_o


def test_smooth_k_and_its_codes():
    cfg, Q, K, V = _slice("mid", B=1, H=1, S=1000)
    K = K + np.float32(3.0) * np.arange(128, dtype=np.float32)[None, :] / 128.0
    K = np.asarray(torch_free_bf16(K))
    xs_c, kb_c = C.smooth_k(K)
    xs_o, kb_o = O.smooth_k(K)
    assert np.array_equal(kb_c.view(np.uint32), kb_o.view(np.uint32))
    assert np.array_equal(xs_c.view(np.uint32), xs_o.view(np.uint32))
    perm = np.random.default_rng(2).permutation(1000).astype(np.int32)
    cc, scc = C.quant_blocks_e4m3(xs_c, perm)
    _, _, kc, ks = O.quant_qk_head(Q, K, perm, smooth=True)
    assert np.array_equal(cc, kc) and np.array_equal(scc.view(np.uint32), ks.view(np.uint32))


def test_zero_slice_and_zero_block():
    X = np.zeros((300, 128), np.float32)
    X[200:, 5] = 1.0          # blocks 0 and 1 all zero, block 2 not
    perm = np.arange(300, dtype=np.int32)
    mu = C.block_means(X, perm)
    vt_c, sv_c, _ = C.residual_e4m3(np.zeros_like(X), perm, mu * 0)
    vt_o, sv_o, _ = O.residual_e4m3(np.zeros_like(X), perm, mu * 0)
    assert np.array_equal(vt_c, vt_o) and sv_c == sv_o == 1.0
    cc, scc = C.quant_blocks_e4m3(X)
    co, sco = O.quant_blocks_e4m3(X)
    assert np.array_equal(cc, co) and np.array_equal(scc, sco)


def test_mx_exponent_boundaries():
    vals = [0.0, 6.0 * 2.0 ** -127, 6.0 * 2.0 ** -130, 6.0 * 2.0 ** 127, 6.0 * 2.0 ** 130, 1e-45, 3.0, 6.0, 6.000001,
            12.0, 12.5, 0.75, 0.7499999]
    for e in range(-20, 21):
        b = 6.0 * 2.0 ** e
        vals += [b, np.nextafter(b, 0.0), np.nextafter(b, np.inf)]
    for v in vals:
        assert C.mx_exponent(v) == O.mx_exponent(v), v


def test_kappa():
    for s in (SCALE, 0.125, 1.0, 0.3):
        assert C.softmax_kappa(s) == O.softmax_kappa(s)


@pytest.mark.parametrize("name,kw,k_p", [("tiny", {}, 8), ("mid", dict(B=1, H=1, S=700), 8),
                                         ("mid", dict(B=1, H=1, S=700), 0)])
def test_vc_attention_rows(name, kw, k_p):
    cfg, Q, K, V = _slice(name, **kw)
    S = cfg["S"]
    ref = O.prepare_v_head(V, cfg["k"], cfg["iters"], 0, 0)
    qc, qs = O.quant_blocks_e4m3(Q)
    kc, ks = O.quant_blocks_e4m3(K, ref["perm"])
    rows = np.unique(np.concatenate([[0, S - 1], np.random.default_rng(3).choice(S, 40, replace=False)]))
    o_o, codes_o, F_o, l_o = O.vc_attention_rows(qc, qs, kc, ks, ref["vres"], ref["mu"], S, rows, SCALE, k_p=k_p,
                                                 return_codes=True)
    o_c, codes_c, l_c = C.vc_attention_rows(qc, qs, kc, ks, ref["vres"], ref["mu"], S, rows, SCALE, k_p=k_p)
    assert np.array_equal(codes_c, codes_o)
    assert np.allclose(l_c, l_o, rtol=1e-13, atol=0)
    assert np.max(np.abs(o_c - o_o)) <= 1e-12 * max(1.0, np.max(np.abs(o_o)))


def test_exact_attention_rows():
    cfg, Q, K, V = _slice("mid", B=1, H=1, S=500)
    rows = np.array([0, 7, 250, 499])
    o_c = C.exact_attention_rows(Q, K, V, rows, SCALE)
    o_o = O.exact_attention_rows(Q, K, V, rows, SCALE)
    assert np.max(np.abs(o_c - o_o)) <= 1e-12 * max(1.0, np.max(np.abs(o_o)))


def test_a_planted_mistake_is_caught():
    # the same comparison fails when one statement drops the block-mean term:
    # a zero mu in the C++ call against the numpy oracle's real one
    cfg, Q, K, V = _slice("tiny")
    S = cfg["S"]
    ref = O.prepare_v_head(V, cfg["k"], cfg["iters"], 0, 0)
    qc, qs = O.quant_blocks_e4m3(Q)
    kc, ks = O.quant_blocks_e4m3(K, ref["perm"])
    rows = np.arange(S)
    o_o = O.vc_attention_rows(qc, qs, kc, ks, ref["vres"], ref["mu"], S, rows, SCALE)
    o_c, _, _ = C.vc_attention_rows(qc, qs, kc, ks, ref["vres"], np.zeros_like(ref["mu"]), S, rows, SCALE)
    assert np.max(np.abs(o_c - o_o)) > 1e-3
