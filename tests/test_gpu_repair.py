"""GPU: the V residual repair. The two planes and the kept positions are
bit-exact with the oracle's two-plane repair; O over the two planes is within the
parity bars of the oracle's VC-Attention on the repaired values."""
import numpy as np
import pytest
import torch

import oracle as O
from parity_helpers import SCALE, assert_o_close, head, make

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def va():
    from bit_fp8_attention_prep_b200 import build, vc_attn
    build.build()
    vc_attn.load()
    return vc_attn


def _oracle_slice(va, V, v, b, h, budget):
    # the oracle in lock-step with the GPU's k-means passes (same config)
    hist = va.prepare_v(v, history=True)["history"].cpu().numpy()
    H = V.shape[2]
    X = head(V, b, h)
    prep = O.prepare_v_head(X, 16, 4, 0, b * H + h, adopt=[hist[t, b, h] for t in range(4)])
    assert prep["stats"]["mismatches"] == 0
    return X, prep, O.residual_repair_planes(X, prep["perm"], prep["mu"], budget)


@pytest.mark.parametrize("budget", [0.0, 0.005, 0.05, 1.0])
def test_prepare_v_repair_bit_exact(va, budget):
    cfg, Q, K, V = make("mid", B=1, H=2, S=1000)
    v = V.cuda()
    g = va.prepare_v_repair(v, budget=budget)
    torch.cuda.synchronize()
    planes, kept = g["v_codes"].cpu().numpy(), g["kept"].cpu().numpy()
    for h in range(2):
        X, prep, (pos, p0, p1, s_v, rep) = _oracle_slice(va, V, v, 0, h, budget)
        assert np.array_equal(g["perm"][0, h].cpu().numpy(), prep["perm"])
        assert g["s_v"][0, h].item() == s_v
        assert np.array_equal(planes[0, 0, h], p0)
        assert np.array_equal(planes[1, 0, h], p1)
        assert np.array_equal(np.nonzero(kept[0, h])[0], pos)


def test_forward_repair_parity(va):
    # O over the two planes against the oracle's VC-Attention on the repaired
    # values (the accuracy gain of the repair is pinned on the oracle in fp64:
    # here the error of the FP8 probabilities and the BF16 output rounding are of
    # the same size as that gain, so only parity is asserted)
    cfg, Q, K, V = make("mid", B=1, H=2, S=1000)
    q, k, v = Q.cuda(), K.cuda(), V.cuda()
    g = va.prepare_v_repair(v, budget=0.05)
    qk = va.quant_qk(q, k, g["perm"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = va.forward_repair(qk, g, va.shape_of(q), SCALE, status=status).float().cpu().numpy()
    assert int(status.item()) == 0
    rows = np.arange(0, 1000, 11)
    for h in range(2):
        X, prep, (pos, p0, p1, s_v, rep) = _oracle_slice(va, V, v, 0, h, 0.05)
        qc, qs, kc, ks = O.quant_qk_head(head(Q, 0, h), head(K, 0, h), prep["perm"])
        assert_o_close(o[0, rows, h], O.vc_attention_rows(qc, qs, kc, ks, rep, prep["mu"], 1000, rows, SCALE))
