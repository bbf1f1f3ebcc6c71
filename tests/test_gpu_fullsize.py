"""GPU: parity at the benchmark's full size and launch configuration.

minimax_h56 (B=1, S=73397, H=56, D=128, the shape the headline metric is quoted
on) is drawn on the GPU with the synthetic recipe and run through the same
library calls and grids that bench.py times. For two heads (the first and the
last) the oracle recomputes the prep from the same inputs: permutation, block
means, residual codes and Q/K codes and scales must be bit-exact (k-means near
ties adopted in lock-step and counted), and the output rows it computes one by
one (a spread of 48 query rows, the last row included) must meet the O
acceptance bars. The preallocated plan (the bench's path) must give the same
output bits as the one-shot calls."""
import numpy as np
import pytest
import torch

import oracle as O
from parity_helpers import SCALE, assert_o_close, assert_prep_bit_exact
from bit_fp8_attention_prep_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def va():
    from bit_fp8_attention_prep_b200 import build, vc_attn
    build.build()
    vc_attn.load()
    return vc_attn


def test_minimax_h56_sampled_heads_and_rows(va):
    cfg, Q, K, V = synth.make_workload("minimax_h56", seed=0, device="cuda")
    B, S, H, k, iters = cfg["B"], cfg["S"], cfg["H"], cfg["k"], cfg["iters"]
    pv = va.prepare_v(V, k=k, iters=iters, history=True)
    qk = va.quant_qk(Q, K, pv["perm"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = va.forward(qk, pv, va.shape_of(Q), SCALE, 8, status=status)
    plan = va.Plan(B, S, H, k=k, iters=iters)
    o_plan = plan.run(Q, K, V)
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and int(plan.status.item()) == 0
    assert torch.equal(o.view(torch.int16), o_plan.view(torch.int16))

    rows = np.unique(np.concatenate([np.linspace(0, S - 1, 47).astype(np.int64), [S - 1]]))
    ties = 0
    for h in (0, H - 1):
        q, kk, v = (X[0, :, h].float().cpu().numpy() for X in (Q, K, V))
        adopt = [pv["history"][t, 0, h].cpu().numpy() for t in range(iters)]
        ref = O.prepare_v_head(v, k, iters, 0, h, adopt=adopt)
        qc, qs, kc, ks = O.quant_qk_head(q, kk, ref["perm"])
        ref.update(q_codes=qc, q_scales=qs, k_codes=kc, k_scales=ks)
        g = dict(perm=pv["perm"][:, h:h + 1].cpu().numpy(), mu=pv["mu"][:, h:h + 1].cpu().numpy(),
                 v_codes=pv["v_codes"][:, h:h + 1].cpu().numpy(), s_v=pv["s_v"][:, h:h + 1].cpu().numpy(),
                 v_scales=None, q_codes=qk["q_codes"][:, h:h + 1].cpu().numpy(),
                 q_scales=qk["q_scales"][:, h:h + 1].cpu().numpy(),
                 k_codes=qk["k_codes"][:, h:h + 1].cpu().numpy(),
                 k_scales=qk["k_scales"][:, h:h + 1].cpu().numpy())
        assert_prep_bit_exact(g, ref, 0, 0)
        ties += ref["stats"]["near_ties"]
        o_ref = O.vc_attention_rows(qc, qs, kc, ks, ref["vres"], ref["mu"], S, rows, SCALE, k_p=8)
        r, m = assert_o_close(o[0, rows, h].float().cpu().numpy(), o_ref)
        print(f"head {h}: rel-L2 vs oracle {r:.2e}, max-abs {m:.2e}")
    print(f"k-means near ties adopted: {ties}")
