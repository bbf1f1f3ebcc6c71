"""GPU: a problem split by heads (vc_attn_prepare_v_shard, as each rank of a
head-split multi-GPU run calls it) gives, bit for bit, those heads of the
single-call prep of the whole problem, and the attention on each shard gives
those heads of the whole problem's output. Run here as several calls on one GPU:
the shards share nothing, so the split needs no exchange between GPUs."""
import numpy as np
import pytest
import torch

from parity_helpers import SCALE, make

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def va():
    from bit_fp8_attention_prep_b200 import build, vc_attn
    build.build()
    vc_attn.load()
    return vc_attn


@pytest.mark.parametrize("B,H,S,world", [(1, 7, 1500, 2), (2, 5, 777, 3)])
def test_head_shards_equal_the_whole_problem(va, B, H, S, world):
    cfg, Q, K, V = make("mid", B=B, H=H, S=S)
    q, k, v = Q.cuda(), K.cuda(), V.cuda()
    whole = va.prepare_v(v)
    o_whole = va.forward(va.quant_qk(q, k, whole["perm"]), whole, va.shape_of(q), SCALE)
    for r in range(world):
        h0, h1 = va.head_range(H, r, world)
        qs, ks, vs = (X[:, :, h0:h1].contiguous() for X in (q, k, v))
        part = va.prepare_v(vs, h_base=h0, H_total=H)
        o_part = va.forward(va.quant_qk(qs, ks, part["perm"]), part, va.shape_of(qs), SCALE)
        torch.cuda.synchronize()
        for key in ("perm", "mu", "v_codes", "s_v"):
            a = part[key].cpu().numpy()
            b = whole[key][:, h0:h1].cpu().numpy()
            assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), (r, key)
        assert torch.equal(o_part.view(torch.int16), o_whole[:, :, h0:h1].contiguous().view(torch.int16)), r


def test_shard_plan_matches_the_calls(va):
    # the preallocated plan of one shard gives the bytes of the separate calls
    cfg, Q, K, V = make("mid", B=1, H=6, S=900)
    h0, h1 = 2, 5
    q, k, v = (X[:, :, h0:h1].contiguous().cuda() for X in (Q, K, V))
    plan = va.Plan(1, 900, h1 - h0, h_base=h0, H_total=6)
    o_plan = plan.run(q, k, v).clone()
    pv = va.prepare_v(v, h_base=h0, H_total=6)
    o_calls = va.forward(va.quant_qk(q, k, pv["perm"]), pv, va.shape_of(q), SCALE)
    torch.cuda.synchronize()
    assert int(plan.status.item()) == 0
    assert torch.equal(o_plan.view(torch.int16), o_calls.view(torch.int16))
