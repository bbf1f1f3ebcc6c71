"""Shared helpers of the GPU parity tests: run the CUDA path through the binding,
run the oracle on the same seeded inputs, compare."""
import math

import numpy as np
import torch

import oracle as O
from bit_fp8_attention_prep_b200 import synth

SCALE = 1.0 / math.sqrt(128)
REL_L2_TOL = 2e-3      # O vs the oracle, relative L2 over the compared elements
MAX_ABS_TOL = 1e-2     # O vs the oracle, max absolute difference


def head(X, b, h):
    return X[b, :, h].float().numpy()


def gpu_pipeline(va, Q, K, V, k, iters, seed=0, fmt="e4m3", k_p=8, history=True, attend=True, mode="vsmooth",
                 smooth_k=False):
    """Q, K, V CPU tensors [B,S,H,128] -> dict of GPU outputs copied to the CPU."""
    q, kk, v = Q.cuda(), K.cuda(), V.cuda()
    pv = va.prepare_v(v, k=k, iters=iters, seed=seed, fmt=fmt, history=history, mode=mode)
    qk = va.quant_qk(q, kk, pv["perm"], smooth_k=smooth_k)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = va.forward(qk, pv, va.shape_of(q), SCALE, k_p, status=status) if attend else None
    torch.cuda.synchronize()
    cpu = lambda t: None if t is None else t.cpu().numpy()
    return dict(perm=cpu(pv["perm"]), mu=cpu(pv["mu"]), v_codes=cpu(pv["v_codes"]), v_scales=cpu(pv["v_scales"]),
                s_v=cpu(pv["s_v"]), history=cpu(pv["history"]), q_codes=cpu(qk["q_codes"]),
                q_scales=cpu(qk["q_scales"]), k_codes=cpu(qk["k_codes"]), k_scales=cpu(qk["k_scales"]),
                o=None if o is None else o.float().cpu().numpy(), status=int(status.item()),
                k_mean=cpu(qk.get("k_mean")))


def oracle_head(g, Q, K, V, b, h, k, iters, seed=0, fmt="e4m3", smooth_k=False):
    """Oracle prep + quantisation for slice (b, h), in lock-step with the GPU's
    per-pass k-means assignments (near ties adopted and counted)."""
    H = V.shape[2]
    adopt = None if g.get("history") is None else [g["history"][t, b, h] for t in range(iters)]
    prep = O.prepare_v_head(head(V, b, h), k, iters, seed, b * H + h, fmt=fmt, adopt=adopt)
    qc, qs, kc, ks = O.quant_qk_head(head(Q, b, h), head(K, b, h), prep["perm"], smooth=smooth_k)
    prep.update(q_codes=qc, q_scales=qs, k_codes=kc, k_scales=ks)
    return prep


def assert_prep_bit_exact(g, ref, b, h, fmt="e4m3"):
    assert ref["stats"]["mismatches"] == 0, ref["stats"]
    assert np.array_equal(g["perm"][b, h], ref["perm"])
    assert np.array_equal(g["mu"][b, h].view(np.uint32), ref["mu"].view(np.uint32))
    if fmt == "mxfp4":
        # the oracle keeps one code per element and exponents as (D, S_pad/32);
        # the library packs two codes a byte and groups exponents per block
        c = ref["v_codes"]
        assert np.array_equal(g["v_codes"][b, h], (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8))
        e8 = ref["v_scales"]
        assert np.array_equal(g["v_scales"][b, h], e8.reshape(e8.shape[0], -1, 4).transpose(1, 0, 2))
        assert g["s_v"][b, h] == 1.0
    else:
        assert np.array_equal(g["v_codes"][b, h], ref["v_codes"])
    if fmt == "e4m3":
        assert g["s_v"][b, h] == ref["s_v"]
    elif fmt == "e4m3c":
        assert np.array_equal(g["s_v"][b, h].view(np.uint32), ref["s_v"].view(np.uint32))
    elif fmt == "nvfp4":
        assert np.array_equal(g["v_scales"][b, h], ref["v_scales"])
        assert g["s_v"][b, h] == ref["g"]
    assert np.array_equal(g["q_codes"][b, h], ref["q_codes"])
    assert np.array_equal(g["k_codes"][b, h], ref["k_codes"])
    assert np.array_equal(g["q_scales"][b, h].view(np.uint32), ref["q_scales"].view(np.uint32))
    assert np.array_equal(g["k_scales"][b, h].view(np.uint32), ref["k_scales"].view(np.uint32))


def oracle_rows(ref, S, rows, k_p=8):
    return O.vc_attention_rows(ref["q_codes"], ref["q_scales"], ref["k_codes"], ref["k_scales"], ref["vres"],
                               ref["mu"], S, rows, SCALE, k_p=k_p)


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def bf16_ulp(x):
    """Spacing of BF16 numbers at |x| (8 significant bits)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return np.exp2(e - 7)


def assert_o_close(o_gpu, o_ref):
    """O within the acceptance bars. Both sides are BF16 (o_ref is the oracle's
    fp64 output rounded to BF16): rel-L2 <= 2e-3 over the compared elements, and
    per element |diff| <= max(1e-2, one BF16 ulp of the reference) -- above
    |O| = 2.56 one BF16 step (2^-6 at [2, 4)) is coarser than 1e-2, so two
    correctly computed outputs on either side of a rounding point differ by it."""
    ref = O.bf16_round(o_ref)
    r = rel_l2(o_gpu, ref)
    diff = np.abs(o_gpu - ref)
    m = float(np.max(diff))
    over = diff > np.maximum(MAX_ABS_TOL, bf16_ulp(ref))
    assert r <= REL_L2_TOL and not over.any(), (r, m, int(over.sum()))
    return r, m


def make(name, **kw):
    return synth.make_workload(name, **kw)
