"""GPU: vc_attn_prepare_v_noalloc, the V-Smooth prep entry point that takes no
workspace (for callers that cannot allocate device memory themselves, e.g. a
plugin handed only its input and output buffers, or a loop that must not call
cudaMalloc), gives exactly the outputs of vc_attn_prepare_v with a caller
workspace. Its scratch is one fixed device array shared by every call and left
holding the previous call's contents, so the check runs two calls in a row on
different problems. The prep outputs are codes, a permutation and fp32 means,
compared bit for bit as everywhere else in these tests.

This file is named to be collected last: if it fails, a run that stops at the
first failure has already run every other test."""
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


def _same(a, b):
    for key in ("perm", "mu", "v_codes", "s_v", "history"):
        x, y = a[key].cpu().numpy(), b[key].cpu().numpy()
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), key


def _same_nvfp4(a, b):
    for key in ("perm", "mu", "v_codes", "v_scales", "s_v"):
        x, y = a[key].cpu().numpy(), b[key].cpu().numpy()
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), key


def test_noalloc_prep_matches_workspace_prep_on_two_calls(va):
    # the mid case fills most of the scratch; the tiny case after it must not see
    # its leftovers (the k-means sums, counts and histograms start at zero)
    cases = [("mid", dict(B=2, H=3, S=2500), 16, 4), ("tiny", {}, 4, 3)]
    for name, kw, k, iters in cases:
        cfg, Q, K, V = make(name, **kw)
        q, kk, v = Q.cuda(), K.cuda(), V.cuda()
        ref = va.prepare_v(v, k=k, iters=iters, history=True)
        got = va.prepare_v_noalloc(v, k=k, iters=iters, history=True)
        torch.cuda.synchronize()
        _same(got, ref)
        # and the attention built on it is the same
        shape = va.shape_of(q)
        o_ref = va.forward(va.quant_qk(q, kk, ref["perm"]), ref, shape, SCALE)
        o_got = va.forward(va.quant_qk(q, kk, got["perm"]), got, shape, SCALE)
        torch.cuda.synchronize()
        assert torch.equal(o_ref, o_got)


def test_noalloc_prep_other_residuals_and_modes(va):
    # the NVFP4, MX-style and per-channel residuals and the MEANONLY / NAIVE modes
    # lay the scratch out differently (one cluster, no second label buffer, an amax
    # per channel); each runs right after a mid-size VSMOOTH call has left its
    # contents in the array
    cfg, Q, K, V = make("mid", B=1, H=4, S=3000)
    v = V.cuda()
    for fmt, mode in (("nvfp4", "vsmooth"), ("e4m3", "meanonly"), ("e4m3", "naive"), ("nvfp4", "meanonly"),
                      ("e4m3c", "vsmooth"), ("mxfp4", "vsmooth")):
        va.prepare_v_noalloc(v, k=16, iters=4)            # leaves VSMOOTH scratch behind
        ref = va.prepare_v(v, k=16, iters=4, fmt=fmt, mode=mode)
        got = va.prepare_v_noalloc(v, k=16, iters=4, fmt=fmt, mode=mode)
        torch.cuda.synchronize()
        if fmt in ("nvfp4", "mxfp4"):
            _same_nvfp4(got, ref)
        else:
            for key in ("perm", "mu", "v_codes", "s_v"):
                assert np.array_equal(got[key].cpu().numpy().view(np.uint8), ref[key].cpu().numpy().view(np.uint8)), (fmt, mode, key)


def test_noalloc_rejects_problems_beyond_its_scratch(va):
    # B=1, S=73397, H=64 with 32 clusters needs about 13 MB of prep scratch. The
    # size check comes before anything touches the device, so the data pointers
    # here are placeholders that are never dereferenced.
    lib = va.load()
    sh = va.Shape(1, 73397, 64, 128, va.VC_DTYPE_BF16)
    cfg = va.VSmoothCfg(32, 4, 0, va.VC_RESIDUAL_E4M3, va.VC_MODE_VSMOOTH)
    need = lib.vc_attn_prepare_v_workspace_bytes(va.ctypes.byref(sh), va.ctypes.byref(cfg))
    assert need > va.NOALLOC_SCRATCH_BYTES
    pv = va.PreparedV(256, 256, 256, 0, 256)
    st = lib.vc_attn_prepare_v_noalloc(va.ctypes.c_void_p(256), va.ctypes.byref(sh), va.ctypes.byref(cfg),
                                       va.ctypes.byref(pv), None, None)
    assert st == va.VC_ERR_WORKSPACE
    msg = lib.vc_attn_last_error().decode()
    assert str(need) in msg and str(va.NOALLOC_SCRATCH_BYTES) in msg
