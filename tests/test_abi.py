"""The C-ABI library loads, exports every symbol its headers declare, and its
host-side validation answers without a GPU (CPU only)."""
import ctypes
import os
import re

import pytest
import torch

from bit_fp8_attention_prep_b200 import build, vc_attn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return vc_attn.load()


def _declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vc_attn_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared("vc_attn.h") + _declared("vc_attn_testing.h")
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert set(_declared("vc_attn.h")) == set(vc_attn.ABI_SYMBOLS)
    assert set(_declared("vc_attn_testing.h")) == set(vc_attn.TEST_SYMBOLS)


def test_version_and_last_error(lib):
    assert lib.vc_attn_version() == 100
    assert lib.vc_attn_last_error() == b""


def _shape(B=1, S=256, H=2, D=128, dt=vc_attn.VC_DTYPE_BF16):
    return vc_attn.Shape(B, S, H, D, dt)


def _cfg(k=4, iters=3, fmt=0, mode=0):
    return vc_attn.VSmoothCfg(k, iters, 0, fmt, mode)


def test_workspace_bytes_and_validation(lib):
    ok = lib.vc_attn_prepare_v_workspace_bytes(ctypes.byref(_shape()), ctypes.byref(_cfg()))
    assert ok > 0 and ok % 256 == 0
    big = lib.vc_attn_prepare_v_workspace_bytes(ctypes.byref(_shape(S=73397, H=56)), ctypes.byref(_cfg(k=16)))
    assert big > ok
    for sh in (_shape(D=64), _shape(S=0), _shape(H=0), _shape(dt=7), _shape(S=1 << 20, H=200)):
        assert lib.vc_attn_prepare_v_workspace_bytes(ctypes.byref(sh), ctypes.byref(_cfg())) == 0
    for cfg in (_cfg(k=0), _cfg(k=33), _cfg(iters=0), _cfg(fmt=4), _cfg(fmt=-1), _cfg(mode=5)):
        assert lib.vc_attn_prepare_v_workspace_bytes(ctypes.byref(_shape()), ctypes.byref(cfg)) == 0


def test_calls_reject_bad_arguments_before_any_launch(lib):
    sh = _shape(D=64)
    pv = vc_attn.PreparedV(16, 16, 16, 16, 16)
    st = lib.vc_attn_prepare_v(ctypes.c_void_p(16), ctypes.byref(sh), ctypes.byref(_cfg()), ctypes.byref(pv),
                               ctypes.c_void_p(256), 1 << 20, None, None)
    assert st == vc_attn.VC_ERR_INVALID_ARG
    assert b"D must be 128" in lib.vc_attn_last_error()
    # NULL output pointer
    pv0 = vc_attn.PreparedV(0, 16, 16, 16, 16)
    st = lib.vc_attn_prepare_v(ctypes.c_void_p(16), ctypes.byref(_shape()), ctypes.byref(_cfg()),
                               ctypes.byref(pv0), ctypes.c_void_p(256), 1 << 20, None, None)
    assert st == vc_attn.VC_ERR_INVALID_ARG
    # misaligned input
    st = lib.vc_attn_prepare_v(ctypes.c_void_p(18), ctypes.byref(_shape()), ctypes.byref(_cfg()),
                               ctypes.byref(pv), ctypes.c_void_p(256), 1 << 20, None, None)
    assert st == vc_attn.VC_ERR_INVALID_ARG and b"aligned" in lib.vc_attn_last_error()
    # workspace too small
    st = lib.vc_attn_prepare_v(ctypes.c_void_p(16), ctypes.byref(_shape()), ctypes.byref(_cfg()),
                               ctypes.byref(pv), ctypes.c_void_p(256), 64, None, None)
    assert st == vc_attn.VC_ERR_WORKSPACE
    qk = vc_attn.QKFP8(16, 16, 16, 16)
    st = lib.vc_attn_quant_qk(ctypes.c_void_p(16), None, ctypes.byref(_shape()), ctypes.c_void_p(16),
                              ctypes.byref(qk), None)
    assert st == vc_attn.VC_ERR_INVALID_ARG
    for kp, scale in ((9, 0.088), (-1, 0.088), (8, 0.0), (8, float("nan"))):
        st = lib.vc_attn_forward(ctypes.byref(qk), ctypes.byref(pv), ctypes.byref(_shape()), scale, kp,
                                 ctypes.c_void_p(16), None, None)
        assert st == vc_attn.VC_ERR_INVALID_ARG
    for fn in (lib.vc_attn_test_e4m3_round, lib.vc_attn_test_e2m1_round):
        assert fn(None, None, -1, None) == vc_attn.VC_ERR_INVALID_ARG
        assert fn(None, None, 0, None) == vc_attn.VC_OK
    assert lib.vc_attn_test_bounded_wait(None, 1000, None) == vc_attn.VC_ERR_INVALID_ARG


def test_nvfp4_forward_workspace_size_and_checks(lib):
    sz = lib.vc_attn_forward_nvfp4v_workspace_bytes
    assert sz(ctypes.byref(_shape(B=1, S=256, H=2))) == 2 * 1 * 2 * 128 * 256
    assert sz(ctypes.byref(_shape(B=2, S=300, H=3))) == 2 * 2 * 3 * 128 * 384  # S padded to 128
    assert sz(ctypes.byref(_shape(D=64))) == 0
    qk = vc_attn.QKFP8(16, 16, 16, 16)
    pv = vc_attn.PreparedV(16, 16, 16, 16, 16)
    need = sz(ctypes.byref(_shape()))
    for ws, nbytes in ((None, need), (ctypes.c_void_p(256), need - 1)):
        st = lib.vc_attn_forward_nvfp4v(ctypes.byref(qk), ctypes.byref(pv), ctypes.byref(_shape()), 0.088, 8,
                                        ctypes.c_void_p(16), ws, nbytes, None, None)
        assert st == vc_attn.VC_ERR_WORKSPACE
        assert str(need).encode() in lib.vc_attn_last_error()
    st = lib.vc_attn_forward_nvfp4v(ctypes.byref(qk), ctypes.byref(pv), ctypes.byref(_shape()), 0.088, 8,
                                    ctypes.c_void_p(16), ctypes.c_void_p(264), need, None, None)
    assert st == vc_attn.VC_ERR_INVALID_ARG and b"aligned" in lib.vc_attn_last_error()
    pv_noscale = vc_attn.PreparedV(16, 16, 16, 0, 16)
    st = lib.vc_attn_forward_nvfp4v(ctypes.byref(qk), ctypes.byref(pv_noscale), ctypes.byref(_shape()), 0.088, 8,
                                    ctypes.c_void_p(16), ctypes.c_void_p(256), need, None, None)
    assert st == vc_attn.VC_ERR_INVALID_ARG


def test_run_host_workspace_and_validation(lib):
    sh, cfg = _shape(S=1000, H=5), _cfg(k=16, iters=4)
    ws = [lib.vc_attn_run_host_workspace_bytes(ctypes.byref(sh), ctypes.byref(cfg), c) for c in (1, 2, 5, 9)]
    assert all(w > 0 and w % 256 == 0 for w in ws)
    assert ws[0] < ws[1] < ws[2] == ws[3]          # head_chunk above H means H
    # two slots of Q, K, V, O chunk buffers are part of it
    assert ws[1] > 8 * 1000 * 2 * 256
    assert lib.vc_attn_run_host_workspace_bytes(ctypes.byref(sh), ctypes.byref(cfg), 0) == 0
    assert lib.vc_attn_run_host_workspace_bytes(ctypes.byref(_shape(D=64)), ctypes.byref(cfg), 2) == 0
    nv = lib.vc_attn_run_host_workspace_bytes(ctypes.byref(sh), ctypes.byref(_cfg(k=16, iters=4, fmt=1)), 2)
    assert nv > ws[1]                               # plus the NVFP4 scales and planes
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    for args, code in (
        ((p, p, p, ctypes.byref(sh), ctypes.byref(cfg), 0.088, 8, p, 0, None, 0, None, None), vc_attn.VC_ERR_INVALID_ARG),
        ((p, p, p, ctypes.byref(sh), ctypes.byref(cfg), -1.0, 8, p, 2, None, 0, None, None), vc_attn.VC_ERR_INVALID_ARG),
        ((p, p, p, ctypes.byref(sh), ctypes.byref(cfg), 0.088, 9, p, 2, None, 0, None, None), vc_attn.VC_ERR_INVALID_ARG),
        ((None, p, p, ctypes.byref(sh), ctypes.byref(cfg), 0.088, 8, p, 2, None, 0, None, None), vc_attn.VC_ERR_INVALID_ARG),
        ((p, p, p, ctypes.byref(sh), ctypes.byref(cfg), 0.088, 8, p, 2, None, 0, None, None), vc_attn.VC_ERR_WORKSPACE),
        ((p, p, p, ctypes.byref(sh), ctypes.byref(cfg), 0.088, 8, p, 2, p, 64, None, None), vc_attn.VC_ERR_WORKSPACE),
    ):
        assert lib.vc_attn_run_host(*args) == code
        assert lib.vc_attn_last_error() != b""


def test_residual_energy_validation(lib):
    # argument checks run on the host before anything is launched
    sh = _shape(S=1000, H=5)
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    odd = ctypes.c_void_p(p.value + 8)
    for args in (
        (p, ctypes.byref(sh), None, None, None, None),              # energy NULL
        (None, ctypes.byref(sh), None, None, p, None),              # v NULL
        (p, ctypes.byref(_shape(D=64)), None, None, p, None),       # D != 128
        (p, ctypes.byref(_shape(S=0)), None, None, p, None),        # empty sequence
        (odd, ctypes.byref(sh), None, None, p, None),               # misaligned v
        (p, ctypes.byref(sh), odd, None, p, None),                  # misaligned perm
    ):
        assert lib.vc_attn_residual_energy(*args) == vc_attn.VC_ERR_INVALID_ARG
        assert lib.vc_attn_last_error() != b""
    v = torch.zeros(1, 300, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        vc_attn.residual_energy(v, perm=torch.zeros(1, 2, 299, dtype=torch.int32))
    with pytest.raises(ValueError):
        vc_attn.residual_energy(v, mu=torch.zeros(1, 2, 3, 128, dtype=torch.float64))


def test_quant_qk_smoothk_workspace_and_validation(lib):
    sh = _shape(B=2, S=1000, H=5)
    assert lib.vc_attn_quant_qk_smoothk_workspace_bytes(ctypes.byref(sh)) == 2 * 5 * 128 * 12
    assert lib.vc_attn_quant_qk_smoothk_workspace_bytes(ctypes.byref(_shape(D=64))) == 0
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    qk = vc_attn.QKFP8(p, p, p, p)
    odd = ctypes.c_void_p(p.value + 4)
    need = 2 * 5 * 128 * 12
    for args, code in (
        ((p, p, ctypes.byref(sh), p, ctypes.byref(qk), None, need, None, None), vc_attn.VC_ERR_WORKSPACE),
        ((p, p, ctypes.byref(sh), p, ctypes.byref(qk), p, need - 1, None, None), vc_attn.VC_ERR_WORKSPACE),
        ((p, None, ctypes.byref(sh), p, ctypes.byref(qk), p, need, None, None), vc_attn.VC_ERR_INVALID_ARG),
        ((p, p, ctypes.byref(sh), None, ctypes.byref(qk), p, need, None, None), vc_attn.VC_ERR_INVALID_ARG),
        ((p, p, ctypes.byref(sh), p, ctypes.byref(qk), odd, need, None, None), vc_attn.VC_ERR_INVALID_ARG),
        ((p, p, ctypes.byref(sh), p, ctypes.byref(qk), p, need, odd, None), vc_attn.VC_ERR_INVALID_ARG),
        ((p, p, ctypes.byref(_shape(S=0)), p, ctypes.byref(qk), p, need, None, None), vc_attn.VC_ERR_INVALID_ARG),
    ):
        assert lib.vc_attn_quant_qk_smoothk(*args) == code
        assert lib.vc_attn_last_error() != b""


def test_too_many_slices_is_refused_before_any_launch(lib):
    # B*H above 65535 fits the element limit when S <= 128 but not one grid row
    # per slice: every entry point refuses it on the host
    sh = _shape(B=2, S=100, H=40000)
    cfg = _cfg(k=4, iters=2)
    assert lib.vc_attn_prepare_v_workspace_bytes(ctypes.byref(sh), ctypes.byref(cfg)) == 0
    assert lib.vc_attn_quant_qk_smoothk_workspace_bytes(ctypes.byref(sh)) == 0
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    assert lib.vc_attn_residual_energy(p, ctypes.byref(sh), None, None, p, None) == vc_attn.VC_ERR_UNSUPPORTED
    assert b"65535" in lib.vc_attn_last_error()
    ok = _shape(B=1, S=100, H=65535)
    assert lib.vc_attn_quant_qk_smoothk_workspace_bytes(ctypes.byref(ok)) == 65535 * 128 * 12


def test_prepare_v_repair_workspace_and_validation(lib):
    sh, cfg = _shape(S=1000, H=5), _cfg(k=16, iters=4)
    base = lib.vc_attn_prepare_v_workspace_bytes(ctypes.byref(sh), ctypes.byref(cfg))
    need = lib.vc_attn_prepare_v_repair_workspace_bytes(ctypes.byref(sh), ctypes.byref(cfg))
    assert need >= base + 5 * 1000 * 4 + 5 * 8 and need % 256 == 0
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    pv = vc_attn.PreparedV(p, p, p, None, p)
    for args, code in (
        ((p, ctypes.byref(sh), ctypes.byref(_cfg(k=16, iters=4, fmt=1)), 0.005, ctypes.byref(pv), None, p, need, None),
         vc_attn.VC_ERR_UNSUPPORTED),
        ((p, ctypes.byref(sh), ctypes.byref(cfg), -0.1, ctypes.byref(pv), None, p, need, None),
         vc_attn.VC_ERR_INVALID_ARG),
        ((p, ctypes.byref(sh), ctypes.byref(cfg), float("nan"), ctypes.byref(pv), None, p, need, None),
         vc_attn.VC_ERR_INVALID_ARG),
        ((p, ctypes.byref(sh), ctypes.byref(cfg), 0.005, ctypes.byref(pv), None, p, need - 1, None),
         vc_attn.VC_ERR_WORKSPACE),
        ((p, ctypes.byref(sh), ctypes.byref(cfg), 0.005, ctypes.byref(pv), None, None, need, None),
         vc_attn.VC_ERR_WORKSPACE),
    ):
        assert lib.vc_attn_prepare_v_repair(*args) == code
        assert lib.vc_attn_last_error() != b""


def test_no_fallback_without_the_library_or_a_gpu(monkeypatch):
    # the binding raises when libvcattn.so is missing ...
    monkeypatch.setattr(vc_attn, "_lib", None)
    monkeypatch.setattr(vc_attn, "LIB_PATH", "/nonexistent/libvcattn.so")
    with pytest.raises(RuntimeError, match="missing"):
        vc_attn.load()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour on a host without a GPU")
def test_product_path_raises_on_a_host_without_gpu():
    # ... and on a machine without a GPU the whole path raises (torch's stream
    # lookup or the library's device check, both RuntimeError) instead of computing
    q = torch.zeros(1, 256, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError):
        vc_attn.attention(q, q, q)


def test_package_never_imports_the_oracle():
    pkg = os.path.dirname(vc_attn.__file__)
    for root, _, files in os.walk(pkg):
        for name in files:
            if name.endswith(".py"):
                src = open(os.path.join(root, name)).read()
                assert not re.search(r"^\s*(import oracle|from oracle)", src, re.M), name


def test_noalloc_prep_checks_arguments_before_the_device(lib):
    # vc_attn_prepare_v_noalloc answers a bad argument exactly as vc_attn_prepare_v
    # does, before it looks at the device or its fixed scratch: on this host there
    # is no GPU, so any device step would give VC_ERR_CUDA or VC_ERR_UNSUPPORTED.
    pv = vc_attn.PreparedV(16, 16, 16, 16, 16)
    st = lib.vc_attn_prepare_v_noalloc(ctypes.c_void_p(16), ctypes.byref(_shape(D=64)), ctypes.byref(_cfg()),
                                       ctypes.byref(pv), None, None)
    assert st == vc_attn.VC_ERR_INVALID_ARG and b"D must be 128" in lib.vc_attn_last_error()
    st = lib.vc_attn_prepare_v_noalloc(None, ctypes.byref(_shape()), ctypes.byref(_cfg()), ctypes.byref(pv),
                                       None, None)
    assert st == vc_attn.VC_ERR_INVALID_ARG and b"non-NULL" in lib.vc_attn_last_error()
    st = lib.vc_attn_prepare_v_noalloc(ctypes.c_void_p(18), ctypes.byref(_shape()), ctypes.byref(_cfg()),
                                       ctypes.byref(pv), None, None)
    assert st == vc_attn.VC_ERR_INVALID_ARG and b"aligned" in lib.vc_attn_last_error()
    pv_nv = vc_attn.PreparedV(16, 16, 16, 0, 16)   # NVFP4 without v_scales
    st = lib.vc_attn_prepare_v_noalloc(ctypes.c_void_p(16), ctypes.byref(_shape()),
                                       ctypes.byref(_cfg(fmt=vc_attn.VC_RESIDUAL_NVFP4)), ctypes.byref(pv_nv),
                                       None, None)
    assert st == vc_attn.VC_ERR_INVALID_ARG and b"v_scales" in lib.vc_attn_last_error()
    # valid arguments: only now does the call reach the device, which this host lacks
    st = lib.vc_attn_prepare_v_noalloc(ctypes.c_void_p(16), ctypes.byref(_shape()), ctypes.byref(_cfg()),
                                       ctypes.byref(pv), None, None)
    assert st in (vc_attn.VC_ERR_CUDA, vc_attn.VC_ERR_UNSUPPORTED)


def test_shard_prep_rejects_head_ranges_outside_the_problem(lib):
    pv = vc_attn.PreparedV(16, 16, 16, 16, 16)
    for h_base, H_total in ((-1, 8), (7, 8), (0, 1), (3, 4)):   # local H = 2
        st = lib.vc_attn_prepare_v_shard(ctypes.c_void_p(16), ctypes.byref(_shape(H=2)), ctypes.byref(_cfg()),
                                         h_base, H_total, ctypes.byref(pv), ctypes.c_void_p(256), 1 << 20, None)
        assert st == vc_attn.VC_ERR_INVALID_ARG and b"H_total" in lib.vc_attn_last_error()
