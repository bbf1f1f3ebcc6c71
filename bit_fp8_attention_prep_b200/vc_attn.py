"""Thin Python binding of libvcattn.so (the C ABI in include/vc_attn.h).

Argument marshalling only: torch provides device memory and the current CUDA
stream; every step of the computation runs in the library's CUDA kernels. There
is no fallback: if the library is missing or the device is not an sm_100 GPU,
the calls raise.
"""
import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libvcattn.so")

VC_OK, VC_ERR_INVALID_ARG, VC_ERR_UNSUPPORTED, VC_ERR_WORKSPACE, VC_ERR_CUDA, VC_ERR_TIMEOUT = range(6)
STATUS_NAMES = ["VC_OK", "VC_ERR_INVALID_ARG", "VC_ERR_UNSUPPORTED", "VC_ERR_WORKSPACE", "VC_ERR_CUDA",
                "VC_ERR_TIMEOUT"]
VC_DTYPE_F16, VC_DTYPE_BF16 = 0, 1
VC_RESIDUAL_E4M3, VC_RESIDUAL_NVFP4, VC_RESIDUAL_E4M3_PER_CHANNEL, VC_RESIDUAL_MXFP4 = 0, 1, 2, 3
# residual formats by name: "e4m3" (one scale per head), "nvfp4", "e4m3c" (one
# E4M3 scale per channel), "mxfp4" (E2M1 with a power of two per 32 tokens)
_FMTS = {"e4m3": VC_RESIDUAL_E4M3, "nvfp4": VC_RESIDUAL_NVFP4, "e4m3c": VC_RESIDUAL_E4M3_PER_CHANNEL,
         "mxfp4": VC_RESIDUAL_MXFP4}
VC_MODE_VSMOOTH, VC_MODE_MEANONLY, VC_MODE_NAIVE = 0, 1, 2
_MODES = {"vsmooth": VC_MODE_VSMOOTH, "meanonly": VC_MODE_MEANONLY, "naive": VC_MODE_NAIVE}

# every symbol declared in include/vc_attn.h and include/vc_attn_testing.h
ABI_SYMBOLS = [
    "vc_attn_version", "vc_attn_last_error", "vc_attn_launch_count", "vc_attn_prepare_v_workspace_bytes",
    "vc_attn_prepare_v",
    "vc_attn_quant_qk", "vc_attn_forward", "vc_attn_forward_nvfp4v_workspace_bytes", "vc_attn_forward_nvfp4v",
    "vc_attn_prepare_v_noalloc", "vc_attn_run_host_workspace_bytes", "vc_attn_run_host",
    "vc_attn_residual_energy", "vc_attn_quant_qk_smoothk_workspace_bytes", "vc_attn_quant_qk_smoothk",
    "vc_attn_prepare_v_repair_workspace_bytes", "vc_attn_prepare_v_repair", "vc_attn_forward_repair",
    "vc_attn_forward_e4m3_per_channel", "vc_attn_forward_mxfp4v", "vc_attn_prepare_v_shard",
]
NOALLOC_SCRATCH_BYTES = 12 << 20  # VC_ATTN_NOALLOC_SCRATCH_BYTES
TEST_SYMBOLS = ["vc_attn_test_e4m3_round", "vc_attn_test_e2m1_round", "vc_attn_test_expcast",
                "vc_attn_test_bounded_wait", "vc_attn_test_forward_exp2"]


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("S", ctypes.c_int32), ("H", ctypes.c_int32), ("D", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


class VSmoothCfg(ctypes.Structure):
    _fields_ = [("k", ctypes.c_int32), ("iters", ctypes.c_int32), ("seed", ctypes.c_uint64),
                ("residual_fmt", ctypes.c_int32), ("mode", ctypes.c_int32)]


class PreparedV(ctypes.Structure):
    _fields_ = [("perm", ctypes.c_void_p), ("mu", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("v_scales", ctypes.c_void_p), ("s_v", ctypes.c_void_p)]


class QKFP8(ctypes.Structure):
    _fields_ = [("q_codes", ctypes.c_void_p), ("q_scales", ctypes.c_void_p), ("k_codes", ctypes.c_void_p),
                ("k_scales", ctypes.c_void_p)]


class VCError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS_NAMES[status] if 0 <= status < 6 else status}: {msg}")
        self.status = status


_lib = None


def load():
    """Load libvcattn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m bit_fp8_attention_prep_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, u64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    P = ctypes.POINTER
    lib.vc_attn_version.restype = i32
    lib.vc_attn_last_error.restype = ctypes.c_char_p
    lib.vc_attn_launch_count.restype = u64
    lib.vc_attn_launch_count.argtypes = []
    lib.vc_attn_prepare_v_workspace_bytes.restype = sz
    lib.vc_attn_prepare_v_workspace_bytes.argtypes = [P(Shape), P(VSmoothCfg)]
    lib.vc_attn_prepare_v.restype = i32
    lib.vc_attn_prepare_v.argtypes = [vp, P(Shape), P(VSmoothCfg), P(PreparedV), vp, sz, vp, vp]
    lib.vc_attn_prepare_v_shard.restype = i32
    lib.vc_attn_prepare_v_shard.argtypes = [vp, P(Shape), P(VSmoothCfg), i32, i32, P(PreparedV), vp, sz, vp]
    lib.vc_attn_prepare_v_noalloc.restype = i32
    lib.vc_attn_prepare_v_noalloc.argtypes = [vp, P(Shape), P(VSmoothCfg), P(PreparedV), vp, vp]
    lib.vc_attn_quant_qk.restype = i32
    lib.vc_attn_quant_qk.argtypes = [vp, vp, P(Shape), vp, P(QKFP8), vp]
    lib.vc_attn_forward.restype = i32
    lib.vc_attn_forward.argtypes = [P(QKFP8), P(PreparedV), P(Shape), ctypes.c_float, i32, vp, vp, vp]
    lib.vc_attn_forward_nvfp4v_workspace_bytes.restype = sz
    lib.vc_attn_forward_nvfp4v_workspace_bytes.argtypes = [P(Shape)]
    lib.vc_attn_forward_nvfp4v.restype = i32
    lib.vc_attn_forward_nvfp4v.argtypes = [P(QKFP8), P(PreparedV), P(Shape), ctypes.c_float, i32, vp, vp, sz,
                                           vp, vp]
    lib.vc_attn_run_host_workspace_bytes.restype = sz
    lib.vc_attn_run_host_workspace_bytes.argtypes = [P(Shape), P(VSmoothCfg), i32]
    lib.vc_attn_run_host.restype = i32
    lib.vc_attn_run_host.argtypes = [vp, vp, vp, P(Shape), P(VSmoothCfg), ctypes.c_float, i32, vp, i32, vp, sz,
                                     vp, vp]
    lib.vc_attn_quant_qk_smoothk_workspace_bytes.restype = sz
    lib.vc_attn_quant_qk_smoothk_workspace_bytes.argtypes = [P(Shape)]
    lib.vc_attn_quant_qk_smoothk.restype = i32
    lib.vc_attn_quant_qk_smoothk.argtypes = [vp, vp, P(Shape), vp, P(QKFP8), vp, sz, vp, vp]
    lib.vc_attn_prepare_v_repair_workspace_bytes.restype = sz
    lib.vc_attn_prepare_v_repair_workspace_bytes.argtypes = [P(Shape), P(VSmoothCfg)]
    lib.vc_attn_prepare_v_repair.restype = i32
    lib.vc_attn_prepare_v_repair.argtypes = [vp, P(Shape), P(VSmoothCfg), ctypes.c_double, P(PreparedV), vp, vp,
                                             sz, vp]
    for name in ("vc_attn_forward_e4m3_per_channel", "vc_attn_forward_mxfp4v"):
        getattr(lib, name).restype = i32
        getattr(lib, name).argtypes = [P(QKFP8), P(PreparedV), P(Shape), ctypes.c_float, i32, vp, vp, vp]
    lib.vc_attn_forward_repair.restype = i32
    lib.vc_attn_forward_repair.argtypes = [P(QKFP8), P(PreparedV), P(Shape), ctypes.c_float, i32, vp, vp, vp]
    lib.vc_attn_residual_energy.restype = i32
    lib.vc_attn_residual_energy.argtypes = [vp, P(Shape), vp, vp, vp, vp]
    lib.vc_attn_test_e4m3_round.restype = i32
    lib.vc_attn_test_e4m3_round.argtypes = [vp, vp, i64, vp]
    lib.vc_attn_test_e2m1_round.restype = i32
    lib.vc_attn_test_e2m1_round.argtypes = [vp, vp, i64, vp]
    lib.vc_attn_test_expcast.restype = i32
    lib.vc_attn_test_expcast.argtypes = [vp, vp, vp, i32, vp, i64, i32, vp]
    lib.vc_attn_test_bounded_wait.restype = i32
    lib.vc_attn_test_bounded_wait.argtypes = [vp, u64, vp]
    lib.vc_attn_test_forward_exp2.restype = i32
    lib.vc_attn_test_forward_exp2.argtypes = [P(QKFP8), P(PreparedV), P(Shape), ctypes.c_float, i32, vp, vp, vp]
    _lib = lib
    return lib


def _check(status):
    if status != VC_OK:
        raise VCError(status, load().vc_attn_last_error().decode())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def shape_of(x):
    """vc_shape_t for a [B,S,H,128] or [S,H,128] FP16/BF16 tensor."""
    if x.dim() == 3:
        B, (S, H, D) = 1, x.shape
    elif x.dim() == 4:
        B, S, H, D = x.shape
    else:
        raise ValueError("expected [S,H,128] or [B,S,H,128]")
    if x.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("Q, K, V must be float16 or bfloat16")
    if not x.is_contiguous():
        raise ValueError("Q, K, V must be contiguous")
    return Shape(B, S, H, D, VC_DTYPE_BF16 if x.dtype == torch.bfloat16 else VC_DTYPE_F16)


def num_blocks(S):
    return (S + 127) // 128


def _fmt_code(fmt):
    if fmt not in _FMTS:
        raise ValueError(f"fmt must be one of {sorted(_FMTS)} (got {fmt!r})")
    return _FMTS[fmt]


def _prepared_buffers(B, S, H, fmt, dev):
    """The caller-owned outputs of the prep for one residual format (layouts as
    in vc_prepared_v_t)."""
    nb = num_blocks(S)
    Sp = nb * 128
    e = lambda shp, dt: torch.empty(shp, dtype=dt, device=dev)
    out = dict(perm=e((B, H, S), torch.int32), mu=e((B, H, nb, 128), torch.float32), fmt=fmt,
               s_v=e((B, H, 128) if fmt == "e4m3c" else (B, H), torch.float32))
    if fmt == "nvfp4":
        out["v_codes"], out["v_scales"] = e((B, H, 128, Sp // 2), torch.uint8), e((B, H, 128, Sp // 16), torch.uint8)
    elif fmt == "mxfp4":
        out["v_codes"], out["v_scales"] = e((B, H, 128, Sp // 2), torch.uint8), e((B, H, nb, 128, 4), torch.uint8)
    else:
        out["v_codes"], out["v_scales"] = e((B, H, 128, Sp), torch.uint8), None
    return out


def head_range(H, rank, world):
    """Heads [h0, h1) of rank ``rank`` when a problem of H heads is split by heads
    over ``world`` ranks: contiguous ranges, sizes differing by at most one, that
    tile [0, H) in rank order."""
    if not (0 <= rank < world):
        raise ValueError("rank must be in [0, world)")
    return (H * rank) // world, (H * (rank + 1)) // world


def seed_slice_index(b, h, H):
    """Index of slice (b, h) of a problem with H heads: the k-means seed's input
    (slice i is seeded with seed ^ (0x9E3779B97F4A7C15 * (i + 1)))."""
    return b * H + h


def prepare_v(v, k=16, iters=4, seed=0, fmt="e4m3", mode="vsmooth", history=False, h_base=0, H_total=None):
    """V-Smooth prep of V (device tensor). Returns a dict of the caller-owned
    outputs (perm, mu, v_codes, v_scales, s_v; plus the per-pass assignments
    when ``history``). With ``H_total``, ``v`` holds heads [h_base, h_base + H)
    of a problem with H_total heads (vc_attn_prepare_v_shard): the outputs are
    those heads of the whole problem's prep, bit for bit."""
    lib = load()
    sh = shape_of(v)
    cfg = VSmoothCfg(k, iters, seed, _fmt_code(fmt), _MODES[mode])
    B, S, H = sh.B, sh.S, sh.H
    dev = v.device
    out = _prepared_buffers(B, S, H, fmt, dev)
    wsb = lib.vc_attn_prepare_v_workspace_bytes(ctypes.byref(sh), ctypes.byref(cfg))
    if wsb == 0:
        raise VCError(VC_ERR_INVALID_ARG, "invalid shape or config")
    ws = torch.empty(wsb + 256, dtype=torch.uint8, device=dev)
    off = (-ws.data_ptr()) % 256
    hist = torch.empty((iters, B, H, S), dtype=torch.uint8, device=dev) if history else None
    pv = PreparedV(_ptr(out["perm"]), _ptr(out["mu"]), _ptr(out["v_codes"]), _ptr(out["v_scales"]), _ptr(out["s_v"]))
    if H_total is not None:
        if history:
            raise ValueError("the shard prep keeps no assignment history")
        _check(lib.vc_attn_prepare_v_shard(_ptr(v), ctypes.byref(sh), ctypes.byref(cfg), int(h_base), int(H_total),
                                           ctypes.byref(pv), ctypes.c_void_p(ws.data_ptr() + off), wsb, _stream()))
    else:
        _check(lib.vc_attn_prepare_v(_ptr(v), ctypes.byref(sh), ctypes.byref(cfg), ctypes.byref(pv),
                                     ctypes.c_void_p(ws.data_ptr() + off), wsb, _ptr(hist), _stream()))
    out["workspace"] = ws
    out["history"] = hist
    return out


def prepare_v_noalloc(v, k=16, iters=4, seed=0, fmt="e4m3", mode="vsmooth", history=False):
    """As ``prepare_v`` but through vc_attn_prepare_v_noalloc: no workspace is
    passed; the library's fixed device scratch is used. The outputs are still
    allocated here (by torch), as the caller's buffers."""
    lib = load()
    sh = shape_of(v)
    cfg = VSmoothCfg(k, iters, seed, _fmt_code(fmt), _MODES[mode])
    B, S, H = sh.B, sh.S, sh.H
    dev = v.device
    out = _prepared_buffers(B, S, H, fmt, dev)
    hist = torch.empty((iters, B, H, S), dtype=torch.uint8, device=dev) if history else None
    pv = PreparedV(_ptr(out["perm"]), _ptr(out["mu"]), _ptr(out["v_codes"]), _ptr(out["v_scales"]), _ptr(out["s_v"]))
    _check(lib.vc_attn_prepare_v_noalloc(_ptr(v), ctypes.byref(sh), ctypes.byref(cfg), ctypes.byref(pv), _ptr(hist),
                                         _stream()))
    out["history"] = hist
    return out


def quant_qk(q, k, perm, smooth_k=False):
    """Per-block E4M3 quantisation of Q and of K gathered through ``perm``.
    ``smooth_k``: K minus its per-channel token mean first (vc_attn_quant_qk_smoothk;
    the mean is returned as ``k_mean``, fp32 [B, H, 128])."""
    lib = load()
    sh = shape_of(q)
    if shape_of(k).S != sh.S or k.shape != q.shape or k.dtype != q.dtype:
        raise ValueError("q and k must have the same shape and dtype")
    B, S, H = sh.B, sh.S, sh.H
    nb = num_blocks(S)
    dev = q.device
    out = dict(
        q_codes=torch.empty((B, H, nb * 128, 128), dtype=torch.uint8, device=dev),
        q_scales=torch.empty((B, H, nb), dtype=torch.float32, device=dev),
        k_codes=torch.empty((B, H, nb * 128, 128), dtype=torch.uint8, device=dev),
        k_scales=torch.empty((B, H, nb), dtype=torch.float32, device=dev),
    )
    qk = QKFP8(_ptr(out["q_codes"]), _ptr(out["q_scales"]), _ptr(out["k_codes"]), _ptr(out["k_scales"]))
    if not smooth_k:
        _check(lib.vc_attn_quant_qk(_ptr(q), _ptr(k), ctypes.byref(sh), _ptr(perm), ctypes.byref(qk), _stream()))
        return out
    wsb = lib.vc_attn_quant_qk_smoothk_workspace_bytes(ctypes.byref(sh))
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    out["k_mean"] = torch.empty((B, H, 128), dtype=torch.float32, device=dev)
    _check(lib.vc_attn_quant_qk_smoothk(_ptr(q), _ptr(k), ctypes.byref(sh), _ptr(perm), ctypes.byref(qk), _ptr(ws),
                                        wsb, _ptr(out["k_mean"]), _stream()))
    out["workspace"] = ws
    return out


def prepare_v_repair(v, budget=0.005, k=16, iters=4, seed=0, mode="vsmooth"):
    """V-Smooth prep with the V residual repair (E4M3 residual): returns the
    prepared-V dict of ``prepare_v`` whose ``v_codes`` holds the two planes
    [2, B, H, 128, S_pad], plus ``kept`` (uint8 [B, H, S], 1 at the repaired
    permuted positions)."""
    lib = load()
    sh = shape_of(v)
    cfg = VSmoothCfg(k, iters, seed, VC_RESIDUAL_E4M3, _MODES[mode])
    B, S, H = sh.B, sh.S, sh.H
    nb = num_blocks(S)
    dev = v.device
    out = dict(perm=torch.empty((B, H, S), dtype=torch.int32, device=dev),
               mu=torch.empty((B, H, nb, 128), dtype=torch.float32, device=dev),
               s_v=torch.empty((B, H), dtype=torch.float32, device=dev),
               v_codes=torch.empty((2, B, H, 128, nb * 128), dtype=torch.uint8, device=dev), v_scales=None,
               kept=torch.empty((B, H, S), dtype=torch.uint8, device=dev), fmt="repair")
    wsb = lib.vc_attn_prepare_v_repair_workspace_bytes(ctypes.byref(sh), ctypes.byref(cfg))
    if wsb == 0:
        raise VCError(VC_ERR_INVALID_ARG, "invalid shape or config")
    ws = torch.empty(wsb + 256, dtype=torch.uint8, device=dev)
    off = (-ws.data_ptr()) % 256
    pv = PreparedV(_ptr(out["perm"]), _ptr(out["mu"]), _ptr(out["v_codes"]), None, _ptr(out["s_v"]))
    _check(lib.vc_attn_prepare_v_repair(_ptr(v), ctypes.byref(sh), ctypes.byref(cfg), float(budget),
                                        ctypes.byref(pv), _ptr(out["kept"]), ctypes.c_void_p(ws.data_ptr() + off),
                                        wsb, _stream()))
    out["workspace"] = ws
    return out


def forward_repair(qk, pv, shape, softmax_scale=None, k_p=8, out=None, status=None):
    """Attention over the two planes of ``prepare_v_repair``; BF16 O in the input
    layout."""
    lib = load()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(128)
    dev = qk["q_codes"].device
    if out is None:
        out = torch.empty((shape.B, shape.S, shape.H, 128), dtype=torch.bfloat16, device=dev)
    q_ = QKFP8(_ptr(qk["q_codes"]), _ptr(qk["q_scales"]), _ptr(qk["k_codes"]), _ptr(qk["k_scales"]))
    p_ = PreparedV(_ptr(pv["perm"]), _ptr(pv["mu"]), _ptr(pv["v_codes"]), None, _ptr(pv["s_v"]))
    _check(lib.vc_attn_forward_repair(ctypes.byref(q_), ctypes.byref(p_), ctypes.byref(shape), float(softmax_scale),
                                      int(k_p), _ptr(out), _ptr(status), _stream()))
    return out


def residual_energy(v, perm=None, mu=None):
    """Per-slice fp64 energy sum ||v[perm[p]] - mu[p // 128]||^2 as a [B, H]
    device tensor (``perm`` None: identity order; ``mu`` None: zero means)."""
    lib = load()
    sh = shape_of(v)
    nb = num_blocks(sh.S)
    for name, t, shp, dt in (("perm", perm, (sh.B, sh.H, sh.S), torch.int32),
                             ("mu", mu, (sh.B, sh.H, nb, 128), torch.float32)):
        if t is not None and (tuple(t.shape) != shp or t.dtype != dt or not t.is_contiguous()
                              or t.device != v.device):
            raise ValueError(f"{name} must be a contiguous {dt} tensor of shape {shp} on {v.device}")
    energy = torch.empty((sh.B, sh.H), dtype=torch.float64, device=v.device)
    _check(lib.vc_attn_residual_energy(_ptr(v), ctypes.byref(sh), _ptr(perm), _ptr(mu), _ptr(energy), _stream()))
    return energy


def forward(qk, pv, shape, softmax_scale=None, k_p=8, out=None, status=None, workspace=None):
    """Fused ExpCast FP8 attention from the two prep outputs; returns BF16 O in
    the input layout. ``shape`` is the vc_shape_t of Q (``shape_of(q)``).
    For an NVFP4 ``pv`` the call needs a device workspace of
    ``forward_nvfp4v_workspace_bytes(shape)`` bytes; one is allocated when
    ``workspace`` is None. The other formats ("e4m3", "e4m3c", "mxfp4") go to
    vc_attn_forward, vc_attn_forward_e4m3_per_channel and vc_attn_forward_mxfp4v."""
    lib = load()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(128)
    dev = qk["q_codes"].device
    if out is None:
        out = torch.empty((shape.B, shape.S, shape.H, 128), dtype=torch.bfloat16, device=dev)
    q_ = QKFP8(_ptr(qk["q_codes"]), _ptr(qk["q_scales"]), _ptr(qk["k_codes"]), _ptr(qk["k_scales"]))
    p_ = PreparedV(_ptr(pv["perm"]), _ptr(pv["mu"]), _ptr(pv["v_codes"]), _ptr(pv.get("v_scales")), _ptr(pv["s_v"]))
    if pv.get("fmt") == "nvfp4":
        if workspace is None:
            workspace = torch.empty(forward_nvfp4v_workspace_bytes(shape), dtype=torch.uint8, device=dev)
        _check(lib.vc_attn_forward_nvfp4v(ctypes.byref(q_), ctypes.byref(p_), ctypes.byref(shape),
                                          float(softmax_scale), int(k_p), _ptr(out), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _ptr(status), _stream()))
    else:
        fn = {"e4m3c": lib.vc_attn_forward_e4m3_per_channel, "mxfp4": lib.vc_attn_forward_mxfp4v}.get(
            pv.get("fmt"), lib.vc_attn_forward)
        _check(fn(ctypes.byref(q_), ctypes.byref(p_), ctypes.byref(shape), float(softmax_scale), int(k_p), _ptr(out),
                  _ptr(status), _stream()))
    return out


def forward_nvfp4v_workspace_bytes(shape):
    """Device bytes vc_attn_forward_nvfp4v needs for this shape (the two E4M3
    planes of the decoded NVFP4 residual)."""
    return int(load().vc_attn_forward_nvfp4v_workspace_bytes(ctypes.byref(shape)))


def attention(q, k, v, softmax_scale=None, k_p=8, kmeans_k=16, iters=4, seed=0, fmt="e4m3", smooth_k=False):
    """One call: V-Smooth prep, Q/K quantisation (K smoothed by its token mean
    when ``smooth_k``) and the fused attention. Q, K, V: [B,S,H,128] or [S,H,128]
    FP16/BF16 on the GPU; returns BF16 O with the same layout."""
    pv = prepare_v(v, k=kmeans_k, iters=iters, seed=seed, fmt=fmt)
    qk = quant_qk(q, k, pv["perm"], smooth_k=smooth_k)
    o = forward(qk, pv, shape_of(q), softmax_scale, k_p)
    return o.view(q.shape)


class Plan:
    """Preallocated buffers for repeated calls on one shape (the form a serving
    loop or the benchmark uses): the prepared V, the Q/K codes, the prep
    workspace, O and a device status word, all owned by this object.

    ``run(q, k, v)`` enqueues the three calls (prepare_v, quant_qk, forward) on
    the current stream and returns O; nothing is allocated per call. With
    ``smooth_k`` the Q/K call is vc_attn_quant_qk_smoothk (K minus its token mean,
    into the preallocated ``k_mean``).
    """

    def __init__(self, B, S, H, dtype=torch.bfloat16, k=16, iters=4, seed=0, fmt="e4m3", k_p=8,
                 softmax_scale=None, device=None, mode="vsmooth", smooth_k=False, h_base=0, H_total=None):
        self.lib = load()
        # a shard of heads [h_base, h_base + H) of a problem with H_total heads
        self.h_base, self.H_total = int(h_base), (None if H_total is None else int(H_total))
        dev = torch.device(device if device is not None else "cuda")
        self.shape = Shape(B, S, H, 128, VC_DTYPE_BF16 if dtype == torch.bfloat16 else VC_DTYPE_F16)
        self.cfg = VSmoothCfg(k, iters, seed, _fmt_code(fmt), _MODES[mode])
        self.fmt, self.k_p = fmt, int(k_p)
        self.softmax_scale = 1.0 / math.sqrt(128) if softmax_scale is None else float(softmax_scale)
        nb = num_blocks(S)
        Sp = nb * 128
        e = lambda shp, dt: torch.empty(shp, dtype=dt, device=dev)
        pb = _prepared_buffers(B, S, H, fmt, dev)
        self.perm, self.mu, self.s_v, self.v_codes, self.v_scales = (pb["perm"], pb["mu"], pb["s_v"], pb["v_codes"],
                                                                     pb["v_scales"])
        self.q_codes, self.k_codes = e((B, H, Sp, 128), torch.uint8), e((B, H, Sp, 128), torch.uint8)
        self.q_scales, self.k_scales = e((B, H, nb), torch.float32), e((B, H, nb), torch.float32)
        self.o = e((B, S, H, 128), torch.bfloat16)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ws_bytes = self.lib.vc_attn_prepare_v_workspace_bytes(ctypes.byref(self.shape), ctypes.byref(self.cfg))
        if self.ws_bytes == 0:
            raise VCError(VC_ERR_INVALID_ARG, "invalid shape or config")
        self._ws = e((self.ws_bytes + 256,), torch.uint8)
        self.ws_ptr = ctypes.c_void_p(self._ws.data_ptr() + (-self._ws.data_ptr()) % 256)
        self._pv = PreparedV(_ptr(self.perm), _ptr(self.mu), _ptr(self.v_codes), _ptr(self.v_scales), _ptr(self.s_v))
        self._qk = QKFP8(_ptr(self.q_codes), _ptr(self.q_scales), _ptr(self.k_codes), _ptr(self.k_scales))
        if fmt == "nvfp4":
            self.fwd_ws_bytes = self.lib.vc_attn_forward_nvfp4v_workspace_bytes(ctypes.byref(self.shape))
            self._fwd_ws = e((self.fwd_ws_bytes,), torch.uint8)
        else:
            self.fwd_ws_bytes, self._fwd_ws = 0, None
        self.smooth_k = bool(smooth_k)
        if self.smooth_k:
            self.smooth_ws_bytes = self.lib.vc_attn_quant_qk_smoothk_workspace_bytes(ctypes.byref(self.shape))
            self._smooth_ws = e((self.smooth_ws_bytes,), torch.uint8)
            self.k_mean = e((B, H, 128), torch.float32)
        else:
            self.smooth_ws_bytes, self._smooth_ws, self.k_mean = 0, None, None

    def prepare_v(self, v):
        if self.H_total is not None:
            _check(self.lib.vc_attn_prepare_v_shard(_ptr(v), ctypes.byref(self.shape), ctypes.byref(self.cfg),
                                                    self.h_base, self.H_total, ctypes.byref(self._pv), self.ws_ptr,
                                                    self.ws_bytes, _stream()))
        else:
            _check(self.lib.vc_attn_prepare_v(_ptr(v), ctypes.byref(self.shape), ctypes.byref(self.cfg),
                                              ctypes.byref(self._pv), self.ws_ptr, self.ws_bytes, None, _stream()))

    def quant_qk(self, q, k):
        if self.smooth_k:
            _check(self.lib.vc_attn_quant_qk_smoothk(_ptr(q), _ptr(k), ctypes.byref(self.shape), _ptr(self.perm),
                                                     ctypes.byref(self._qk), _ptr(self._smooth_ws),
                                                     self.smooth_ws_bytes, _ptr(self.k_mean), _stream()))
        else:
            _check(self.lib.vc_attn_quant_qk(_ptr(q), _ptr(k), ctypes.byref(self.shape), _ptr(self.perm),
                                             ctypes.byref(self._qk), _stream()))

    def forward(self, out=None):
        o = self.o if out is None else out
        if self.fmt == "nvfp4":
            _check(self.lib.vc_attn_forward_nvfp4v(ctypes.byref(self._qk), ctypes.byref(self._pv),
                                                   ctypes.byref(self.shape), self.softmax_scale, self.k_p, _ptr(o),
                                                   _ptr(self._fwd_ws), self.fwd_ws_bytes, _ptr(self.status),
                                                   _stream()))
        else:
            fn = {"e4m3c": self.lib.vc_attn_forward_e4m3_per_channel, "mxfp4": self.lib.vc_attn_forward_mxfp4v}.get(
                self.fmt, self.lib.vc_attn_forward)
            _check(fn(ctypes.byref(self._qk), ctypes.byref(self._pv), ctypes.byref(self.shape), self.softmax_scale,
                      self.k_p, _ptr(o), _ptr(self.status), _stream()))
        return o

    def run(self, q, k, v, out=None):
        self.prepare_v(v)
        self.quant_qk(q, k)
        return self.forward(out)


class HostPlan:
    """The whole path for Q, K, V and O in host memory (``vc_attn_run_host``):
    the device workspace for one shape and head chunk is allocated once here;
    ``run(q, k, v, o)`` takes CPU tensors of shape [B,S,H,128] (page-locked for
    the copies to overlap the compute; ``o`` bf16) and enqueues the chunked
    copies and the three calls on the current stream. ``o`` is complete once
    the stream has passed the call."""

    def __init__(self, B, S, H, dtype=torch.bfloat16, k=16, iters=4, seed=0, fmt="e4m3", k_p=8,
                 softmax_scale=None, head_chunk=4, device=None, mode="vsmooth"):
        self.lib = load()
        dev = torch.device(device if device is not None else "cuda")
        self.dtype = dtype
        self.shape = Shape(B, S, H, 128, VC_DTYPE_BF16 if dtype == torch.bfloat16 else VC_DTYPE_F16)
        self.cfg = VSmoothCfg(k, iters, seed, _fmt_code(fmt), _MODES[mode])
        self.k_p, self.head_chunk = int(k_p), int(head_chunk)
        self.softmax_scale = 1.0 / math.sqrt(128) if softmax_scale is None else float(softmax_scale)
        self.ws_bytes = self.lib.vc_attn_run_host_workspace_bytes(ctypes.byref(self.shape), ctypes.byref(self.cfg),
                                                                   self.head_chunk)
        if self.ws_bytes == 0:
            raise VCError(VC_ERR_INVALID_ARG, "invalid shape, config or head chunk")
        self._ws = torch.empty((self.ws_bytes + 256,), dtype=torch.uint8, device=dev)
        self.ws_ptr = ctypes.c_void_p(self._ws.data_ptr() + (-self._ws.data_ptr()) % 256)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def run(self, q, k, v, o):
        want = (self.shape.B, self.shape.S, self.shape.H, 128)
        for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
            if t.device.type != "cpu" or not t.is_contiguous() or tuple(t.reshape(want).shape) != want:
                raise ValueError(f"{name} must be a contiguous CPU tensor of shape {want}")
        if q.dtype != self.dtype or k.dtype != self.dtype or v.dtype != self.dtype or o.dtype != torch.bfloat16:
            raise ValueError("q, k, v must have the plan's dtype and o must be bfloat16")
        _check(self.lib.vc_attn_run_host(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(self.shape), ctypes.byref(self.cfg),
                                         self.softmax_scale, self.k_p, _ptr(o), self.head_chunk, self.ws_ptr,
                                         self.ws_bytes, _ptr(self.status), _stream()))
        return o


def launch_count():
    """Kernels the library has enqueued since it was loaded."""
    return int(load().vc_attn_launch_count())


# ------------------------------------------------------------------ test hooks
def test_e4m3_round(x):
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(load().vc_attn_test_e4m3_round(_ptr(x), _ptr(out), x.numel(), _stream()))
    return out


def test_e2m1_round(x):
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(load().vc_attn_test_e2m1_round(_ptr(x), _ptr(out), x.numel(), _stream()))
    return out


def test_expcast(t, c, M, bias_b, hot=False):
    out = torch.empty(t.shape, dtype=torch.uint8, device=t.device)
    _check(load().vc_attn_test_expcast(_ptr(t), _ptr(c), _ptr(M), int(bias_b), _ptr(out), t.numel(), int(hot),
                                       _stream()))
    return out


def test_forward_exp2(qk, pv, shape, softmax_scale=None, k_p=8, out=None, status=None):
    """The E4M3-V forward with exp2 + E4M3 conversion instead of ExpCast (the
    comparison kernel of vc_attn_test_forward_exp2)."""
    lib = load()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(128)
    dev = qk["q_codes"].device
    if out is None:
        out = torch.empty((shape.B, shape.S, shape.H, 128), dtype=torch.bfloat16, device=dev)
    q_ = QKFP8(_ptr(qk["q_codes"]), _ptr(qk["q_scales"]), _ptr(qk["k_codes"]), _ptr(qk["k_scales"]))
    p_ = PreparedV(_ptr(pv["perm"]), _ptr(pv["mu"]), _ptr(pv["v_codes"]), _ptr(pv.get("v_scales")), _ptr(pv["s_v"]))
    _check(lib.vc_attn_test_forward_exp2(ctypes.byref(q_), ctypes.byref(p_), ctypes.byref(shape), float(softmax_scale),
                                         int(k_p), _ptr(out), _ptr(status), _stream()))
    return out


def test_bounded_wait(status, limit_ns):
    _check(load().vc_attn_test_bounded_wait(_ptr(status), int(limit_ns), _stream()))
