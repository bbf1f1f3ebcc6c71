"""Loader and numpy wrappers of the C++ statement of the oracle (vc_oracle_ref.cpp).

TEST INFRASTRUCTURE ONLY, like the rest of this package: only ``tests/``,
``__graft_entry__`` (which compiles it) and the benchmark's CPU legs may use it.
It is a second CPU statement of the same definitions as ``vc_oracle.py``, written
as plain loops; the tests hold the two against each other bit for bit.
"""
import ctypes
import os
import shutil
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "vc_oracle_ref.cpp")
LIB = os.path.join(_HERE, "_build", "libvcoracle.so")
_lib = None


def build(force=False):
    """Compile the C++ oracle with g++ (no fused multiply-add contraction)."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cxx = os.environ.get("CXX") or shutil.which("g++")
    if not cxx:
        raise RuntimeError("g++ not found")
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [cxx, "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c++17", "-shared", "-fPIC", "-o", tmp, SRC]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("building the C++ oracle failed:\n" + r.stdout + r.stderr)
    os.replace(tmp, LIB)
    return LIB


def load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIB)
        P = ctypes.c_void_p
        i32, i64, u64, f32 = ctypes.c_int, ctypes.c_long, ctypes.c_uint64, ctypes.c_float
        lib.orc_version.restype = i32
        lib.orc_e4m3_round.argtypes = [P, i64, P]
        lib.orc_e2m1_round.argtypes = [P, i64, P]
        lib.orc_kmeans_init.argtypes = [i32, i32, u64, i64, P]
        lib.orc_kmeans_lloyd.argtypes = [P, i32, i32, i32, i32, u64, i64, P, P, P]
        lib.orc_cluster_perm.argtypes = [P, i32, i32, P]
        lib.orc_block_means.argtypes = [P, i32, i32, P, P]
        lib.orc_residual_e4m3.argtypes = [P, i32, i32, P, P, P, P, P]
        lib.orc_residual_nvfp4.argtypes = [P, i32, i32, P, P, P, P, P, P]
        lib.orc_vres_from_e4m3.argtypes = [P, i32, i32, i32, f32, P]
        lib.orc_residual_e4m3_per_channel.argtypes = [P, i32, i32, P, P, P, P, P]
        lib.orc_mx_exponent.argtypes = [ctypes.c_double]
        lib.orc_mx_exponent.restype = i32
        lib.orc_residual_mxfp4.argtypes = [P, i32, i32, P, P, P, P]
        lib.orc_residual_repair_planes.argtypes = [P, i32, i32, P, P, ctypes.c_double, P, P, P, P]
        lib.orc_residual_repair_planes.restype = i32
        lib.orc_residual_energy.argtypes = [P, i32, i32, P, P]
        lib.orc_residual_energy.restype = ctypes.c_double
        lib.orc_smooth_k.argtypes = [P, i32, i32, P, P]
        lib.orc_quant_blocks_e4m3.argtypes = [P, i32, i32, P, P, P]
        lib.orc_softmax_kappa.argtypes = [f32]
        lib.orc_softmax_kappa.restype = f32
        lib.orc_vc_attention_rows.argtypes = [P, P, P, P, P, P, i32, i32, P, i32, f32, i32, P, P, P]
        lib.orc_exact_attention_rows.argtypes = [P, P, P, i32, i32, P, i32, ctypes.c_double, P]
        _lib = lib
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _f32(x):
    return np.ascontiguousarray(np.asarray(x, np.float32))


def _i32(x):
    return np.ascontiguousarray(np.asarray(x, np.int32))


def nblocks(S):
    return (S + 127) // 128


def e4m3_round(x):
    x = _f32(x)
    out = np.empty(x.shape, np.uint8)
    load().orc_e4m3_round(_p(x), x.size, _p(out))
    return out


def e2m1_round(x):
    x = _f32(x)
    out = np.empty(x.shape, np.uint8)
    load().orc_e2m1_round(_p(x), x.size, _p(out))
    return out


def kmeans_init_indices(S, k, seed, bh):
    out = np.empty(k, np.int32)
    load().orc_kmeans_init(S, k, seed, bh, _p(out))
    return [int(v) for v in out]


def kmeans_lloyd(X, k, iters, seed, bh):
    """Returns (final assignment, final centroids, per-pass assignments)."""
    X = _f32(X)
    S, D = X.shape
    a = np.empty(S, np.int32)
    C = np.empty((k, D), np.float32)
    hist = np.empty((iters, S), np.int32)
    load().orc_kmeans_lloyd(_p(X), S, D, k, iters, seed, bh, _p(a), _p(C), _p(hist))
    return a, C, list(hist)


def cluster_permutation(a, k):
    a = _i32(a)
    perm = np.empty(a.size, np.int32)
    load().orc_cluster_perm(_p(a), a.size, k, _p(perm))
    return perm


def block_means(X, perm):
    X, perm = _f32(X), _i32(perm)
    S, D = X.shape
    mu = np.empty((nblocks(S), D), np.float32)
    load().orc_block_means(_p(X), S, D, _p(perm), _p(mu))
    return mu


def residual_e4m3(X, perm, mu):
    X, perm, mu = _f32(X), _i32(perm), _f32(mu)
    S, D = X.shape
    vt = np.empty((D, nblocks(S) * 128), np.uint8)
    s_v, amax = np.empty(1, np.float32), np.empty(1, np.float32)
    load().orc_residual_e4m3(_p(X), S, D, _p(perm), _p(mu), _p(vt), _p(s_v), _p(amax))
    return vt, np.float32(s_v[0]), np.float32(amax[0])


def residual_nvfp4(X, perm, mu):
    X, perm, mu = _f32(X), _i32(perm), _f32(mu)
    S, D = X.shape
    Sp = nblocks(S) * 128
    packed = np.empty((D, Sp // 2), np.uint8)
    scales = np.empty((D, Sp // 16), np.uint8)
    g, amax = np.empty(1, np.float32), np.empty(1, np.float32)
    load().orc_residual_nvfp4(_p(X), S, D, _p(perm), _p(mu), _p(packed), _p(scales), _p(g), _p(amax))
    return packed, scales, np.float32(g[0]), np.float32(amax[0])


def residual_e4m3_per_channel(X, perm, mu):
    X, perm, mu = _f32(X), _i32(perm), _f32(mu)
    S, D = X.shape
    vt = np.empty((D, nblocks(S) * 128), np.uint8)
    s_v, amax = np.empty(D, np.float32), np.empty(D, np.float32)
    load().orc_residual_e4m3_per_channel(_p(X), S, D, _p(perm), _p(mu), _p(vt), _p(s_v), _p(amax))
    return vt, s_v, amax


def mx_exponent(amax):
    return int(load().orc_mx_exponent(float(amax)))


def residual_mxfp4(X, perm, mu):
    X, perm, mu = _f32(X), _i32(perm), _f32(mu)
    S, D = X.shape
    Sp = nblocks(S) * 128
    codes = np.empty((D, Sp), np.uint8)
    e8 = np.empty((D, Sp // 32), np.uint8)
    load().orc_residual_mxfp4(_p(X), S, D, _p(perm), _p(mu), _p(codes), _p(e8))
    return codes, e8


def residual_repair_planes(X, perm, mu, budget):
    """Returns (kept positions ascending, plane 0 (D, S_pad), plane 1 (D, S_pad), s_v)."""
    X, perm, mu = _f32(X), _i32(perm), _f32(mu)
    S, D = X.shape
    Sp = nblocks(S) * 128
    vt = np.empty((D, Sp), np.uint8)
    lo = np.empty((D, Sp), np.uint8)
    s_v = np.empty(1, np.float32)
    pos = np.empty(max(S, 1), np.int32)
    m = load().orc_residual_repair_planes(_p(X), S, D, _p(perm), _p(mu), float(budget), _p(vt), _p(lo), _p(s_v),
                                         _p(pos))
    return pos[:m].copy(), vt, lo, np.float32(s_v[0])


def residual_energy(X, perm, mu):
    X, perm, mu = _f32(X), _i32(perm), _f32(mu)
    S, D = X.shape
    return float(load().orc_residual_energy(_p(X), S, D, _p(perm), _p(mu)))


def vres_from_e4m3(vt, s_v, S):
    vt = np.ascontiguousarray(vt, np.uint8)
    D, Sp = vt.shape
    out = np.empty((S, D), np.float64)
    load().orc_vres_from_e4m3(_p(vt), Sp, S, D, float(s_v), _p(out))
    return out


def quant_blocks_e4m3(X, order=None):
    X = _f32(X)
    S, D = X.shape
    codes = np.empty((nblocks(S) * 128, D), np.uint8)
    scales = np.empty(nblocks(S), np.float32)
    o = _i32(order) if order is not None else None
    load().orc_quant_blocks_e4m3(_p(X), S, D, _p(o), _p(codes), _p(scales))
    return codes, scales


def smooth_k(K):
    """Returns (K - kbar, kbar)."""
    K = _f32(K)
    S, D = K.shape
    kbar = np.empty(D, np.float32)
    xs = np.empty((S, D), np.float32)
    load().orc_smooth_k(_p(K), S, D, _p(kbar), _p(xs))
    return xs, kbar


def softmax_kappa(softmax_scale):
    return np.float32(load().orc_softmax_kappa(float(softmax_scale)))


def vc_attention_rows(q_codes, q_scales, k_codes, k_scales, vres, mu, S, rows, softmax_scale, k_p=8):
    """Returns (O (rows, D) fp64, codes (rows, S) uint8, l (rows,) fp64)."""
    q_codes, k_codes = np.ascontiguousarray(q_codes, np.uint8), np.ascontiguousarray(k_codes, np.uint8)
    q_scales, k_scales, mu = _f32(q_scales), _f32(k_scales), _f32(mu)
    vres = np.ascontiguousarray(vres, np.float64)
    rows = _i32(rows)
    D = q_codes.shape[1]
    O = np.empty((rows.size, D), np.float64)
    codes = np.empty((rows.size, S), np.uint8)
    l = np.empty(rows.size, np.float64)
    load().orc_vc_attention_rows(_p(q_codes), _p(q_scales), _p(k_codes), _p(k_scales), _p(vres), _p(mu), S, D,
                                 _p(rows), rows.size, float(softmax_scale), int(k_p), _p(O), _p(codes), _p(l))
    return O, codes, l


def exact_attention_rows(Q, K, V, rows, softmax_scale):
    Q, K, V, rows = _f32(Q), _f32(K), _f32(V), _i32(rows)
    S, D = K.shape
    O = np.empty((rows.size, D), np.float64)
    load().orc_exact_attention_rows(_p(Q), _p(K), _p(V), S, D, _p(rows), rows.size, float(softmax_scale), _p(O))
    return O
