"""Seeded synthetic Q/K/V workloads (torch CPU generators only).

This module draws random numbers and nothing else: it holds none of the
method's arithmetic, so both the CUDA path's tests and the CPU oracle can take
their inputs from it.

Workloads (shapes of the video-DiT attention calls the method targets):
  tiny        B=1, H=2,  S=256    N(0,1) Q/K/V; 4 V tokens per head scaled x16
  mid         B=2, H=8,  S=4096   mixture recipe (below)
  wan         B=1, H=40, S=75600  mixture recipe, [S,H,128] (21 x 45 x 80 latents)
  minimax_hN  B=1, H=N,  S=73397  mixture recipe, N in {7, 14, 56}
  nvfp4_sN    B=1, H=24, S=N      mixture recipe, N in {1024 ... 131072}

Mixture recipe: Q, K ~ N(0,1) * lambda[h, d] with lambda ~ LogNormal(0, 0.5)
drawn per (tensor, head, channel); V from a 16-centre Gaussian mixture with
centres ~ N(0, 2^2) per (batch, head, centre, channel), each token's centre
uniform i.i.d., spread 0.3; 1% of tokens per (batch, head), at positions drawn
per (batch, head), are scaled x20 (whole vector).

Stream ids (seed offsets): Q=1, K=2, V=3, outliers=4, lambda=5, centres=6,
centre choice=7.
"""
import math

import torch

D_HEAD = 128

WORKLOADS = {
    "tiny": dict(B=1, H=2, S=256, recipe="normal", k=4, iters=3, fmt="e4m3", layout="BSHD"),
    "mid": dict(B=2, H=8, S=4096, recipe="mixture", k=16, iters=4, fmt="e4m3", layout="BSHD"),
    "wan": dict(B=1, H=40, S=75600, recipe="mixture", k=16, iters=4, fmt="e4m3", layout="SHD"),
}
for _h in (7, 14, 56):
    WORKLOADS[f"minimax_h{_h}"] = dict(B=1, H=_h, S=73397, recipe="mixture", k=16, iters=4,
                                       fmt="e4m3", layout="SHD")
for _s in (1024, 4096, 16384, 32768, 65536, 131072):
    WORKLOADS[f"nvfp4_s{_s}"] = dict(B=1, H=24, S=_s, recipe="mixture", k=16, iters=4,
                                     fmt="nvfp4", layout="SHD")

STREAM = dict(q=1, k=2, v=3, outliers=4, lam=5, centres=6, choice=7)


def softmax_scale(d=D_HEAD):
    return 1.0 / math.sqrt(d)


def _gen(seed, stream, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000 + STREAM[stream])
    return g


def workload(name, **overrides):
    cfg = dict(WORKLOADS[name])
    cfg.update(overrides)
    cfg["name"] = name
    return cfg


def make_qkv(B, S, H, recipe="mixture", seed=0, dtype=torch.bfloat16, chunk=8192, device="cpu", **_):
    """Return tensors Q, K, V of shape [B, S, H, 128] in ``dtype`` on ``device``.

    Drawn chunk by chunk along S (fixed chunk size, so the values do not depend
    on available memory) and converted to ``dtype`` as they are drawn. The values
    depend on the device's generator: the same seed gives the same recipe but not
    the same numbers on "cpu" and "cuda" (tests use "cpu"; the benchmark draws
    its large workloads on the GPU).
    """
    D = D_HEAD
    shape = (B, S, H, D)
    Q = torch.empty(shape, dtype=dtype, device=device)
    K = torch.empty(shape, dtype=dtype, device=device)
    V = torch.empty(shape, dtype=dtype, device=device)
    g = lambda name: _gen(seed, name, device)
    gq, gk, gv = g("q"), g("k"), g("v")
    if recipe == "normal":
        for s0 in range(0, S, chunk):
            n = min(chunk, S - s0)
            Q[:, s0:s0 + n] = torch.randn((B, n, H, D), generator=gq, device=device).to(dtype)
            K[:, s0:s0 + n] = torch.randn((B, n, H, D), generator=gk, device=device).to(dtype)
            V[:, s0:s0 + n] = torch.randn((B, n, H, D), generator=gv, device=device).to(dtype)
        go = g("outliers")
        for b in range(B):
            for h in range(H):
                pos = torch.randperm(S, generator=go, device=device)[: min(4, S)]
                V[b, pos, h] = (V[b, pos, h].float() * 16.0).to(dtype)
        return Q, K, V
    if recipe != "mixture":
        raise ValueError(recipe)
    gl = g("lam")
    lam_q = torch.exp(0.5 * torch.randn((H, D), generator=gl, device=device))
    lam_k = torch.exp(0.5 * torch.randn((H, D), generator=gl, device=device))
    centres = 2.0 * torch.randn((B, H, 16, D), generator=g("centres"), device=device)
    gc = g("choice")
    hidx = torch.arange(H, device=device).view(1, 1, H)
    for s0 in range(0, S, chunk):
        n = min(chunk, S - s0)
        Q[:, s0:s0 + n] = (torch.randn((B, n, H, D), generator=gq, device=device) * lam_q).to(dtype)
        K[:, s0:s0 + n] = (torch.randn((B, n, H, D), generator=gk, device=device) * lam_k).to(dtype)
        choice = torch.randint(0, 16, (B, n, H), generator=gc, device=device)
        bidx = torch.arange(B, device=device).view(B, 1, 1)
        v = centres[bidx, hidx, choice] + 0.3 * torch.randn((B, n, H, D), generator=gv, device=device)
        V[:, s0:s0 + n] = v.to(dtype)
    go = g("outliers")
    n_out = max(1, round(0.01 * S))
    for b in range(B):
        for h in range(H):
            pos = torch.randperm(S, generator=go, device=device)[:n_out]
            V[b, pos, h] = (V[b, pos, h].float() * 20.0).to(dtype)
    return Q, K, V


def make_workload(name, seed=0, dtype=torch.bfloat16, device="cpu", **overrides):
    cfg = workload(name, **overrides)
    Q, K, V = make_qkv(cfg["B"], cfg["S"], cfg["H"], recipe=cfg["recipe"], seed=seed, dtype=dtype, device=device)
    return cfg, Q, K, V
