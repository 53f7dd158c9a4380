"""Seeded synthetic inputs for LLA decode attention (workload recipes only).

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no encode, reconstruction, RoPE or attention), so both
the FP64 oracle's tests and the CUDA library's tests and benchmark can take
their inputs from it.

Workloads follow the shapes the paper serves: Ouro-1.4B (D=24 layers, T=4
loops, H=16 heads, d_head=128) at ratios 4 and 21.3, its head-folded LLA-2D
variant, and a Huginn-like T=32 recurrence ("Looped Latent Attention:
Cross-Loop KV Compression for Looped Transformers", §1 and abstract).  No
model activations are available, so smooth low-rank loop trajectories stand
in for teacher K/V stacks (recipe in ``smooth_stacks``).
"""

from __future__ import annotations

import hashlib
import math

import numpy as np

BASE_SEED = 0x11A

# name -> shape recipe.  `context` is the number of cached tokens per sequence.
CONFIGS = {
    "tiny_d16_t4": dict(D=1, T=4, H=2, d_head=16, r_k=4, r_v=8, variant=0, batch=1, context=64,
                        rope_base=10000.0, traj_rank=6, noise_var=1e-3, calib=512),
    "ouro_rho4_b32_n4096": dict(D=24, T=4, H=16, d_head=128, r_k=96, r_v=160, variant=0, batch=32,
                                context=4096, rope_base=10000.0, mu_var=0.1),
    "ouro_rho21_b768_n4096": dict(D=24, T=4, H=16, d_head=128, r_k=16, r_v=32, variant=0, batch=768,
                                  context=4096, rope_base=10000.0, mu_var=0.1),
    "ouro_2d_b256_n8192": dict(D=24, T=4, H=16, d_head=128, r_k=64, r_v=128, variant=1, batch=256,
                               context=8192, rope_base=10000.0, mu_var=0.1),
    "huginn_t32_b16_n32768": dict(D=4, T=32, H=16, d_head=128, r_k=96, r_v=160, variant=0, batch=16,
                                  context=32768, rope_base=10000.0, traj_rank=24, noise_var=1e-2,
                                  mu_var=0.1),
    # matched-axis baseline at the ratio-21.3 cache budget: per-loop MLA, a latent over the head
    # axis of each (layer, loop) with no sharing across loops.  The 24 layers x 4 loops become 96
    # single-loop slots; 4 loops x 192 elements = 16 heads x 48 elements per token and layer.
    "mla_perloop_b768_n4096": dict(D=96, T=1, H=16, d_head=128, r_k=64, r_v=128, variant=1, batch=768,
                                   context=4096, rope_base=10000.0, mu_var=0.1),
}


def sub_seed(name: str, base: int = BASE_SEED) -> int:
    """Stable 63-bit seed for a named tensor."""
    h = hashlib.sha256(f"{base:x}/{name}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def rng(name: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(sub_seed(name)))


def torch_generator(name: str, device="cpu"):
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(sub_seed(name))
    return g


def loop_basis(T: int, R: int) -> np.ndarray:
    """phi_m(t) = cos(pi * m * (t + 1/2) / (2T)), m < R: smooth in t, none identically zero."""
    t = np.arange(T, dtype=np.float64)
    return np.stack([np.cos(math.pi * m * (t + 0.5) / (2 * T)) for m in range(R)])  # [R, T]


def smooth_stacks(name: str, n: int, T: int, d: int, R: int, noise_var: float, mu=None,
                  basis_name: str | None = None) -> np.ndarray:
    """n loop stacks x = mu + sum_m g_m (phi_m (x) u_m) + eps, shape [n, T*d].

    u_m ~ N(0, I/d) is fixed per basis name (a (layer, head, axis) slot), the
    coefficients g_m ~ N(0, (1+m)^-2) are drawn per token, eps ~ N(0, noise_var).
    Before noise the stacks are exactly rank <= R around mu.
    """
    r_b = rng((basis_name or name) + "/basis")
    u = r_b.standard_normal((R, d)) / math.sqrt(d)
    phi = loop_basis(T, R)
    r = rng(name)
    g = r.standard_normal((n, R)) / (1.0 + np.arange(R))
    x = np.einsum("nm,mt,md->ntd", g, phi, u).reshape(n, T * d)
    if noise_var > 0:
        x = x + math.sqrt(noise_var) * r.standard_normal((n, T * d))
    if mu is not None:
        x = x + np.asarray(mu)[None, :]
    return x


def gaussian(name: str, shape, var: float = 1.0) -> np.ndarray:
    return math.sqrt(var) * rng(name).standard_normal(shape)


def orthonormal_columns(name: str, S: int, r: int) -> np.ndarray:
    """Seeded S x r matrix with orthonormal columns (QR of a Gaussian, sign-fixed)."""
    a = rng(name).standard_normal((S, r))
    q, rr = np.linalg.qr(a)
    return q * np.where(np.diag(rr) < 0, -1.0, 1.0)[None, :]


def seeded_codec(cfg: dict, tag: str = "codec", layers=None) -> dict:
    """A seeded codec: stacked W_up orthonormal, W_down equal to that stack, mu ~ N(0, mu_var).

    Per-head (variant 0): w_down [D,H,S,r], w_up [D,H,T,d,r], mu [D,H,S] with S = T*d.
    LLA-2D (variant 1):   w_down [D,S2,r],  w_up [D,T,H,d,r], mu [D,S2] with S2 = T*H*d,
    the stack ordered (loop, head, d).
    Every (layer, head, axis) slot draws from its own seed, so `layers` (default: all) may name
    the layers to draw; the others are left at zero.
    """
    D, T, H, d = cfg["D"], cfg["T"], cfg["H"], cfg["d_head"]
    mu_var = cfg.get("mu_var", 0.1)
    layers = range(D) if layers is None else layers
    out = {}
    for axis, r in (("k", cfg["r_k"]), ("v", cfg["r_v"])):
        if cfg["variant"] == 0:
            S = T * d
            wd = np.zeros((D, H, S, r))
            mu = np.zeros((D, H, S))
            for l in layers:
                for h in range(H):
                    wd[l, h] = orthonormal_columns(f"{tag}/{axis}/l{l}/h{h}/w", S, r)
                    mu[l, h] = gaussian(f"{tag}/{axis}/l{l}/h{h}/mu", S, mu_var)
            wu = wd.reshape(D, H, T, d, r).copy()
        else:
            S2 = T * H * d
            wd = np.zeros((D, S2, r))
            mu = np.zeros((D, S2))
            for l in layers:
                wd[l] = orthonormal_columns(f"{tag}/{axis}/l{l}/w", S2, r)
                mu[l] = gaussian(f"{tag}/{axis}/l{l}/mu", S2, mu_var)
            wu = wd.reshape(D, T, H, d, r).copy()
        out[f"w_down_{axis}"] = wd
        out[f"w_up_{axis}"] = wu
        out[f"mu_{axis}"] = mu
    return out


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (nearest-even, via float32) and return them as float64.

    Infinities and NaNs pass through unchanged; for every other float32 bit pattern the
    increment cannot carry out of 32 bits."""
    f = np.array(a, dtype=np.float32)
    u = f.view(np.uint32)
    special = (u & np.uint32(0x7F800000)) == np.uint32(0x7F800000)
    kept = u[special] if special.any() else None
    inc = (u >> np.uint32(16)) & np.uint32(1)
    inc += np.uint32(0x7FFF)
    u += inc
    u &= np.uint32(0xFFFF0000)
    if kept is not None:
        u[special] = kept
    return f.astype(np.float64)


def round_f32(a: np.ndarray) -> np.ndarray:
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def fill_gaussian_bf16_(t, name: str, chunk_elems: int = 1 << 28):
    """Fill a (possibly huge) CUDA bf16 tensor with seeded N(0,1) values in chunks."""
    import torch

    flat = t.view(-1)
    g = torch_generator(name, device=t.device)
    for s in range(0, flat.numel(), chunk_elems):
        e = min(flat.numel(), s + chunk_elems)
        flat[s:e].normal_(0.0, 1.0, generator=g)
    return t
