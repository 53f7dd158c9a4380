"""Shared helpers for the GPU parity tests: codecs, stores, comparisons.

Inputs come from ``lla_synth`` (random numbers only) and, where the method
itself is needed to make an input (an SVD-fitted codec, oracle-encoded
latents), from the FP64 oracle.  Nothing here takes a value from the CUDA
path as an input or an expected value.
"""

from __future__ import annotations

import math

import numpy as np

import lla_synth as syn
from oracle import lla_oracle as O

# Acceptance bar for attention outputs and latents (bf16 storage, fp32 accumulation).
REL_L2_TOL = 5e-3
MAX_ABS_TOL = 2e-2


def rel_l2(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def assert_close(got, ref, what=""):
    e = rel_l2(got, ref)
    m = float(np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64)).max()) if np.size(ref) else 0.0
    assert e <= REL_L2_TOL and m <= MAX_ABS_TOL, f"{what}: rel_l2={e:.3e} max_abs={m:.3e}"
    return e, m


def rounded_codec(codec: dict) -> dict:
    """The values both sides use: W_down rounded to bf16, W_up and mu to float32."""
    out = {}
    for k, v in codec.items():
        out[k] = syn.round_bf16(v) if k.startswith("w_down") else syn.round_f32(v)
    return out


def make_lib_codec(lla, desc_kw: dict, codec: dict):
    desc = lla.Desc(**desc_kw)
    return lla.Codec(desc, codec["w_down_k"], codec["w_down_v"], codec["w_up_k"], codec["w_up_v"],
                     codec["mu_k"], codec["mu_v"])


def svd_codec(cfg: dict, tag: str) -> dict:
    """Per-head codec fitted by the oracle's SVD on seeded calibration stacks."""
    D, T, H, d = cfg["D"], cfg["T"], cfg["H"], cfg["d_head"]
    S = T * d
    out = {k: [] for k in ("w_down_k", "w_down_v", "w_up_k", "w_up_v", "mu_k", "mu_v")}
    for axis, r in (("k", cfg["r_k"]), ("v", cfg["r_v"])):
        wd = np.empty((D, H, S, r))
        mu = np.empty((D, H, S))
        for l in range(D):
            for h in range(H):
                slot = f"{tag}/{axis}/l{l}/h{h}"
                m0 = syn.gaussian(slot + "/mu", S, cfg.get("mu_var", 0.1))
                X = syn.smooth_stacks(slot + "/calib", cfg.get("calib", 512), T, d, cfg["traj_rank"],
                                      cfg["noise_var"], m0, basis_name=slot)
                mu[l, h], wd[l, h], _ = O.fit_codec_svd(X, r)
        out[f"w_down_{axis}"] = wd
        out[f"w_up_{axis}"] = wd.reshape(D, H, T, d, r).copy()
        out[f"mu_{axis}"] = mu
    return out


def to_bf16_bits(a) -> np.ndarray:
    """float64 array -> bf16 bit patterns (uint16), nearest-even."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF
    return u.astype(np.uint16)


def from_bf16_bits(u) -> np.ndarray:
    return (np.asarray(u, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def pack_store(cK, cV, variant: int) -> np.ndarray:
    """Per-head: cK [B,D,N,H,rk], cV [B,D,N,H,rv] -> bf16 bits [B,D,N,H,rk+rv].
    2D: cK [B,D,N,rk], cV [B,D,N,rv] -> [B,D,N,rk+rv]."""
    return to_bf16_bits(np.concatenate([cK, cV], axis=-1))


def unpack_layer(store_bits: np.ndarray, layer: int, rk: int):
    """bf16 store bits -> (cK, cV) float64 of one layer."""
    s = from_bf16_bits(store_bits[:, layer])
    return s[..., :rk], s[..., rk:]


def oracle_decode(codec: dict, cfg: dict, cK, cV, q, layer, loop, seq_lens, q_pos, scale, k_self=None, v_self=None):
    """Oracle output for one (layer, loop) call; codec is the rounded dict; optional self slot."""
    T, H, d = cfg["T"], cfg["H"], cfg["d_head"]
    base = cfg.get("rope_base", 10000.0)
    if cfg["variant"] == 0:
        muK = codec["mu_k"][layer].reshape(H, T, d)
        muV = codec["mu_v"][layer].reshape(H, T, d)
        return O.lla_decode(q, cK, cV, muK, codec["w_up_k"][layer], muV, codec["w_up_v"][layer], loop,
                            seq_lens, q_pos, scale, base, k_self, v_self)
    muK = codec["mu_k"][layer].reshape(T, H, d)
    muV = codec["mu_v"][layer].reshape(T, H, d)
    return O.lla_decode_2d(q, cK, cV, muK, codec["w_up_k"][layer], muV, codec["w_up_v"][layer], loop,
                           seq_lens, q_pos, scale, base, k_self, v_self)


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
