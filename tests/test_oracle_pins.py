"""Pins for the FP64 oracle: printed numbers, closed forms, special cases.

Each check here compares the oracle with something other than itself: the
numbers the LLA pages print (tests/golden/serving_capacity.json), library
routines (torch's scaled-dot-product attention in float64, NumPy complex
exponentials for RoPE), exactness that linear algebra guarantees, and the
pure-Python brute force in ``oracle/bruteforce.py``.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import lla_synth as syn
from oracle import bruteforce as bf
from oracle import lla_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "serving_capacity.json")
GiB = 1 << 30


def golden():
    with open(GOLDEN) as f:
        return json.load(f)


# --------------------------------------------------------------------------------------
# independent references (not the oracle's formulas)
# --------------------------------------------------------------------------------------

def rope_complex(x, pos, base):
    """RoPE as a complex rotation of (x_i + i x_{i+d/2}) by exp(i * pos / base^(2i/d))."""
    x = np.asarray(x, np.float64)
    h = x.shape[-1] // 2
    inv = np.exp(-np.log(base) * (2.0 * np.arange(h)) / x.shape[-1])
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * np.asarray(pos, np.float64)[..., None] * inv)
    return np.concatenate([z.real, z.imag], axis=-1)


def sdpa(q, K, V, scale):
    """torch scaled_dot_product_attention in float64 for one query."""
    qt = torch.tensor(q, dtype=torch.float64)[None, None, None, :]
    Kt = torch.tensor(K, dtype=torch.float64)[None, None]
    Vt = torch.tensor(V, dtype=torch.float64)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)[0, 0, 0].numpy()


# --------------------------------------------------------------------------------------
# printed numbers
# --------------------------------------------------------------------------------------

def test_printed_cache_sizes_at_1m_context():
    g = golden()
    m = g["ouro_1p4b"]
    full = O.uncompressed_cache_bytes(1, 1 << 20, m["D"], m["T"], m["H"], m["d_head"])
    lla = O.store_bytes(1, 1 << 20, m["D"], m["H"], 16, 32)
    assert full == g["kv_cache_1m_context_uncompressed_gib"]["value"] * GiB
    assert lla == g["kv_cache_1m_context_lla_gib"]["value"] * GiB
    rho = O.compression_ratio(m["T"], m["d_head"], 16, 32)
    assert round(rho, g["compression_ratio_serving"]["decimals"]) == g["compression_ratio_serving"]["value"]
    assert full / lla == pytest.approx(rho, rel=1e-12)


def test_printed_decoder_equivalent_and_final_loop_ratio():
    g = golden()
    m = g["ouro_1p4b"]
    per_loop_layer = 2 * m["H"] * m["d_head"]  # one ordinary decoder layer's K+V per token
    assert O.uncompressed_scalars_per_token_layer(m["T"], m["H"], m["d_head"]) * m["D"] == \
        g["decoder_layers_equivalent"]["value"] * per_loop_layer
    # caching only the final loop keeps 2*H*d per token per layer: ratio T
    assert O.uncompressed_scalars_per_token_layer(m["T"], m["H"], m["d_head"]) / per_loop_layer == \
        g["final_loop_reuse_ratio_t4"]["value"]


def test_printed_batch_capacity_is_consistent():
    """32 uncompressed and 768 latent sequences at 4k fit the same device; 2x each does not."""
    g = golden()
    m = g["ouro_1p4b"]
    full32 = O.uncompressed_cache_bytes(g["max_batch_uncompressed_4k"]["value"], 4096, m["D"], m["T"], m["H"], m["d_head"])
    lla768 = O.store_bytes(g["max_batch_lla_4k"]["value"], 4096, m["D"], m["H"], 16, 32)
    assert full32 == 96 * GiB
    assert lla768 == 108 * GiB
    # same ratio as the cache-size figure: 768/32 = 24 sequences per uncompressed one
    assert lla768 / 768 * 32 == pytest.approx(full32 / O.compression_ratio(4, 128, 16, 32), rel=1e-12)
    assert O.store_bytes(2 * 768, 4096, m["D"], m["H"], 16, 32) > 2 * lla768 - 1


def test_ratio_2d_and_per_head_sizes():
    # LLA-2D stores H times fewer scalars than per-head LLA at equal ranks
    assert O.latent_scalars_per_token_layer(16, 64, 128, 0) == 16 * O.latent_scalars_per_token_layer(16, 64, 128, 1)
    assert O.compression_ratio_2d(4, 16, 128, 64, 128) == pytest.approx(16 * O.compression_ratio(4, 128, 64, 128))
    for name, cfg in syn.CONFIGS.items():
        v = cfg["variant"]
        bytes_ = O.store_bytes(cfg["batch"], cfg["context"], cfg["D"], cfg["H"], cfg["r_k"], cfg["r_v"], v)
        full = O.uncompressed_cache_bytes(cfg["batch"], cfg["context"], cfg["D"], cfg["T"], cfg["H"], cfg["d_head"])
        rho = O.compression_ratio(cfg["T"], cfg["d_head"], cfg["r_k"], cfg["r_v"]) if v == 0 else \
            O.compression_ratio_2d(cfg["T"], cfg["H"], cfg["d_head"], cfg["r_k"], cfg["r_v"])
        assert full / bytes_ == pytest.approx(rho, rel=1e-12), name


# --------------------------------------------------------------------------------------
# codec exactness
# --------------------------------------------------------------------------------------

def test_full_rank_codec_is_exact():
    T, d = 3, 4
    S = T * d
    X = syn.gaussian("pin/fullrank/calib", (200, S))
    mu, W, _ = O.fit_codec_svd(X, S)
    assert np.allclose(W.T @ W, np.eye(S), atol=1e-12)
    x = syn.gaussian("pin/fullrank/x", (7, S))
    c = O.encode(x, mu, W)
    Wt, mut = O.loop_slices(W, T), O.loop_slices(mu, T)
    for t in range(T):
        assert np.abs(O.reconstruct(c, Wt[t], mut[t]) - x[:, t * d:(t + 1) * d]).max() < 1e-12


@pytest.mark.parametrize("R,r", [(3, 3), (3, 5), (6, 6)])
def test_exact_recovery_on_rank_r_data(R, r):
    T, d = 4, 8
    mu = syn.gaussian("pin/rank/mu", T * d, 0.1)
    X = syn.smooth_stacks("pin/rank/calib", 300, T, d, R, 0.0, mu, basis_name="pin/rank")
    m, W, s = O.fit_codec_svd(X, r)
    assert s[R - 1] > 1e-6 and (len(s) <= R or s[R] < 1e-10)  # exactly rank R around the mean
    x = syn.smooth_stacks("pin/rank/fresh", 20, T, d, R, 0.0, mu, basis_name="pin/rank")
    c = O.encode(x, m, W)
    for t in range(T):
        xt = O.reconstruct(c, O.loop_slices(W, T)[t], O.loop_slices(m, T)[t])
        assert np.abs(xt - x[:, t * d:(t + 1) * d]).max() < 1e-10


def test_truncation_error_decreases_with_rank():
    T, d, R = 4, 8, 6
    X = syn.smooth_stacks("pin/trunc/calib", 400, T, d, R, 1e-4, None, basis_name="pin/trunc")
    x = syn.smooth_stacks("pin/trunc/fresh", 50, T, d, R, 1e-4, None, basis_name="pin/trunc")
    errs = []
    for r in range(1, 9):
        m, W, _ = O.fit_codec_svd(X, r)
        xh = np.concatenate([O.reconstruct(O.encode(x, m, W), O.loop_slices(W, T)[t], O.loop_slices(m, T)[t])
                             for t in range(T)], axis=1)
        errs.append(np.linalg.norm(xh - x))
    assert all(a >= b - 1e-12 for a, b in zip(errs, errs[1:]))
    noise_norm = math.sqrt(50 * T * d * 1e-4)
    assert errs[R - 1] < 1.1 * noise_norm < errs[R - 2] / 1.5  # rank R reaches the noise floor


def test_svd_sign_convention_and_subspace_vs_jacobi():
    X = syn.gaussian("pin/jacobi/X", (40, 6)) @ np.diag([3, 2.5, 2, 1, 0.5, 0.1])
    mu, W, _ = O.fit_codec_svd(X, 3)
    for a in range(3):
        assert W[np.argmax(np.abs(W[:, a])), a] > 0
    mu_b, W_b = bf.fit_codec(X.tolist(), 3)
    assert np.allclose(mu, mu_b, atol=1e-13)
    Wb = np.array(W_b)
    assert np.allclose(W @ W.T, Wb @ Wb.T, atol=1e-9)  # same rank-3 subspace


# --------------------------------------------------------------------------------------
# RoPE
# --------------------------------------------------------------------------------------

def test_rope_matches_complex_rotation():
    x = syn.gaussian("pin/rope/x", (9, 16))
    pos = np.arange(9) * 37.0 + 5
    assert np.allclose(O.apply_rope(x, pos, 10000.0), rope_complex(x, pos, 10000.0), atol=1e-12)
    assert np.allclose(O.apply_rope(x[0], 4096.0, 500.0), rope_complex(x[0], 4096.0, 500.0), atol=1e-12)


def test_rope_norm_identity_and_relative_positions():
    q = syn.gaussian("pin/rope/q", 32)
    k = syn.gaussian("pin/rope/k", 32)
    assert np.allclose(O.apply_rope(q, 0.0, 10000.0), q, atol=0)
    for p in (1.0, 77.0, 32767.0):
        assert np.linalg.norm(O.apply_rope(q, p, 10000.0)) == pytest.approx(np.linalg.norm(q), rel=1e-13)
    ref = O.apply_rope(q, 10.0, 10000.0) @ O.apply_rope(k, 3.0, 10000.0)
    for shift in (0.0, 1.0, 100.0, 5000.0):
        got = O.apply_rope(q, 10.0 + shift, 10000.0) @ O.apply_rope(k, 3.0 + shift, 10000.0)
        assert got == pytest.approx(ref, rel=1e-9, abs=1e-9)


# --------------------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------------------

def _codec_from_fit(X, r, T):
    mu, W, _ = O.fit_codec_svd(X, r)
    return mu, W, O.loop_slices(W, T), O.loop_slices(mu, T)


def test_lla_equals_uncompressed_attention_on_exact_data():
    """With lossless codecs, LLA attention is ordinary RoPE attention over the teacher K/V."""
    T, d, R, n = 4, 8, 5, 33
    base, scale = 10000.0, 1 / math.sqrt(8)
    muK, muV = syn.gaussian("pin/eq/muK", T * d, 0.1), syn.gaussian("pin/eq/muV", T * d, 0.1)
    XK = syn.smooth_stacks("pin/eq/calK", 300, T, d, R, 0.0, muK, basis_name="pin/eq/K")
    XV = syn.smooth_stacks("pin/eq/calV", 300, T, d, R, 0.0, muV, basis_name="pin/eq/V")
    mK, WK, WKt, mKt = _codec_from_fit(XK, R, T)
    mV, WV, WVt, mVt = _codec_from_fit(XV, R + 2, T)
    xK = syn.smooth_stacks("pin/eq/K", n, T, d, R, 0.0, muK, basis_name="pin/eq/K")
    xV = syn.smooth_stacks("pin/eq/V", n, T, d, R, 0.0, muV, basis_name="pin/eq/V")
    cK, cV = O.encode(xK, mK, WK), O.encode(xV, mV, WV)
    q = syn.gaussian("pin/eq/q", d)
    for t in range(T):
        got = O.lla_decode_head(q, cK, cV, mKt[t], WKt[t], mVt[t], WVt[t], n, scale, base)
        Kt = rope_complex(xK[:, t * d:(t + 1) * d], np.arange(n), base)
        ref = sdpa(rope_complex(q, n, base), Kt, xV[:, t * d:(t + 1) * d], scale)
        assert np.abs(got - ref).max() < 1e-10


def test_single_loop_full_rank_is_textbook_rope_attention():
    d, n = 16, 20
    W = syn.orthonormal_columns("pin/t1/W", d, d)
    mu = syn.gaussian("pin/t1/mu", d, 0.1)
    K = syn.gaussian("pin/t1/K", (n, d))
    V = syn.gaussian("pin/t1/V", (n, d))
    q = syn.gaussian("pin/t1/q", d)
    cK, cV = O.encode(K, mu, W), O.encode(V, mu, W)
    got = O.lla_decode_head(q, cK, cV, mu, W, mu, W, 27.0, 0.25, 10000.0)
    ref = sdpa(rope_complex(q, 27.0, 10000.0), rope_complex(K, np.arange(n), 10000.0), V, 0.25)
    assert np.abs(got - ref).max() < 1e-12


def test_v_identity_in_latent_space():
    """sum_j p_j x_hat_j = (sum_j p_j c_j) W_up^T + mu_t, because the p_j sum to one."""
    T, d, rk, rv, n = 4, 16, 4, 8, 40
    cK = syn.gaussian("pin/vid/cK", (n, rk))
    cV = syn.gaussian("pin/vid/cV", (n, rv))
    WK = syn.gaussian("pin/vid/WK", (d, rk), 0.1)
    WV = syn.gaussian("pin/vid/WV", (d, rv), 0.1)
    muK, muV = syn.gaussian("pin/vid/muK", d), syn.gaussian("pin/vid/muV", d)
    q = syn.gaussian("pin/vid/q", d)
    got = O.lla_decode_head(q, cK, cV, muK, WK, muV, WV, n, 0.25, 10000.0)
    Krot = rope_complex(cK @ WK.T + muK, np.arange(n), 10000.0)
    logits = 0.25 * Krot @ rope_complex(q, n, 10000.0)
    p = np.exp(logits - logits.max())
    p /= p.sum()
    assert np.abs(got - ((p @ cV) @ WV.T + muV)).max() < 1e-13


def test_self_slot_with_empty_cache_is_its_value():
    """With no cached token the softmax has the self slot alone: the output is v_self."""
    d, rk, rv = 8, 3, 5
    q = syn.gaussian("pin/self0/q", d)
    ks, vs = syn.gaussian("pin/self0/k", d), syn.gaussian("pin/self0/v", d)
    W = syn.gaussian("pin/self0/W", (d, rk))
    got = O.lla_decode_head(q, np.zeros((0, rk)), np.zeros((0, rv)), np.zeros(d), W, np.zeros(d),
                            np.zeros((d, rv)), 11.0, 0.5, 10000.0, ks, vs)
    assert np.abs(got - vs).max() < 1e-15


def test_self_slot_matches_sdpa_over_the_appended_token():
    """Self slot = one more key/value row, the key rotated at the query's position."""
    d, rk, rv, n, pos = 16, 4, 6, 25, 31.0
    cK, cV = syn.gaussian("pin/self/cK", (n, rk)), syn.gaussian("pin/self/cV", (n, rv))
    WK, WV = syn.gaussian("pin/self/WK", (d, rk), 0.3), syn.gaussian("pin/self/WV", (d, rv), 0.3)
    muK, muV = syn.gaussian("pin/self/muK", d), syn.gaussian("pin/self/muV", d)
    q = syn.gaussian("pin/self/q", d)
    ks, vs = syn.gaussian("pin/self/k", d), syn.gaussian("pin/self/v", d)
    got = O.lla_decode_head(q, cK, cV, muK, WK, muV, WV, pos, 0.3, 10000.0, ks, vs)
    K = np.vstack([rope_complex(cK @ WK.T + muK, np.arange(n), 10000.0), rope_complex(ks, pos, 10000.0)[None]])
    V = np.vstack([cV @ WV.T + muV, vs[None]])
    ref = sdpa(rope_complex(q, pos, 10000.0), K, V, 0.3)
    assert np.abs(got - ref).max() < 1e-12
    # query and self key share one rotation, which cancels: the self logit is scale * <q, k_self>
    lg = np.append(0.3 * K[:n] @ rope_complex(q, pos, 10000.0), 0.3 * q @ ks)
    p = np.exp(lg - lg.max())
    assert np.abs(got - (p / p.sum()) @ V).max() < 1e-12


def test_full_cache_decode_equals_lla_on_the_reconstructed_cache():
    """The comparator over the cache a fast path would build (keys reconstructed and rotated at
    their positions, values reconstructed) gives the LLA result; and it is SDPA per head."""
    B, n, H, d, rk, rv, T, t = 2, 30, 3, 16, 4, 6, 3, 1
    cK = syn.gaussian("pin/full/cK", (B, n, H, rk))
    cV = syn.gaussian("pin/full/cV", (B, n, H, rv))
    WK, WV = syn.gaussian("pin/full/WK", (H, T, d, rk), 0.3), syn.gaussian("pin/full/WV", (H, T, d, rv), 0.3)
    muK, muV = syn.gaussian("pin/full/muK", (H, T, d)), syn.gaussian("pin/full/muV", (H, T, d))
    q = syn.gaussian("pin/full/q", (B, H, d))
    lens, qpos = np.array([n, 17]), np.array([n, 40])
    K = np.einsum("bnha,hda->bnhd", cK, WK[:, t]) + muK[None, None, :, t]
    V = np.einsum("bnha,hda->bnhd", cV, WV[:, t]) + muV[None, None, :, t]
    K_rot = rope_complex(K, np.arange(n)[None, :, None], 10000.0)
    got = O.full_decode(q, K_rot, V, lens, qpos, 0.25, 10000.0)
    ref = O.lla_decode(q, cK, cV, muK, WK, muV, WV, t, lens, qpos, 0.25, 10000.0)
    assert np.abs(got - ref).max() < 1e-12
    for b in range(B):
        for h in range(H):
            r = sdpa(rope_complex(q[b, h], float(qpos[b]), 10000.0), K_rot[b, :lens[b], h], V[b, :lens[b], h], 0.25)
            assert np.abs(got[b, h] - r).max() < 1e-12


def test_softmax_special_cases():
    d, n = 8, 12
    V = syn.gaussian("pin/sm/V", (n, d))
    K = syn.gaussian("pin/sm/K", (n, d))
    assert np.allclose(O.softmax_attention(np.zeros(d), K, V, 1.0), V.mean(0), atol=1e-14)
    q = 1e3 * K[5] / np.linalg.norm(K[5])
    Kn = K / np.linalg.norm(K, axis=1, keepdims=True)
    assert np.allclose(O.softmax_attention(q, Kn, V, 1.0), V[5], atol=1e-12)
    assert np.all(O.softmax_attention(q, Kn[:0], V[:0], 1.0) == 0)


def test_2d_with_one_head_equals_per_head():
    T, d, rk, rv, n, B = 3, 8, 5, 6, 10, 2
    WK = syn.gaussian("pin/2d/WK", (T, 1, d, rk), 0.2)
    WV = syn.gaussian("pin/2d/WV", (T, 1, d, rv), 0.2)
    muK, muV = syn.gaussian("pin/2d/muK", (T, 1, d)), syn.gaussian("pin/2d/muV", (T, 1, d))
    cK, cV = syn.gaussian("pin/2d/cK", (B, n, rk)), syn.gaussian("pin/2d/cV", (B, n, rv))
    q = syn.gaussian("pin/2d/q", (B, 1, d))
    lens, qpos = np.array([n, 7]), np.array([n, 9])
    for t in range(T):
        a = O.lla_decode_2d(q, cK, cV, muK, WK, muV, WV, t, lens, qpos, 0.3, 10000.0)
        b = O.lla_decode(q, cK[:, :, None], cV[:, :, None], muK.transpose(1, 0, 2), WK.transpose(1, 0, 2, 3),
                         muV.transpose(1, 0, 2), WV.transpose(1, 0, 2, 3), t, lens, qpos, 0.3, 10000.0)
        assert np.abs(a - b).max() == 0.0


# --------------------------------------------------------------------------------------
# brute force
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("case", [dict(T=2, d=4, rk=2, rv=3, n=8, H=2, B=2),
                                  dict(T=4, d=16, rk=4, rv=8, n=64, H=2, B=1)])
def test_vectorised_oracle_matches_brute_force(case):
    T, d, rk, rv, n, H, B = (case[k] for k in ("T", "d", "rk", "rv", "n", "H", "B"))
    S = T * d
    base, scale = 10000.0, 1 / math.sqrt(d)
    tag = f"pin/bf/{T}/{d}"
    XK = syn.smooth_stacks(tag + "/calK", 64, T, d, 3, 1e-3, syn.gaussian(tag + "/muK", S, 0.1), basis_name=tag + "K")
    XV = syn.smooth_stacks(tag + "/calV", 64, T, d, 3, 1e-3, syn.gaussian(tag + "/muV", S, 0.1), basis_name=tag + "V")
    mK, WK, _ = O.fit_codec_svd(XK, rk)
    mV, WV, _ = O.fit_codec_svd(XV, rv)
    x = syn.smooth_stacks(tag + "/x", 3, T, d, 3, 1e-3, None, basis_name=tag + "K")
    cv = O.encode(x, mK, WK)
    cb = [bf.encode(row, mK.tolist(), WK.tolist()) for row in x.tolist()]
    assert np.abs(cv - np.array(cb)).max() < 1e-12
    WKt, mKt = O.loop_slices(WK, T), O.loop_slices(mK, T)
    WVt, mVt = O.loop_slices(WV, T), O.loop_slices(mV, T)
    cK = syn.gaussian(tag + "/cK", (B, n, H, rk))
    cV = syn.gaussian(tag + "/cV", (B, n, H, rv))
    q = syn.gaussian(tag + "/q", (B, H, d))
    lens = np.array([n - b for b in range(B)])
    qpos = lens + 1
    muK = np.stack([mKt] * H)
    muV = np.stack([mVt] * H)
    WupK = np.stack([WKt] * H)
    WupV = np.stack([WVt] * H)
    ks, vs = syn.gaussian(tag + "/ks", (B, H, d)), syn.gaussian(tag + "/vs", (B, H, d))
    for t in range(T):
        got = O.lla_decode(q, cK, cV, muK, WupK, muV, WupV, t, lens, qpos, scale, base)
        got_self = O.lla_decode(q, cK, cV, muK, WupK, muV, WupV, t, lens, qpos, scale, base, ks, vs)
        for b in range(B):
            for h in range(H):
                args = (q[b, h].tolist(), cK[b, :lens[b], h].tolist(), cV[b, :lens[b], h].tolist(),
                        mKt[t].tolist(), WKt[t].tolist(), mVt[t].tolist(), WVt[t].tolist(), float(qpos[b]), scale,
                        base)
                ref = bf.decode_head(*args)
                assert np.abs(got[b, h] - np.array(ref)).max() < 1e-12
                ref_self = bf.decode_head(*args, ks[b, h].tolist(), vs[b, h].tolist())
                assert np.abs(got_self[b, h] - np.array(ref_self)).max() < 1e-12


def test_tiny_workload_codec_properties():
    """The tiny workload's V codec (r_v=8 >= trajectory rank 6) leaves only noise-level error."""
    cfg = syn.CONFIGS["tiny_d16_t4"]
    T, d = cfg["T"], cfg["d_head"]
    S = T * d
    mu = syn.gaussian("pin/tiny/mu", S, 0.1)
    X = syn.smooth_stacks("pin/tiny/calib", cfg["calib"], T, d, cfg["traj_rank"], cfg["noise_var"], mu, basis_name="pin/tiny")
    x = syn.smooth_stacks("pin/tiny/x", 64, T, d, cfg["traj_rank"], cfg["noise_var"], mu, basis_name="pin/tiny")
    noise_rms = math.sqrt(cfg["noise_var"])
    errs = {}
    for r in (cfg["r_k"], cfg["r_v"]):
        m, W, _ = O.fit_codec_svd(X, r)
        xh = np.concatenate([O.reconstruct(O.encode(x, m, W), O.loop_slices(W, T)[t], O.loop_slices(m, T)[t])
                             for t in range(T)], axis=1)
        errs[r] = np.sqrt(np.mean((xh - x) ** 2))
    assert errs[cfg["r_v"]] < 1.2 * noise_rms
    assert errs[cfg["r_k"]] > errs[cfg["r_v"]]
