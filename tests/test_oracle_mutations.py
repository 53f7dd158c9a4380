"""Planted mistakes in the oracle must be caught by its pins.

Each mutation below is a plausible slip in restating the LLA equations (a
dropped term, a wrong sign, index or operand).  It is planted in the oracle
module on the CPU, and the pin tests of ``test_oracle_pins.py`` are run
against the mutated oracle: at least one of them has to fail.
"""

import numpy as np
import pytest

import test_oracle_pins as pins
from oracle import lla_oracle as O

PIN_TESTS = [
    pins.test_printed_cache_sizes_at_1m_context,
    pins.test_printed_decoder_equivalent_and_final_loop_ratio,
    pins.test_printed_batch_capacity_is_consistent,
    pins.test_full_rank_codec_is_exact,
    lambda: pins.test_exact_recovery_on_rank_r_data(3, 5),
    pins.test_svd_sign_convention_and_subspace_vs_jacobi,
    pins.test_rope_matches_complex_rotation,
    pins.test_rope_norm_identity_and_relative_positions,
    pins.test_lla_equals_uncompressed_attention_on_exact_data,
    pins.test_single_loop_full_rank_is_textbook_rope_attention,
    pins.test_v_identity_in_latent_space,
    pins.test_softmax_special_cases,
    pins.test_self_slot_with_empty_cache_is_its_value,
    pins.test_self_slot_matches_sdpa_over_the_appended_token,
    pins.test_full_cache_decode_equals_lla_on_the_reconstructed_cache,
    lambda: pins.test_vectorised_oracle_matches_brute_force(dict(T=2, d=4, rk=2, rv=3, n=8, H=2, B=2)),
]

_orig = {k: getattr(O, k) for k in ("reconstruct", "encode", "apply_rope", "rope_frequencies",
                                      "softmax_attention", "fit_codec_svd", "lla_decode_head",
                                      "store_bytes", "uncompressed_scalars_per_token_layer")}


def _drop_mu(c, W, mu):
    return np.asarray(c, np.float64) @ np.asarray(W, np.float64).T


def _flip_rows(c, W, mu):
    return _orig["reconstruct"](c, np.asarray(W)[::-1], mu)


def _no_centering(x, mu, W):
    return np.asarray(x, np.float64) @ np.asarray(W, np.float64)


def _rope_sign(x, positions, base):
    return _orig["apply_rope"](x, -np.asarray(positions, np.float64), base)


def _rope_freq(d, base):
    return np.power(float(base), -1.0 * np.arange(d // 2) / d)


def _rope_pairing(x, positions, base):
    """Adjacent pairs (2i, 2i+1) instead of (i, i + d/2)."""
    x = np.asarray(x, np.float64)
    perm = np.concatenate([np.arange(0, x.shape[-1], 2), np.arange(1, x.shape[-1], 2)])
    inv = np.argsort(perm)
    return _orig["apply_rope"](x[..., perm], positions, base)[..., inv]


def _softmax_unscaled(q, K, V, scale):
    return _orig["softmax_attention"](q, K, V, 1.0)


def _softmax_unnormalised(q, K, V, scale):
    K = np.asarray(K, np.float64)
    if K.shape[0] == 0:
        return np.zeros(np.asarray(V).shape[-1])
    lg = scale * K @ q
    return np.exp(lg - lg.max()) @ V


def _fit_uncentred(X, r):
    X = np.asarray(X, np.float64)
    mu, W, s = _orig["fit_codec_svd"](X, r)
    _, s2, vt = np.linalg.svd(X, full_matrices=False)
    return mu, vt[:r].T.copy(), s2


def _with_self(K, V, k_self, v_self, pos_q, base, self_pos=None):
    if k_self is None:
        return K, V
    p = pos_q if self_pos is None else self_pos
    return (np.vstack([K, O.apply_rope(k_self, p, base)[None]]),
            np.vstack([V, np.asarray(v_self, np.float64)[None]]))


def _decode_shift_positions(q, cK, cV, muK_t, WupK_t, muV_t, WupV_t, pos_q, scale, base, k_self=None, v_self=None):
    n = np.asarray(cK).shape[0]
    K = O.apply_rope(O.reconstruct(cK, WupK_t, muK_t), np.arange(1, n + 1), base)
    V = O.reconstruct(cV, WupV_t, muV_t)
    K, V = _with_self(K, V, k_self, v_self, pos_q, base)
    return O.softmax_attention(O.apply_rope(q, pos_q, base), K, V, scale)


def _decode_rope_on_v(q, cK, cV, muK_t, WupK_t, muV_t, WupV_t, pos_q, scale, base, k_self=None, v_self=None):
    n = np.asarray(cK).shape[0]
    K = O.apply_rope(O.reconstruct(cK, WupK_t, muK_t), np.arange(n), base)
    V = O.apply_rope(O.reconstruct(cV, WupV_t, muV_t), np.arange(n), base)
    K, V = _with_self(K, V, k_self, v_self, pos_q, base)
    return O.softmax_attention(O.apply_rope(q, pos_q, base), K, V, scale)


def _decode_self_unrotated(q, cK, cV, muK_t, WupK_t, muV_t, WupV_t, pos_q, scale, base, k_self=None, v_self=None):
    """The self key enters at position 0 instead of the query's position."""
    n = np.asarray(cK).shape[0]
    K = O.apply_rope(O.reconstruct(cK, WupK_t, muK_t), np.arange(n), base)
    V = O.reconstruct(cV, WupV_t, muV_t)
    K, V = _with_self(K, V, k_self, v_self, pos_q, base, self_pos=0.0)
    return O.softmax_attention(O.apply_rope(q, pos_q, base), K, V, scale)


def _decode_self_dropped(q, cK, cV, muK_t, WupK_t, muV_t, WupV_t, pos_q, scale, base, k_self=None, v_self=None):
    return _orig["lla_decode_head"](q, cK, cV, muK_t, WupK_t, muV_t, WupV_t, pos_q, scale, base)


def _store_bytes_fp32(batch, tokens, D, H, r_k, r_v, variant=0, bytes_per_scalar=2):
    return _orig["store_bytes"](batch, tokens, D, H, r_k, r_v, variant, 4)


def _scalars_one_axis(T, H, d_head):
    return T * H * d_head


MUTATIONS = {
    "reconstruct drops mu_t": ("reconstruct", _drop_mu),
    "reconstruct reads W_up rows reversed": ("reconstruct", _flip_rows),
    "encode skips centring": ("encode", _no_centering),
    "RoPE rotates the wrong way": ("apply_rope", _rope_sign),
    "RoPE frequency exponent -i/d": ("rope_frequencies", _rope_freq),
    "RoPE pairs adjacent lanes": ("apply_rope", _rope_pairing),
    "softmax ignores the scale": ("softmax_attention", _softmax_unscaled),
    "softmax not normalised": ("softmax_attention", _softmax_unnormalised),
    "SVD fit on uncentred stacks": ("fit_codec_svd", _fit_uncentred),
    "keys at positions 1..n": ("lla_decode_head", _decode_shift_positions),
    "RoPE applied to values": ("lla_decode_head", _decode_rope_on_v),
    "self key not rotated to the query position": ("lla_decode_head", _decode_self_unrotated),
    "self slot dropped": ("lla_decode_head", _decode_self_dropped),
    "store counted in fp32": ("store_bytes", _store_bytes_fp32),
    "teacher cache counts one axis": ("uncompressed_scalars_per_token_layer", _scalars_one_axis),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = 0
    for t in PIN_TESTS:
        try:
            t()
        except Exception:  # AssertionError or a shape error: the pin caught it
            failed += 1
    assert failed > 0, f"no pin catches: {name}"
