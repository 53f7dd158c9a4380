"""FP64 CPU oracle for Looped Latent Attention (LLA) decode attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
links this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.  It
shares no code with the CUDA library in ``decode_attention_lla_b200``.

Source.  "Looped Latent Attention: Cross-Loop KV Compression for Looped
Transformers" (O'Neill & Reid, arXiv 2607.15456).  Citations below name the
section and equation of that paper's HTML rendering, written [LLA §3 eq. (2)]
and so on; [LLA abstract] is its abstract and [LLA summary, Serving Capacity]
is the "Technical Summary" page about the same paper.

Everything is plain NumPy in float64.  A library matmul or SVD serves as a
step; nothing is blocked, fused or reordered beyond what the equations state.

Readings of points the paper leaves open:

* RoPE convention: rotate-half pairs (i, i + d/2), frequencies
  theta_i = base ** (-2 i / d).  The paper only cites Su et al. for RoPE.
* Softmax scale: passed explicitly (1/sqrt(d_head) in every workload).
* Positions: cached token j sits at RoPE position j; the query position is
  an argument.  Only cached tokens are attended (the current token's latent
  cannot exist before its last loop, eq. (2) needs the full loop stack).
* mu_t is the loop-t slice of mu; W_up,t is independent of W_down (they
  coincide only at SVD initialisation).
* An empty context (seq_len == 0) yields a zero output.
* Self slot (optional): the current token's latent is written only after
  its last loop, so at decode time its own loop-t key and value are the
  loop's exact vectors; when given, they join the attention as one more
  slot at the query's position.

Parity pins: every public function here is checked by ``tests/test_oracle_*``
against closed forms, printed numbers, special cases that reduce to library
routines, an independent complex-number RoPE, and pure-Python brute force.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "compression_ratio",
    "compression_ratio_2d",
    "uncompressed_scalars_per_token_layer",
    "latent_scalars_per_token_layer",
    "store_bytes",
    "uncompressed_cache_bytes",
    "fit_codec_svd",
    "loop_slices",
    "encode",
    "reconstruct",
    "rope_frequencies",
    "apply_rope",
    "softmax_attention",
    "lla_decode_head",
    "lla_decode",
    "lla_decode_2d",
    "encode_2d",
    "full_decode",
]


# ---------------------------------------------------------------------------
# Cache sizes: [LLA §3, "Teacher cache", eq. (1)] and [LLA §3 eq. (4)]
# ---------------------------------------------------------------------------

def uncompressed_scalars_per_token_layer(T: int, H: int, d_head: int) -> int:
    """K and V for every loop and head: 2*T*H*d_head scalars [LLA §3, eq. (1)]."""
    return 2 * T * H * d_head


def latent_scalars_per_token_layer(H: int, r_k: int, r_v: int, variant: int = 0) -> int:
    """Scalars the latent store keeps per token per layer.

    Per-head LLA keeps (r_k + r_v) * H [LLA §3 eq. (4)]; LLA-2D keeps one
    latent per token and layer, (r_k + r_v) [LLA §3, "LLA-2D variant"].
    """
    if variant == 0:
        return (r_k + r_v) * H
    if variant == 1:
        return r_k + r_v
    raise ValueError("variant must be 0 (per-head) or 1 (2D)")


def compression_ratio(T: int, d_head: int, r_k: int, r_v: int) -> float:
    """rho = 2*T*H*d_head / ((r_k + r_v) * H) [LLA §3 eq. (4)], written as that ratio."""
    H = 1  # cancels; kept to follow the equation's own form
    return uncompressed_scalars_per_token_layer(T, H, d_head) / latent_scalars_per_token_layer(H, r_k, r_v, 0)


def compression_ratio_2d(T: int, H: int, d_head: int, r_k: int, r_v: int) -> float:
    """LLA-2D ratio: the full 2*T*H*d_head cache over r_k + r_v [LLA §3, "LLA-2D variant"]."""
    return uncompressed_scalars_per_token_layer(T, H, d_head) / latent_scalars_per_token_layer(H, r_k, r_v, 1)


def store_bytes(batch: int, tokens: int, D: int, H: int, r_k: int, r_v: int,
                variant: int = 0, bytes_per_scalar: int = 2) -> int:
    """Bytes of a latent store for `batch` sequences of `tokens` cached tokens over D layers."""
    return batch * tokens * D * latent_scalars_per_token_layer(H, r_k, r_v, variant) * bytes_per_scalar


def uncompressed_cache_bytes(batch: int, tokens: int, D: int, T: int, H: int, d_head: int,
                             bytes_per_scalar: int = 2) -> int:
    """Bytes of the loop-indexed teacher cache [LLA §3, "Teacher cache"]."""
    return batch * tokens * D * uncompressed_scalars_per_token_layer(T, H, d_head) * bytes_per_scalar


# ---------------------------------------------------------------------------
# Codec fit: [LLA §3, "Initialisation and conversion"]
# ---------------------------------------------------------------------------

def fit_codec_svd(X: np.ndarray, r: int):
    """SVD initialisation of one (layer, head, axis) codec.

    The calibration stacks X (n x S, S = T*d_head) are centred with their
    mean; W_down is the top-r right singular vectors of the centred matrix
    [LLA §3, "Initialisation and conversion"].  Singular vectors are unique
    only up to sign, so each column is flipped to make its entry of largest
    magnitude positive.

    Returns (mu [S], W_down [S, r], singular_values [min(n, S)]).
    """
    X = np.asarray(X, dtype=np.float64)
    mu = X.mean(axis=0)
    _, s, vt = np.linalg.svd(X - mu, full_matrices=False)
    W = vt[:r].T.copy()
    for a in range(W.shape[1]):
        k = int(np.argmax(np.abs(W[:, a])))
        if W[k, a] < 0:
            W[:, a] = -W[:, a]
    return mu, W, s


def loop_slices(M: np.ndarray, T: int) -> np.ndarray:
    """Split a stacked [T*d, ...] array into its T loop slices [T, d, ...].

    At SVD initialisation the loop-t up-projection is the loop-t row slice of
    W_down, and mu_t is the loop-t slice of mu [LLA §3, "Initialisation and
    conversion"; eq. (3)].
    """
    M = np.asarray(M, dtype=np.float64)
    S = M.shape[0]
    if S % T:
        raise ValueError("leading dimension is not a multiple of T")
    return M.reshape((T, S // T) + M.shape[1:])


# ---------------------------------------------------------------------------
# Encode and reconstruct: [LLA §3 eq. (2)], [LLA §3 eq. (3)]
# ---------------------------------------------------------------------------

def encode(x: np.ndarray, mu: np.ndarray, W_down: np.ndarray) -> np.ndarray:
    """c = (x - mu) W_down  [LLA §3 eq. (2)].  x: [..., S]; returns [..., r]."""
    return (np.asarray(x, np.float64) - np.asarray(mu, np.float64)) @ np.asarray(W_down, np.float64)


def reconstruct(c: np.ndarray, W_up_t: np.ndarray, mu_t: np.ndarray) -> np.ndarray:
    """x_hat_t = c W_up,t^T + mu_t  [LLA §3 eq. (3)].  c: [..., r]; W_up_t: [d, r]."""
    return np.asarray(c, np.float64) @ np.asarray(W_up_t, np.float64).T + np.asarray(mu_t, np.float64)


# ---------------------------------------------------------------------------
# RoPE after reconstruction: [LLA §3, "RoPE and reconstruction"]
# ---------------------------------------------------------------------------

def rope_frequencies(d_head: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/d) for i < d/2 (rotate-half convention)."""
    i = np.arange(d_head // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d_head)


def apply_rope(x: np.ndarray, positions, base: float) -> np.ndarray:
    """Rotate each (i, i + d/2) pair of x by angle position * theta_i.

    The phase depends on the token's position only, which is the same in
    every loop, so it is applied to the reconstructed x_hat_t [LLA §3,
    "RoPE and reconstruction"].  x: [..., n, d] with positions [n], or
    [..., d] with a scalar position.
    """
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    h = d // 2
    theta = rope_frequencies(d, base)
    ang = np.asarray(positions, np.float64)[..., None] * theta  # [n, h] or [h]
    cos, sin = np.cos(ang), np.sin(ang)
    lo, hi = x[..., :h], x[..., h:]
    return np.concatenate([lo * cos - hi * sin, hi * cos + lo * sin], axis=-1)


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def softmax_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """o = sum_j softmax_j(scale * q.k_j) v_j for one query q [d] over K [n, d], V [n, dv].

    The paper keeps the attention computation itself unchanged and only
    changes what the cache stores [LLA §3, opening paragraph].  An empty
    context returns zeros.
    """
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    if K.shape[0] == 0:
        return np.zeros(V.shape[-1], np.float64)
    logits = scale * (K @ np.asarray(q, np.float64))
    w = np.exp(logits - logits.max())
    return (w / w.sum()) @ V


def lla_decode_head(q, cK, cV, muK_t, WupK_t, muV_t, WupV_t, pos_q, scale, base, k_self=None, v_self=None):
    """Loop-t decode attention for one (sequence, head) from latents.

    cK [n, r_k], cV [n, r_v] are the cached latents of tokens 0..n-1 (token j
    at position j).  K and V are fully reconstructed with eq. (3), RoPE is
    applied to the reconstructed keys and to the query, and softmax attention
    follows [LLA §3 eq. (3); "RoPE and reconstruction"].  The latent-space
    shortcut for V is deliberately NOT used here.

    k_self, v_self [d] (optional): the current token's exact loop-t key
    (pre-RoPE) and value.  Its latent does not exist yet (eq. (2) needs the
    whole loop stack), so it joins as one more slot, key rotated at the
    query's position.
    """
    cK = np.asarray(cK, np.float64)
    n = cK.shape[0]
    K_hat = reconstruct(cK, WupK_t, muK_t)
    V_hat = reconstruct(cV, WupV_t, muV_t)
    K_rot = apply_rope(K_hat, np.arange(n), base)
    q_rot = apply_rope(q, pos_q, base)
    if k_self is not None:
        K_rot = np.vstack([K_rot, apply_rope(k_self, pos_q, base)[None]])
        V_hat = np.vstack([V_hat, np.asarray(v_self, np.float64)[None]])
    return softmax_attention(q_rot, K_rot, V_hat, scale)


def lla_decode(q, cK, cV, muK, WupK, muV, WupV, loop, seq_lens, q_pos, scale, base, k_self=None, v_self=None):
    """Per-head LLA decode attention for one (layer, loop) call.

    q       [B, H, d]          pre-RoPE queries
    cK      [B, N, H, r_k]     K latents of the layer (token-major, as cached)
    cV      [B, N, H, r_v]     V latents of the layer
    muK     [H, T, d]          mu_t slices of the K codec   (muV alike)
    WupK    [H, T, d, r_k]     W_up,t of the K codec        (WupV alike)
    loop    t in [0, T)
    seq_lens[B], q_pos[B]      context length and query position per sequence
    k_self, v_self [B, H, d]   optional self slot (see lla_decode_head)
    Returns out [B, H, d].
    """
    q = np.asarray(q, np.float64)
    B, H, d = q.shape
    out = np.zeros((B, H, WupV.shape[2]), np.float64)
    for b in range(B):
        n = int(seq_lens[b])
        for h in range(H):
            ks = None if k_self is None else k_self[b, h]
            vs = None if v_self is None else v_self[b, h]
            out[b, h] = lla_decode_head(q[b, h], cK[b, :n, h], cV[b, :n, h],
                                        muK[h, loop], WupK[h, loop], muV[h, loop], WupV[h, loop],
                                        float(q_pos[b]), scale, base, ks, vs)
    return out


# ---------------------------------------------------------------------------
# LLA-2D (loop x head): [LLA §3, "LLA-2D variant"], Fig. 1(b)
# ---------------------------------------------------------------------------

def encode_2d(x, mu, W_down):
    """One latent per token and layer from the full T*H*d_head stack.

    The stack is ordered (loop, head, d) and encoded with eq. (2) as a whole
    [LLA §3, "LLA-2D variant"].
    """
    return encode(x, mu, W_down)


def lla_decode_2d(q, cK, cV, muK, WupK, muV, WupV, loop, seq_lens, q_pos, scale, base, k_self=None, v_self=None):
    """LLA-2D decode attention: one latent per token decodes all H heads.

    q    [B, H, d]
    cK   [B, N, r_k], cV [B, N, r_v]   one latent per token (per layer)
    muK  [T, H, d], WupK [T, H, d, r_k] per-(loop, head) slices (V alike)
    Head h at loop t reconstructs x_hat_{t,h} = c W_up,(t,h)^T + mu_{t,h}
    [LLA §3, "LLA-2D variant"]; RoPE, attention and the optional self slot
    (k_self, v_self [B, H, d]) as in the per-head case.
    """
    q = np.asarray(q, np.float64)
    B, H, d = q.shape
    out = np.zeros((B, H, WupV.shape[2]), np.float64)
    for b in range(B):
        n = int(seq_lens[b])
        for h in range(H):
            ks = None if k_self is None else k_self[b, h]
            vs = None if v_self is None else v_self[b, h]
            out[b, h] = lla_decode_head(q[b, h], cK[b, :n], cV[b, :n],
                                        muK[loop, h], WupK[loop, h], muV[loop, h], WupV[loop, h],
                                        float(q_pos[b]), scale, base, ks, vs)
    return out


# ---------------------------------------------------------------------------
# Comparator: decode over a full (uncompressed) K/V cache
# ---------------------------------------------------------------------------

def full_decode(q, K_rot, V, seq_lens, q_pos, scale, base):
    """Decode attention over a full cache, the comparator of the latent store.

    The "fast path" the summary page contrasts with the latent path keeps, for
    each cached token, the loop-t key and value themselves [LLA summary,
    "Serving Capacity"; LLA §3, "Teacher cache"]; keys are cached already
    rotated at their positions, so only the query is rotated here.
    q [B, H, d] pre-RoPE; K_rot, V [B, N, H, d]; returns out [B, H, d].
    """
    q = np.asarray(q, np.float64)
    B, H, d = q.shape
    out = np.zeros((B, H, np.asarray(V).shape[-1]), np.float64)
    for b in range(B):
        n = int(seq_lens[b])
        for h in range(H):
            out[b, h] = softmax_attention(apply_rope(q[b, h], float(q_pos[b]), base),
                                          np.asarray(K_rot[b, :n, h], np.float64),
                                          np.asarray(V[b, :n, h], np.float64), scale)
    return out
