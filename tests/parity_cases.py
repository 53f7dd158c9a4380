"""Decode parity input sets, shared by the GPU parity tests and the CPU sensitivity test.

Seeded latents and codecs come from ``lla_synth``.  The queries are aimed: for each (sequence,
head) the query is solved so that three of the cached keys (the last one and two others) get
logits of L = ln(n) + 7, 0.85 L and 0.7 L, and the mean of all the rotated keys gets logit 0; a
seeded N(0, 1) query is added on top.  The keys are the oracle's reconstructed, rotated keys
[LLA §3 eq. (3); "RoPE and reconstruction"], so this module uses the FP64 oracle to make inputs
(never the CUDA path).

Why aim the queries: with q ~ N(0, 1), latents ~ N(0, 1) and mu ~ N(0, 0.1) the logits spread by
about 0.3, attention is almost uniform and the output is dominated by mu^V_t.  A kernel that
scored every token alike, put the query one position off or dropped a sequence's last token then
still met the acceptance bar.  With aimed queries the logits spread by 2.4-5, three tokens carry
most of the weight, and each of those mistakes misses the bar by a wide margin (pinned on the CPU
by ``test_parity_sensitivity.py`` for every set listed in ``SETS``).

Every set is also checked on the attention-dependent part of the output, out - mu^V_t, and some
use a codec with mu^V = 0, where the whole output depends on the attention.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

import lla_synth as syn
from lla_testutil import (MAX_ABS_TOL, REL_L2_TOL, oracle_decode, rel_l2, rounded_codec, svd_codec,
                          to_bf16_bits)
from oracle import lla_oracle as O

ROPE_BASE = 10000.0
PEAK_MARGIN_NATS = 7.0          # L = ln(n) + 7 for the last cached token
TARGET_LEVELS = (1.0, 0.85, 0.7)  # relative logit of the three aimed keys


# ---------------------------------------------------------------------------------------------
# aimed queries
# ---------------------------------------------------------------------------------------------

def aim_query(keys_rot: np.ndarray, q_pos: float, scale: float, rng: np.random.Generator,
              noise: np.ndarray) -> np.ndarray:
    """One (sequence, head): a pre-RoPE query whose logits peak on a few of the n rotated keys.

    keys_rot [n, d] are the keys as the attention sees them (token j rotated at position j).
    Targets: token n-1 and, when n >= 3, two other tokens drawn by `rng`.  The rotated query is
    the least-norm solution of <q', k_t> = levels_t * L / scale for the targets and
    <q', mean_j k_j> = 0 (so the bulk of the logits sits near 0), plus `noise`; it is rotated back
    by -q_pos, so that RoPE at q_pos gives q' again.
    """
    n, d = keys_rot.shape
    if n == 0:
        return noise.copy()
    targets = [n - 1]
    if n >= 3:
        targets += [int(t) for t in rng.choice(n - 1, size=2, replace=False)]
    L = math.log(n) + PEAK_MARGIN_NATS
    rows = [keys_rot[targets]]
    rhs = [np.asarray(TARGET_LEVELS[:len(targets)]) * L / scale]
    if n > 3:
        rows.append(keys_rot.mean(axis=0)[None])
        rhs.append(np.zeros(1))
    A = np.vstack(rows)
    y = np.concatenate(rhs)
    q_rot = A.T @ np.linalg.solve(A @ A.T, y) + noise
    return O.apply_rope(q_rot, -float(q_pos), ROPE_BASE)


def key_slices(codec: dict, cfg: dict, layer: int, loop: int, h: int):
    """(W^K_up of loop `loop` and head h [d, r_k], mu^K of that loop and head [d])."""
    T, H, d = cfg["T"], cfg["H"], cfg["d_head"]
    if cfg["variant"] == 0:
        return codec["w_up_k"][layer][h, loop], codec["mu_k"][layer].reshape(H, T, d)[h, loop]
    return codec["w_up_k"][layer][loop, h], codec["mu_k"][layer].reshape(T, H, d)[loop, h]


def mu_v_t(codec: dict, cfg: dict, layer: int, loop: int) -> np.ndarray:
    """mu^V of loop `loop` for every head [H, d]."""
    T, H, d = cfg["T"], cfg["H"], cfg["d_head"]
    if cfg["variant"] == 0:
        return codec["mu_v"][layer].reshape(H, T, d)[:, loop]
    return codec["mu_v"][layer].reshape(T, H, d)[loop]


def aimed_queries(codec: dict, cfg: dict, cK: np.ndarray, layer: int, loop: int, lens, q_pos, scale: float,
                  tag: str) -> np.ndarray:
    """Aimed pre-RoPE queries [B, H, d] for one (layer, loop) call over latents cK of that layer
    ([B, N, H, r_k] per-head, [B, N, r_k] 2D), rounded to float32."""
    B, H, d = len(lens), cfg["H"], cfg["d_head"]
    rng = syn.rng(tag + "/targets")
    noise = syn.gaussian(tag + "/q", (B, H, d))
    q = np.empty((B, H, d))
    for b in range(B):
        n = int(lens[b])
        for h in range(H):
            W, mu = key_slices(codec, cfg, layer, loop, h)
            c = cK[b, :n, h] if cfg["variant"] == 0 else cK[b, :n]
            keys = O.apply_rope(O.reconstruct(c, W, mu), np.arange(n), ROPE_BASE)
            q[b, h] = aim_query(keys, q_pos[b], scale, rng, noise[b, h])
    return syn.round_f32(q)


# ---------------------------------------------------------------------------------------------
# decode cases
# ---------------------------------------------------------------------------------------------

@dataclass
class DecodeCase:
    """One (layer, loop) decode call: what the GPU gets and what the oracle recomputes."""
    name: str
    cfg: dict                 # D, T, H, d_head, r_k, r_v, variant
    codec: dict               # rounded codec (W_down bf16 values, W_up and mu float32 values)
    cK: np.ndarray            # latents of the layer under test [B, N, (H,) r_k], bf16 values
    cV: np.ndarray
    q: np.ndarray             # [B, H, d] pre-RoPE, float32 values
    lens: list
    qpos: list
    scale: float
    layer: int
    loop: int
    k_self: np.ndarray | None = None
    v_self: np.ndarray | None = None
    extra: dict = field(default_factory=dict)

    def reference(self, lens=None, qpos=None, scale=None) -> np.ndarray:
        return oracle_decode(self.codec, self.cfg, self.cK, self.cV, self.q, self.layer, self.loop,
                             self.lens if lens is None else lens, self.qpos if qpos is None else qpos,
                             self.scale if scale is None else scale, k_self=self.k_self, v_self=self.v_self)

    def mu_v(self) -> np.ndarray:
        return mu_v_t(self.codec, self.cfg, self.layer, self.loop)


def decode_errors(got, ref, mu_v) -> tuple[float, float, float]:
    """(rel-L2 of the output, rel-L2 of out - mu^V_t, max-abs of the output)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    mv = np.asarray(mu_v, np.float64)[None]
    m = float(np.abs(got - ref).max()) if ref.size else 0.0
    return rel_l2(got, ref), rel_l2(got - mv, ref - mv), m


def assert_decode_close(got, ref, mu_v, what: str = "") -> tuple[float, float, float]:
    """The acceptance bar on the output and on its attention-dependent part out - mu^V_t."""
    e_out, e_att, m = decode_errors(got, ref, mu_v)
    ok = e_out <= REL_L2_TOL and e_att <= REL_L2_TOL and m <= MAX_ABS_TOL
    assert ok, f"{what}: rel_l2={e_out:.3e} rel_l2(out-mu_v)={e_att:.3e} max_abs={m:.3e}"
    return e_out, e_att, m


class LatentSet:
    """A seeded codec and store: latents of every layer, ragged lengths."""

    def __init__(self, cfg: dict, codec: dict, cK: np.ndarray, cV: np.ndarray, lens, tag: str):
        self.cfg, self.codec, self.cK, self.cV, self.lens, self.tag = cfg, codec, cK, cV, list(lens), tag

    @property
    def bits(self) -> np.ndarray:
        """bf16 store bits [B, D, N, (H,) r_k + r_v]."""
        return to_bf16_bits(np.concatenate([self.cK, self.cV], -1))

    def desc_kw(self, max_pos: int) -> dict:
        c = self.cfg
        return dict(D=c["D"], T=c["T"], H=c["H"], d_head=c["d_head"], r_k=c["r_k"], r_v=c["r_v"],
                    variant=c["variant"], rope_base=ROPE_BASE, max_pos=max_pos)

    def case(self, layer: int, loop: int, qpos=None, lens=None, self_slot: bool = False) -> DecodeCase:
        lens = self.lens if lens is None else list(lens)
        qpos = lens if qpos is None else list(qpos)
        scale = 1.0 / math.sqrt(self.cfg["d_head"])
        tag = f"{self.tag}/l{layer}/t{loop}"
        cK, cV = self.cK[:, layer], self.cV[:, layer]
        q = aimed_queries(self.codec, self.cfg, cK, layer, loop, lens, qpos, scale, tag)
        ks = vs = None
        if self_slot:
            B, H, d = len(lens), self.cfg["H"], self.cfg["d_head"]
            ks = syn.round_f32(syn.gaussian(tag + "/ks", (B, H, d)))
            vs = syn.round_f32(syn.gaussian(tag + "/vs", (B, H, d)))
        return DecodeCase(f"{self.tag}/l{layer}/t{loop}", self.cfg, self.codec, cK, cV, q, lens, qpos, scale,
                          layer, loop, ks, vs)


def seeded_latent_set(c: dict, tag: str, mu_v_zero: bool = False, codec_tag: str | None = None) -> LatentSet:
    """Seeded orthonormal codec (mu ~ N(0, 0.1)) and N(0, 1) bf16 latents for every layer.
    c: D, T, H, d_head, r_k, r_v, variant, B, N, lens.  The codec is drawn from `codec_tag`
    (default `tag`), the latents from `tag`."""
    cfg = dict(D=c["D"], T=c["T"], H=c["H"], d_head=c["d_head"], r_k=c["r_k"], r_v=c["r_v"],
               variant=c.get("variant", 0), rope_base=ROPE_BASE, mu_var=0.1)
    codec = rounded_codec(syn.seeded_codec(cfg, codec_tag or tag))
    if mu_v_zero:
        codec["mu_v"] = np.zeros_like(codec["mu_v"])
    B, N, D, H = c["B"], c["N"], c["D"], c["H"]
    head = () if cfg["variant"] == 1 else (H,)
    cK = syn.round_bf16(syn.gaussian(tag + "/cK", (B, D, N) + head + (c["r_k"],)))
    cV = syn.round_bf16(syn.gaussian(tag + "/cV", (B, D, N) + head + (c["r_v"],)))
    return LatentSet(cfg, codec, cK, cV, c["lens"], tag)


# ragged contexts (0, 1, a tile boundary, odd tails) for four per-head codec shapes
RAGGED = [
    dict(D=2, T=4, H=3, d_head=32, r_k=8, r_v=24, B=6, N=300, lens=[0, 1, 127, 128, 300, 259]),
    dict(D=1, T=4, H=16, d_head=128, r_k=16, r_v=32, B=3, N=520, lens=[520, 129, 384]),
    dict(D=1, T=4, H=16, d_head=128, r_k=96, r_v=160, B=2, N=400, lens=[400, 255]),
    dict(D=1, T=2, H=4, d_head=64, r_k=16, r_v=40, B=4, N=700, lens=[700, 1, 2, 333]),
]

# LLA-2D codecs; the last has T = 1 (per-loop MLA, the head-axis latent of one loop)
TWO_D = [
    dict(D=2, T=2, H=4, d_head=16, r_k=12, r_v=20, B=3, N=200, lens=[200, 0, 77], variant=1),
    dict(D=1, T=4, H=16, d_head=128, r_k=64, r_v=128, B=2, N=300, lens=[300, 130], variant=1),
    dict(D=2, T=4, H=16, d_head=128, r_k=64, r_v=128, B=5, N=900, lens=[900, 0, 1, 385, 640], variant=1),
    dict(D=3, T=1, H=16, d_head=128, r_k=64, r_v=128, B=3, N=400, lens=[400, 5, 256], variant=1),
]

# self slot: per-head (two shapes), LLA-2D, and a small per-head codec
SELF = [
    dict(variant=0, D=1, T=4, H=16, d_head=128, r_k=16, r_v=32, B=4, N=300, lens=[300, 0, 129, 77]),
    dict(variant=0, D=1, T=4, H=16, d_head=128, r_k=96, r_v=160, B=3, N=260, lens=[260, 1, 128]),
    dict(variant=1, D=1, T=4, H=16, d_head=128, r_k=64, r_v=128, B=3, N=400, lens=[400, 0, 131]),
    dict(variant=0, D=2, T=2, H=3, d_head=32, r_k=8, r_v=24, B=3, N=90, lens=[90, 0, 33]),
]

# paged stores: pages of 128 tokens, max_pages per sequence
PAGED = [
    dict(variant=0, D=2, T=4, H=16, d_head=128, r_k=16, r_v=32, B=3, max_pages=4, lens=[512, 130, 0]),
    dict(variant=0, D=1, T=4, H=16, d_head=128, r_k=96, r_v=160, B=2, max_pages=3, lens=[300, 257]),
    dict(variant=1, D=2, T=4, H=16, d_head=128, r_k=64, r_v=128, B=3, max_pages=4, lens=[400, 1, 384]),
    dict(variant=0, D=1, T=2, H=3, d_head=32, r_k=8, r_v=24, B=2, max_pages=3, lens=[200, 75]),
]
PAGE_TOKENS = 128


def paged_set(ci: int, tag: str | None = None) -> LatentSet:
    c = PAGED[ci]
    return seeded_latent_set(dict(c, N=c["max_pages"] * PAGE_TOKENS), tag or f"paged{ci}")


# the three codec shapes the tensor-core kernels cover, with NaN bits / a stale workspace
TC_SHAPES = [(0, 16, 32), (0, 96, 160), (1, 64, 128)]


def ragged_set(ci: int, mu_v_zero: bool = False) -> LatentSet:
    return seeded_latent_set(RAGGED[ci], f"ragged{ci}" + ("/muv0" if mu_v_zero else ""), mu_v_zero)


def ragged_case(ci: int, mu_v_zero: bool = False) -> tuple[LatentSet, DecodeCase]:
    s = ragged_set(ci, mu_v_zero)
    c = RAGGED[ci]
    N = c["N"]
    return s, s.case(c["D"] - 1, c["T"] - 1, qpos=[min(n + 3, N + 7) for n in c["lens"]])


def two_d_set(ci: int, mu_v_zero: bool = False) -> LatentSet:
    c = TWO_D[ci]
    return seeded_latent_set(c, f"2d{ci}/{c['d_head']}/{c['T']}" + ("/muv0" if mu_v_zero else ""), mu_v_zero)


def two_d_calls(ci: int):
    c = TWO_D[ci]
    return ((0, 0), (c["D"] - 1, c["T"] - 1))


def self_set(ci: int) -> LatentSet:
    return seeded_latent_set(SELF[ci], f"self{ci}")


def self_calls(ci: int):
    c = SELF[ci]
    return ((0, 1), (c["D"] - 1, c["T"] - 1))


def tc_shape_set(variant: int, rk: int, rv: int, tag: str, lens=(300, 77, 130)) -> LatentSet:
    c = dict(D=1, T=2, H=16, d_head=128, r_k=rk, r_v=rv, variant=variant, B=len(lens), N=300, lens=list(lens))
    return seeded_latent_set(c, tag)


def tiny_set() -> LatentSet:
    """The tiny workload: codec fitted by the oracle's SVD, teacher stacks encoded by the oracle."""
    cfg = dict(syn.CONFIGS["tiny_d16_t4"])
    D, T, H, d, rk, rv, N = cfg["D"], cfg["T"], cfg["H"], cfg["d_head"], cfg["r_k"], cfg["r_v"], cfg["context"]
    codec = rounded_codec(svd_codec(cfg, "tiny"))
    S = T * d
    cK = np.empty((1, D, N, H, rk))
    cV = np.empty((1, D, N, H, rv))
    for l in range(D):
        for h in range(H):
            for axis, arr in (("k", cK), ("v", cV)):
                slot = f"tiny/{axis}/l{l}/h{h}"
                x = syn.smooth_stacks(slot + "/teacher", N, T, d, cfg["traj_rank"], cfg["noise_var"],
                                      syn.gaussian(slot + "/mu", S, 0.1), basis_name=slot)
                arr[0, l, :, h] = O.encode(x, codec[f"mu_{axis}"][l, h], codec[f"w_down_{axis}"][l, h])
    cK, cV = syn.round_bf16(cK), syn.round_bf16(cV)
    return LatentSet(dict(cfg, rope_base=ROPE_BASE), codec, cK, cV, [N], "tiny/aimed")


# ---------------------------------------------------------------------------------------------
# encode -> decode pipeline: teacher stacks encoded by the oracle (and by the GPU)
# ---------------------------------------------------------------------------------------------

PIPE_B, PIPE_N, PIPE_LENS = 2, 300, [300, 171]


def pipeline_inputs(variant: int, rk: int, rv: int, T: int = 4, H: int = 16, d: int = 128):
    """Teacher stacks (bf16 values) for a one-layer pipeline case, the codec, and the oracle's
    latents of those stacks (rounded to bf16, as the store holds them)."""
    tag = f"pipe/{variant}/{rk}"
    cfg = dict(D=1, T=T, H=H, d_head=d, r_k=rk, r_v=rv, variant=variant, rope_base=ROPE_BASE, mu_var=0.1)
    codec = rounded_codec(syn.seeded_codec(cfg, tag))
    B, N = PIPE_B, PIPE_N
    n = B * N
    S = T * d if variant == 0 else T * H * d
    if variant == 0:
        x = np.empty((n, 1, H, 2, S))
        for h in range(H):
            for a in range(2):
                x[:, 0, h, a] = syn.smooth_stacks(f"{tag}/x/{h}/{a}", n, T, d, 8, 1e-2,
                                                  codec[f"mu_{'kv'[a]}"][0, h], basis_name=f"{tag}/b/{h}/{a}")
    else:
        x = np.empty((n, 1, 2, S))
        for a in range(2):
            x[:, 0, a] = syn.smooth_stacks(f"{tag}/x/{a}", n, T, H * d, 8, 1e-2, codec[f"mu_{'kv'[a]}"][0],
                                           basis_name=f"{tag}/b/{a}")
    x = syn.round_bf16(x)
    if variant == 0:
        cK = np.empty((n, H, rk))
        cV = np.empty((n, H, rv))
        for h in range(H):
            cK[:, h] = O.encode(x[:, 0, h, 0], codec["mu_k"][0, h], codec["w_down_k"][0, h])
            cV[:, h] = O.encode(x[:, 0, h, 1], codec["mu_v"][0, h], codec["w_down_v"][0, h])
        cK, cV = cK.reshape(B, 1, N, H, rk), cV.reshape(B, 1, N, H, rv)
    else:
        cK = O.encode(x[:, 0, 0], codec["mu_k"][0], codec["w_down_k"][0]).reshape(B, 1, N, rk)
        cV = O.encode(x[:, 0, 1], codec["mu_v"][0], codec["w_down_v"][0]).reshape(B, 1, N, rv)
    lat = LatentSet(cfg, codec, syn.round_bf16(cK), syn.round_bf16(cV), PIPE_LENS, tag)
    return x, lat


# ---------------------------------------------------------------------------------------------
# full-size workloads, sampled
# ---------------------------------------------------------------------------------------------

# name -> (layer, loop, sampled sequences, tokens cut from the last sampled sequence)
FULL_SIZE = {
    "ouro_rho21_b768_n4096": (5, 3, [0, 1, 383, 767], 77),
    "ouro_rho4_b32_n4096": (23, 0, [0, 17, 31], 77),
    "huginn_t32_b16_n32768": (2, 31, [0, 15], 77),
    "ouro_2d_b256_n8192": (11, 2, [0, 1, 128, 255], 1000),
    # per-loop MLA at the ratio-21.3 budget: 96 single-loop slots, 116 GB store
    "mla_perloop_b768_n4096": (57, 0, [0, 300, 767], 1000),
}


def full_size_sample(name: str, mu_v_zero: bool = False, all_layers: bool = True) -> DecodeCase:
    """The sampled sequences of a full-size call.  Latent rows of the layer under test for the
    sampled sequences are drawn here (seeded per sequence and head, bf16 values, float32 arrays),
    for all cap = N + 1 slots; the GPU test writes them into the full store over the rest of the
    batch's rows.  extra: batch, cap, sample, lens of the whole batch.  all_layers=False draws the
    codec of the layer under test only (all the oracle reads; the GPU codec needs every layer)."""
    cfg0 = syn.CONFIGS[name]
    layer, loop, sample, cut = FULL_SIZE[name]
    cfg = dict(D=cfg0["D"], T=cfg0["T"], H=cfg0["H"], d_head=cfg0["d_head"], r_k=cfg0["r_k"], r_v=cfg0["r_v"],
               variant=cfg0["variant"], rope_base=ROPE_BASE, mu_var=cfg0.get("mu_var", 0.1))
    codec = rounded_codec(syn.seeded_codec(cfg, f"full/{name}/codec", None if all_layers else [layer]))
    if mu_v_zero:
        codec["mu_v"] = np.zeros_like(codec["mu_v"])
    B, N = cfg0["batch"], cfg0["context"]
    cap = N + 1
    H, rk, rv = cfg["H"], cfg["r_k"], cfg["r_v"]
    S = len(sample)
    if cfg["variant"] == 0:
        lat = np.empty((S, cap, H, rk + rv), np.float32)
        for i, b in enumerate(sample):
            for h in range(H):
                lat[i, :, h] = syn.round_bf16(syn.gaussian(f"full/{name}/lat/s{b}/h{h}", (cap, rk + rv)))
    else:
        lat = np.empty((S, cap, rk + rv), np.float32)
        for i, b in enumerate(sample):
            lat[i] = syn.round_bf16(syn.gaussian(f"full/{name}/lat/s{b}", (cap, rk + rv)))
    lens_all = np.full(B, N, np.int32)
    lens_all[sample[-1]] = N - cut
    lens = [int(lens_all[b]) for b in sample]
    scale = 1.0 / math.sqrt(cfg["d_head"])
    cK, cV = lat[..., :rk], lat[..., rk:]
    q = aimed_queries(codec, cfg, cK, layer, loop, lens, lens, scale, f"full/{name}/aim")
    return DecodeCase(f"full/{name}" + ("/muv0" if mu_v_zero else ""), cfg, codec, cK, cV, q, lens, list(lens),
                      scale, layer, loop,
                      extra=dict(batch=B, cap=cap, sample=list(sample), lens_all=lens_all, latents=lat))


# ---------------------------------------------------------------------------------------------
# full-cache comparator
# ---------------------------------------------------------------------------------------------

FULL_CACHE = [dict(B=3, L=1, N=520, H=16, lens=[520, 0, 129]),
              dict(B=4, L=2, N=300, H=3, lens=[1, 300, 255, 77]),
              dict(B=2, L=1, N=1, H=1, lens=[1, 0])]  # one cached token: out = v_0


def full_cache_inputs(ci: int):
    """Rotated keys and values [B, L, N, H, d] (bf16 values) and aimed queries for layer L-1."""
    c = FULL_CACHE[ci]
    B, L, N, H, d = c["B"], c["L"], c["N"], c["H"], 128
    tag = f"full/{B}/{H}"
    K = syn.gaussian(tag + "/K", (B, L, N, H, d))
    pos = np.arange(N, dtype=np.float64)
    Kr = np.stack([np.stack([O.apply_rope(K[b, l].transpose(1, 0, 2), pos, ROPE_BASE).transpose(1, 0, 2)
                             for l in range(L)]) for b in range(B)])
    Kr, V = syn.round_bf16(Kr), syn.round_bf16(syn.gaussian(tag + "/V", (B, L, N, H, d)))
    qpos = [n + 3 for n in c["lens"]]
    scale = 1.0 / math.sqrt(d)
    rng = syn.rng(tag + "/targets")
    noise = syn.gaussian(tag + "/q", (B, H, d))
    q = np.empty((B, H, d))
    for b, n in enumerate(c["lens"]):
        for h in range(H):
            q[b, h] = aim_query(Kr[b, L - 1, :n, h], qpos[b], scale, rng, noise[b, h])
    return c, Kr, V, syn.round_f32(q), qpos, scale


# the comparator at the bench's size: batch 32 x 4096, 16 heads; sampled sequences (one ragged)
FULL_CACHE_SIZE = dict(B=32, H=16, d=128, N=4096, sample=[0, 17, 31], cut={17: 333})


def full_cache_full_size_sample():
    """Keys (taken as cached already rotated) and values of the sampled sequences, in the kernel's
    head-major layout [sample][H][N + 1][d] (bf16 values, float32 arrays), lengths and aimed
    queries.  The GPU test writes these rows over a device-filled cache of the whole batch."""
    c = FULL_CACHE_SIZE
    B, H, d, N, sample = c["B"], c["H"], c["d"], c["N"], c["sample"]
    cap = N + 1
    K = np.empty((len(sample), H, cap, d), np.float32)
    V = np.empty((len(sample), H, cap, d), np.float32)
    for i, b in enumerate(sample):
        K[i] = syn.round_bf16(syn.gaussian(f"fullcache/size/K/s{b}", (H, cap, d)))
        V[i] = syn.round_bf16(syn.gaussian(f"fullcache/size/V/s{b}", (H, cap, d)))
    lens_all = np.full(B, N, np.int32)
    for b, cut in c["cut"].items():
        lens_all[b] = N - cut
    lens = [int(lens_all[b]) for b in sample]
    qpos = [n + 1 for n in lens]
    scale = 1.0 / math.sqrt(d)
    rng = syn.rng("fullcache/size/targets")
    noise = syn.gaussian("fullcache/size/q", (len(sample), H, d))
    q = np.empty((len(sample), H, d))
    for i, n in enumerate(lens):
        for h in range(H):
            q[i, h] = aim_query(K[i, h, :n].astype(np.float64), qpos[i], scale, rng, noise[i, h])
    return dict(K=K, V=V, lens_all=lens_all, lens=lens, qpos=qpos, q=syn.round_f32(q), scale=scale, cap=cap)


# ---------------------------------------------------------------------------------------------
# registry of every decode input set the GPU parity tests compare with the oracle
# ---------------------------------------------------------------------------------------------

def decode_sets():
    """name -> zero-argument builder of the DecodeCase list of that set."""
    sets = {}
    tiny = lambda: [tiny_set().case(0, t, qpos=[syn.CONFIGS["tiny_d16_t4"]["context"]]) for t in range(4)]
    sets["tiny/aimed"] = tiny
    for ci in range(len(RAGGED)):
        sets[f"ragged{ci}"] = lambda ci=ci: [ragged_case(ci)[1]]
    sets["ragged1/muv0"] = lambda: [ragged_case(1, mu_v_zero=True)[1]]
    for ci in range(len(TWO_D)):
        sets[f"2d{ci}"] = lambda ci=ci: [two_d_set(ci).case(l, t) for l, t in two_d_calls(ci)]
    sets["2d2/muv0"] = lambda: [two_d_set(2, mu_v_zero=True).case(l, t) for l, t in two_d_calls(2)]
    for ci in range(len(SELF)):
        sets[f"self{ci}"] = lambda ci=ci: [self_set(ci).case(l, t, self_slot=True) for l, t in self_calls(ci)]
    for v, rk, rv in TC_SHAPES:
        sets[f"nan_tail/{v}/{rk}"] = lambda v=v, rk=rk, rv=rv: [tc_shape_set(v, rk, rv, f"nan_tail/{v}/{rk}").case(0, 1)]
        sets[f"stale_ws/{v}/{rk}"] = lambda v=v, rk=rk, rv=rv: [
            tc_shape_set(v, rk, rv, f"stale_ws/{v}/{rk}").case(0, loop, lens=lens) for loop, lens in STALE_CALLS]
        sets[f"pipe/{v}/{rk}"] = lambda v=v, rk=rk, rv=rv: [pipeline_inputs(v, rk, rv)[1].case(0, t) for t in range(4)]
    for name in FULL_SIZE:
        sets[f"full/{name}"] = lambda name=name: [full_size_sample(name, all_layers=False)]
    for name in ("ouro_rho21_b768_n4096", "ouro_2d_b256_n8192"):
        sets[f"full/{name}/muv0"] = lambda name=name: [full_size_sample(name, mu_v_zero=True, all_layers=False)]
    for ci in range(len(PAGED)):
        sets[f"paged{ci}"] = lambda ci=ci: [paged_set(ci).case(PAGED[ci]["D"] - 1, 1)]
    sets["paged_self"] = lambda: [paged_set(0, "paged_self").case(0, 2, self_slot=True)]
    for v in (0, 1):
        sets[f"noalloc/{v}"] = lambda v=v: [noalloc_set(v, i).case(layer, loop)
                                            for i, (_, _, _, layer, loop) in enumerate(NOALLOC_CALLS)]
    return sets


# workspace reuse: the same workspace, other lengths (the first call empties a sequence)
STALE_CALLS = ((1, [300, 1, 0]), (0, [129, 300, 5]))

# allocation-free entry point: two calls in a row, the second smaller
NOALLOC_CALLS = [(3, 700, [700, 129, 1], 1, 2), (2, 300, [17, 300], 0, 3)]


def noalloc_set(variant: int, i: int) -> LatentSet:
    B, N, lens, _, _ = NOALLOC_CALLS[i]
    c = dict(D=2, T=4, H=16, d_head=128, r_k=16, r_v=32, variant=variant, B=B, N=N, lens=lens)
    if variant == 1:
        c.update(H=4, r_k=24, r_v=40)
    return seeded_latent_set(c, f"noalloc/{variant}/{i}", codec_tag=f"noalloc/{variant}")
