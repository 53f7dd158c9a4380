"""The fast path's cache, rebuilt from the latent store (lla_reconstruct_cache), against the oracle.

For one (layer, loop) the cache must hold k_hat_j = RoPE_j(c^K_j W^K_up,t^T + mu^K_t) and
v_hat_j = c^V_j W^V_up,t^T + mu^V_t for every cached token [LLA §3 eq. (3); "RoPE and
reconstruction"], in the head-major layout the full-cache comparator reads, and nothing else:
rows past each sequence's length keep their previous bits.  The expected rows come from the
oracle's reconstruct and apply_rope in float64; the cache is bf16, so the bar is the acceptance
bar (rel-L2 5e-3, max-abs 2e-2).  Then the comparator over the rebuilt cache is checked against
the oracle's LLA decode over the latents: the two paths of the pages give the same attention.
Both kernels run where they apply (tensor cores for d_head 128 at the decode kernels' ranks).
"""

import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
import parity_cases as PC  # noqa: E402
from lla_testutil import assert_close, from_bf16_bits, make_lib_codec  # noqa: E402
from oracle import lla_oracle as O  # noqa: E402

DEV = "cuda"
SENTINEL = 0x7FC3  # a bf16 NaN pattern: rows the call must not write

CASES = [
    dict(variant=0, D=2, T=4, H=16, d_head=128, r_k=16, r_v=32, B=3, N=300, lens=[300, 0, 129]),
    dict(variant=0, D=1, T=4, H=16, d_head=128, r_k=96, r_v=160, B=2, N=260, lens=[260, 1]),
    dict(variant=1, D=2, T=4, H=16, d_head=128, r_k=64, r_v=128, B=3, N=200, lens=[200, 77, 128]),
    dict(variant=0, D=2, T=2, H=3, d_head=32, r_k=8, r_v=24, B=4, N=150, lens=[150, 1, 0, 64]),
]


def expected_rows(s, layer, loop, b, n):
    """Oracle rows of sequence b: (K rotated, V) [H, n, d]."""
    cfg, codec = s.cfg, s.codec
    H = cfg["H"]
    K = np.zeros((H, n, cfg["d_head"]))
    V = np.zeros_like(K)
    for h in range(H):
        W, mu = PC.key_slices(codec, cfg, layer, loop, h)
        if cfg["variant"] == 0:
            Wv, muv = codec["w_up_v"][layer][h, loop], PC.mu_v_t(codec, cfg, layer, loop)[h]
            cK, cV = s.cK[b, layer, :n, h], s.cV[b, layer, :n, h]
        else:
            Wv, muv = codec["w_up_v"][layer][loop, h], PC.mu_v_t(codec, cfg, layer, loop)[h]
            cK, cV = s.cK[b, layer, :n], s.cV[b, layer, :n]
        K[h] = O.apply_rope(O.reconstruct(cK, W, mu), np.arange(n), PC.ROPE_BASE)
        V[h] = O.reconstruct(cV, Wv, muv)
    return K, V


def _impls(lib, c):
    tc = c["d_head"] == 128 and ((c["variant"] == 0 and (c["r_k"], c["r_v"]) in ((16, 32), (96, 160))) or
                                 (c["variant"] == 1 and (c["r_k"], c["r_v"]) == (64, 128)))
    return [lla.IMPL_SIMT] + ([lla.IMPL_TC] if tc else [])


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_reconstructed_cache_matches_oracle(ci):
    c = CASES[ci]
    s = PC.seeded_latent_set(c, f"recon{ci}")
    B, N, H, d = c["B"], c["N"], c["H"], c["d_head"]
    lib = make_lib_codec(lla, s.desc_kw(N + 8), s.codec)
    store = torch.from_numpy(s.bits.view(np.int16)).to(DEV)
    lens = torch.tensor(c["lens"], dtype=torch.int32, device=DEV)
    cap = N + 5                          # cache rows per (sequence, head): more than max_tokens
    slices = 2                           # two (layer, loop) slices per sequence: the call writes the second
    stride = slices * H * cap * d
    for impl in _impls(lib, c):
        for layer, loop in ((0, 1), (c["D"] - 1, c["T"] - 1)):
            kc = torch.full((B * stride,), SENTINEL, dtype=torch.int16, device=DEV)
            vc = torch.full_like(kc, SENTINEL)
            off = H * cap * d
            lla.reconstruct_cache(lib, store, B, N, layer, loop, lens, kc.data_ptr() + 2 * off,
                                  vc.data_ptr() + 2 * off, stride, cap, impl=impl)
            torch.cuda.synchronize()
            kh = kc.cpu().numpy().view(np.uint16).reshape(B, slices, H, cap, d)
            vh = vc.cpu().numpy().view(np.uint16).reshape(B, slices, H, cap, d)
            assert np.all(kh[:, 0] == SENTINEL) and np.all(vh[:, 0] == SENTINEL), "wrote outside its slice"
            for b, n in enumerate(c["lens"]):
                assert np.all(kh[b, 1, :, n:] == SENTINEL) and np.all(vh[b, 1, :, n:] == SENTINEL), \
                    f"impl {impl}: rows past the length of sequence {b} written"
                if n == 0:
                    continue
                K, V = expected_rows(s, layer, loop, b, n)
                assert_close(from_bf16_bits(kh[b, 1, :, :n]), K, f"impl {impl} layer {layer} loop {loop} K seq {b}")
                assert_close(from_bf16_bits(vh[b, 1, :, :n]), V, f"impl {impl} layer {layer} loop {loop} V seq {b}")
    lib.close()


@pytest.mark.parametrize("ci", [0, 1])
def test_full_cache_decode_over_the_rebuilt_cache_equals_lla(ci):
    """Both paths of the pages on the same latents: the comparator over the rebuilt cache and LLA
    decode over the store agree with the oracle's LLA decode (queries aimed at cached keys)."""
    c = CASES[ci]
    s = PC.seeded_latent_set(c, f"recon{ci}")
    B, N, H, d = c["B"], c["N"], c["H"], c["d_head"]
    lib = make_lib_codec(lla, s.desc_kw(N + 8), s.codec)
    store = torch.from_numpy(s.bits.view(np.int16)).to(DEV)
    lens = torch.tensor(c["lens"], dtype=torch.int32, device=DEV)
    layer, loop = c["D"] - 1, c["T"] - 1
    case = s.case(layer, loop)
    kc = torch.zeros(B * H * N * d, dtype=torch.int16, device=DEV)
    vc = torch.zeros_like(kc)
    lla.reconstruct_cache(lib, store, B, N, layer, loop, lens, kc, vc, H * N * d, N)
    q = torch.from_numpy(case.q.astype(np.float32)).to(DEV)
    qpos = torch.tensor(case.qpos, dtype=torch.int32, device=DEV)
    out = torch.full((B, H, d), float("nan"), device=DEV)
    ws = torch.empty(lla.full_decode_workspace_bytes(H, d, B), dtype=torch.uint8, device=DEV)
    lla.full_decode_attn(H, d, PC.ROPE_BASE, kc, vc, H * N * d, B, N, q, qpos, lens, case.scale, out, ws)
    torch.cuda.synchronize()
    PC.assert_decode_close(out.cpu().numpy().astype(np.float64), case.reference(), case.mu_v(), "comparator")
    lib.close()


@pytest.mark.slow
def test_reconstruct_full_size_sampled():
    """The ratio-4 workload's shape (batch 32 x 4096 x 16 heads, r 96/160) in the launch
    configuration bench.py times, one (layer, loop), sampled sequences (one ragged) checked."""
    cfg = syn.CONFIGS["ouro_rho4_b32_n4096"]
    D, T, H, d, rk, rv, B, N = (cfg[k] for k in ("D", "T", "H", "d_head", "r_k", "r_v", "batch", "context"))
    layer, loop = 7, 2
    codec = PC.rounded_codec(syn.seeded_codec(cfg, "recon/full/codec"))
    lib = lla.Codec(lla.Desc(D, T, H, d, rk, rv, 0, PC.ROPE_BASE, N + 1), codec["w_down_k"], codec["w_down_v"],
                    codec["w_up_k"], codec["w_up_v"], codec["mu_k"], codec["mu_v"])
    store = torch.empty(lla.store_bytes(lib.desc, B, N) // 2, dtype=torch.bfloat16, device=DEV)
    view = store.view(B, D, N, H, rk + rv)
    view[:, layer].normal_(generator=syn.torch_generator("recon/full/lat", DEV))
    lens_np = np.full(B, N, np.int32)
    lens_np[9] = N - 333
    lens = torch.from_numpy(lens_np).to(DEV)
    kc = torch.empty(B * H * N * d, dtype=torch.int16, device=DEV)
    vc = torch.empty_like(kc)
    lla.reconstruct_cache(lib, store, B, N, layer, loop, lens, kc, vc, H * N * d, N)
    torch.cuda.synchronize()
    for b in (0, 9, 31):
        n = int(lens_np[b])
        lat = view[b, layer, :n].float().cpu().numpy().astype(np.float64)  # [n, H, rk+rv]
        kh = from_bf16_bits(kc.view(B, H, N, d)[b, :, :n].cpu().numpy().view(np.uint16))
        vh = from_bf16_bits(vc.view(B, H, N, d)[b, :, :n].cpu().numpy().view(np.uint16))
        for h in range(H):
            mk = codec["mu_k"][layer, h].reshape(T, d)[loop]
            mv = codec["mu_v"][layer, h].reshape(T, d)[loop]
            Kx = O.apply_rope(O.reconstruct(lat[:, h, :rk], codec["w_up_k"][layer, h, loop], mk), np.arange(n),
                              PC.ROPE_BASE)
            Vx = O.reconstruct(lat[:, h, rk:], codec["w_up_v"][layer, h, loop], mv)
            assert_close(kh[h], Kx, f"K seq {b} head {h}")
            assert_close(vh[h], Vx, f"V seq {b} head {h}")
    del store, view, kc, vc
    lib.close()
    torch.cuda.empty_cache()


def test_reconstruct_argument_errors():
    c = CASES[0]
    s = PC.seeded_latent_set(c, "recon0")
    lib = make_lib_codec(lla, s.desc_kw(c["N"] + 8), s.codec)
    buf = torch.zeros(1 << 20, dtype=torch.int16, device=DEV)
    p = buf.data_ptr()
    H, d = c["H"], c["d_head"]
    with pytest.raises(lla.LLAError) as e:  # beyond the RoPE table
        lla.reconstruct_cache(lib, p, 1, c["N"] + 9, 0, 0, p, p, p, H * 1000 * d, 1000)
    assert e.value.status == 1
    with pytest.raises(lla.LLAError) as e:  # sequence stride shorter than a sequence's rows
        lla.reconstruct_cache(lib, p, 1, 100, 0, 0, p, p, p, 100, 100)
    assert e.value.status == 1
    with pytest.raises(lla.LLAError) as e:  # misaligned cache
        lla.reconstruct_cache(lib, p, 1, 100, 0, 0, p, p + 2, p, H * 100 * d, 100)
    assert e.value.status == 3
    lib.close()
