"""GPU decode attention vs the FP64 oracle, through the C ABI.

Small shapes that span several 128-token tiles, ragged context lengths
(0, 1, a tile boundary and odd tails), several split counts, both kernels
(CUDA-core reference and tcgen05), both LLA variants, and the device-side
range flags.  The acceptance bar is rel-L2 <= 5e-3 and max-abs <= 2e-2.
"""

import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
from oracle import lla_oracle as O  # noqa: E402
from lla_testutil import (assert_close, from_bf16_bits, make_lib_codec, oracle_decode, rounded_codec,  # noqa: E402
                          svd_codec, to_bf16_bits)

DEV = "cuda"


def _impls(codec):
    out = [lla.IMPL_SIMT]
    probe = getattr(codec, "_tc_ok", None)
    return out if probe is False else out + [lla.IMPL_TC]


def _run(codec, store_bits, B, N, layer, loop, q, q_pos, lens, scale, impl=lla.IMPL_AUTO, num_ctas=0):
    d = codec.desc
    store = torch.from_numpy(store_bits.view(np.int16)).to(DEV)
    qd = torch.from_numpy(np.ascontiguousarray(q, np.float32)).to(DEV)
    qp = torch.tensor(q_pos, dtype=torch.int32, device=DEV)
    ln = torch.tensor(lens, dtype=torch.int32, device=DEV)
    out = torch.full((B, d.H, d.d_head), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.empty(codec.workspace_bytes(B, N), dtype=torch.uint8, device=DEV)
    lla.decode_attn(codec, store, B, N, layer, loop, qd, qp, ln, scale, out, ws, impl=impl, num_ctas=num_ctas)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), lla.workspace_flags(ws)


def _tc_supported(codec, B, N):
    d = codec.desc
    store = torch.zeros(max(1, lla.store_bytes(d, B, N) // 2), dtype=torch.int16, device=DEV)
    q = torch.zeros(B, d.H, d.d_head, device=DEV)
    z = torch.zeros(B, dtype=torch.int32, device=DEV)
    out = torch.empty_like(q)
    ws = torch.empty(codec.workspace_bytes(B, N), dtype=torch.uint8, device=DEV)
    try:
        lla.decode_attn(codec, store, B, N, 0, 0, q, z, z, 1.0, out, ws, impl=lla.IMPL_TC)
        return True
    except lla.LLAError as e:
        if e.status == 2:
            return False
        raise


# ---------------------------------------------------------------------------------------------
# tiny workload: SVD codec fitted by the oracle, teacher stacks encoded by the oracle
# ---------------------------------------------------------------------------------------------

@pytest.fixture(scope="module")
def tiny():
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
    store_bits = to_bf16_bits(np.concatenate([cK, cV], -1))
    lib = make_lib_codec(lla, dict(D=D, T=T, H=H, d_head=d, r_k=rk, r_v=rv, variant=0,
                                   rope_base=cfg["rope_base"], max_pos=N + 1), codec)
    q = syn.round_f32(syn.gaussian("tiny/q", (T, 1, H, d)))
    yield cfg, codec, lib, store_bits, q
    lib.close()


@pytest.mark.parametrize("impl", [lla.IMPL_SIMT, lla.IMPL_TC])
def test_tiny_workload_all_loops(tiny, impl):
    cfg, codec, lib, store_bits, q = tiny
    N, d = cfg["context"], cfg["d_head"]
    if impl == lla.IMPL_TC and not _tc_supported(lib, 1, N):
        pytest.skip("tcgen05 kernel does not cover this shape")
    s = from_bf16_bits(store_bits)
    cK, cV = s[:, 0, ..., :cfg["r_k"]], s[:, 0, ..., cfg["r_k"]:]
    for t in range(cfg["T"]):
        got, flags = _run(lib, store_bits, 1, N, 0, t, q[t], [N], [N], 1 / math.sqrt(d), impl=impl)
        ref = oracle_decode(codec, cfg, cK, cV, q[t], 0, t, [N], [N], 1 / math.sqrt(d))
        assert flags == 0
        assert_close(got, ref, f"loop {t}")


# ---------------------------------------------------------------------------------------------
# ragged contexts, several splits, seeded orthonormal codecs
# ---------------------------------------------------------------------------------------------

RAGGED = [
    dict(D=2, T=4, H=3, d_head=32, r_k=8, r_v=24, B=6, N=300, lens=[0, 1, 127, 128, 300, 259]),
    dict(D=1, T=4, H=16, d_head=128, r_k=16, r_v=32, B=3, N=520, lens=[520, 129, 384]),
    dict(D=1, T=4, H=16, d_head=128, r_k=96, r_v=160, B=2, N=400, lens=[400, 255]),
    dict(D=1, T=2, H=4, d_head=64, r_k=16, r_v=40, B=4, N=700, lens=[700, 1, 2, 333]),
]


def _ragged_case(c, tag):
    cfg = dict(c, variant=0, rope_base=10000.0, mu_var=0.1)
    codec = rounded_codec(syn.seeded_codec(cfg, tag))
    B, N, D, H = c["B"], c["N"], c["D"], c["H"]
    cK = syn.round_bf16(syn.gaussian(tag + "/cK", (B, D, N, H, c["r_k"])))
    cV = syn.round_bf16(syn.gaussian(tag + "/cV", (B, D, N, H, c["r_v"])))
    q = syn.round_f32(syn.gaussian(tag + "/q", (B, H, c["d_head"])))
    lib = make_lib_codec(lla, dict(D=D, T=c["T"], H=H, d_head=c["d_head"], r_k=c["r_k"], r_v=c["r_v"], variant=0,
                                   rope_base=10000.0, max_pos=N + 8), codec)
    return cfg, codec, lib, to_bf16_bits(np.concatenate([cK, cV], -1)), cK, cV, q


@pytest.mark.parametrize("ci", range(len(RAGGED)))
def test_ragged_contexts_match_oracle(ci):
    c = RAGGED[ci]
    cfg, codec, lib, bits, cK, cV, q = _ragged_case(c, f"ragged{ci}")
    B, N = c["B"], c["N"]
    qpos = [min(n + 3, N + 7) for n in c["lens"]]
    scale = 1 / math.sqrt(c["d_head"])
    impls = [lla.IMPL_SIMT] + ([lla.IMPL_TC] if _tc_supported(lib, B, N) else [])
    layer, loop = c["D"] - 1, c["T"] - 1
    ref = oracle_decode(codec, cfg, cK[:, layer], cV[:, layer], q, layer, loop, c["lens"], qpos, scale)
    for impl in impls:
        got, flags = _run(lib, bits, B, N, layer, loop, q, qpos, c["lens"], scale, impl=impl)
        assert flags == 0
        assert_close(got, ref, f"impl {impl}")
        assert np.all(got[np.array(c["lens"]) == 0] == 0)
    lib.close()


@pytest.mark.parametrize("ci", [1, 2])
@pytest.mark.parametrize("impl,ctas", [(lla.IMPL_SIMT, 1), (lla.IMPL_SIMT, 2), (lla.IMPL_SIMT, 7),
                                       (lla.IMPL_TC, 1), (lla.IMPL_TC, 2), (lla.IMPL_TC, 7), (lla.IMPL_TC, 300)])
def test_split_count_invariance(impl, ctas, ci):
    c = RAGGED[ci]
    cfg, codec, lib, bits, cK, cV, q = _ragged_case(c, f"ragged{ci}")
    if impl == lla.IMPL_TC and not _tc_supported(lib, c["B"], c["N"]):
        pytest.skip("tcgen05 kernel does not cover this shape")
    scale = 1 / math.sqrt(c["d_head"])
    base, _ = _run(lib, bits, c["B"], c["N"], 0, 2, q, c["lens"], c["lens"], scale, impl=impl, num_ctas=1)
    got, _ = _run(lib, bits, c["B"], c["N"], 0, 2, q, c["lens"], c["lens"], scale, impl=impl, num_ctas=ctas)
    assert np.abs(got - base).max() < 1e-4
    lib.close()


# ---------------------------------------------------------------------------------------------
# LLA-2D
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("c", [dict(D=2, T=2, H=4, d_head=16, r_k=12, r_v=20, B=3, N=200, lens=[200, 0, 77]),
                               dict(D=1, T=4, H=16, d_head=128, r_k=64, r_v=128, B=2, N=300, lens=[300, 130]),
                               dict(D=2, T=4, H=16, d_head=128, r_k=64, r_v=128, B=5, N=900,
                                    lens=[900, 0, 1, 385, 640]),
                               # T = 1: per-loop MLA, the head-axis latent of one loop
                               dict(D=3, T=1, H=16, d_head=128, r_k=64, r_v=128, B=3, N=400, lens=[400, 5, 256])])
def test_2d_matches_oracle(c):
    tag = f"2d/{c['d_head']}/{c['T']}"
    cfg = dict(c, variant=1, rope_base=10000.0, mu_var=0.1)
    codec = rounded_codec(syn.seeded_codec(cfg, tag))
    B, N, D = c["B"], c["N"], c["D"]
    cK = syn.round_bf16(syn.gaussian(tag + "/cK", (B, D, N, c["r_k"])))
    cV = syn.round_bf16(syn.gaussian(tag + "/cV", (B, D, N, c["r_v"])))
    q = syn.round_f32(syn.gaussian(tag + "/q", (B, c["H"], c["d_head"])))
    lib = make_lib_codec(lla, dict(D=D, T=c["T"], H=c["H"], d_head=c["d_head"], r_k=c["r_k"], r_v=c["r_v"],
                                   variant=1, rope_base=10000.0, max_pos=N + 4), codec)
    bits = to_bf16_bits(np.concatenate([cK, cV], -1))
    scale = 1 / math.sqrt(c["d_head"])
    impls = [lla.IMPL_SIMT] + ([lla.IMPL_TC] if _tc_supported(lib, B, N) else [])
    for layer, loop in ((0, 0), (D - 1, c["T"] - 1)):
        ref = oracle_decode(codec, cfg, cK[:, layer], cV[:, layer], q, layer, loop, c["lens"], c["lens"], scale)
        for impl in impls:
            got, flags = _run(lib, bits, B, N, layer, loop, q, c["lens"], c["lens"], scale, impl=impl)
            assert flags == 0
            assert_close(got, ref, f"2d impl {impl} layer {layer} loop {loop}")
            assert np.all(got[np.array(c["lens"]) == 0] == 0)
        if lla.IMPL_TC in impls:  # result independent of the persistent grid
            for ctas in (4, 8, 300):
                got, _ = _run(lib, bits, B, N, layer, loop, q, c["lens"], c["lens"], scale, impl=lla.IMPL_TC,
                              num_ctas=ctas)
                assert_close(got, ref, f"2d tc ctas {ctas}")
    lib.close()


@pytest.mark.parametrize("variant,rk,rv", [(0, 16, 32), (0, 96, 160), (1, 64, 128)])
def test_rows_past_the_context_may_hold_nan(variant, rk, rv):
    """Store rows at or beyond a sequence's length are outside the attention [LLA §3 eq. (3)
    sums over the cached tokens only]: a quiet-NaN pattern there must not reach the output."""
    B, N, D, T, H, d = 3, 300, 1, 2, 16, 128
    lens = [300, 77, 130]
    tag = f"nan_tail/{variant}/{rk}"
    cfg = dict(D=D, T=T, H=H, d_head=d, r_k=rk, r_v=rv, variant=variant, rope_base=10000.0, mu_var=0.1)
    codec = rounded_codec(syn.seeded_codec(cfg, tag))
    head = () if variant == 1 else (H,)
    cK = syn.round_bf16(syn.gaussian(tag + "/cK", (B, D, N) + head + (rk,)))
    cV = syn.round_bf16(syn.gaussian(tag + "/cV", (B, D, N) + head + (rv,)))
    q = syn.round_f32(syn.gaussian(tag + "/q", (B, H, d)))
    bits = to_bf16_bits(np.concatenate([cK, cV], -1))
    for b, n in enumerate(lens):
        bits[b, :, n:] = 0x7FC0  # bf16 quiet NaN
    lib = make_lib_codec(lla, dict(D=D, T=T, H=H, d_head=d, r_k=rk, r_v=rv, variant=variant, rope_base=10000.0,
                                   max_pos=N + 4), codec)
    scale = 1 / math.sqrt(d)
    ref = oracle_decode(codec, cfg, cK[:, 0], cV[:, 0], q, 0, 1, lens, lens, scale)
    impls = [lla.IMPL_SIMT] + ([lla.IMPL_TC] if _tc_supported(lib, B, N) else [])
    assert lla.IMPL_TC in impls
    for impl in impls:
        got, flags = _run(lib, bits, B, N, 0, 1, q, lens, lens, scale, impl=impl)
        assert flags == 0
        assert np.isfinite(got).all(), f"impl {impl}"
        assert_close(got, ref, f"nan tail impl {impl}")
    lib.close()


@pytest.mark.parametrize("variant,rk,rv", [(0, 16, 32), (0, 96, 160), (1, 64, 128)])
def test_stale_workspace_does_not_reach_the_output(variant, rk, rv):
    """The workspace is not cleared between calls: every split record the combine reads is
    written by the same call, and a CTA group whose share of the tiles is empty (a batch with
    fewer tiles than groups) is skipped.  A workspace full of NaN bytes, then the same workspace
    reused with other lengths, gives the oracle's outputs both times."""
    B, N, D, T, H, d = 3, 300, 1, 2, 16, 128
    tag = f"stale_ws/{variant}/{rk}"
    cfg = dict(D=D, T=T, H=H, d_head=d, r_k=rk, r_v=rv, variant=variant, rope_base=10000.0, mu_var=0.1)
    codec = rounded_codec(syn.seeded_codec(cfg, tag))
    head = () if variant == 1 else (H,)
    cK = syn.round_bf16(syn.gaussian(tag + "/cK", (B, D, N) + head + (rk,)))
    cV = syn.round_bf16(syn.gaussian(tag + "/cV", (B, D, N) + head + (rv,)))
    q = syn.round_f32(syn.gaussian(tag + "/q", (B, H, d)))
    lib = make_lib_codec(lla, dict(D=D, T=T, H=H, d_head=d, r_k=rk, r_v=rv, variant=variant, rope_base=10000.0,
                                   max_pos=N + 4), codec)
    assert _tc_supported(lib, B, N)
    store = torch.from_numpy(to_bf16_bits(np.concatenate([cK, cV], -1)).view(np.int16)).to(DEV)
    qd = torch.from_numpy(np.ascontiguousarray(q, np.float32)).to(DEV)
    ws = torch.full((lib.workspace_bytes(B, N),), 0xFF, dtype=torch.uint8, device=DEV)
    scale = 1 / math.sqrt(d)
    for loop, lens in ((1, [300, 1, 0]), (0, [129, 300, 5])):
        ln = torch.tensor(lens, dtype=torch.int32, device=DEV)
        out = torch.full((B, H, d), float("nan"), dtype=torch.float32, device=DEV)
        lla.decode_attn(lib, store, B, N, 0, loop, qd, ln, ln, scale, out, ws, impl=lla.IMPL_TC)
        torch.cuda.synchronize()
        assert lla.workspace_flags(ws) == 0
        got = out.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all(), lens
        assert_close(got, oracle_decode(codec, cfg, cK[:, 0], cV[:, 0], q, 0, loop, lens, lens, scale), f"lens {lens}")
    lib.close()


# ---------------------------------------------------------------------------------------------
# range flags
# ---------------------------------------------------------------------------------------------

def test_out_of_range_lengths_and_positions_are_clamped_and_flagged():
    c = RAGGED[0]
    cfg, codec, lib, bits, cK, cV, q = _ragged_case(c, "ragged0")
    B, N = c["B"], c["N"]
    scale = 1 / math.sqrt(c["d_head"])
    lens = [N + 50] + c["lens"][1:]
    got, flags = _run(lib, bits, B, N, 0, 0, q, c["lens"], lens, scale, impl=lla.IMPL_SIMT)
    assert flags & lla.FLAG_SEQ_LEN_CLAMPED
    ref = oracle_decode(codec, cfg, cK[:, 0], cV[:, 0], q, 0, 0, [N] + c["lens"][1:], c["lens"], scale)
    assert_close(got, ref, "clamped length")
    qpos = [N + 100] + c["lens"][1:]
    _, flags = _run(lib, bits, B, N, 0, 0, q, qpos, c["lens"], scale, impl=lla.IMPL_SIMT)
    assert flags & lla.FLAG_POS_CLAMPED
    lib.close()


def test_host_validation_without_launch():
    c = RAGGED[0]
    cfg, codec, lib, bits, cK, cV, q = _ragged_case(c, "ragged0")
    d = lib.desc
    B, N = c["B"], c["N"]
    store = torch.zeros(lla.store_bytes(d, B, N) // 2, dtype=torch.int16, device=DEV)
    qd = torch.zeros(B, d.H, d.d_head, device=DEV)
    z = torch.zeros(B, dtype=torch.int32, device=DEV)
    out = torch.empty_like(qd)
    ws = torch.empty(lib.workspace_bytes(B, N), dtype=torch.uint8, device=DEV)
    with pytest.raises(lla.LLAError) as e:
        lla.decode_attn(lib, store, B, N, d.D, 0, qd, z, z, 1.0, out, ws)  # layer out of range
    assert e.value.status == 1
    with pytest.raises(lla.LLAError) as e:
        lla.decode_attn(lib, store, B, N, 0, 0, qd, z, z, 1.0, out, ws, workspace_bytes=16)
    assert e.value.status == 6
    with pytest.raises(lla.LLAError) as e:
        lla.decode_attn(lib, store.data_ptr() + 2, B, N, 0, 0, qd, z, z, 1.0, out, ws)
    assert e.value.status == 3
    with pytest.raises(lla.LLAError) as e:
        lla.decode_attn_2d(lib, store, B, N, 0, 0, qd, z, z, 1.0, out, ws)  # variant mismatch
    assert e.value.status == 1
    lib.close()
