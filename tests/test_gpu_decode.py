"""GPU decode attention vs the FP64 oracle, through the C ABI.

Small shapes that span several 128-token tiles, ragged context lengths
(0, 1, a tile boundary and odd tails), several split counts, both kernels
(CUDA-core reference and tcgen05), both LLA variants, and the device-side
range flags.  The acceptance bar is rel-L2 <= 5e-3 and max-abs <= 2e-2, on
the output and on its attention-dependent part out - mu^V_t.

The queries are aimed at a few cached keys (``parity_cases``), so attention is
peaked and a mistake in the score path (query or key position, a dropped
token, the scale, scores ignored) misses the bar; ``test_parity_sensitivity``
pins that on the CPU for every input set used here.
"""

import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
from oracle import lla_oracle as O  # noqa: E402
import parity_cases as PC  # noqa: E402
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


def _run_case(lib, bits, case, N, impl=lla.IMPL_AUTO, num_ctas=0):
    return _run(lib, bits, len(case.lens), N, case.layer, case.loop, case.q, case.qpos, case.lens, case.scale,
                impl=impl, num_ctas=num_ctas)


# ---------------------------------------------------------------------------------------------
# tiny workload: SVD codec fitted by the oracle, teacher stacks encoded by the oracle
# ---------------------------------------------------------------------------------------------

@pytest.fixture(scope="module")
def tiny():
    cfg = dict(syn.CONFIGS["tiny_d16_t4"])
    D, T, H, d, rk, rv, N = cfg["D"], cfg["T"], cfg["H"], cfg["d_head"], cfg["r_k"], cfg["r_v"], cfg["context"]
    s = PC.tiny_set()
    lib = make_lib_codec(lla, s.desc_kw(N + 1), s.codec)
    q = syn.round_f32(syn.gaussian("tiny/q", (T, 1, H, d)))
    yield cfg, s, lib, q
    lib.close()


@pytest.mark.parametrize("impl", [lla.IMPL_SIMT, lla.IMPL_TC])
def test_tiny_workload_all_loops(tiny, impl):
    """The tiny workload as configured: query ~ N(0, 1), scale 1/sqrt(d_head), query at position N."""
    cfg, s, lib, q = tiny
    N, d = cfg["context"], cfg["d_head"]
    if impl == lla.IMPL_TC and not _tc_supported(lib, 1, N):
        pytest.skip("tcgen05 kernel does not cover this shape")
    bits = s.bits
    for t in range(cfg["T"]):
        got, flags = _run(lib, bits, 1, N, 0, t, q[t], [N], [N], 1 / math.sqrt(d), impl=impl)
        ref = oracle_decode(s.codec, s.cfg, s.cK[:, 0], s.cV[:, 0], q[t], 0, t, [N], [N], 1 / math.sqrt(d))
        assert flags == 0
        PC.assert_decode_close(got, ref, PC.mu_v_t(s.codec, s.cfg, 0, t), f"loop {t}")


def test_tiny_workload_aimed_queries(tiny):
    """The tiny workload's store and codec with queries aimed at a few cached keys, every loop."""
    cfg, s, lib, _ = tiny
    N = cfg["context"]
    bits = s.bits
    for t in range(cfg["T"]):
        case = s.case(0, t, qpos=[N])
        got, flags = _run_case(lib, bits, case, N, impl=lla.IMPL_SIMT)
        assert flags == 0
        PC.assert_decode_close(got, case.reference(), case.mu_v(), f"aimed loop {t}")


# ---------------------------------------------------------------------------------------------
# ragged contexts, several splits, seeded orthonormal codecs
# ---------------------------------------------------------------------------------------------

RAGGED = PC.RAGGED


@pytest.mark.parametrize("ci,mu_v_zero", [(0, False), (1, False), (2, False), (3, False), (1, True)])
def test_ragged_contexts_match_oracle(ci, mu_v_zero):
    c = RAGGED[ci]
    s, case = PC.ragged_case(ci, mu_v_zero)
    lib = make_lib_codec(lla, s.desc_kw(c["N"] + 8), s.codec)
    B, N = c["B"], c["N"]
    impls = [lla.IMPL_SIMT] + ([lla.IMPL_TC] if _tc_supported(lib, B, N) else [])
    ref = case.reference()
    bits = s.bits
    for impl in impls:
        got, flags = _run_case(lib, bits, case, N, impl=impl)
        assert flags == 0
        PC.assert_decode_close(got, ref, case.mu_v(), f"impl {impl}")
        assert np.all(got[np.array(c["lens"]) == 0] == 0)
    lib.close()


@pytest.mark.parametrize("ci", [1, 2])
@pytest.mark.parametrize("impl,ctas", [(lla.IMPL_SIMT, 1), (lla.IMPL_SIMT, 2), (lla.IMPL_SIMT, 7),
                                       (lla.IMPL_TC, 1), (lla.IMPL_TC, 2), (lla.IMPL_TC, 7), (lla.IMPL_TC, 300)])
def test_split_count_invariance(impl, ctas, ci):
    c = RAGGED[ci]
    s = PC.ragged_set(ci)
    lib = make_lib_codec(lla, s.desc_kw(c["N"] + 8), s.codec)
    if impl == lla.IMPL_TC and not _tc_supported(lib, c["B"], c["N"]):
        pytest.skip("tcgen05 kernel does not cover this shape")
    case = s.case(0, 2)
    bits = s.bits
    base, _ = _run_case(lib, bits, case, c["N"], impl=impl, num_ctas=1)
    got, _ = _run_case(lib, bits, case, c["N"], impl=impl, num_ctas=ctas)
    assert np.abs(got - base).max() < 1e-4
    lib.close()


# ---------------------------------------------------------------------------------------------
# LLA-2D
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("ci,mu_v_zero", [(0, False), (1, False), (2, False), (3, False), (2, True)])
def test_2d_matches_oracle(ci, mu_v_zero):
    """LLA-2D codecs (the last with T = 1: per-loop MLA, the head-axis latent of one loop)."""
    c = PC.TWO_D[ci]
    s = PC.two_d_set(ci, mu_v_zero)
    B, N = c["B"], c["N"]
    lib = make_lib_codec(lla, s.desc_kw(N + 4), s.codec)
    bits = s.bits
    impls = [lla.IMPL_SIMT] + ([lla.IMPL_TC] if _tc_supported(lib, B, N) else [])
    for layer, loop in PC.two_d_calls(ci):
        case = s.case(layer, loop)
        ref = case.reference()
        for impl in impls:
            got, flags = _run_case(lib, bits, case, N, impl=impl)
            assert flags == 0
            PC.assert_decode_close(got, ref, case.mu_v(), f"2d impl {impl} layer {layer} loop {loop}")
            assert np.all(got[np.array(c["lens"]) == 0] == 0)
        if lla.IMPL_TC in impls:  # result independent of the persistent grid
            for ctas in (4, 8, 300):
                got, _ = _run_case(lib, bits, case, N, impl=lla.IMPL_TC, num_ctas=ctas)
                PC.assert_decode_close(got, ref, case.mu_v(), f"2d tc ctas {ctas}")
    lib.close()


@pytest.mark.parametrize("variant,rk,rv", PC.TC_SHAPES)
def test_rows_past_the_context_may_hold_nan(variant, rk, rv):
    """Store rows at or beyond a sequence's length are outside the attention [LLA §3 eq. (3)
    sums over the cached tokens only]: a quiet-NaN pattern there must not reach the output."""
    s = PC.tc_shape_set(variant, rk, rv, f"nan_tail/{variant}/{rk}")
    N = 300
    case = s.case(0, 1)
    bits = s.bits
    for b, n in enumerate(case.lens):
        bits[b, :, n:] = 0x7FC0  # bf16 quiet NaN
    lib = make_lib_codec(lla, s.desc_kw(N + 4), s.codec)
    ref = case.reference()
    impls = [lla.IMPL_SIMT] + ([lla.IMPL_TC] if _tc_supported(lib, len(case.lens), N) else [])
    assert lla.IMPL_TC in impls
    for impl in impls:
        got, flags = _run_case(lib, bits, case, N, impl=impl)
        assert flags == 0
        assert np.isfinite(got).all(), f"impl {impl}"
        PC.assert_decode_close(got, ref, case.mu_v(), f"nan tail impl {impl}")
    lib.close()


@pytest.mark.parametrize("variant,rk,rv", PC.TC_SHAPES)
def test_stale_workspace_does_not_reach_the_output(variant, rk, rv):
    """The workspace is not cleared between calls: every split record the combine reads is
    written by the same call, and a CTA group whose share of the tiles is empty (a batch with
    fewer tiles than groups) is skipped.  A workspace full of NaN bytes, then the same workspace
    reused with other lengths, gives the oracle's outputs both times."""
    s = PC.tc_shape_set(variant, rk, rv, f"stale_ws/{variant}/{rk}")
    B, N, H, d = 3, 300, 16, 128
    lib = make_lib_codec(lla, s.desc_kw(N + 4), s.codec)
    assert _tc_supported(lib, B, N)
    store = torch.from_numpy(s.bits.view(np.int16)).to(DEV)
    ws = torch.full((lib.workspace_bytes(B, N),), 0xFF, dtype=torch.uint8, device=DEV)
    for loop, lens in PC.STALE_CALLS:
        case = s.case(0, loop, lens=lens)
        qd = torch.from_numpy(np.ascontiguousarray(case.q, np.float32)).to(DEV)
        ln = torch.tensor(lens, dtype=torch.int32, device=DEV)
        out = torch.full((B, H, d), float("nan"), dtype=torch.float32, device=DEV)
        lla.decode_attn(lib, store, B, N, 0, loop, qd, ln, ln, case.scale, out, ws, impl=lla.IMPL_TC)
        torch.cuda.synchronize()
        assert lla.workspace_flags(ws) == 0
        got = out.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all(), lens
        PC.assert_decode_close(got, case.reference(), case.mu_v(), f"lens {lens}")
    lib.close()


# ---------------------------------------------------------------------------------------------
# range flags
# ---------------------------------------------------------------------------------------------

def test_out_of_range_lengths_and_positions_are_clamped_and_flagged():
    c = RAGGED[0]
    s, case = PC.ragged_case(0)
    lib = make_lib_codec(lla, s.desc_kw(c["N"] + 8), s.codec)
    B, N = c["B"], c["N"]
    bits = s.bits
    lens = [N + 50] + c["lens"][1:]
    got, flags = _run(lib, bits, B, N, case.layer, case.loop, case.q, case.qpos, lens, case.scale,
                      impl=lla.IMPL_SIMT)
    assert flags & lla.FLAG_SEQ_LEN_CLAMPED
    ref = case.reference(lens=[N] + c["lens"][1:])
    PC.assert_decode_close(got, ref, case.mu_v(), "clamped length")
    qpos = [N + 100] + case.qpos[1:]
    _, flags = _run(lib, bits, B, N, case.layer, case.loop, case.q, qpos, c["lens"], case.scale, impl=lla.IMPL_SIMT)
    assert flags & lla.FLAG_POS_CLAMPED
    lib.close()


def test_host_validation_without_launch():
    c = RAGGED[0]
    s = PC.ragged_set(0)
    lib = make_lib_codec(lla, s.desc_kw(c["N"] + 8), s.codec)
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
