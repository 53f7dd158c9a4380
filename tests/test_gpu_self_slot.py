"""Decode attention with the current token as a self slot, against the oracle.

A token's latent is written only after its last loop [LLA §3 eq. (2)], so while it is decoded
its own loop-t key and value are exact and join the softmax as one more slot at the query's
position.  lla_decode_attn_self is checked against the oracle's lla_decode(..., k_self, v_self)
on both kernels, for per-head and LLA-2D codecs, ragged contexts and empty ones.
"""

import ctypes
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
import parity_cases as PC  # noqa: E402
from lla_testutil import assert_close, make_lib_codec, oracle_decode, rounded_codec, to_bf16_bits  # noqa: E402

DEV = "cuda"

CASES = PC.SELF


def _case(c, tag):
    cfg = dict(c, rope_base=10000.0, mu_var=0.1)
    codec = rounded_codec(syn.seeded_codec(cfg, tag))
    B, N, D, H, d = c["B"], c["N"], c["D"], c["H"], c["d_head"]
    head = () if c["variant"] == 1 else (H,)
    cK = syn.round_bf16(syn.gaussian(tag + "/cK", (B, D, N) + head + (c["r_k"],)))
    cV = syn.round_bf16(syn.gaussian(tag + "/cV", (B, D, N) + head + (c["r_v"],)))
    q = syn.round_f32(syn.gaussian(tag + "/q", (B, H, d)))
    ks = syn.round_f32(syn.gaussian(tag + "/ks", (B, H, d)))
    vs = syn.round_f32(syn.gaussian(tag + "/vs", (B, H, d)))
    lib = make_lib_codec(lla, dict(D=D, T=c["T"], H=H, d_head=d, r_k=c["r_k"], r_v=c["r_v"], variant=c["variant"],
                                   rope_base=10000.0, max_pos=N + 8), codec)
    return cfg, codec, lib, to_bf16_bits(np.concatenate([cK, cV], -1)), cK, cV, q, ks, vs


def _run_self(lib, bits, B, N, layer, loop, q, lens, ks, vs, scale, impl):
    d = lib.desc
    store = torch.from_numpy(bits.view(np.int16)).to(DEV)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(DEV)
    ln = torch.tensor(lens, dtype=torch.int32, device=DEV)
    out = torch.full((B, d.H, d.d_head), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.empty(lib.workspace_bytes(B, N), dtype=torch.uint8, device=DEV)
    lla.decode_attn_self(lib, store, B, N, layer, loop, t(q), ln, ln, t(ks), t(vs), scale, out, ws, impl=impl)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), lla.workspace_flags(ws)


def _tc_ok(c):
    return c["d_head"] == 128 and c["H"] == 16


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_self_slot_matches_oracle(ci):
    """Queries aimed at a few cached keys (the self slot's logit is scale * <q, k_self>)."""
    c = CASES[ci]
    s = PC.self_set(ci)
    lib = make_lib_codec(lla, s.desc_kw(c["N"] + 8), s.codec)
    bits = s.bits
    B, N = c["B"], c["N"]
    impls = [lla.IMPL_SIMT] + ([lla.IMPL_TC] if _tc_ok(c) else [])
    for layer, loop in PC.self_calls(ci):
        case = s.case(layer, loop, self_slot=True)
        ref = case.reference()
        for impl in impls:
            got, flags = _run_self(lib, bits, B, N, layer, loop, case.q, case.lens, case.k_self, case.v_self,
                                   case.scale, impl)
            assert flags == 0
            PC.assert_decode_close(got, ref, case.mu_v(), f"self slot impl {impl} layer {layer} loop {loop}")
            # a sequence with no cached token attends to the self slot alone
            empty = np.array(c["lens"]) == 0
            assert np.abs(got[empty] - case.v_self[empty]).max(initial=0.0) < 1e-6
    lib.close()


def test_self_slot_without_cache_is_the_value():
    c = CASES[0]
    cfg, codec, lib, bits, cK, cV, q, ks, vs = _case(c, "self_nocache")
    B = c["B"]
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(DEV)
    store = torch.zeros(8, dtype=torch.int16, device=DEV)
    ln = torch.zeros(B, dtype=torch.int32, device=DEV)
    out = torch.full((B, 16, 128), float("nan"), device=DEV)
    ws = torch.empty(lib.workspace_bytes(B, 0), dtype=torch.uint8, device=DEV)
    lla.decode_attn_self(lib, store, B, 0, 0, 0, t(q), ln, ln, t(ks), t(vs), 0.1, out, ws)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), vs.astype(np.float32))
    lib.close()


def test_self_slot_argument_errors_without_launch():
    c = CASES[0]
    cfg, codec, lib, bits, cK, cV, q, ks, vs = _case(c, "self_args")
    B, N = c["B"], c["N"]
    buf = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    p = buf.data_ptr()
    ws_bytes = lib.workspace_bytes(B, N)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=DEV)
    opts = lla.DecodeOpts(0, 0, None, None)
    common = (lib.handle, p, B, N, 0, 0, p, p, p)
    # a missing k_self or v_self is an argument error; so is a misaligned one (alignment)
    assert lla.raw_decode_status("lla_decode_attn_self", *common, None, p, 0.1, p, ws.data_ptr(), ws_bytes,
                                 ctypes.byref(opts), None) == 1
    assert lla.raw_decode_status("lla_decode_attn_self", *common, p, None, 0.1, p, ws.data_ptr(), ws_bytes,
                                 ctypes.byref(opts), None) == 1
    assert lla.raw_decode_status("lla_decode_attn_self", *common, p + 4, p, 0.1, p, ws.data_ptr(), ws_bytes,
                                 ctypes.byref(opts), None) == 3
    lib.close()
