"""Paged latent stores: the same rows in shuffled pages of LLA_PAGE_TOKENS tokens give the same results.

A paged store only changes where a latent row is kept [LLA §3 eqs. (2)-(3) are unchanged], so
decode over a paged pool must equal, bit for bit, decode over the contiguous store holding the
same rows (same kernel, same work split), and match the oracle; unused pages and slots past each
sequence's length hold NaN bits, which must never be read into the result.  Encode into a paged
pool must write exactly the rows the contiguous encode writes.
"""

import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
import parity_cases as PC  # noqa: E402
from lla_testutil import make_lib_codec, rounded_codec, to_bf16_bits  # noqa: E402

DEV = "cuda"
P = lla.PAGE_TOKENS
NAN_BF16 = 0x7FC0

CASES = PC.PAGED


def _setup(c, ci, tag):
    s = PC.paged_set(ci, tag)
    B, D, mp = c["B"], c["D"], c["max_pages"]
    N = mp * P
    bits = s.bits  # [B, D, N, (H,) row]
    for b, n in enumerate(c["lens"]):
        bits[b, :, n:] = NAN_BF16
    # pool: every sequence's pages in a shuffled order, plus spare pages of NaN
    num_pages = B * mp + 3
    perm = syn.rng(tag + "/perm").permutation(num_pages)
    table = perm[:B * mp].reshape(B, mp).astype(np.int32)
    pool = np.full((num_pages, D, P) + bits.shape[3:], NAN_BF16, np.uint16)
    for b in range(B):
        for pg in range(mp):
            pool[table[b, pg]] = bits[b, :, pg * P:(pg + 1) * P]
    lib = make_lib_codec(lla, s.desc_kw(N + 8), s.codec)
    return s, lib, bits, pool, table, num_pages


def _t(a, dt=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device=DEV, dtype=dt)


def _decode_both(lib, c, bits, pool, table, num_pages, q, lens, layer, loop, impl, ks=None, vs=None):
    B, mp = c["B"], c["max_pages"]
    N = mp * P
    ln = torch.tensor(lens, dtype=torch.int32, device=DEV)
    qd = _t(q)
    ws = torch.empty(lib.workspace_bytes(B, N), dtype=torch.uint8, device=DEV)
    scale = 1 / math.sqrt(c["d_head"])
    out_c = torch.full((B, c["H"], c["d_head"]), float("nan"), device=DEV)
    store = torch.from_numpy(bits.view(np.int16)).to(DEV)
    if ks is None:
        lla.decode_attn(lib, store, B, N, layer, loop, qd, ln, ln, scale, out_c, ws, impl=impl)
    else:
        lla.decode_attn_self(lib, store, B, N, layer, loop, qd, ln, ln, _t(ks), _t(vs), scale, out_c, ws, impl=impl)
    torch.cuda.synchronize()
    flags_c = lla.workspace_flags(ws)
    out_p = torch.full_like(out_c, float("nan"))
    pool_d = torch.from_numpy(pool.view(np.int16)).to(DEV)
    tab = _t(table, torch.int32)
    lla.decode_attn_paged(lib, pool_d, num_pages, tab, mp, B, layer, loop, qd, ln, ln, scale, out_p, ws,
                          k_self=None if ks is None else _t(ks), v_self=None if vs is None else _t(vs), impl=impl)
    torch.cuda.synchronize()
    return out_c.cpu().numpy(), flags_c, out_p.cpu().numpy(), lla.workspace_flags(ws)


def _impls(c):
    return [lla.IMPL_SIMT] + ([lla.IMPL_TC] if c["d_head"] == 128 and c["H"] == 16 else [])


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_paged_decode_equals_contiguous_and_oracle(ci):
    c = CASES[ci]
    s, lib, bits, pool, table, num_pages = _setup(c, ci, f"paged{ci}")
    case = s.case(c["D"] - 1, 1)
    ref = case.reference()
    for impl in _impls(c):
        out_c, fc, out_p, fp = _decode_both(lib, c, bits, pool, table, num_pages, case.q, c["lens"], case.layer,
                                            case.loop, impl)
        assert fc == 0 and fp == 0
        assert np.array_equal(out_c, out_p), f"impl {impl}: paged differs from contiguous"
        PC.assert_decode_close(out_p.astype(np.float64), ref, case.mu_v(), f"paged impl {impl}")
    lib.close()


def test_paged_decode_with_self_slot():
    c = CASES[0]
    s, lib, bits, pool, table, num_pages = _setup(c, 0, "paged_self")
    case = s.case(0, 2, self_slot=True)
    ref = case.reference()
    for impl in _impls(c):
        out_c, _, out_p, _ = _decode_both(lib, c, bits, pool, table, num_pages, case.q, c["lens"], 0, 2, impl,
                                          case.k_self, case.v_self)
        assert np.array_equal(out_c, out_p)
        PC.assert_decode_close(out_p.astype(np.float64), ref, case.mu_v(), f"paged self impl {impl}")
    lib.close()


def test_invalid_page_cuts_the_sequence_and_is_flagged():
    c = CASES[0]
    s, lib, bits, pool, table, num_pages = _setup(c, 0, "paged_bad")
    bad = table.copy()
    bad[0, 2] = num_pages + 5  # sequence 0 (512 tokens) loses pages 2 and 3: 256 tokens remain
    cut = list(c["lens"])
    cut[0] = 2 * P
    case = s.case(1, 0, lens=cut, qpos=c["lens"])
    for impl in _impls(c):
        B, mp = c["B"], c["max_pages"]
        ln = torch.tensor(c["lens"], dtype=torch.int32, device=DEV)
        ws = torch.empty(lib.workspace_bytes(B, mp * P), dtype=torch.uint8, device=DEV)
        out = torch.empty(B, 16, 128, device=DEV)
        lla.decode_attn_paged(lib, _t(pool.view(np.int16), torch.int16), num_pages, _t(bad, torch.int32), mp, B, 1, 0,
                              _t(case.q), ln, ln, case.scale, out, ws, impl=impl)
        torch.cuda.synchronize()
        assert lla.workspace_flags(ws) & lla.FLAG_PAGE_INVALID
        PC.assert_decode_close(out.cpu().numpy().astype(np.float64), case.reference(), case.mu_v(), f"cut impl {impl}")
    lib.close()


@pytest.mark.parametrize("shape", [(0, 16, 32, 16), (0, 96, 160, 16), (1, 64, 128, 16), (0, 8, 24, 3)])
def test_paged_encode_writes_the_same_rows(shape):
    variant, rk, rv, H = shape
    D, T, d, B, mp = 2, 4, 128 if H == 16 else 32, 3, 2
    N = mp * P
    cfg = dict(D=D, T=T, H=H, d_head=d, r_k=rk, r_v=rv, variant=variant, rope_base=10000.0, mu_var=0.1)
    codec = rounded_codec(syn.seeded_codec(cfg, f"penc/{shape}"))
    lib = make_lib_codec(lla, dict(D=D, T=T, H=H, d_head=d, r_k=rk, r_v=rv, variant=variant, rope_base=10000.0,
                                   max_pos=N + 8), codec)
    S = T * d if variant == 0 else T * H * d
    n = 150
    xs = (n, D, H, 2, S) if variant == 0 else (n, D, 2, S)
    x = _t(to_bf16_bits(syn.gaussian(f"penc/{shape}/x", xs)).view(np.int16), torch.int16)
    r = syn.rng(f"penc/{shape}/idx")
    seq = r.integers(0, B, n).astype(np.int32)
    tok = r.integers(0, N, n).astype(np.int32)
    keys = seq.astype(np.int64) * N + tok
    _, first = np.unique(keys, return_index=True)  # one write per slot
    seq, tok = seq[np.sort(first)], tok[np.sort(first)]
    n = len(seq)
    x = x[:n]
    row = (rk + rv) * (H if variant == 0 else 1)
    store = torch.zeros(B * D * N * row, dtype=torch.int16, device=DEV)
    lla.encode(lib, x, n, 0, D, _t(seq, torch.int32), _t(tok, torch.int32), store, B, N)
    num_pages = B * mp + 2
    table = syn.rng(f"penc/{shape}/perm").permutation(num_pages)[:B * mp].reshape(B, mp).astype(np.int32)
    pool = torch.zeros(num_pages * D * P * row, dtype=torch.int16, device=DEV)
    lla.encode_paged(lib, x, n, 0, D, _t(seq, torch.int32), _t(tok, torch.int32), pool, num_pages,
                     _t(table, torch.int32), mp, B)
    torch.cuda.synchronize()
    s = store.cpu().numpy().reshape(B, D, N, row)
    pl = pool.cpu().numpy().reshape(num_pages, D, P, row)
    for b in range(B):
        for pg in range(mp):
            assert np.array_equal(s[b, :, pg * P:(pg + 1) * P], pl[table[b, pg]]), (b, pg)
    lib.close()
