"""The full-cache comparator (lla_full_decode_attn) against the oracle's full_decode.

Keys are cached already rotated at their positions; the kernel rotates the query.  Checked on
ragged contexts (empty ones included), NaN bits past each sequence's length, a slice of a larger
multi-layer cache (sequence stride above max_tokens * H * d), several persistent grid sizes, and
argument errors.
"""

import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
import parity_cases as PC  # noqa: E402
from lla_testutil import to_bf16_bits  # noqa: E402
from oracle import lla_oracle as O  # noqa: E402

DEV = "cuda"
NAN_BF16 = 0x7FC0


def _run(kb, vb, layer, B, L, N, H, d, q, qpos, lens, scale, num_ctas=0):
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(device=DEV, dtype=dt)
    # the kernel's head-major layout [B][L][H][N][d]
    K = t(kb.view(np.int16).transpose(0, 1, 3, 2, 4), torch.int16)
    V = t(vb.view(np.int16).transpose(0, 1, 3, 2, 4), torch.int16)
    off = layer * N * H * d  # elements: the layer's slice of sequence 0
    out = torch.full((B, H, d), float("nan"), device=DEV)
    ws = torch.empty(lla.full_decode_workspace_bytes(H, d, B), dtype=torch.uint8, device=DEV)
    lla.full_decode_attn(H, d, 10000.0, K.data_ptr() + 2 * off, V.data_ptr() + 2 * off, L * N * H * d, B, N,
                         t(q, torch.float32), t(np.array(qpos, np.int32), torch.int32),
                         t(np.array(lens, np.int32), torch.int32), scale, out, ws, num_ctas=num_ctas)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), lla.workspace_flags(ws)


@pytest.mark.parametrize("ci", range(len(PC.FULL_CACHE)))
def test_full_decode_matches_oracle(ci):
    """Queries aimed at a few cached keys (the last one included), so the scores decide the result."""
    c, Kr, V, q, qpos, scale = PC.full_cache_inputs(ci)
    B, L, N, H, d = c["B"], c["L"], c["N"], c["H"], 128
    kb, vb = to_bf16_bits(Kr), to_bf16_bits(V)
    for b, n in enumerate(c["lens"]):
        kb[b, :, n:] = NAN_BF16
        vb[b, :, n:] = NAN_BF16
    layer = L - 1
    ref = O.full_decode(q, Kr[:, layer], V[:, layer], c["lens"], qpos, scale, PC.ROPE_BASE)
    zero = np.zeros((H, d))
    for ctas in (0, 1, 7, 300):
        got, flags = _run(kb, vb, layer, B, L, N, H, d, q, qpos, c["lens"], scale, ctas)
        assert flags == 0
        PC.assert_decode_close(got, ref, zero, f"full decode ctas {ctas}")
        assert np.all(got[np.array(c["lens"]) == 0] == 0)


def test_full_decode_argument_errors():
    buf = torch.zeros(1 << 16, dtype=torch.uint8, device=DEV)
    p = buf.data_ptr()
    ws = torch.empty(lla.full_decode_workspace_bytes(16, 128, 2), dtype=torch.uint8, device=DEV)
    with pytest.raises(lla.LLAError) as e:  # only d_head 128 is built
        lla.full_decode_attn(16, 64, 10000.0, p, p, 1 << 12, 2, 4, p, p, p, 0.1, p, ws)
    assert e.value.status == 2
    with pytest.raises(lla.LLAError) as e:  # sequence stride shorter than one sequence
        lla.full_decode_attn(16, 128, 10000.0, p, p, 100, 2, 4, p, p, p, 0.1, p, ws)
    assert e.value.status == 1


def test_full_decode_full_size_sampled():
    """The comparator at the bench's size and launch configuration: batch 32 x 4096 x 16 heads, one
    (layer, loop) slice of a cache with a larger sequence stride, one persistent CTA per SM.  The
    cache is filled on the device; the sampled sequences' rows (one ragged) are overwritten with
    host-drawn keys and values, their queries aimed at a few cached keys, and they are checked
    against the oracle."""
    f = PC.full_cache_full_size_sample()
    c = PC.FULL_CACHE_SIZE
    B, H, d, cap, sample = c["B"], c["H"], c["d"], f["cap"], c["sample"]
    stride = 2 * cap * H * d  # two slices per sequence: the call reads the second
    g = torch.Generator(device=DEV)
    g.manual_seed(syn.sub_seed("full/fullsize"))
    K = torch.empty(B * stride, dtype=torch.bfloat16, device=DEV).normal_(generator=g)
    V = torch.empty(B * stride, dtype=torch.bfloat16, device=DEV).normal_(generator=g)
    for T, host in ((K, f["K"]), (V, f["V"])):
        view = T.view(B, 2, H, cap, d)
        for i, b in enumerate(sample):
            view[b, 1] = torch.from_numpy(host[i]).to(device=DEV, dtype=torch.bfloat16)
    q = torch.empty(B, H, d, device=DEV).normal_(generator=g) * 8.0
    q[torch.tensor(sample, device=DEV)] = torch.from_numpy(f["q"].astype(np.float32)).to(DEV)
    lens = torch.from_numpy(f["lens_all"]).to(DEV)
    qpos = lens + 1
    out = torch.full((B, H, d), float("nan"), device=DEV)
    ws = torch.empty(lla.full_decode_workspace_bytes(H, d, B), dtype=torch.uint8, device=DEV)
    off = cap * H * d
    lla.full_decode_attn(H, d, 10000.0, K.data_ptr() + 2 * off, V.data_ptr() + 2 * off, stride, B, cap, q, qpos, lens,
                         f["scale"], out, ws)
    torch.cuda.synchronize()
    assert lla.workspace_flags(ws) == 0
    ref = O.full_decode(f["q"], f["K"].transpose(0, 2, 1, 3), f["V"].transpose(0, 2, 1, 3), f["lens"], f["qpos"],
                        f["scale"], PC.ROPE_BASE)
    e = PC.assert_decode_close(out[sample].cpu().numpy().astype(np.float64), ref, np.zeros((H, d)),
                               "full size sampled")
    print(f"full cache, full size: rel_l2={e[0]:.3e} max_abs={e[2]:.3e}")
