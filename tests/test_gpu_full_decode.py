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
from lla_testutil import assert_close, from_bf16_bits, to_bf16_bits  # noqa: E402
from oracle import lla_oracle as O  # noqa: E402

DEV = "cuda"
NAN_BF16 = 0x7FC0


def _cache(tag, B, L, N, H, d, lens):
    """bf16 bits of [B][L][N][H][d] rotated keys and values (the oracle's order), NaN past lens."""
    K = syn.gaussian(tag + "/K", (B, L, N, H, d))
    pos = np.arange(N, dtype=np.float64)[None, None, :, None]
    half = d // 2
    th = pos[..., None] * np.power(10000.0, -2.0 * np.arange(half) / d)  # [1,1,N,1,half]
    c, s = np.cos(th), np.sin(th)
    Kr = np.concatenate([K[..., :half] * c - K[..., half:] * s, K[..., half:] * c + K[..., :half] * s], -1)
    kb, vb = to_bf16_bits(Kr), to_bf16_bits(syn.gaussian(tag + "/V", (B, L, N, H, d)))
    for b, n in enumerate(lens):
        kb[b, :, n:] = NAN_BF16
        vb[b, :, n:] = NAN_BF16
    return kb, vb


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


@pytest.mark.parametrize("c", [dict(B=3, L=1, N=520, H=16, lens=[520, 0, 129]),
                               dict(B=4, L=2, N=300, H=3, lens=[1, 300, 255, 77]),
                               dict(B=2, L=1, N=1, H=1, lens=[1, 0])])  # one cached token: out = v_0
def test_full_decode_matches_oracle(c):
    B, L, N, H, d = c["B"], c["L"], c["N"], c["H"], 128
    tag = f"full/{B}/{H}"
    kb, vb = _cache(tag, B, L, N, H, d, c["lens"])
    q = syn.round_f32(syn.gaussian(tag + "/q", (B, H, d)))
    qpos = [n + 3 for n in c["lens"]]
    scale = 1 / math.sqrt(d)
    layer = L - 1
    ref = O.full_decode(q, from_bf16_bits(kb[:, layer]), from_bf16_bits(vb[:, layer]), c["lens"], qpos, scale,
                        10000.0)
    for ctas in (0, 1, 7, 300):
        got, flags = _run(kb, vb, layer, B, L, N, H, d, q, qpos, c["lens"], scale, ctas)
        assert flags == 0
        assert_close(got, ref, f"full decode ctas {ctas}")
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
    (layer, loop) slice of a cache with a larger sequence stride, one persistent CTA per SM;
    sampled sequences (one ragged) checked against the oracle."""
    B, H, d, N = 32, 16, 128, 4096
    cap = N + 1
    stride = 2 * cap * H * d  # two slices per sequence: the call reads the second
    g = torch.Generator(device=DEV)
    g.manual_seed(syn.sub_seed("full/fullsize"))
    K = torch.empty(B * stride, dtype=torch.bfloat16, device=DEV).normal_(generator=g)
    V = torch.empty(B * stride, dtype=torch.bfloat16, device=DEV).normal_(generator=g)
    q = torch.empty(B, H, d, device=DEV).normal_(generator=g)
    lens = torch.full((B,), N, dtype=torch.int32, device=DEV)
    lens[17] = N - 333
    qpos = lens + 1
    out = torch.full((B, H, d), float("nan"), device=DEV)
    ws = torch.empty(lla.full_decode_workspace_bytes(H, d, B), dtype=torch.uint8, device=DEV)
    off = cap * H * d
    scale = 1 / math.sqrt(d)
    lla.full_decode_attn(H, d, 10000.0, K.data_ptr() + 2 * off, V.data_ptr() + 2 * off, stride, B, cap, q, qpos, lens,
                         scale, out, ws)
    torch.cuda.synchronize()
    assert lla.workspace_flags(ws) == 0
    sample = [0, 17, 31]
    kv = lambda T: T.view(B, 2, H, cap, d)[sample, 1].float().cpu().numpy().astype(np.float64).transpose(0, 2, 1, 3)
    ref = O.full_decode(q[sample].cpu().numpy().astype(np.float64), kv(K), kv(V), lens[sample].cpu().numpy(),
                        qpos[sample].cpu().numpy(), scale, 10000.0)
    assert_close(out[sample].cpu().numpy().astype(np.float64), ref, "full size sampled")
