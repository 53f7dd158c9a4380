"""The GPU path end to end: teacher stacks -> lla_encode -> store -> lla_decode_attn, against the
oracle's encode [LLA §3 eq. (2)] followed by its decode [LLA §3 eq. (3), RoPE after
reconstruction, softmax attention], on the same seeded stacks and codec.

The oracle consumes the latents rounded to bf16, as the store holds them; the GPU encode rounds
to nearest-even too, so the two latent sets agree to within an ulp and the outputs within the
acceptance bar (on the output and on out - mu^V_t; queries aimed at a few cached keys, so the
score path is exercised).  Also: repeated decode calls on the same inputs are bit-identical.
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

SHAPES = [  # (variant, r_k, r_v): the three shapes the tensor-core kernels cover
    (0, 16, 32),
    (0, 96, 160),
    (1, 64, 128),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_encode_then_decode_matches_oracle(shape):
    """Queries aimed at a few cached keys of the oracle's latents, one decode call per loop."""
    variant, rk, rv = shape
    H, d, T = 16, 128, 4
    B, N, lens = PC.PIPE_B, PC.PIPE_N, PC.PIPE_LENS
    x, lat = PC.pipeline_inputs(variant, rk, rv, T, H, d)
    lib = make_lib_codec(lla, lat.desc_kw(N + 8), lat.codec)
    # GPU: every (sequence, token) stack encoded into its slot, then one decode call per loop
    seq = np.repeat(np.arange(B), N).astype(np.int32)
    tok = np.tile(np.arange(N), B).astype(np.int32)
    store = torch.zeros(lla.store_bytes(lib.desc, B, N) // 2, dtype=torch.int16, device=DEV)
    xd = torch.from_numpy(to_bf16_bits(x).view(np.int16)).to(DEV)
    lla.encode(lib, xd, B * N, 0, 1, torch.from_numpy(seq).to(DEV), torch.from_numpy(tok).to(DEV), store, B, N)
    ln = torch.tensor(lens, dtype=torch.int32, device=DEV)
    ws = torch.empty(lib.workspace_bytes(B, N), dtype=torch.uint8, device=DEV)
    # oracle: encode [LLA §3 eq. (2)] (the store's bf16 rounding included), then decode
    for t in range(T):
        case = lat.case(0, t)
        out = torch.full((B, H, d), float("nan"), device=DEV)
        qd = torch.from_numpy(case.q.astype(np.float32)).to(DEV)
        lla.decode_attn(lib, store, B, N, 0, t, qd, ln, ln, case.scale, out, ws, impl=lla.IMPL_TC)
        torch.cuda.synchronize()
        assert lla.workspace_flags(ws) == 0
        PC.assert_decode_close(out.cpu().numpy().astype(np.float64), case.reference(), case.mu_v(), f"loop {t}")
    lib.close()


@pytest.mark.parametrize("shape", SHAPES)
def test_decode_is_deterministic(shape):
    """Same inputs, same grid: bit-identical outputs (the split-combine order is fixed)."""
    variant, rk, rv = shape
    B, N, H, d = 3, 700, 16, 128
    tag = f"det/{variant}/{rk}"
    cfg = dict(D=1, T=4, H=H, d_head=d, r_k=rk, r_v=rv, variant=variant, rope_base=10000.0, mu_var=0.1)
    codec = rounded_codec(syn.seeded_codec(cfg, tag))
    lib = make_lib_codec(lla, dict(D=1, T=4, H=H, d_head=d, r_k=rk, r_v=rv, variant=variant, rope_base=10000.0,
                                   max_pos=N + 8), codec)
    g = torch.Generator(device=DEV)
    g.manual_seed(syn.sub_seed(tag))
    store = torch.empty(lla.store_bytes(lib.desc, B, N) // 2, dtype=torch.bfloat16, device=DEV).normal_(generator=g)
    q = torch.empty(B, H, d, device=DEV).normal_(generator=g)
    ln = torch.tensor([700, 333, 129], dtype=torch.int32, device=DEV)
    ws = torch.empty(lib.workspace_bytes(B, N), dtype=torch.uint8, device=DEV)
    outs = []
    for _ in range(3):
        out = torch.empty(B, H, d, device=DEV)
        lla.decode_attn(lib, store, B, N, 0, 2, q, ln, ln, 1 / math.sqrt(d), out, ws, impl=lla.IMPL_TC)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy())
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])
    lib.close()
