"""GPU encode c = (x - mu) W_down vs the FP64 oracle, through the C ABI.

The oracle encodes the same bf16 teacher stacks with the same bf16 W_down
and float32 mu; the library's bf16 latents must match within rel-L2 5e-3 and
max-abs 2e-2.  Rows are scattered to (sequence, token) slots; slots nobody
writes keep their previous contents.
"""

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
from oracle import lla_oracle as O  # noqa: E402
from lla_testutil import assert_close, from_bf16_bits, make_lib_codec, rounded_codec, to_bf16_bits  # noqa: E402

DEV = "cuda"
SENTINEL = 0x7FC1  # a bf16 NaN bit pattern


def _stacks(tag, n, nl, H, T, d, R, noise, variant):
    """Teacher stacks [n][nl][H][2][S] (per-head) or [n][nl][2][S2] (2D), rounded to bf16."""
    if variant == 0:
        x = np.empty((n, nl, H, 2, T * d))
        for l in range(nl):
            for h in range(H):
                for a in range(2):
                    x[:, l, h, a] = syn.smooth_stacks(f"{tag}/x/{l}/{h}/{a}", n, T, d, R, noise,
                                                      syn.gaussian(f"{tag}/mu/{l}/{h}/{a}", T * d, 0.1))
    else:
        x = np.empty((n, nl, 2, T * H * d))
        for l in range(nl):
            for a in range(2):
                x[:, l, a] = syn.smooth_stacks(f"{tag}/x/{l}/{a}", n, T, H * d, R, noise,
                                               syn.gaussian(f"{tag}/mu/{l}/{a}", T * H * d, 0.1))
    return syn.round_bf16(x)


CASES = [
    dict(D=2, T=4, H=2, d_head=16, r_k=4, r_v=8, variant=0, n=300, B=3, N=128, layers=(0, 2)),
    dict(D=3, T=4, H=4, d_head=128, r_k=16, r_v=32, variant=0, n=200, B=2, N=160, layers=(1, 2)),
    dict(D=1, T=4, H=2, d_head=128, r_k=96, r_v=160, variant=0, n=130, B=1, N=130, layers=(0, 1)),
    dict(D=1, T=32, H=2, d_head=128, r_k=96, r_v=160, variant=0, n=70, B=2, N=64, layers=(0, 1)),
    # several 256-token items of the wide codec, the last one ragged
    dict(D=3, T=4, H=2, d_head=128, r_k=96, r_v=160, variant=0, n=700, B=2, N=400, layers=(1, 3)),
    dict(D=2, T=2, H=4, d_head=16, r_k=12, r_v=20, variant=1, n=150, B=2, N=100, layers=(0, 2)),
    dict(D=1, T=4, H=16, d_head=128, r_k=64, r_v=128, variant=1, n=100, B=1, N=128, layers=(0, 1)),
    # T = 1: per-loop MLA, the head-axis latent of one loop
    dict(D=2, T=1, H=16, d_head=128, r_k=64, r_v=128, variant=1, n=90, B=1, N=128, layers=(0, 2)),
]


@pytest.mark.parametrize("ci", range(len(CASES)))
def test_encode_matches_oracle(ci):
    c = CASES[ci]
    tag = f"enc{ci}"
    D, T, H, d, rk, rv, v = c["D"], c["T"], c["H"], c["d_head"], c["r_k"], c["r_v"], c["variant"]
    lb, nl = c["layers"][0], c["layers"][1] - c["layers"][0]
    codec = rounded_codec(syn.seeded_codec(dict(c, mu_var=0.1), tag))
    lib = make_lib_codec(lla, dict(D=D, T=T, H=H, d_head=d, r_k=rk, r_v=rv, variant=v, rope_base=10000.0,
                                   max_pos=c["N"] + 1), codec)
    x = _stacks(tag, c["n"], nl, H, T, d, 6, 1e-2, v)
    rng = syn.rng(tag + "/slots")
    slots = rng.permutation(c["B"] * c["N"])[: c["n"]]
    seq_idx, tok_idx = slots // c["N"], slots % c["N"]
    seq_idx[0] = -1  # out of range: skipped
    tok_idx[1] = c["N"]  # out of range: skipped
    nbytes = lla.store_bytes(lib.desc, c["B"], c["N"])
    store = torch.full((nbytes // 2,), SENTINEL, dtype=torch.int16, device=DEV)
    xd = torch.from_numpy(to_bf16_bits(x).view(np.int16)).to(DEV)
    sd = torch.tensor(seq_idx, dtype=torch.int32, device=DEV)
    td = torch.tensor(tok_idx, dtype=torch.int32, device=DEV)
    lla.encode(lib, xd, c["n"], lb, nl, sd, td, store, c["B"], c["N"])
    torch.cuda.synchronize()
    rowlen = (rk + rv) * (H if v == 0 else 1)
    got_bits = store.cpu().numpy().view(np.uint16).reshape(c["B"], D, c["N"], rowlen)
    written = np.zeros((c["B"], c["N"]), bool)
    errs = []
    for i in range(c["n"]):
        b, j = seq_idx[i], tok_idx[i]
        if not (0 <= b < c["B"] and 0 <= j < c["N"]):
            continue
        written[b, j] = True
        for L in range(nl):
            l = lb + L
            row = from_bf16_bits(got_bits[b, l, j])
            if v == 0:
                row = row.reshape(H, rk + rv)
                for h in range(H):
                    for a, (r, off) in enumerate(((rk, 0), (rv, rk))):
                        ref = O.encode(x[i, L, h, a], codec[f"mu_{'kv'[a]}"][l, h], codec[f"w_down_{'kv'[a]}"][l, h])
                        errs.append((row[h, off:off + r], ref))
            else:
                for a, (r, off) in enumerate(((rk, 0), (rv, rk))):
                    ref = O.encode(x[i, L, a], codec[f"mu_{'kv'[a]}"][l], codec[f"w_down_{'kv'[a]}"][l])
                    errs.append((row[off:off + r], ref))
    got = np.concatenate([g for g, _ in errs])
    ref = np.concatenate([r for _, r in errs])
    assert_close(got, ref, "latents")
    # untouched rows and layers keep the sentinel
    for l in range(D):
        mask = ~written if lb <= l < lb + nl else np.ones_like(written)
        assert np.all(got_bits[:, l][mask] == SENTINEL)
    lib.close()
