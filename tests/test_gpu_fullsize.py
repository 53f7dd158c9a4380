"""Full-size workloads in the launch configuration bench.py times, checked on samples.

The store is allocated at its full size (116 GB for batch 768 x 4096 at ratio
21.3); only the layer under test is filled, since a decode call reads no other
layer: seeded N(0, 1) latents drawn on the device for the whole batch, then the
rows of a few sampled sequences overwritten with latents drawn on the host
(``parity_cases.full_size_sample``).  The sampled sequences get queries aimed
at a few of their cached keys, so attention is peaked and the score path
decides the result; the other sequences get N(0, 64) queries.  The default
entry point runs (the tensor-core kernel where it applies) and the oracle
recomputes the sampled sequences, all heads.  Where a codec with mu^V = 0 is
listed, the same store is decoded through it too (the whole output then
depends on the attention).
"""

import dataclasses

import numpy as np
import pytest

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

torch = pytest.importorskip("torch")
import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
import parity_cases as PC  # noqa: E402

DEV = "cuda"
MU_V_ZERO = ("ouro_rho21_b768_n4096", "ouro_2d_b256_n8192")


def _codec(case, cap):
    c, k = case.cfg, case.codec
    return lla.Codec(lla.Desc(c["D"], c["T"], c["H"], c["d_head"], c["r_k"], c["r_v"], c["variant"], PC.ROPE_BASE,
                              cap + 1), k["w_down_k"], k["w_down_v"], k["w_up_k"], k["w_up_v"], k["mu_k"], k["mu_v"])


@pytest.mark.parametrize("name", list(PC.FULL_SIZE))
def test_full_size_sampled(name):
    case = PC.full_size_sample(name)
    cfg, x = case.cfg, case.extra
    D, H, d, rk, rv, variant = cfg["D"], cfg["H"], cfg["d_head"], cfg["r_k"], cfg["r_v"], cfg["variant"]
    B, cap, sample, layer = x["batch"], x["cap"], x["sample"], case.layer
    cases = [case]
    if name in MU_V_ZERO:
        cases.append(dataclasses.replace(case, name=case.name + "/muv0",
                                         codec=dict(case.codec, mu_v=np.zeros_like(case.codec["mu_v"]))))
    libs = [_codec(c, cap) for c in cases]
    store = torch.empty(lla.store_bytes(libs[0].desc, B, cap) // 2, dtype=torch.bfloat16, device=DEV)
    view = store.view((B, D, cap) + ((H,) if variant == 0 else ()) + (rk + rv,))
    g = syn.torch_generator(f"full/{name}/lat", DEV)
    for b0 in range(0, B, 64):
        view[b0:b0 + 64, layer].normal_(generator=g)
    for i, b in enumerate(sample):
        view[b, layer] = torch.from_numpy(x["latents"][i]).to(device=DEV, dtype=torch.bfloat16)
    q = torch.empty(B, H, d, device=DEV).normal_(generator=syn.torch_generator(f"full/{name}/q", DEV)) * 8.0
    idx = torch.tensor(sample, device=DEV)
    q[idx] = torch.from_numpy(case.q.astype(np.float32)).to(DEV)
    lens = torch.from_numpy(x["lens_all"]).to(DEV)
    ws = torch.empty(libs[0].workspace_bytes(B, cap), dtype=torch.uint8, device=DEV)
    decode = lla.decode_attn if variant == 0 else lla.decode_attn_2d
    for c, lib in zip(cases, libs):
        out = torch.full((B, H, d), float("nan"), device=DEV)
        decode(lib, store, B, cap, layer, case.loop, q, lens, lens, case.scale, out, ws)
        torch.cuda.synchronize()
        assert lla.workspace_flags(ws) == 0
        got = out.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        e_out, e_att, m = PC.assert_decode_close(got[sample], c.reference(), c.mu_v(), c.name)
        print(f"{c.name}: rel_l2={e_out:.3e} rel_l2(out-mu_v)={e_att:.3e} max_abs={m:.3e}")
    del store, view
    for lib in libs:
        lib.close()
    torch.cuda.empty_cache()
