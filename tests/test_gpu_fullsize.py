"""Full-size workloads in the launch configuration bench.py times, checked on samples.

The store is allocated at its full size (116 GB for batch 768 x 4096 at ratio
21.3); only the layer under test is filled with seeded latents, since a
decode call reads no other layer.  The default entry point runs (the
tensor-core kernel where it applies) and the oracle recomputes a sample of
sequences, all heads, one by one.
"""

import math

import numpy as np
import pytest

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

torch = pytest.importorskip("torch")
import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
from lla_testutil import assert_close, oracle_decode, rounded_codec  # noqa: E402

DEV = "cuda"


@pytest.mark.parametrize("name,layer,loop,sample", [
    ("ouro_rho21_b768_n4096", 5, 3, [0, 1, 383, 767]),
    ("ouro_rho4_b32_n4096", 23, 0, [0, 17, 31]),
    ("huginn_t32_b16_n32768", 2, 31, [0, 15]),
])
def test_full_size_sampled(name, layer, loop, sample):
    cfg = syn.CONFIGS[name]
    D, T, H, d, rk, rv = cfg["D"], cfg["T"], cfg["H"], cfg["d_head"], cfg["r_k"], cfg["r_v"]
    B, N = cfg["batch"], cfg["context"]
    cap = N + 1
    codec_np = syn.seeded_codec(cfg, f"full/{name}/codec")
    codec = rounded_codec(codec_np)
    lib = lla.Codec(lla.Desc(D, T, H, d, rk, rv, 0, cfg["rope_base"], cap + 1), codec["w_down_k"],
                    codec["w_down_v"], codec["w_up_k"], codec["w_up_v"], codec["mu_k"], codec["mu_v"])
    store = torch.empty(lla.store_bytes(lib.desc, B, cap) // 2, dtype=torch.bfloat16, device=DEV)
    view = store.view(B, D, cap, H, rk + rv)
    g = syn.torch_generator(f"full/{name}/lat", DEV)
    for b0 in range(0, B, 64):
        view[b0:b0 + 64, layer].normal_(generator=g)
    q = torch.empty(B, H, d, device=DEV).normal_(generator=syn.torch_generator(f"full/{name}/q", DEV))
    lens_np = np.full(B, N, np.int32)
    lens_np[sample[-1]] = N - 77  # one ragged sequence in the sample
    lens = torch.from_numpy(lens_np).to(DEV)
    qpos = lens.clone()
    out = torch.empty(B, H, d, device=DEV)
    ws = torch.empty(lib.workspace_bytes(B, cap), dtype=torch.uint8, device=DEV)
    scale = 1 / math.sqrt(d)
    lla.decode_attn(lib, store, B, cap, layer, loop, q, qpos, lens, scale, out, ws)
    torch.cuda.synchronize()
    assert lla.workspace_flags(ws) == 0
    got = out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    idx = torch.tensor(sample, device=DEV)
    lat = view[idx, layer].float().cpu().numpy().astype(np.float64)  # [S, cap, H, rk+rv]
    qs = q[idx].cpu().numpy().astype(np.float64)
    ref = oracle_decode(codec, cfg, lat[..., :rk], lat[..., rk:], qs, layer, loop, lens_np[sample],
                        lens_np[sample], scale)
    assert_close(got[sample], ref, name)
    del store, view
    lib.close()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,layer,loop,sample", [
    ("ouro_2d_b256_n8192", 11, 2, [0, 1, 128, 255]),
    # per-loop MLA at the ratio-21.3 budget: 96 single-loop slots, 116 GB store
    ("mla_perloop_b768_n4096", 57, 0, [0, 300, 767]),
])
def test_full_size_2d_sampled(name, layer, loop, sample):
    """LLA-2D (batch 256 x 8192, 19.3 GB store) and per-loop MLA (T = 1, batch 768 x 4096), one
    layer slot filled, sampled sequences."""
    cfg = syn.CONFIGS[name]
    D, T, H, d, rk, rv = cfg["D"], cfg["T"], cfg["H"], cfg["d_head"], cfg["r_k"], cfg["r_v"]
    B, N = cfg["batch"], cfg["context"]
    cap = N + 1
    codec = rounded_codec(syn.seeded_codec(cfg, f"full/{name}/codec"))
    lib = lla.Codec(lla.Desc(D, T, H, d, rk, rv, 1, cfg["rope_base"], cap + 1), codec["w_down_k"],
                    codec["w_down_v"], codec["w_up_k"], codec["w_up_v"], codec["mu_k"], codec["mu_v"])
    store = torch.empty(lla.store_bytes(lib.desc, B, cap) // 2, dtype=torch.bfloat16, device=DEV)
    view = store.view(B, D, cap, rk + rv)
    view[:, layer].normal_(generator=syn.torch_generator(f"full/{name}/lat", DEV))
    q = torch.empty(B, H, d, device=DEV).normal_(generator=syn.torch_generator(f"full/{name}/q", DEV))
    lens_np = np.full(B, N, np.int32)
    lens_np[sample[-1]] = N - 1000
    lens = torch.from_numpy(lens_np).to(DEV)
    out = torch.empty(B, H, d, device=DEV)
    ws = torch.empty(lib.workspace_bytes(B, cap), dtype=torch.uint8, device=DEV)
    scale = 1 / math.sqrt(d)
    lla.decode_attn_2d(lib, store, B, cap, layer, loop, q, lens, lens, scale, out, ws)
    torch.cuda.synchronize()
    assert lla.workspace_flags(ws) == 0
    got = out.cpu().numpy().astype(np.float64)
    idx = torch.tensor(sample, device=DEV)
    lat = view[idx, layer].float().cpu().numpy().astype(np.float64)  # [S, cap, rk+rv]
    qs = q[idx].cpu().numpy().astype(np.float64)
    ref = oracle_decode(codec, cfg, lat[..., :rk], lat[..., rk:], qs, layer, loop, lens_np[sample],
                        lens_np[sample], scale)
    assert_close(got[sample], ref, name)
    del store, view
    lib.close()
    torch.cuda.empty_cache()
