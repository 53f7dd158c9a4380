"""The allocation-free decode entry point agrees with the workspace one.

lla_decode_attn_noalloc serves callers that may not allocate device memory
(a running serving loop, or a host that owns all device memory): it keeps
its scratch in a fixed array inside the library.  This file is collected
last so a stop at its first failure has already run every other test.
Calls go through the C ABI; outputs are compared with lla_decode_attn's on
the same inputs, on two calls in a row, within the parity tolerance.
"""

import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
from lla_testutil import assert_close, make_lib_codec, rounded_codec, to_bf16_bits  # noqa: E402

DEV = "cuda"


def _case(tag, variant=0):
    c = dict(D=2, T=4, H=16, d_head=128, r_k=16, r_v=32, variant=variant, rope_base=10000.0, mu_var=0.1)
    if variant == 1:
        c.update(H=4, r_k=24, r_v=40)
    codec = rounded_codec(syn.seeded_codec(c, tag))
    lib = make_lib_codec(lla, dict(D=c["D"], T=c["T"], H=c["H"], d_head=c["d_head"], r_k=c["r_k"], r_v=c["r_v"],
                                   variant=variant, rope_base=10000.0, max_pos=1024), codec)
    return c, lib


def _inputs(tag, c, B, N, lens):
    shape = (B, c["D"], N, c["H"], c["r_k"] + c["r_v"]) if c["variant"] == 0 else (B, c["D"], N, c["r_k"] + c["r_v"])
    store = torch.from_numpy(to_bf16_bits(syn.gaussian(tag + "/lat", shape)).view(np.int16)).to(DEV)
    q = torch.from_numpy(syn.gaussian(tag + "/q", (B, c["H"], c["d_head"])).astype(np.float32)).to(DEV)
    ln = torch.tensor(lens, dtype=torch.int32, device=DEV)
    return store, q, ln


@pytest.mark.parametrize("variant", [0, 1])
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(variant):
    c, lib = _case(f"noalloc/{variant}", variant)
    scale = 1 / math.sqrt(c["d_head"])
    calls = [(3, 700, [700, 129, 1], 1, 2), (2, 300, [17, 300], 0, 3)]  # second call is smaller: no stale state
    for i, (B, N, lens, layer, loop) in enumerate(calls):
        store, q, ln = _inputs(f"noalloc/{variant}/{i}", c, B, N, lens)
        ref = torch.empty(B, c["H"], c["d_head"], device=DEV)
        ws = torch.empty(lib.workspace_bytes(B, N), dtype=torch.uint8, device=DEV)
        lla.decode_attn(lib, store, B, N, layer, loop, q, ln, ln, scale, ref, ws)
        got = torch.full_like(ref, float("nan"))
        lla.decode_attn_noalloc(lib, store, B, N, layer, loop, q, ln, ln, scale, got)
        torch.cuda.synchronize()
        assert_close(got.cpu().numpy(), ref.cpu().numpy(), f"call {i}")
    lib.close()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    c, lib = _case("noalloc/big")
    B, N = 8, 64
    store, q, ln = _inputs("noalloc/big", c, B, N, [N] * B)
    out = torch.empty(B, c["H"], c["d_head"], device=DEV)
    with pytest.raises(lla.LLAError) as e:
        # a batch whose split records alone exceed the fixed scratch; rejected before any launch
        lla.decode_attn_noalloc(lib, store, 100000, N, 0, 0, q, ln, ln, 1.0, out)
    assert e.value.status == 6
    lib.close()
