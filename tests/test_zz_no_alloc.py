"""The allocation-free decode entry point agrees with the workspace one and with the oracle.

lla_decode_attn_noalloc serves callers that may not allocate device memory
(a running serving loop, or a host that owns all device memory): it keeps
its scratch in a fixed array inside the library.  This file is collected
last so a stop at its first failure has already run every other test.
Calls go through the C ABI; outputs are compared with lla_decode_attn's on
the same inputs, on two calls in a row, within the parity tolerance, and
with the FP64 oracle (queries aimed at a few cached keys).  The size limit
is checked at its edge: the call runs at its automatic split count, so a
shape fits when that split count's records do, even where the workspace of
lla_decode_attn would reserve room for more splits than the array holds.
"""

import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
import parity_cases as PC  # noqa: E402
from lla_testutil import assert_close, make_lib_codec, rounded_codec  # noqa: E402

DEV = "cuda"
SCRATCH_BYTES = 8 << 20
HEADER_BYTES = 256


def _dev(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device=DEV, dtype=dtype)


@pytest.mark.parametrize("variant", [0, 1])
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(variant):
    lib = None
    for i, (B, N, lens, layer, loop) in enumerate(PC.NOALLOC_CALLS):  # second call smaller: no stale state
        s = PC.noalloc_set(variant, i)
        if lib is None:  # one codec for both calls
            lib = make_lib_codec(lla, s.desc_kw(1024), s.codec)
        case = s.case(layer, loop)
        store = _dev(s.bits.view(np.int16), torch.int16)
        q = _dev(case.q, torch.float32)
        ln = torch.tensor(lens, dtype=torch.int32, device=DEV)
        ref = torch.empty(B, s.cfg["H"], s.cfg["d_head"], device=DEV)
        ws = torch.empty(lib.workspace_bytes(B, N), dtype=torch.uint8, device=DEV)
        lla.decode_attn(lib, store, B, N, layer, loop, q, ln, ln, case.scale, ref, ws)
        got = torch.full_like(ref, float("nan"))
        lla.decode_attn_noalloc(lib, store, B, N, layer, loop, q, ln, ln, case.scale, got)
        torch.cuda.synchronize()
        got = got.cpu().numpy().astype(np.float64)
        assert_close(got, ref.cpu().numpy(), f"call {i} vs lla_decode_attn")
        PC.assert_decode_close(got, case.reference(), case.mu_v(), f"call {i} vs oracle")
    lib.close()


def _ratio21_codec(tag):
    c = dict(D=1, T=4, H=16, d_head=128, r_k=16, r_v=32, variant=0, rope_base=10000.0, mu_var=0.1)
    codec = rounded_codec(syn.seeded_codec(c, tag))
    return c, make_lib_codec(lla, dict(D=1, T=4, H=16, d_head=128, r_k=16, r_v=32, variant=0, rope_base=10000.0,
                                       max_pos=2048), codec)


def _auto_scratch_bytes(B, N, H=16, r_v=32):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    splits = max(1, min(-(-4 * sms // (B * H)), -(-N // 128)))
    return HEADER_BYTES + B * splits * H * (r_v + 2) * 4


@pytest.mark.parametrize("B,N", [(512, 1024), (3854, 128)])
def test_noalloc_accepts_shapes_whose_automatic_splits_fit(B, N):
    """(512, 1024): one automatic split (1.1 MB of records), where room for 8 splits would need
    8.9 MB.  (3854, 128): the largest batch whose records fit the 8 MiB array at H 16, r_v 32."""
    c, lib = _ratio21_codec("noalloc/edge")
    assert _auto_scratch_bytes(B, N) <= SCRATCH_BYTES
    g = syn.torch_generator(f"noalloc/edge/{B}", DEV)
    store = torch.empty(lla.store_bytes(lib.desc, B, N) // 2, dtype=torch.bfloat16, device=DEV).normal_(generator=g)
    q = torch.empty(B, 16, 128, device=DEV).normal_(generator=g) * 8.0
    ln = torch.randint(0, N + 1, (B,), dtype=torch.int32, device=DEV, generator=g)
    scale = 1 / math.sqrt(128)
    ref = torch.empty(B, 16, 128, device=DEV)
    ws = torch.empty(lib.workspace_bytes(B, N), dtype=torch.uint8, device=DEV)
    lla.decode_attn(lib, store, B, N, 0, 1, q, ln, ln, scale, ref, ws)
    for _ in range(2):
        got = torch.full_like(ref, float("nan"))
        lla.decode_attn_noalloc(lib, store, B, N, 0, 1, q, ln, ln, scale, got)
        torch.cuda.synchronize()
        assert_close(got.cpu().numpy(), ref.cpu().numpy(), f"batch {B} x {N}")
    lib.close()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    c, lib = _ratio21_codec("noalloc/big")
    B, N = 8, 64
    buf = torch.zeros(1 << 20, dtype=torch.uint8, device=DEV)
    p = buf.data_ptr()
    # one sequence past the largest batch that fits (its records alone exceed the array), and a
    # batch far beyond it; both rejected before any launch
    for batch in (3855, 100000):
        assert _auto_scratch_bytes(batch, 1024) > SCRATCH_BYTES
        with pytest.raises(lla.LLAError) as e:
            lla.decode_attn_noalloc(lib, p, batch, 1024, 0, 0, p, p, p, 1.0, p)
        assert e.value.status == 6
    lib.close()
