"""Host-side checks of the C ABI that need no GPU: symbols, sizes, validation."""

import ctypes
import os
import re

import pytest

import __graft_entry__

__graft_entry__._build_module().build()

import decode_attention_lla_b200 as lla  # noqa: E402
import lla_synth as syn  # noqa: E402
from oracle import lla_oracle as O  # noqa: E402

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "lla.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lla_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_function():
    lib = ctypes.CDLL(lla.LIB_PATH)
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"{n} declared in lla.h but not exported"
    assert sorted(lla.EXPORTED) == names


def test_status_strings_and_version():
    assert lla.version().startswith("lla-b200")
    for s in range(7):
        assert lla.status_string(s)
    assert lla.status_string(99) == "unknown status"


@pytest.mark.parametrize("name", sorted(syn.CONFIGS))
def test_store_bytes_matches_the_ratio(name):
    cfg = syn.CONFIGS[name]
    desc = lla.Desc(cfg["D"], cfg["T"], cfg["H"], cfg["d_head"], cfg["r_k"], cfg["r_v"], cfg["variant"],
                    cfg["rope_base"], cfg["context"] + 1)
    got = lla.store_bytes(desc, cfg["batch"], cfg["context"])
    assert got == O.store_bytes(cfg["batch"], cfg["context"], cfg["D"], cfg["H"], cfg["r_k"], cfg["r_v"],
                                cfg["variant"])


def test_store_bytes_printed_figures():
    d = lla.Desc(24, 4, 16, 128, 16, 32, 0, 10000.0, 4097)
    assert lla.store_bytes(d, 1, 1 << 20) == 36 << 30
    assert lla.store_bytes(d, 768, 4096) == 108 << 30


@pytest.mark.parametrize("bad", [dict(D=0), dict(T=0), dict(d_head=3), dict(r_k=0), dict(r_v=10**6),
                                 dict(variant=2), dict(rope_base=1.0), dict(max_pos=0)])
def test_invalid_descriptions_are_rejected(bad):
    kw = dict(D=2, T=4, H=2, d_head=16, r_k=4, r_v=8, variant=0, rope_base=10000.0, max_pos=64)
    kw.update(bad)
    assert lla.store_bytes(lla.Desc(**kw), 1, 10) == 0


def test_null_and_out_of_range_arguments_return_status():
    # null codec: rejected before any CUDA call
    args = [None, None, 1, 16, 0, 0, None, None, None, 1.0, None, None, 0, None]
    assert lla.raw_decode_status("lla_decode_attn", *args) == 1
    assert lla.raw_decode_status("lla_decode_attn_2d", *args) == 1
    assert lla._ws_bytes(None, 1, 1) == 0
    assert lla._encode(None, None, 1, 0, 1, None, None, None, 1, 1, None) == 1
    assert lla._destroy(None) == 0
    assert lla._flags(None, None, None) == 1


def test_codec_shape_mismatch_is_caught_before_the_abi():
    d = lla.Desc(1, 2, 1, 4, 2, 2)
    z = lambda *s: __import__("numpy").zeros(s)  # noqa: E731
    with pytest.raises(ValueError):
        lla.Codec(d, z(1, 1, 8, 3), z(1, 1, 8, 2), z(1, 1, 2, 4, 2), z(1, 1, 2, 4, 2), z(1, 1, 8), z(1, 1, 8))


def test_fit_workspace_size_rules():
    """lla_fit_codec_workspace_bytes: zero for what lla_fit_codec rejects, else enough for the
    fp64 Gram (m x m, m = min(n, S)) and the subspace blocks of every problem."""
    assert lla.fit_codec_workspace_bytes(1, 10, 8, 9) == 0        # r > min(n, S)
    assert lla.fit_codec_workspace_bytes(1, 4096, 4096, 600) == 0  # block of 1200 > 1024 columns
    assert lla.fit_codec_workspace_bytes(0, 512, 512, 16) == 0
    assert lla.fit_codec_workspace_bytes(65536, 64, 64, 4) == 0  # problems index a grid dimension
    one = lla.fit_codec_workspace_bytes(1, 1024, 512, 96)
    assert one >= 512 * 512 * 8 + 2 * 512 * 192 * 8
    assert lla.fit_codec_workspace_bytes(3, 1024, 512, 96) > 2 * one
    # n < S uses the n x n Gram
    assert lla.fit_codec_workspace_bytes(1, 200, 4096, 40) < lla.fit_codec_workspace_bytes(1, 4096, 4096, 40)
