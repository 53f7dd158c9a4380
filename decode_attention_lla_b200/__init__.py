"""Python binding of the B200 LLA library (liblla_b200.so), argument marshalling only.

Every function mirrors one entry point of ``include/lla.h``.  Tensors are
torch tensors on the current CUDA device (torch provides device memory and
the stream); their data pointers are passed straight to the C ABI, and every
step of the computation runs in the library's CUDA kernels.  There is no
fallback: if the shared library is missing or a call fails, an exception is
raised.

Looped Latent Attention: "Looped Latent Attention: Cross-Loop KV Compression
for Looped Transformers" (arXiv 2607.15456).
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblla_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python decode_attention_lla_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

LLA_OK = 0
STATUS_NAMES = {0: "LLA_OK", 1: "LLA_ERR_INVALID_ARG", 2: "LLA_ERR_UNSUPPORTED_SHAPE", 3: "LLA_ERR_ALIGNMENT",
                4: "LLA_ERR_CUDA", 5: "LLA_ERR_OOM", 6: "LLA_ERR_WORKSPACE"}
FLAG_SEQ_LEN_CLAMPED = 1
FLAG_POS_CLAMPED = 2
IMPL_AUTO, IMPL_SIMT, IMPL_TC = 0, 1, 2


class CodecDesc(ctypes.Structure):
    _fields_ = [("D", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("d_head", ctypes.c_int),
                ("r_k", ctypes.c_int), ("r_v", ctypes.c_int), ("variant", ctypes.c_int),
                ("rope_base", ctypes.c_float), ("max_pos", ctypes.c_int)]


class DecodeOpts(ctypes.Structure):
    _fields_ = [("impl", ctypes.c_int), ("num_ctas", ctypes.c_int), ("ev_begin", ctypes.c_void_p),
                ("ev_end", ctypes.c_void_p)]


_vp, _sz, _i, _f = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float


def _sig(name, res, args):
    fn = getattr(_lib, name)
    fn.restype = res
    fn.argtypes = args
    return fn


_status_string = _sig("lla_status_string", ctypes.c_char_p, [_i])
_version = _sig("lla_version", ctypes.c_char_p, [])
_create = _sig("lla_create_codec", _i, [ctypes.POINTER(_vp), ctypes.POINTER(CodecDesc)] + [_vp] * 6 + [_vp])
_destroy = _sig("lla_destroy_codec", _i, [_vp])
_get_desc = _sig("lla_codec_get_desc", _i, [_vp, ctypes.POINTER(CodecDesc)])
_store_bytes = _sig("lla_store_bytes", _sz, [ctypes.POINTER(CodecDesc), _i, _i])
_encode = _sig("lla_encode", _i, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _i, _i, _vp])
_ws_bytes = _sig("lla_decode_workspace_bytes", _sz, [_vp, _i, _i])
_decode_args = [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _f, _vp, _vp, _sz]
_decode = _sig("lla_decode_attn", _i, _decode_args + [_vp])
_decode_2d = _sig("lla_decode_attn_2d", _i, _decode_args + [_vp])
_decode_ex = _sig("lla_decode_attn_ex", _i, _decode_args + [ctypes.POINTER(DecodeOpts), _vp])
_flags = _sig("lla_workspace_flags", _i, [_vp, ctypes.POINTER(ctypes.c_uint32), _vp])
_decode_noalloc = _sig("lla_decode_attn_noalloc", _i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _f, _vp, _vp])
_paged_bytes = _sig("lla_paged_store_bytes", _sz, [ctypes.POINTER(CodecDesc), _i])
_encode_paged = _sig("lla_encode_paged", _i, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _i, _vp, _i, _i, _vp])
_decode_paged = _sig("lla_decode_attn_paged", _i, [_vp, _vp, _i, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _f,
                                                   _vp, _vp, _sz, ctypes.POINTER(DecodeOpts), _vp])
_full_ws = _sig("lla_full_decode_workspace_bytes", _sz, [_i, _i, _i])
_full_decode = _sig("lla_full_decode_attn", _i, [_i, _i, _f, _vp, _vp, ctypes.c_longlong, _i, _i, _vp, _vp, _vp, _f,
                                                 _vp, _vp, _sz, _i, _vp])
_fit_ws = _sig("lla_fit_codec_workspace_bytes", _sz, [_i, _i, _i, _i])
_fit = _sig("lla_fit_codec", _i, [_i, _i, _i, _i, _vp, _vp, _vp, _vp, _i, _vp, _sz, _vp])
_reconstruct = _sig("lla_reconstruct_cache", _i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, ctypes.c_longlong, _i, _i,
                                                  _vp])
_decode_self = _sig("lla_decode_attn_self", _i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _sz,
                                                 ctypes.POINTER(DecodeOpts), _vp])

EXPORTED = ["lla_status_string", "lla_version", "lla_create_codec", "lla_destroy_codec", "lla_codec_get_desc",
            "lla_store_bytes", "lla_encode", "lla_decode_workspace_bytes", "lla_decode_attn",
            "lla_decode_attn_2d", "lla_decode_attn_ex", "lla_workspace_flags", "lla_decode_attn_noalloc",
            "lla_decode_attn_self", "lla_paged_store_bytes", "lla_encode_paged", "lla_decode_attn_paged",
            "lla_full_decode_workspace_bytes", "lla_full_decode_attn", "lla_fit_codec_workspace_bytes",
            "lla_fit_codec", "lla_reconstruct_cache"]
PAGE_TOKENS = 128
FLAG_PAGE_INVALID = 4
FLAG_FIT_BREAKDOWN = 8


class LLAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


def status_string(status: int) -> str:
    return _status_string(int(status)).decode()


def version() -> str:
    return _version().decode()


def _check(status: int, where: str):
    if status != LLA_OK:
        raise LLAError(status, where)


def _ptr(x) -> int | None:
    """Device/host address of a torch tensor, a NumPy array, or a raw integer pointer."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)}")


def _stream(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


@dataclass
class Desc:
    D: int
    T: int
    H: int
    d_head: int
    r_k: int
    r_v: int
    variant: int = 0
    rope_base: float = 10000.0
    max_pos: int = 8192

    def c(self) -> CodecDesc:
        return CodecDesc(self.D, self.T, self.H, self.d_head, self.r_k, self.r_v, self.variant,
                         float(self.rope_base), self.max_pos)


def store_bytes(desc: Desc, batch: int, max_tokens: int) -> int:
    return int(_store_bytes(ctypes.byref(desc.c()), batch, max_tokens))


class Codec:
    """Device-resident codec (owns its device copies; `close()` frees them)."""

    def __init__(self, desc: Desc, w_down_k, w_down_v, w_up_k, w_up_v, mu_k, mu_v, stream=None):
        self.desc = desc
        arrs = [np.ascontiguousarray(a, dtype=np.float32) for a in (w_down_k, w_down_v, w_up_k, w_up_v, mu_k, mu_v)]
        S = desc.T * desc.d_head * (desc.H if desc.variant == 1 else 1)
        lead = (desc.D,) if desc.variant == 1 else (desc.D, desc.H)
        ups = (desc.D, desc.T, desc.H) if desc.variant == 1 else (desc.D, desc.H, desc.T)
        want = [lead + (S, desc.r_k), lead + (S, desc.r_v), ups + (desc.d_head, desc.r_k),
                ups + (desc.d_head, desc.r_v), lead + (S,), lead + (S,)]
        for a, w, nm in zip(arrs, want, ("w_down_k", "w_down_v", "w_up_k", "w_up_v", "mu_k", "mu_v")):
            if a.shape != w:
                raise ValueError(f"{nm}: expected shape {w}, got {a.shape}")
        h = _vp()
        _check(_create(ctypes.byref(h), ctypes.byref(desc.c()), *[a.ctypes.data for a in arrs], _stream(stream)),
               "lla_create_codec")
        self._h = h
        self._keep = arrs  # alive until the synchronous copy is done (it is, on return)

    @property
    def handle(self) -> int:
        if self._h is None or not self._h.value:
            raise RuntimeError("codec is closed")
        return self._h.value

    def get_desc(self) -> Desc:
        out = CodecDesc()
        _check(_get_desc(self.handle, ctypes.byref(out)), "lla_codec_get_desc")
        return Desc(out.D, out.T, out.H, out.d_head, out.r_k, out.r_v, out.variant, out.rope_base, out.max_pos)

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            _check(_destroy(self._h), "lla_destroy_codec")
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_bytes(self, batch: int, max_tokens: int) -> int:
        return int(_ws_bytes(self.handle, batch, max_tokens))


def encode(codec: Codec, x, n: int, layer_begin: int, num_layers: int, seq_idx, tok_idx, store, batch: int,
           max_tokens: int, stream=None):
    _check(_encode(codec.handle, _ptr(x), n, layer_begin, num_layers, _ptr(seq_idx), _ptr(tok_idx), _ptr(store),
                   batch, max_tokens, _stream(stream)), "lla_encode")


def decode_workspace_bytes(codec: Codec, batch: int, max_tokens: int) -> int:
    return codec.workspace_bytes(batch, max_tokens)


def _decode_call(fn, codec, store, batch, max_tokens, layer, loop, q, q_pos, seq_lens, scale, out, workspace,
                 workspace_bytes, stream, opts=None):
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    args = [codec.handle, _ptr(store), batch, max_tokens, layer, loop, _ptr(q), _ptr(q_pos), _ptr(seq_lens),
            float(scale), _ptr(out), _ptr(workspace), int(workspace_bytes)]
    if opts is not None:
        args.append(ctypes.byref(opts))
    args.append(_stream(stream))
    return fn(*args)


def decode_attn(codec, store, batch, max_tokens, layer, loop, q, q_pos, seq_lens, scale, out, workspace,
                workspace_bytes=None, stream=None, impl=IMPL_AUTO, num_ctas=0, events=None):
    """lla_decode_attn; impl / num_ctas / events (a pair of raw cudaEvent_t handles) go through
    lla_decode_attn_ex."""
    if impl == IMPL_AUTO and num_ctas == 0 and events is None:
        fn = _decode_2d if codec.desc.variant == 1 else _decode
        st = _decode_call(fn, codec, store, batch, max_tokens, layer, loop, q, q_pos, seq_lens, scale, out,
                          workspace, workspace_bytes, stream)
    else:
        st = _decode_call(_decode_ex, codec, store, batch, max_tokens, layer, loop, q, q_pos, seq_lens, scale, out,
                          workspace, workspace_bytes, stream,
                          DecodeOpts(impl, num_ctas, *(events if events is not None else (None, None))))
    _check(st, "lla_decode_attn")


def decode_attn_2d(codec, store, batch, max_tokens, layer, loop, q, q_pos, seq_lens, scale, out, workspace,
                   workspace_bytes=None, stream=None):
    _check(_decode_call(_decode_2d, codec, store, batch, max_tokens, layer, loop, q, q_pos, seq_lens, scale, out,
                        workspace, workspace_bytes, stream), "lla_decode_attn_2d")


def decode_attn_self(codec, store, batch, max_tokens, layer, loop, q, q_pos, seq_lens, k_self, v_self, scale, out,
                     workspace, workspace_bytes=None, stream=None, impl=IMPL_AUTO, num_ctas=0, events=None):
    """lla_decode_attn_self: decode attention with the current token's exact loop-t key and value
    (k_self, v_self [batch][H][d_head] float32) as one more softmax slot; either codec variant."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    opts = DecodeOpts(impl, num_ctas, *(events if events is not None else (None, None)))
    st = _decode_self(codec.handle, _ptr(store), batch, max_tokens, layer, loop, _ptr(q), _ptr(q_pos),
                      _ptr(seq_lens), _ptr(k_self), _ptr(v_self), float(scale), _ptr(out), _ptr(workspace),
                      int(workspace_bytes), ctypes.byref(opts), _stream(stream))
    _check(st, "lla_decode_attn_self")


def paged_store_bytes(desc: Desc, num_pages: int) -> int:
    return int(_paged_bytes(ctypes.byref(desc.c()), num_pages))


def encode_paged(codec, x, n, layer_begin, num_layers, seq_idx, tok_idx, pool, num_pages, block_table, max_pages,
                 batch, stream=None):
    """lla_encode_paged: write latents into a paged store (pages of PAGE_TOKENS tokens)."""
    _check(_encode_paged(codec.handle, _ptr(x), n, layer_begin, num_layers, _ptr(seq_idx), _ptr(tok_idx), _ptr(pool),
                         num_pages, _ptr(block_table), max_pages, batch, _stream(stream)), "lla_encode_paged")


def decode_attn_paged(codec, pool, num_pages, block_table, max_pages, batch, layer, loop, q, q_pos, seq_lens, scale,
                      out, workspace, k_self=None, v_self=None, workspace_bytes=None, stream=None, impl=IMPL_AUTO,
                      num_ctas=0, events=None):
    """lla_decode_attn_paged: decode attention over a paged store, optional self slot."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    opts = DecodeOpts(impl, num_ctas, *(events if events is not None else (None, None)))
    st = _decode_paged(codec.handle, _ptr(pool), num_pages, _ptr(block_table), max_pages, batch, layer, loop, _ptr(q),
                       _ptr(q_pos), _ptr(seq_lens), _ptr(k_self), _ptr(v_self), float(scale), _ptr(out),
                       _ptr(workspace), int(workspace_bytes), ctypes.byref(opts), _stream(stream))
    _check(st, "lla_decode_attn_paged")


def full_decode_workspace_bytes(H: int, d_head: int, batch: int) -> int:
    return int(_full_ws(H, d_head, batch))


def full_decode_attn(H, d_head, rope_base, k_cache, v_cache, seq_stride, batch, max_tokens, q, q_pos, seq_lens, scale,
                     out, workspace, workspace_bytes=None, num_ctas=0, stream=None):
    """lla_full_decode_attn: the full-cache comparator (keys cached rotated; d_head 128)."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(_full_decode(H, d_head, float(rope_base), _ptr(k_cache), _ptr(v_cache), int(seq_stride), batch, max_tokens,
                        _ptr(q), _ptr(q_pos), _ptr(seq_lens), float(scale), _ptr(out), _ptr(workspace),
                        int(workspace_bytes), num_ctas, _stream(stream)), "lla_full_decode_attn")


def reconstruct_cache(codec, store, batch, max_tokens, layer, loop, seq_lens, k_cache, v_cache, seq_stride,
                      cache_tokens, impl=IMPL_AUTO, stream=None):
    """lla_reconstruct_cache: one (layer, loop) slice of the full K/V cache (keys rotated) rebuilt from
    the latent store, in the layout full_decode_attn reads."""
    _check(_reconstruct(codec.handle, _ptr(store), batch, max_tokens, layer, loop, _ptr(seq_lens), _ptr(k_cache),
                        _ptr(v_cache), int(seq_stride), cache_tokens, impl, _stream(stream)), "lla_reconstruct_cache")


def fit_codec_workspace_bytes(problems: int, n: int, S: int, r: int) -> int:
    return int(_fit_ws(problems, n, S, r))


def fit_codec(problems, n, S, r, X, mu, w_down, sigma, workspace, iters=0, workspace_bytes=None, stream=None):
    """lla_fit_codec: mu, W_down (top-r right singular vectors of the centred stacks) and the top
    singular values of `problems` calibration sets X [problems][n][S] (device float32)."""
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(_fit(problems, n, S, r, _ptr(X), _ptr(mu), _ptr(w_down), _ptr(sigma) if sigma is not None else None,
                iters, _ptr(workspace), int(workspace_bytes), _stream(stream)), "lla_fit_codec")


def raw_decode_status(fn_name, *args) -> int:
    """Call a decode entry point with raw arguments and return its status (for ABI tests)."""
    return {"lla_decode_attn": _decode, "lla_decode_attn_2d": _decode_2d, "lla_decode_attn_ex": _decode_ex,
            "lla_decode_attn_self": _decode_self, "lla_decode_attn_paged": _decode_paged}[fn_name](*args)


def workspace_flags(workspace, stream=None) -> int:
    f = ctypes.c_uint32(0)
    _check(_flags(_ptr(workspace), ctypes.byref(f), _stream(stream)), "lla_workspace_flags")
    return int(f.value)


def decode_attn_noalloc(codec, store, batch, max_tokens, layer, loop, q, q_pos, seq_lens, scale, out, stream=None):
    """lla_decode_attn_noalloc: decode without a caller workspace, for hosts that cannot allocate.

    The library keeps the scratch in a fixed 8 MiB device array shared by all
    calls on a device; calls that overlap on the GPU race on it.
    """
    _check(_decode_noalloc(codec.handle, _ptr(store), batch, max_tokens, layer, loop, _ptr(q), _ptr(q_pos),
                           _ptr(seq_lens), float(scale), _ptr(out), _stream(stream)), "lla_decode_attn_noalloc")
