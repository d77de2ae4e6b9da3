"""ctypes binding of libkvq.so: the C ABI of include/kvq.h under the same names.

Argument marshalling only: every step of quantisation and attention runs in
the library's CUDA kernels.  Pointers may be passed as ints or as torch
tensors (their data_ptr() is used); streams as ints, torch.cuda.Stream or
None (the current torch stream when torch is loaded, else the default
stream).  Nothing here computes a result on the host.

If the shared library is missing this module raises ImportError; build it
with ``python -m kv_cache_quantization_03_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkvq.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError("libkvq.so is not built (run: python -m kv_cache_quantization_03_b200.build)")
lib = ctypes.CDLL(_LIB_PATH)

# ---- enums and constants (include/kvq.h)
KVQ_OK = 0
KVQ_ERR_INVALID_ARG = 1
KVQ_ERR_UNSUPPORTED = 2
KVQ_ERR_WORKSPACE_TOO_SMALL = 3
KVQ_ERR_PARTIAL_TILE = 4
KVQ_ERR_BAD_PAGE = 5
KVQ_ERR_TIMEOUT = 6
KVQ_ERR_CUDA = 7

KVQ_DEVERR_BAD_PAGE = 0x1
KVQ_DEVERR_PARTIAL_TILE = 0x2
KVQ_DEVERR_TIMEOUT = 0x4
KVQ_DEVERR_BAD_SEQ = 0x8

KVQ_F16, KVQ_BF16, KVQ_F32 = 0, 1, 2

EXPORTED = (
    "kvq_config_from_string", "kvq_cache_layout", "kvq_quantize_append", "kvq_dequantize",
    "kvq_decode_workspace_bytes", "kvq_decode_attention", "kvq_decode_attention_tail", "kvq_decode_attention_fill",
    "kvq_decode_attention_noalloc", "kvq_read_error", "kvq_set_test_wait",
    "kvq_status_string", "kvq_version",
)


class kvq_config(ctypes.Structure):
    _fields_ = [
        ("head_dim", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("tile_tokens", ctypes.c_int32),
        ("bits_k", ctypes.c_int32), ("bits_v", ctypes.c_int32), ("sinkhorn_iters", ctypes.c_int32),
        ("hadamard_block", ctypes.c_int32), ("mla", ctypes.c_int32), ("rope_dim", ctypes.c_int32),
        ("num_layers", ctypes.c_int32), ("num_pages", ctypes.c_int64), ("in_dtype", ctypes.c_int),
        ("meta_f16", ctypes.c_int32), ("k_per_channel", ctypes.c_int32),
    ]


class kvq_cache_view(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("k_codes", "k_tok_scale", "k_chan_scale", "v_codes", "v_tok_scale", "v_chan_scale", "rope")]


_P = ctypes.c_void_p
_cfgp = ctypes.POINTER(kvq_config)
_viewp = ctypes.POINTER(kvq_cache_view)
_sig = {
    "kvq_config_from_string": (ctypes.c_int, [ctypes.c_char_p, _cfgp]),
    "kvq_cache_layout": (ctypes.c_int, [_cfgp, ctypes.POINTER(ctypes.c_size_t)]),
    "kvq_quantize_append": (ctypes.c_int, [_cfgp, _viewp, _P, _P, _P, ctypes.c_int64, _P, _P, _P]),
    "kvq_dequantize": (ctypes.c_int, [_cfgp, _viewp, ctypes.c_int32, _P, ctypes.c_int64, ctypes.c_int32,
                                      _P, _P, _P, _P]),
    "kvq_decode_workspace_bytes": (ctypes.c_int, [_cfgp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                  ctypes.POINTER(ctypes.c_size_t)]),
    "kvq_decode_attention": (ctypes.c_int, [_cfgp, _viewp, ctypes.c_int32, _P, _P, ctypes.c_int32, _P,
                                            ctypes.c_int32, ctypes.c_int32, ctypes.c_float, _P, _P,
                                            ctypes.c_size_t, _P, _P]),
    "kvq_decode_attention_tail": (ctypes.c_int, [_cfgp, _viewp, ctypes.c_int32, _P, _P, ctypes.c_int32, _P,
                                                 _P, _P, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_float, _P,
                                                 _P, ctypes.c_size_t, _P, _P]),
    "kvq_decode_attention_fill": (ctypes.c_int, [_cfgp, _viewp, ctypes.c_int32, _P, _P, ctypes.c_int32, _P,
                                                 _P, _P, _P, _P, ctypes.c_int32, ctypes.c_int32, ctypes.c_float, _P,
                                                 _P, ctypes.c_size_t, _P, _P]),
    "kvq_decode_attention_noalloc": (ctypes.c_int, [_cfgp, _viewp, ctypes.c_int32, _P, _P, ctypes.c_int32, _P,
                                                    ctypes.c_int32, ctypes.c_int32, ctypes.c_float, _P, _P, _P]),
    "kvq_read_error": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_uint32), _P]),
    "kvq_set_test_wait": (None, [ctypes.c_uint32]),
    "kvq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kvq_version": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class KvqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__("%s failed: %s" % (fn, lib.kvq_status_string(status).decode()))


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except ImportError:  # pragma: no cover
            pass
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn: str, st: int, raise_on_error: bool) -> int:
    if st != KVQ_OK and raise_on_error:
        raise KvqError(fn, st)
    return st


def status_string(status: int) -> str:
    return lib.kvq_status_string(status).decode()


def kvq_version() -> str:
    return lib.kvq_version().decode()


def make_config(head_dim=128, num_kv_heads=1, tile_tokens=16, bits_k=4, bits_v=4, sinkhorn_iters=4,
                mla=False, rope_dim=0, num_layers=1, num_pages=0, in_dtype="bf16",
                hadamard_block=None, meta_f16=False, k_per_channel=False) -> kvq_config:
    return kvq_config(head_dim, num_kv_heads, tile_tokens, bits_k, bits_v, sinkhorn_iters,
                      head_dim if hadamard_block is None else hadamard_block, int(bool(mla)), rope_dim,
                      num_layers, num_pages, {"fp16": KVQ_F16, "bf16": KVQ_BF16}.get(in_dtype, in_dtype),
                      int(bool(meta_f16)), int(bool(k_per_channel)))


def make_view(ptrs: Sequence) -> kvq_cache_view:
    return kvq_cache_view(*[_ptr(p) for p in ptrs])


def kvq_config_from_string(name: str, cfg: kvq_config, raise_on_error=True) -> int:
    return _check("kvq_config_from_string", lib.kvq_config_from_string(name.encode(), ctypes.byref(cfg)),
                  raise_on_error)


def kvq_cache_layout(cfg: kvq_config):
    out = (ctypes.c_size_t * 7)()
    _check("kvq_cache_layout", lib.kvq_cache_layout(ctypes.byref(cfg), out), True)
    return list(out)


def kvq_quantize_append(cfg, view, k_new, v_new, rope_new, n_tok, dst_page, dev_error, stream=None,
                        raise_on_error=True) -> int:
    st = lib.kvq_quantize_append(ctypes.byref(cfg), ctypes.byref(view), _ptr(k_new), _ptr(v_new),
                                 _ptr(rope_new), n_tok, _ptr(dst_page), _ptr(dev_error), _stream(stream))
    return _check("kvq_quantize_append", st, raise_on_error)


def kvq_dequantize(cfg, view, layer, pages, n_pages, unrotate, k_out, v_out, dev_error, stream=None,
                   raise_on_error=True) -> int:
    st = lib.kvq_dequantize(ctypes.byref(cfg), ctypes.byref(view), layer, _ptr(pages), n_pages,
                            int(bool(unrotate)), _ptr(k_out), _ptr(v_out), _ptr(dev_error), _stream(stream))
    return _check("kvq_dequantize", st, raise_on_error)


def kvq_decode_workspace_bytes(cfg, batch, num_q_heads, max_seq_len) -> int:
    n = ctypes.c_size_t(0)
    _check("kvq_decode_workspace_bytes",
           lib.kvq_decode_workspace_bytes(ctypes.byref(cfg), batch, num_q_heads, max_seq_len, ctypes.byref(n)),
           True)
    return n.value


def kvq_decode_attention(cfg, view, layer, q, block_table, max_pages_per_seq, seq_lens, batch, num_q_heads,
                         softmax_scale, out, workspace, workspace_bytes, dev_error, stream=None,
                         raise_on_error=True) -> int:
    st = lib.kvq_decode_attention(ctypes.byref(cfg), ctypes.byref(view), layer, _ptr(q), _ptr(block_table),
                                  max_pages_per_seq, _ptr(seq_lens), batch, num_q_heads, float(softmax_scale),
                                  _ptr(out), _ptr(workspace), workspace_bytes, _ptr(dev_error), _stream(stream))
    return _check("kvq_decode_attention", st, raise_on_error)


def kvq_decode_attention_tail(cfg, view, layer, q, block_table, max_pages_per_seq, seq_lens, k_tail, v_tail,
                              tail_lens, batch, num_q_heads, softmax_scale, out, workspace, workspace_bytes,
                              dev_error, stream=None, raise_on_error=True) -> int:
    st = lib.kvq_decode_attention_tail(ctypes.byref(cfg), ctypes.byref(view), layer, _ptr(q), _ptr(block_table),
                                       max_pages_per_seq, _ptr(seq_lens), _ptr(k_tail), _ptr(v_tail),
                                       _ptr(tail_lens), batch, num_q_heads, float(softmax_scale), _ptr(out),
                                       _ptr(workspace), workspace_bytes, _ptr(dev_error), _stream(stream))
    return _check("kvq_decode_attention_tail", st, raise_on_error)


def kvq_decode_attention_fill(cfg, view, layer, q, block_table, max_pages_per_seq, seq_lens, k_tail, v_tail,
                              tail_lens, fill_page, batch, num_q_heads, softmax_scale, out, workspace,
                              workspace_bytes, dev_error, stream=None, raise_on_error=True) -> int:
    """Quantise this layer's full tails into fill_page (-1: none), then decode with the remaining tails."""
    st = lib.kvq_decode_attention_fill(ctypes.byref(cfg), ctypes.byref(view), layer, _ptr(q), _ptr(block_table),
                                       max_pages_per_seq, _ptr(seq_lens), _ptr(k_tail), _ptr(v_tail),
                                       _ptr(tail_lens), _ptr(fill_page), batch, num_q_heads, float(softmax_scale),
                                       _ptr(out), _ptr(workspace), workspace_bytes, _ptr(dev_error), _stream(stream))
    return _check("kvq_decode_attention_fill", st, raise_on_error)


def kvq_decode_attention_noalloc(cfg, view, layer, q, block_table, max_pages_per_seq, seq_lens, batch,
                                 num_q_heads, softmax_scale, out, dev_error, stream=None, raise_on_error=True) -> int:
    """kvq_decode_attention with the library's fixed scratch array instead of a workspace.

    For callers that cannot allocate device memory when they decode; see
    include/kvq.h for the size limit and the sharing rules."""
    st = lib.kvq_decode_attention_noalloc(ctypes.byref(cfg), ctypes.byref(view), layer, _ptr(q), _ptr(block_table),
                                          max_pages_per_seq, _ptr(seq_lens), batch, num_q_heads,
                                          float(softmax_scale), _ptr(out), _ptr(dev_error), _stream(stream))
    return _check("kvq_decode_attention_noalloc", st, raise_on_error)


def kvq_set_test_wait(ns: int) -> None:
    """Testing hook: later GQA decode calls first wait up to ns nanoseconds on a
    device flag that nothing sets, report a timeout and skip their tiles (0: off)."""
    lib.kvq_set_test_wait(int(ns))


def kvq_read_error(dev_error, stream=None):
    """Returns (status, bits) and clears the device word."""
    bits = ctypes.c_uint32(0)
    st = lib.kvq_read_error(_ptr(dev_error), ctypes.byref(bits), _stream(stream))
    return st, bits.value
