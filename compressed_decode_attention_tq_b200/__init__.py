"""Python binding of the TurboQuant compressed-KV library (include/tq.h).

Argument marshalling only: every step of compression and decode runs in the CUDA
kernels of libtq.so.  PyTorch supplies device memory and streams.  If the shared
library is missing this module raises on import - there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libtq.so")

TQ_OK = 0
TQ_ERR_INVALID_ARG = 1
TQ_ERR_UNSUPPORTED = 2
TQ_ERR_CUDA = 3
TQ_ERR_OVERFLOW = 4
TQ_ERR_TIMEOUT = 5
TQ_ERR_BOUNDS = 6

TQ_DENSITY_BETA = 0
TQ_DENSITY_GAUSS = 1
TQ_ROT_HADAMARD = 0
TQ_ROT_DENSE = 1
TQ_F16 = 0
TQ_F32 = 1

# Every function include/tq.h declares.
EXPORTS = ("tq_version", "tq_status_str", "tq_last_error", "tq_check", "tq_validate_config", "tq_page_bytes",
           "tq_codebook", "tq_compress_kv", "tq_decode_workspace_bytes", "tq_attend_decode",
           "tq_decode_scores", "tq_decompress", "tq_attend_decode_noalloc", "tq_operand_bytes",
           "tq_prepare_operands", "tq_append_kv", "tq_append_attend_decode", "tq_dither_codebook",
           "tq_compress_kv_dithered", "tq_append_kv_dithered", "tq_append_attend_decode_dithered")


class tq_config(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int32), ("key_bits", ctypes.c_int32),
                ("key_qjl", ctypes.c_int32), ("qjl_m", ctypes.c_int32),
                ("value_bits", ctypes.c_int32), ("page_tokens", ctypes.c_int32),
                ("rotation", ctypes.c_int32), ("value_qjl", ctypes.c_int32),
                ("dither", ctypes.c_int32), ("key_corrected_norm", ctypes.c_int32)]


class tq_params(ctypes.Structure):
    _fields_ = [("signs", ctypes.c_void_p), ("pi", ctypes.c_void_p), ("s", ctypes.c_void_p),
                ("k_centroids", ctypes.c_void_p), ("k_boundaries", ctypes.c_void_p),
                ("v_centroids", ctypes.c_void_p), ("v_boundaries", ctypes.c_void_p),
                ("operands", ctypes.c_void_p)]


class tq_cache(ctypes.Structure):
    _fields_ = [("pages", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("num_pages", ctypes.c_int32), ("max_pages", ctypes.c_int32),
                ("batch", ctypes.c_int32), ("kv_heads", ctypes.c_int32),
                ("num_layers", ctypes.c_int32)]


class TQError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {status_str(status)}" + (f" ({detail})" if detail else ""))


# The same library with the kernels' index checks compiled in (built beside libtq.so): a
# failed check records TQ_ERR_BOUNDS in dev_status.
DEBUG_LIB_PATH = os.path.join(PKG, "libtq_debug.so")


def _load(path: Optional[str] = None) -> ctypes.CDLL:
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} not built at {path}; run __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    cfgp, parp, cachep = ctypes.POINTER(tq_config), ctypes.POINTER(tq_params), ctypes.POINTER(tq_cache)
    sig = {
        "tq_version": (I32, []),
        "tq_status_str": (ctypes.c_char_p, [I32]),
        "tq_last_error": (ctypes.c_char_p, []),
        "tq_check": (I32, [ctypes.POINTER(ctypes.c_int32)]),
        "tq_validate_config": (I32, [cfgp]),
        "tq_page_bytes": (SZ, [cfgp]),
        "tq_codebook": (I32, [I32, I32, I32, P, P]),
        "tq_dither_codebook": (I32, [I32, I32, I32, P, P]),
        "tq_compress_kv": (I32, [cfgp, parp, cachep, I32, P, P, I32, I32, P, P, P]),
        "tq_compress_kv_dithered": (I32, [cfgp, parp, cachep, I32, P, P, P, P, I32, I32, P, P, P]),
        "tq_decode_workspace_bytes": (SZ, [cfgp, I32, I32, I32, I32]),
        "tq_attend_decode": (I32, [cfgp, parp, cachep, I32, P, I32, I32, I32, P, I32, P, SZ, P, P, P]),
        "tq_decode_scores": (I32, [cfgp, parp, cachep, I32, P, I32, I32, I32, P, I32, P, SZ, P, P, P]),
        "tq_decompress": (I32, [cfgp, parp, cachep, I32, P, I32, P, P, P, P]),
        "tq_attend_decode_noalloc": (I32, [cfgp, parp, cachep, I32, P, I32, I32, I32, P, I32, P, P, P]),
        "tq_operand_bytes": (SZ, [cfgp]),
        "tq_prepare_operands": (I32, [cfgp, parp, P, P]),
        "tq_append_kv": (I32, [cfgp, parp, cachep, I32, P, P, I32, I32, P, P, P]),
        "tq_append_attend_decode": (I32, [cfgp, parp, cachep, I32, P, P, I32, I32, P, I32, I32, I32, P, I32,
                                          P, SZ, P, P, P]),
        "tq_append_kv_dithered": (I32, [cfgp, parp, cachep, I32, P, P, P, P, I32, I32, P, P, P]),
        "tq_append_attend_decode_dithered": (I32, [cfgp, parp, cachep, I32, P, P, P, P, I32, I32, P, I32, I32,
                                                   I32, P, I32, P, SZ, P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def status_str(st: int) -> str:
    return lib.tq_status_str(st).decode()


def last_error() -> str:
    return lib.tq_last_error().decode()


def check_status(dev_status_value: int) -> int:
    """tq_check on a host copy of a dev_status word: the recorded status code."""
    v = ctypes.c_int32(int(dev_status_value))
    return lib.tq_check(ctypes.byref(v))


def _check(st: int, where: str):
    if st != TQ_OK:
        raise TQError(st, where, last_error())


def make_config(head_dim=128, key_bits=3, key_qjl=True, qjl_m=128, value_bits=3, page_tokens=256,
                rotation=TQ_ROT_HADAMARD, value_qjl=False, dither=False, key_corrected_norm=False) -> tq_config:
    return tq_config(head_dim, key_bits, int(bool(key_qjl)), qjl_m, value_bits, page_tokens, rotation,
                     int(bool(value_qjl)), int(bool(dither)), int(bool(key_corrected_norm)))


def validate_config(cfg: tq_config) -> int:
    return lib.tq_validate_config(ctypes.byref(cfg))


def page_bytes(cfg: tq_config) -> int:
    return lib.tq_page_bytes(ctypes.byref(cfg))


def codebook(bits: int, head_dim: int = 128, density: int = TQ_DENSITY_BETA):
    """Host Lloyd-Max codebook -> (centroids, boundaries) as numpy float32 arrays."""
    import numpy as np
    c = np.zeros(1 << bits, dtype=np.float32)
    b = np.zeros((1 << bits) - 1, dtype=np.float32)
    _check(lib.tq_codebook(bits, head_dim, density, c.ctypes.data, b.ctypes.data), "tq_codebook")
    return c, b


def dither_codebook(bits: int, head_dim: int = 128, density: int = TQ_DENSITY_BETA):
    """Uniform grid of the dithered quantizer -> (centroids, boundaries), numpy float32."""
    import numpy as np
    c = np.zeros(1 << bits, dtype=np.float32)
    b = np.zeros((1 << bits) - 1, dtype=np.float32)
    _check(lib.tq_dither_codebook(bits, head_dim, density, c.ctypes.data, b.ctypes.data), "tq_dither_codebook")
    return c, b


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def make_params(signs=None, pi=None, s=None, k_centroids=None, k_boundaries=None, v_centroids=None,
                v_boundaries=None, operands=None) -> tq_params:
    """Device fp32 tensors -> tq_params (the tensors must outlive every call using it);
    operands: None or a device buffer filled by prepare_operands."""
    return tq_params(_ptr(signs), _ptr(pi), _ptr(s), _ptr(k_centroids), _ptr(k_boundaries),
                     _ptr(v_centroids), _ptr(v_boundaries), _ptr(operands))


def operand_bytes(cfg: tq_config) -> int:
    return lib.tq_operand_bytes(ctypes.byref(cfg))


def prepare_operands(cfg, params, operands, stream=None):
    """Fill operands (device uint8 tensor of operand_bytes(cfg) bytes) for params' signs/s."""
    _check(lib.tq_prepare_operands(ctypes.byref(cfg), ctypes.byref(params), _ptr(operands),
                                   _stream(stream)), "tq_prepare_operands")


def make_cache(pages, block_table, num_pages, max_pages, batch, kv_heads, num_layers=1) -> tq_cache:
    return tq_cache(_ptr(pages), _ptr(block_table), num_pages, max_pages, batch, kv_heads, num_layers)


def dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return TQ_F16
    if t.dtype == torch.float32:
        return TQ_F32
    raise TypeError("inputs must be float16 or float32")


def compress_kv(cfg, params, cache, layer, k, v, seq_lens, status, stream=None):
    """k, v: device [batch][kv_heads][max_len][d] of one dtype; seq_lens: device int32 [batch]."""
    if v.shape != k.shape or v.dtype != k.dtype:
        raise ValueError("k and v must have the same shape and dtype")
    if k.dim() != 4:
        raise ValueError("k and v must be [batch][kv_heads][max_len][d]")
    max_len = k.shape[2]
    _check(lib.tq_compress_kv(ctypes.byref(cfg), ctypes.byref(params), ctypes.byref(cache), layer,
                              _ptr(k), _ptr(v), dtype_code(k), max_len, _ptr(seq_lens), _ptr(status),
                              _stream(stream)), "tq_compress_kv")


def compress_kv_dithered(cfg, params, cache, layer, k, v, k_offsets, v_offsets, seq_lens, status, stream=None):
    """compress_kv for a dithered configuration; k_offsets, v_offsets: device float32
    [batch][kv_heads][max_len], the offset of each vector."""
    if v.shape != k.shape or v.dtype != k.dtype:
        raise ValueError("k and v must have the same shape and dtype")
    if k.dim() != 4:
        raise ValueError("k and v must be [batch][kv_heads][max_len][d]")
    import torch
    for o in (k_offsets, v_offsets):
        if tuple(o.shape) != tuple(k.shape[:3]) or o.dtype != torch.float32 or not o.is_contiguous():
            raise ValueError("offsets must be contiguous float32 [batch][kv_heads][max_len]")
    _check(lib.tq_compress_kv_dithered(ctypes.byref(cfg), ctypes.byref(params), ctypes.byref(cache), layer,
                                       _ptr(k), _ptr(v), _ptr(k_offsets), _ptr(v_offsets), dtype_code(k),
                                       k.shape[2], _ptr(seq_lens), _ptr(status), _stream(stream)),
           "tq_compress_kv_dithered")


def decode_workspace_bytes(cfg, batch, q_heads, seq_q, n_splits) -> int:
    return lib.tq_decode_workspace_bytes(ctypes.byref(cfg), batch, q_heads, seq_q, n_splits)


def attend_decode(cfg, params, cache, layer, q, seq_lens, n_splits, workspace, out, status,
                  stream=None):
    """q: device [batch][q_heads][seq_q][d]; out: device float32, same shape."""
    _check(lib.tq_attend_decode(ctypes.byref(cfg), ctypes.byref(params), ctypes.byref(cache), layer,
                                _ptr(q), dtype_code(q), q.shape[1], q.shape[2], _ptr(seq_lens),
                                n_splits, _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _ptr(out), _ptr(status), _stream(stream)), "tq_attend_decode")


def attend_decode_noalloc(cfg, params, cache, layer, q, seq_lens, n_splits, out, status,
                          stream=None):
    """tq_attend_decode without a workspace: the library's built-in 8 MiB device array is
    used instead, for callers that cannot allocate device memory (see include/tq.h)."""
    _check(lib.tq_attend_decode_noalloc(ctypes.byref(cfg), ctypes.byref(params), ctypes.byref(cache),
                                        layer, _ptr(q), dtype_code(q), q.shape[1], q.shape[2],
                                        _ptr(seq_lens), n_splits, _ptr(out), _ptr(status),
                                        _stream(stream)), "tq_attend_decode_noalloc")


def append_kv(cfg, params, cache, layer, k_new, v_new, seq_lens, status, stream=None):
    """k_new, v_new: device [batch][kv_heads][n_new][d]; seq_lens: device int32 [batch], the
    lengths after the append (new token n goes to position seq_lens[b] - n_new + n)."""
    if v_new.shape != k_new.shape or v_new.dtype != k_new.dtype:
        raise ValueError("k_new and v_new must have the same shape and dtype")
    _check(lib.tq_append_kv(ctypes.byref(cfg), ctypes.byref(params), ctypes.byref(cache), layer,
                            _ptr(k_new), _ptr(v_new), dtype_code(k_new), k_new.shape[2], _ptr(seq_lens),
                            _ptr(status), _stream(stream)), "tq_append_kv")


def _check_offsets(k_offsets, v_offsets, shape):
    import torch
    for o in (k_offsets, v_offsets):
        if tuple(o.shape) != tuple(shape) or o.dtype != torch.float32 or not o.is_contiguous():
            raise ValueError("offsets must be contiguous float32 [batch][kv_heads][n]")


def append_kv_dithered(cfg, params, cache, layer, k_new, v_new, k_offsets, v_offsets, seq_lens, status,
                       stream=None):
    """append_kv for a dithered configuration; k_offsets, v_offsets: device float32
    [batch][kv_heads][n_new], the new tokens' offsets."""
    if v_new.shape != k_new.shape or v_new.dtype != k_new.dtype:
        raise ValueError("k_new and v_new must have the same shape and dtype")
    _check_offsets(k_offsets, v_offsets, k_new.shape[:3])
    _check(lib.tq_append_kv_dithered(ctypes.byref(cfg), ctypes.byref(params), ctypes.byref(cache), layer,
                                     _ptr(k_new), _ptr(v_new), _ptr(k_offsets), _ptr(v_offsets),
                                     dtype_code(k_new), k_new.shape[2], _ptr(seq_lens), _ptr(status),
                                     _stream(stream)), "tq_append_kv_dithered")


def append_attend_decode_dithered(cfg, params, cache, layer, k_new, v_new, k_offsets, v_offsets, q, seq_lens,
                                  n_splits, workspace, out, status, stream=None):
    """append_attend_decode for a dithered configuration (offsets as for append_kv_dithered)."""
    if v_new.shape != k_new.shape or v_new.dtype != k_new.dtype:
        raise ValueError("k_new and v_new must have the same shape and dtype")
    _check_offsets(k_offsets, v_offsets, k_new.shape[:3])
    _check(lib.tq_append_attend_decode_dithered(ctypes.byref(cfg), ctypes.byref(params), ctypes.byref(cache),
                                                layer, _ptr(k_new), _ptr(v_new), _ptr(k_offsets),
                                                _ptr(v_offsets), dtype_code(k_new), k_new.shape[2], _ptr(q),
                                                dtype_code(q), q.shape[1], q.shape[2], _ptr(seq_lens), n_splits,
                                                _ptr(workspace), workspace.numel() * workspace.element_size(),
                                                _ptr(out), _ptr(status), _stream(stream)),
           "tq_append_attend_decode_dithered")


def append_attend_decode(cfg, params, cache, layer, k_new, v_new, q, seq_lens, n_splits, workspace,
                         out, status, stream=None):
    """append_kv then attend_decode in one call; seq_lens are the lengths after the append."""
    if v_new.shape != k_new.shape or v_new.dtype != k_new.dtype:
        raise ValueError("k_new and v_new must have the same shape and dtype")
    _check(lib.tq_append_attend_decode(ctypes.byref(cfg), ctypes.byref(params), ctypes.byref(cache), layer,
                                       _ptr(k_new), _ptr(v_new), dtype_code(k_new), k_new.shape[2],
                                       _ptr(q), dtype_code(q), q.shape[1], q.shape[2], _ptr(seq_lens),
                                       n_splits, _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _ptr(out),
                                       _ptr(status), _stream(stream)), "tq_append_attend_decode")


def decode_scores(cfg, params, cache, layer, q, seq_lens, workspace, scores, status, stream=None):
    """scores: device float32 [batch][q_heads][seq_q][max_len]."""
    _check(lib.tq_decode_scores(ctypes.byref(cfg), ctypes.byref(params), ctypes.byref(cache), layer,
                                _ptr(q), dtype_code(q), q.shape[1], q.shape[2], _ptr(seq_lens),
                                scores.shape[3], _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _ptr(scores),
                                _ptr(status), _stream(stream)), "tq_decode_scores")


def decompress(cfg, params, cache, layer, seq_lens, max_len, k_hat, v_hat, status, stream=None):
    _check(lib.tq_decompress(ctypes.byref(cfg), ctypes.byref(params), ctypes.byref(cache), layer,
                             _ptr(seq_lens), max_len, _ptr(k_hat), _ptr(v_hat), _ptr(status),
                             _stream(stream)), "tq_decompress")
