"""Device-memory plumbing around the C ABI: a paged cache plus its parameters.

Owns nothing but PyTorch tensors; every computation is a call into libtq.so.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import (TQ_ROT_DENSE, TQ_ROT_HADAMARD, TQError, append_attend_decode, append_attend_decode_dithered,
               append_kv, append_kv_dithered, attend_decode,
               check_status, codebook, compress_kv, compress_kv_dithered, dither_codebook, last_error,
               decode_scores, decode_workspace_bytes, decompress, make_cache, make_config, make_params,
               operand_bytes, page_bytes, prepare_operands)


def _f32(x, device):
    if x is None:
        return None
    return torch.as_tensor(x, dtype=torch.float32).to(device).contiguous()


def splits_for(batch: int, kv_heads: int, sms: int, rows: int = 1, max_len: Optional[int] = None) -> int:
    """Split count that fills a GPU of `sms` SMs once: the tensor-core decode kernel keeps two
    CTAs per SM, one CTA per (split, kv head, sequence, run of query rows); a KV head's
    rows = G * seq_q query rows are taken four at a time, or eight when there are more than
    four.  A batch of several sequences gets twice that: when their lengths differ the kernel
    cuts the longest into more splits and the shorter ones into fewer (at most this count).
    With max_len, no more splits than 128-token units of the longest sequence."""
    runs = -(-max(1, rows) // (8 if rows > 4 else 4))
    n = (2 * sms) // max(1, batch * kv_heads * runs)
    if batch > 1:
        n *= 2
    if max_len is not None:
        n = min(n, -(-max(1, max_len) // 128))
    return max(1, min(1024, n))


def default_splits(batch: int, kv_heads: int, device=None, rows: int = 1, max_len: Optional[int] = None) -> int:
    """splits_for on the current (or given) GPU."""
    sms = torch.cuda.get_device_properties(device if device is not None else 0).multi_processor_count
    return splits_for(batch, kv_heads, sms, rows, max_len)


class PagedKV:
    """A packed TurboQuant cache for `num_layers` layers sharing one block table."""

    def __init__(self, *, batch: int, kv_heads: int, num_pages: int, block_table, key_bits: int,
                 key_qjl: bool, value_bits: int, rotation: int = TQ_ROT_HADAMARD,
                 num_layers: int = 1, signs=None, pi=None, s=None, codebooks=None,
                 device: str = "cuda", prepared_operands: bool = True, value_qjl: bool = False,
                 dither: bool = False, key_corrected_norm: bool = False):
        self.device = torch.device(device)
        self.cfg = make_config(key_bits=key_bits, key_qjl=key_qjl, value_bits=value_bits,
                               rotation=rotation, value_qjl=value_qjl, dither=dither,
                               key_corrected_norm=key_corrected_norm)
        self.dither = bool(dither)
        self.block_bytes = page_bytes(self.cfg)
        if self.block_bytes == 0:
            raise TQError(2, "PagedKV", "unsupported configuration")
        self.batch, self.kv_heads, self.num_pages, self.num_layers = batch, kv_heads, num_pages, num_layers
        self.block_table = torch.as_tensor(block_table, dtype=torch.int32).to(self.device).contiguous()
        self.max_pages = self.block_table.shape[1]
        nbytes = num_layers * num_pages * kv_heads * self.block_bytes
        self.pages = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        if codebooks is None:
            book = dither_codebook if dither else codebook
            kc, kb = book(key_bits)
            vc, vb = book(value_bits)
        else:
            kc, kb, vc, vb = codebooks
        self.tensors = {
            "signs": _f32(signs, self.device), "pi": _f32(pi, self.device), "s": _f32(s, self.device),
            "kc": _f32(kc, self.device), "kb": _f32(kb, self.device),
            "vc": _f32(vc, self.device), "vb": _f32(vb, self.device),
        }
        t = self.tensors
        # the compress kernel's tensor-core operands (H D, S D H; or sqrt(d) Pi), formed once
        # for the cache instead of in every thread block of every call
        t["ops"] = None
        nops = operand_bytes(self.cfg)
        if rotation == TQ_ROT_DENSE:
            have = t["pi"] is not None
        else:
            have = t["signs"] is not None and (not (key_qjl or value_qjl) or t["s"] is not None)
        if prepared_operands and nops and have:
            t["ops"] = torch.empty(nops, dtype=torch.uint8, device=self.device)
            prepare_operands(self.cfg, make_params(t["signs"], t["pi"], s=t["s"]), t["ops"])
        self.params = make_params(t["signs"], t["pi"], t["s"], t["kc"], t["kb"], t["vc"], t["vb"], t["ops"])
        self.cache = make_cache(self.pages, self.block_table, num_pages, self.max_pages, batch, kv_heads,
                                num_layers)
        self._ws = {}

    # ---- calls -----------------------------------------------------------------------------
    def compress(self, layer: int, k: torch.Tensor, v: torch.Tensor, seq_lens: torch.Tensor, stream=None,
                 k_offsets: Optional[torch.Tensor] = None, v_offsets: Optional[torch.Tensor] = None):
        """A dithered cache takes each vector's offset (device float32 [batch][kv_heads][max_len])."""
        if self.dither:
            if k_offsets is None or v_offsets is None:
                raise ValueError("a dithered cache needs k_offsets and v_offsets")
            compress_kv_dithered(self.cfg, self.params, self.cache, layer, k, v, k_offsets, v_offsets,
                                 seq_lens, self.status, stream)
        else:
            compress_kv(self.cfg, self.params, self.cache, layer, k, v, seq_lens, self.status, stream)

    def append(self, layer: int, k_new: torch.Tensor, v_new: torch.Tensor, seq_lens: torch.Tensor,
               stream=None, k_offsets: Optional[torch.Tensor] = None, v_offsets: Optional[torch.Tensor] = None):
        """Compresses k_new, v_new [batch][kv_heads][n_new][d] into positions
        seq_lens[b] - n_new .. seq_lens[b] - 1 (seq_lens: the lengths after the append); a
        dithered cache takes the new tokens' offsets [batch][kv_heads][n_new]."""
        if self.dither:
            if k_offsets is None or v_offsets is None:
                raise ValueError("a dithered cache needs k_offsets and v_offsets")
            append_kv_dithered(self.cfg, self.params, self.cache, layer, k_new, v_new, k_offsets, v_offsets,
                               seq_lens, self.status, stream)
        else:
            append_kv(self.cfg, self.params, self.cache, layer, k_new, v_new, seq_lens, self.status, stream)

    def workspace(self, q_heads: int, seq_q: int, n_splits: int) -> torch.Tensor:
        key = (q_heads, seq_q, n_splits)
        if key not in self._ws:
            nb = decode_workspace_bytes(self.cfg, self.batch, q_heads, seq_q, n_splits)
            self._ws[key] = torch.empty(nb, dtype=torch.uint8, device=self.device)
        return self._ws[key]

    def decode(self, layer: int, q: torch.Tensor, seq_lens: torch.Tensor, n_splits: int,
               out: Optional[torch.Tensor] = None, stream=None, k_new: Optional[torch.Tensor] = None,
               v_new: Optional[torch.Tensor] = None, k_offsets: Optional[torch.Tensor] = None,
               v_offsets: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Attention of q over the first seq_lens[b] tokens.  With k_new and v_new the step's
        new tokens are appended first, in the same call (seq_lens count them)."""
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=self.device)
        ws = self.workspace(q.shape[1], q.shape[2], n_splits)
        if k_new is not None and self.dither:
            if k_offsets is None or v_offsets is None:
                raise ValueError("a dithered cache needs k_offsets and v_offsets")
            append_attend_decode_dithered(self.cfg, self.params, self.cache, layer, k_new, v_new, k_offsets,
                                          v_offsets, q, seq_lens, n_splits, ws, out, self.status, stream)
        elif k_new is not None:
            append_attend_decode(self.cfg, self.params, self.cache, layer, k_new, v_new, q, seq_lens,
                                 n_splits, ws, out, self.status, stream)
        else:
            attend_decode(self.cfg, self.params, self.cache, layer, q, seq_lens, n_splits, ws, out,
                          self.status, stream)
        return out

    def scores(self, layer: int, q: torch.Tensor, seq_lens: torch.Tensor, max_len: int, stream=None):
        sc = torch.full((q.shape[0], q.shape[1], q.shape[2], max_len), float("nan"),
                        dtype=torch.float32, device=self.device)
        ws = self.workspace(q.shape[1], q.shape[2], 1)
        decode_scores(self.cfg, self.params, self.cache, layer, q, seq_lens, ws, sc, self.status, stream)
        return sc

    def decompress(self, layer: int, seq_lens: torch.Tensor, max_len: int, stream=None):
        kh = torch.zeros((self.batch, self.kv_heads, max_len, 128), dtype=torch.float32, device=self.device)
        vh = torch.zeros_like(kh)
        decompress(self.cfg, self.params, self.cache, layer, seq_lens, max_len, kh, vh, self.status, stream)
        return kh, vh

    def check(self) -> int:
        """Synchronise, read the device status word through tq_check and reset it; returns
        the recorded status (0 = ok)."""
        torch.cuda.synchronize(self.device)
        st = check_status(int(self.status.item()))
        self.status.zero_()
        return st

    def raise_on_error(self, where: str = "device"):
        st = self.check()
        if st:
            raise TQError(st, where, last_error())

    def pages_numpy(self):
        """Host copy of the cache as [num_layers][num_pages][kv_heads][block_bytes] uint8."""
        return self.pages.view(self.num_layers, self.num_pages, self.kv_heads, self.block_bytes).cpu().numpy()
