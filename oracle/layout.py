"""The packed, paged cache format, written out independently of the library (oracle).

The pages fix what is stored per token - b-bit centroid indices, a 16-bit norm,
for keys m QJL sign bits and ||r|| ("TurboQuant explained", section "QJL: Inner
Product Recovery from a Single Sign Bit": m sign bits plus 16 bits for the norm,
no scale or zero point) - and that serving uses a packed paged cache with a page
table ("TurboQuant" limits page, section "Operational Assumptions": vLLM-style
packed paged decode).  How the bits are laid out is left open; this module
states the layout the library documents in include/tq.h, reading it from the
format description only.

Format (d = 128, m = 128, P tokens per page, one block per (layer, physical
page, kv head); the cache is [layer][physical page][kv head][block]):

  region  content                               bytes
  KN      stored ||k|| as fp16, one per token    2P
  KR      stored ||r|| as fp16 (keys with QJL)   2P
  VN      stored ||v|| as fp16                   2P
  KC      key codes, b_k*d/8 bytes per token     b_k*16*P  (merged keys: 4*16*P)
  KS      QJL sign bits, m/8 bytes per token     16*P   (keys with QJL, not merged)
  VC      value codes, b_v*d/8 bytes per token   b_v*16*P
  VS      QJL sign bits of the value residual    16*P   (values with QJL)
  VR      stored ||r_v|| as fp16                 2P     (values with QJL)
  KD      key dither offset xi as fp16           2P     (dithered configurations)
  VD      value dither offset xi as fp16         2P     (dithered configurations)

Each code region is a sequence of 16-byte chunks per token, stored chunk-major:
chunk c of token t sits at byte (c*P + t)*16 of the region.  Token t's chunks,
concatenated, form its bit string; bit k of the bit string is bit (k mod 8) of
byte k/8 (little endian).

Stored code of a centroid index idx in [0, 2^b) ("sign-magnitude"): with
h = 2^(b-1), the sign bit s = [idx >= h] and the rank r = idx - h if s else
h - 1 - idx (0 = the centroid nearest zero).  Because the codebook is symmetric,
c[idx] = (+1 if s else -1) * c[h + r].  Fields of coordinate j in the bit string:
  b = 1:  bit j = s
  b = 2:  bits 2j, 2j+1 = r, s
  b = 3:  bits 2j, 2j+1 = r (2-bit rank); the sign plane follows at bit 2d: with
          j = 32q + 8a + 4h + t (a in 0..3, h in 0..1, t in 0..3) the sign sits at
          bit 2d + 32q + 4a + t + 16h (a fixed permutation inside each group of 32)
  b = 4:  bits 4j..4j+2 = r (3-bit rank), bit 4j + 3 = s
Keys with b_k = 3 and QJL ("merged keys") store one 4-bit field per coordinate,
bits 4j..4j+3 = r0, r1, s, sigma_j, and have no KS region; other keys with QJL keep
the sign bits in KS, bit i = sigma_i.

Values with QJL (TurboQuant_prod applied to the value cache: "TurboQuant explained",
section "Two-Stage Approach: MSE Approximation + QJL Correction", which reconstructs a
vector as x_mse + sqrt(pi/2)/d ||r|| S^T sign(S r) and notes that this serves the value
cache too) store the residual's signs in VS (bit i = sigma_i, as KS) and its norm in VR;
the two regions come last, so every other offset is the same with or without them.

Dithered configurations (the "Minimum Distortion Quantization with Specified Output
Distribution" page, third abstract: a random scalar offset per vector) keep each vector's
offset, which the reconstruction adds back, in KD and VD after everything else.
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass
class Format:
    head_dim: int = 128
    key_bits: int = 3
    key_qjl: bool = True
    qjl_m: int = 128
    value_bits: int = 3
    page_tokens: int = 256
    value_qjl: bool = False
    dither: bool = False

    @property
    def merged_keys(self) -> bool:
        return bool(self.key_qjl) and self.key_bits == 3

    @property
    def key_bytes(self) -> int:
        """Bytes of one token's key bit string in KC."""
        return (4 if self.merged_keys else self.key_bits) * self.head_dim // 8

    def regions(self) -> dict:
        P, d, m = self.page_tokens, self.head_dim, self.qjl_m
        ks = m // 8 * P if (self.key_qjl and not self.merged_keys) else 0
        sizes = [("KN", 2 * P), ("KR", 2 * P if self.key_qjl else 0), ("VN", 2 * P),
                 ("KC", self.key_bytes * P), ("KS", ks),
                 ("VC", self.value_bits * d // 8 * P),
                 ("VS", m // 8 * P if self.value_qjl else 0),
                 ("VR", 2 * P if self.value_qjl else 0),
                 ("KD", 2 * P if self.dither else 0),
                 ("VD", 2 * P if self.dither else 0)]
        out, off = {}, 0
        for name, sz in sizes:
            out[name] = (off, sz)
            off += sz
        out["total"] = (0, off)
        return out

    @property
    def block_bytes(self) -> int:
        return self.regions()["total"][1]


def stored_code(idx, bits: int):
    idx = np.asarray(idx, dtype=np.int64)
    h = 1 << (bits - 1)
    s = (idx >= h).astype(np.int64)
    r = np.where(s == 1, idx - h, h - 1 - idx)
    return s, r


def index_from_code(s, r, bits: int):
    h = 1 << (bits - 1)
    s = np.asarray(s, dtype=np.int64)
    r = np.asarray(r, dtype=np.int64)
    return np.where(s == 1, h + r, h - 1 - r)


def sign_plane_position(j):
    """Bit offset inside the b = 3 sign plane of coordinate j (see the format above)."""
    j = np.asarray(j)
    q, e = j // 32, j % 32
    a, h, t = e // 8, (e // 4) % 2, e % 4
    return 32 * q + 4 * a + t + 16 * h


def code_bits(idx, bits: int) -> np.ndarray:
    """[N, d] indices -> [N, bits*d] uint8 bit strings."""
    idx = np.asarray(idx, dtype=np.int64)
    n, d = idx.shape
    s, r = stored_code(idx, bits)
    out = np.zeros((n, bits * d), dtype=np.uint8)
    j = np.arange(d)
    if bits == 1:
        out[:, j] = s
    elif bits == 2:
        out[:, 2 * j] = r & 1
        out[:, 2 * j + 1] = s
    elif bits == 3:
        out[:, 2 * j] = r & 1
        out[:, 2 * j + 1] = (r >> 1) & 1
        out[:, 2 * d + sign_plane_position(j)] = s
    elif bits == 4:
        out[:, 4 * j] = r & 1
        out[:, 4 * j + 1] = (r >> 1) & 1
        out[:, 4 * j + 2] = (r >> 2) & 1
        out[:, 4 * j + 3] = s
    else:
        raise ValueError("bits must be 1..4")
    return out


def merged_key_bits(idx, sigma) -> np.ndarray:
    """[N, d] 3-bit indices and [N, d] QJL bits -> [N, 4d] merged key bit strings."""
    idx = np.asarray(idx, dtype=np.int64)
    n, d = idx.shape
    s, r = stored_code(idx, 3)
    out = np.zeros((n, 4 * d), dtype=np.uint8)
    j = np.arange(d)
    out[:, 4 * j] = r & 1
    out[:, 4 * j + 1] = (r >> 1) & 1
    out[:, 4 * j + 2] = s
    out[:, 4 * j + 3] = np.asarray(sigma, dtype=np.uint8)
    return out


def merged_key_from_bits(bitstr, d: int):
    b = np.asarray(bitstr, dtype=np.int64)
    j = np.arange(d)
    r = b[:, 4 * j] | (b[:, 4 * j + 1] << 1)
    return index_from_code(b[:, 4 * j + 2], r, 3), b[:, 4 * j + 3].astype(bool)


def index_from_bits(bitstr, bits: int, d: int) -> np.ndarray:
    """[N, bits*d] bit strings -> [N, d] indices."""
    b = np.asarray(bitstr, dtype=np.int64)
    j = np.arange(d)
    if bits == 1:
        s, r = b[:, j], np.zeros_like(b[:, j])
    elif bits == 2:
        r, s = b[:, 2 * j], b[:, 2 * j + 1]
    elif bits == 3:
        r = b[:, 2 * j] | (b[:, 2 * j + 1] << 1)
        s = b[:, 2 * d + sign_plane_position(j)]
    elif bits == 4:
        r = b[:, 4 * j] | (b[:, 4 * j + 1] << 1) | (b[:, 4 * j + 2] << 2)
        s = b[:, 4 * j + 3]
    else:
        raise ValueError("bits must be 1..4")
    return index_from_code(s, r, bits)


def bits_to_bytes(bitstr) -> np.ndarray:
    return np.packbits(np.asarray(bitstr, dtype=np.uint8), axis=-1, bitorder="little")


def bytes_to_bits(by) -> np.ndarray:
    return np.unpackbits(np.asarray(by, dtype=np.uint8), axis=-1, bitorder="little")


def _put_chunked(region: np.ndarray, tok_bytes: np.ndarray, t0: int, P: int):
    """Write [n, nbytes] per-token byte strings into a chunk-major region for tokens t0.."""
    n, nb = tok_bytes.shape
    nch = nb // 16
    view = region.reshape(nch, P, 16)
    view[:, t0:t0 + n, :] = tok_bytes.reshape(n, nch, 16).transpose(1, 0, 2)


def _get_chunked(region: np.ndarray, n: int, nb: int, P: int) -> np.ndarray:
    nch = nb // 16
    return region.reshape(nch, P, 16)[:, :n, :].transpose(1, 0, 2).reshape(n, nb)


def fp16_bytes(values) -> np.ndarray:
    return np.asarray(values, dtype=np.float64).astype(np.float16).view(np.uint8)


def empty_cache(fmt: Format, num_pages: int, kv_heads: int, num_layers: int = 1) -> np.ndarray:
    return np.zeros((num_layers, num_pages, kv_heads, fmt.block_bytes), dtype=np.uint8)


def write_sequence(cache: np.ndarray, fmt: Format, layer: int, head: int, pages_of_seq,
                   kcomp, vcomp):
    """Write one (sequence, kv head): kcomp/vcomp hold idx, norm (and rnorm, sigma for keys)
    for its tokens 0..n-1; pages_of_seq lists the physical pages in logical order."""
    P, d = fmt.page_tokens, fmt.head_dim
    reg = fmt.regions()
    n = kcomp.idx.shape[0]
    if fmt.merged_keys:
        kbytes = bits_to_bytes(merged_key_bits(kcomp.idx, kcomp.sigma))
        sbytes = None
    else:
        kbytes = bits_to_bytes(code_bits(kcomp.idx, fmt.key_bits))
        sbytes = bits_to_bytes(kcomp.sigma.astype(np.uint8)) if fmt.key_qjl else None
    vbytes = bits_to_bytes(code_bits(vcomp.idx, fmt.value_bits))
    vsbytes = bits_to_bytes(vcomp.sigma.astype(np.uint8)) if fmt.value_qjl else None
    for lp in range((n + P - 1) // P):
        t0, t1 = lp * P, min(n, (lp + 1) * P)
        blk = cache[layer, pages_of_seq[lp], head]

        def region(name):
            o, sz = reg[name]
            return blk[o:o + sz]

        region("KN")[2 * 0:2 * (t1 - t0)] = fp16_bytes(kcomp.norm[t0:t1])
        region("VN")[0:2 * (t1 - t0)] = fp16_bytes(vcomp.norm[t0:t1])
        if fmt.key_qjl:
            region("KR")[0:2 * (t1 - t0)] = fp16_bytes(kcomp.rnorm[t0:t1])
        if sbytes is not None:
            _put_chunked(region("KS"), sbytes[t0:t1], 0, P)
        _put_chunked(region("KC"), kbytes[t0:t1], 0, P)
        _put_chunked(region("VC"), vbytes[t0:t1], 0, P)
        if fmt.value_qjl:
            region("VR")[0:2 * (t1 - t0)] = fp16_bytes(vcomp.rnorm[t0:t1])
            _put_chunked(region("VS"), vsbytes[t0:t1], 0, P)
        if fmt.dither:
            region("KD")[0:2 * (t1 - t0)] = fp16_bytes(kcomp.offset[t0:t1])
            region("VD")[0:2 * (t1 - t0)] = fp16_bytes(vcomp.offset[t0:t1])


@dataclasses.dataclass
class Unpacked:
    k_idx: np.ndarray
    k_norm: np.ndarray
    v_idx: np.ndarray
    v_norm: np.ndarray
    k_rnorm: np.ndarray = None
    k_sigma: np.ndarray = None
    v_rnorm: np.ndarray = None
    v_sigma: np.ndarray = None
    k_offset: np.ndarray = None
    v_offset: np.ndarray = None


def read_sequence(cache: np.ndarray, fmt: Format, layer: int, head: int, pages_of_seq,
                  n: int) -> Unpacked:
    """Read tokens 0..n-1 of one (sequence, kv head) back into indices, norms and signs."""
    P, d, m = fmt.page_tokens, fmt.head_dim, fmt.qjl_m
    reg = fmt.regions()
    kb, vb = fmt.key_bytes, fmt.value_bits * d // 8
    parts = {k: [] for k in ("kn", "vn", "kr", "kc", "ks", "vc", "vr", "vs", "kd", "vd")}
    for lp in range((n + P - 1) // P):
        cnt = min(n, (lp + 1) * P) - lp * P
        blk = cache[layer, pages_of_seq[lp], head]

        def region(name):
            o, sz = reg[name]
            return blk[o:o + sz]

        parts["kn"].append(region("KN")[:2 * cnt].view(np.float16).astype(np.float64))
        parts["vn"].append(region("VN")[:2 * cnt].view(np.float16).astype(np.float64))
        parts["kc"].append(_get_chunked(region("KC"), cnt, kb, P))
        parts["vc"].append(_get_chunked(region("VC"), cnt, vb, P))
        if fmt.key_qjl:
            parts["kr"].append(region("KR")[:2 * cnt].view(np.float16).astype(np.float64))
        if fmt.key_qjl and not fmt.merged_keys:
            parts["ks"].append(_get_chunked(region("KS"), cnt, m // 8, P))
        if fmt.value_qjl:
            parts["vr"].append(region("VR")[:2 * cnt].view(np.float16).astype(np.float64))
            parts["vs"].append(_get_chunked(region("VS"), cnt, m // 8, P))
        if fmt.dither:
            parts["kd"].append(region("KD")[:2 * cnt].view(np.float16).astype(np.float64))
            parts["vd"].append(region("VD")[:2 * cnt].view(np.float16).astype(np.float64))
    cat = lambda k, w: np.concatenate(parts[k]) if parts[k] else np.zeros((0,) + w)
    kc = cat("kc", (kb,))
    vc = cat("vc", (vb,))
    if fmt.merged_keys:
        k_idx, k_sigma = merged_key_from_bits(bytes_to_bits(kc), d)
    else:
        k_idx, k_sigma = index_from_bits(bytes_to_bits(kc), fmt.key_bits, d), None
    out = Unpacked(k_idx=k_idx, k_norm=cat("kn", ()),
                   v_idx=index_from_bits(bytes_to_bits(vc), fmt.value_bits, d),
                   v_norm=cat("vn", ()))
    if fmt.key_qjl:
        out.k_rnorm = cat("kr", ())
        out.k_sigma = k_sigma if fmt.merged_keys else bytes_to_bits(cat("ks", (m // 8,))).astype(bool)
    if fmt.value_qjl:
        out.v_rnorm = cat("vr", ())
        out.v_sigma = bytes_to_bits(cat("vs", (m // 8,))).astype(bool)
    if fmt.dither:
        out.k_offset = cat("kd", ())
        out.v_offset = cat("vd", ())
    return out
