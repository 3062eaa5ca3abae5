"""Seeded synthetic inputs shared by the oracle-side tests, the GPU tests and the bench.

This module only draws random numbers and arranges them in the shapes of the
workloads below. It holds none of the method's arithmetic: no rotation is
applied, nothing is normalised, quantised or sketched here.

Random inputs of the method that both sides must agree on are drawn here and
passed to both:

* the Rademacher diagonal D of the randomized Hadamard rotation HD
  ("TurboQuant explained", section "How JL Matrices Evolved": D is a random
  +-1 diagonal),
* the Gaussian QJL matrix S (m x d, iid N(0,1)), rounded to fp16-representable
  values so that an fp16 tensor-core operand holds it exactly
  ("TurboQuant explained", section "QJL: Inner Product Recovery from a Single
  Sign Bit"),
* the dense Haar-orthogonal rotation Pi = Q of the QR factorisation of a
  Gaussian matrix, with the column signs fixed by diag(R) so that Q is
  Haar-distributed ("turboquant_cutile" function list: "Haar-distributed random
  orthogonal matrix via QR of Gaussian"), rounded to fp32-representable values
  because that is what the device receives.

The data distributions follow the workloads named for this path: iid Gaussian
with a few outlier channels, Gaussian with log-normal per-channel scales,
Student-t heavy tails, ragged batch lengths and permuted page tables.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

HEAD_DIM = 128
QJL_M = 128
PAGE_TOKENS = 256

ROT_HADAMARD = 0
ROT_DENSE = 1


# ---------------------------------------------------------------------------
# rotation / sketch inputs
# ---------------------------------------------------------------------------

def hadamard_signs(d: int, seed: int) -> np.ndarray:
    """Rademacher diagonal of D, as float64 +-1 values."""
    rng = np.random.default_rng(seed)
    return (rng.integers(0, 2, size=d) * 2 - 1).astype(np.float64)


def qjl_matrix(m: int, d: int, seed: int) -> np.ndarray:
    """iid N(0,1) m x d matrix rounded to the nearest fp16 value (returned as float64)."""
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((m, d))
    return s.astype(np.float16).astype(np.float64)


def haar_matrix(d: int, seed: int) -> np.ndarray:
    """Haar-orthogonal d x d matrix (QR of a Gaussian, signs fixed), fp32-rounded, as float64."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((d, d))
    q, r = np.linalg.qr(z)
    q = q * np.sign(np.diag(r))[None, :]
    return q.astype(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# workload descriptions
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    name: str
    batch: int
    kv_heads: int
    q_heads: int
    seq_q: int
    max_len: int
    key_bits: int
    key_qjl: bool
    value_bits: int
    rotation: int
    n_splits: int
    num_layers: int = 1
    in_dtype: str = "f16"          # "f16" or "f32"
    data_seed: int = 0
    rot_seed: int = 0
    s_seed: int = 1
    ragged: bool = False
    permute_pages: bool = False
    kind: str = "gauss_lognormal"  # data recipe, see make_kv
    outlier_channels: int = 0
    outlier_scale: float = 1.0
    outlier_seed: int = 3
    min_len: int = 0
    value_qjl: bool = False        # values carry the QJL sketch of their residual too
    dither: bool = False           # dithered HD: one random offset per key and per value
    key_corrected_norm: bool = False  # keys store the corrected norm

    @property
    def group(self) -> int:
        return self.q_heads // self.kv_heads


def config1(**kw) -> Workload:
    """Single head, 4096 tokens, fp32 N(0,1) K/V with 4 outlier channels x8, HD rotation,
    keys 2-bit + QJL, values 2-bit."""
    w = Workload(name="c1_single_head_4k", batch=1, kv_heads=1, q_heads=1, seq_q=1,
                 max_len=4096, key_bits=2, key_qjl=True, value_bits=2,
                 rotation=ROT_HADAMARD, n_splits=4, in_dtype="f32", data_seed=3,
                 rot_seed=0, s_seed=1, kind="gauss_outliers", outlier_channels=4,
                 outlier_scale=8.0, outlier_seed=3)
    return dataclasses.replace(w, **kw)


def config2(**kw) -> Workload:
    """Llama-3-8B-shaped layer: 32 q heads / 8 KV heads, 32768 tokens, fp16 K/V Gaussian with
    log-normal(0,0.5) channel std and 2% outlier channels x10, keys 3-bit + QJL, values 3-bit."""
    w = Workload(name="c2_llama3_8b_32k", batch=1, kv_heads=8, q_heads=32, seq_q=1,
                 max_len=32768, key_bits=3, key_qjl=True, value_bits=3,
                 rotation=ROT_HADAMARD, n_splits=16, in_dtype="f16", data_seed=4,
                 kind="gauss_lognormal_outliers",
                 outlier_channels=int(round(0.02 * HEAD_DIM)), outlier_scale=10.0)
    return dataclasses.replace(w, **kw)


def config3(**kw) -> Workload:
    """Qwen2.5-3B-shaped: batch 16, 16 q heads / 2 KV heads, ragged lengths U[4096,16384],
    fp16 Gaussian with log-normal channel scales, keys 4-bit (no QJL), values 3-bit,
    dense Haar rotation, permuted page table."""
    w = Workload(name="c3_qwen25_3b_ragged", batch=16, kv_heads=2, q_heads=16, seq_q=1,
                 max_len=16384, min_len=4096, key_bits=4, key_qjl=False, value_bits=3,
                 rotation=ROT_DENSE, n_splits=8, in_dtype="f16", data_seed=5, rot_seed=7,
                 ragged=True, permute_pages=True, kind="gauss_lognormal")
    return dataclasses.replace(w, **kw)


def config4(**kw) -> Workload:
    """Long context: batch 4, 32 q heads / 8 KV heads, 131072 tokens, fp16 K Student-t(3),
    V Gaussian, keys 2-bit + QJL, values 2-bit, 64 splits."""
    w = Workload(name="c4_long_128k", batch=4, kv_heads=8, q_heads=32, seq_q=1,
                 max_len=131072, key_bits=2, key_qjl=True, value_bits=2,
                 rotation=ROT_HADAMARD, n_splits=64, in_dtype="f16", data_seed=6,
                 kind="student_t_keys")
    return dataclasses.replace(w, **kw)


def config5(**kw) -> Workload:
    """Prefill compress of 32 layers x 8 KV heads x 32768 tokens fp16 (Gaussian, log-normal
    channel scales), keys 3-bit + QJL, values 3-bit, then seq_q=8 multi-query decode."""
    w = Workload(name="c5_prefill_32l_multiquery", batch=1, kv_heads=8, q_heads=32, seq_q=8,
                 max_len=32768, key_bits=3, key_qjl=True, value_bits=3,
                 rotation=ROT_HADAMARD, n_splits=16, num_layers=32, in_dtype="f16",
                 data_seed=7, kind="gauss_lognormal")
    return dataclasses.replace(w, **kw)


CONFIGS = {1: config1, 2: config2, 3: config3, 4: config4, 5: config5}


# ---------------------------------------------------------------------------
# data
# ---------------------------------------------------------------------------

def seq_lens(w: Workload) -> np.ndarray:
    if not w.ragged:
        return np.full(w.batch, w.max_len, dtype=np.int32)
    rng = np.random.default_rng(w.data_seed + 1000)
    lo = w.min_len if w.min_len else 1
    return rng.integers(lo, w.max_len + 1, size=w.batch).astype(np.int32)


def pages_per_seq(w: Workload) -> int:
    return (w.max_len + PAGE_TOKENS - 1) // PAGE_TOKENS


def block_table(w: Workload, lens: Optional[np.ndarray] = None) -> tuple[np.ndarray, int]:
    """[batch][max_pages] int32 logical->physical page map and the number of physical pages.

    Pages are handed out densely to the pages each sequence needs; with
    permute_pages the physical ids are a seeded permutation (exercises paging)."""
    if lens is None:
        lens = seq_lens(w)
    mp = pages_per_seq(w)
    need = [(int(n) + PAGE_TOKENS - 1) // PAGE_TOKENS for n in lens]
    total = int(sum(need))
    ids = np.arange(total, dtype=np.int32)
    if w.permute_pages:
        ids = np.random.default_rng(w.data_seed + 2000).permutation(total).astype(np.int32)
    bt = np.full((w.batch, mp), -1, dtype=np.int32)
    k = 0
    for b in range(w.batch):
        bt[b, :need[b]] = ids[k:k + need[b]]
        k += need[b]
    return bt, max(total, 1)


def _channel_scales(rng, heads, d, sigma=0.5):
    return np.exp(rng.normal(0.0, sigma, size=(heads, d)))


def make_kv(w: Workload, layer: int = 0, heads: Optional[list[int]] = None,
            tokens: Optional[int] = None) -> tuple[np.ndarray, np.ndarray]:
    """K and V for one layer as float64 arrays [batch][kv_heads][max_len][d], already rounded
    to the input dtype (fp16 or fp32) so both sides see identical values.

    heads/tokens restrict the draw to a sub-block (same values as the full draw for
    those heads and the first `tokens` positions)."""
    d = HEAD_DIM
    T = w.max_len if tokens is None else tokens
    hs = list(range(w.kv_heads)) if heads is None else heads
    kout = np.zeros((w.batch, len(hs), T, d))
    vout = np.zeros((w.batch, len(hs), T, d))
    for bi in range(w.batch):
        for j, h in enumerate(hs):
            seed = [w.data_seed, layer, bi, h]
            rk = np.random.default_rng(seed + [0])
            rv = np.random.default_rng(seed + [1])
            rs = np.random.default_rng([w.data_seed, layer, h, 7])
            if w.kind == "gauss_outliers":
                k = rk.standard_normal((T, d))
                v = rv.standard_normal((T, d))
                oc = np.random.default_rng(w.outlier_seed).choice(d, w.outlier_channels,
                                                                  replace=False)
                k[:, oc] *= w.outlier_scale
                v[:, oc] *= w.outlier_scale
            elif w.kind in ("gauss_lognormal", "gauss_lognormal_outliers"):
                sk = _channel_scales(rs, 1, d)[0]
                sv = _channel_scales(rs, 1, d)[0]
                if w.kind == "gauss_lognormal_outliers":
                    oc_k = rs.choice(d, w.outlier_channels, replace=False)
                    oc_v = rs.choice(d, w.outlier_channels, replace=False)
                    sk[oc_k] *= w.outlier_scale
                    sv[oc_v] *= w.outlier_scale
                k = rk.standard_normal((T, d)) * sk
                v = rv.standard_normal((T, d)) * sv
            elif w.kind == "student_t_keys":
                k = rk.standard_t(3.0, size=(T, d))
                v = rv.standard_normal((T, d))
            else:
                raise ValueError(w.kind)
            kout[bi, j] = k
            vout[bi, j] = v
    dt = np.float16 if w.in_dtype == "f16" else np.float32
    return kout.astype(dt).astype(np.float64), vout.astype(dt).astype(np.float64)


def make_q(w: Workload, layer: int = 0) -> np.ndarray:
    """Queries [batch][q_heads][seq_q][d], N(0,1), rounded to the input dtype, as float64."""
    rng = np.random.default_rng([w.data_seed, layer, 99])
    q = rng.standard_normal((w.batch, w.q_heads, w.seq_q, HEAD_DIM))
    dt = np.float16 if w.in_dtype == "f16" else np.float32
    return q.astype(dt).astype(np.float64)


def dither_offsets(w: Workload, layer: int, half_k: float, half_v: float) -> tuple[np.ndarray, np.ndarray]:
    """The random offsets of a dithered workload ("Minimum Distortion Quantization with
    Specified Output Distribution" page: a random scalar offset per vector): iid uniform on
    [-half, half) for every (sequence, kv head, position), keys and values drawn apart,
    rounded to fp32 (what the device receives), as float64 [batch][kv_heads][max_len]."""
    rng = np.random.default_rng([w.data_seed, layer, 31])
    shape = (w.batch, w.kv_heads, w.max_len)
    k = rng.uniform(-half_k, half_k, shape)
    v = rng.uniform(-half_v, half_v, shape)
    return k.astype(np.float32).astype(np.float64), v.astype(np.float32).astype(np.float64)


def dither_offsets_device(w: Workload, layer: int, half_k: float, half_v: float, device):
    """dither_offsets drawn with torch on `device` (a different random stream), float32."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(w.data_seed) * 104729 + layer + 31)
    shape = (w.batch, w.kv_heads, w.max_len)
    k = (torch.rand(shape, generator=g, device=device) * 2.0 - 1.0) * half_k
    v = (torch.rand(shape, generator=g, device=device) * 2.0 - 1.0) * half_v
    return k, v


def rotation_inputs(w: Workload) -> dict:
    """The random rotation and sketch inputs of a workload (float64 arrays)."""
    d = HEAD_DIM
    out = {"signs": hadamard_signs(d, w.rot_seed), "s": qjl_matrix(QJL_M, d, w.s_seed)}
    out["pi"] = haar_matrix(d, w.rot_seed) if w.rotation == ROT_DENSE else None
    return out


def np_dtype(w: Workload):
    return np.float16 if w.in_dtype == "f16" else np.float32


# ---------------------------------------------------------------------------
# large inputs drawn directly on the device (bench sizes)
# ---------------------------------------------------------------------------

def make_kv_device(w: Workload, layer: int, device, dtype=None):
    """K, V [batch][kv_heads][max_len][d] drawn with torch on `device` (same recipe as make_kv,
    a different random stream): Gaussian times per-(head, channel) log-normal(0, 0.5) scales,
    optional outlier channels, or Student-t keys.  Used where the host draw would be too slow."""
    import torch
    dt = dtype or (torch.float16 if w.in_dtype == "f16" else torch.float32)
    g = torch.Generator(device=device)
    g.manual_seed(int(w.data_seed) * 1000003 + layer)
    shape = (w.batch, w.kv_heads, w.max_len, HEAD_DIM)
    if w.kind == "student_t_keys":
        # Student-t(3) = N / sqrt(chi2_3 / 3), chi2_3 = sum of three squared normals
        n = torch.randn(shape, generator=g, device=device)
        chi = sum(torch.randn(shape, generator=g, device=device) ** 2 for _ in range(3))
        k = n / torch.sqrt(chi / 3.0)
        v = torch.randn(shape, generator=g, device=device)
        return k.to(dt), v.to(dt)
    sk = torch.exp(0.5 * torch.randn((w.kv_heads, HEAD_DIM), generator=g, device=device))
    sv = torch.exp(0.5 * torch.randn((w.kv_heads, HEAD_DIM), generator=g, device=device))
    if w.outlier_channels:
        for h in range(w.kv_heads):
            ok = torch.randperm(HEAD_DIM, generator=g, device=device)[:w.outlier_channels]
            ov = torch.randperm(HEAD_DIM, generator=g, device=device)[:w.outlier_channels]
            sk[h, ok] *= w.outlier_scale
            sv[h, ov] *= w.outlier_scale
    k = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    k.mul_(sk[None, :, None, :])
    k = k.to(dt)
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    v.mul_(sv[None, :, None, :])
    return k, v.to(dt)


def make_q_device(w: Workload, layer: int, device, dtype=None):
    import torch
    dt = dtype or (torch.float16 if w.in_dtype == "f16" else torch.float32)
    g = torch.Generator(device=device)
    g.manual_seed(int(w.data_seed) * 7919 + layer + 17)
    return torch.randn((w.batch, w.q_heads, w.seq_q, HEAD_DIM), generator=g, device=device).to(dt)
