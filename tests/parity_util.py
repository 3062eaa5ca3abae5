"""Shared pieces of the GPU parity tests: run the library on a workload, run the oracle on
the same seeded inputs, compare with the stated tolerances.

Tolerances (the acceptance contract of this library):
  * packed indices and QJL sign bits bit-exact, except coordinates whose rotated value
    lies within 1e-6 of a codebook boundary, and sign bits whose projection (S r)_i lies
    within 1e-6 * sum_j |S_ij r_j| of zero (both counted and reported);
  * norms, scores and attention outputs |gpu - oracle| <= 1e-3 + 2e-3 |oracle|.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import workloads as wl
from oracle import attention as oatt
from oracle import codebook as ocb
from oracle import layout as olay
from oracle import quant as oq
from oracle import rotation as orot

ATOL, RTOL = 1e-3, 2e-3
BOUNDARY_BAND = 1e-6
SIGN_BAND = 1e-6


def close(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return np.abs(got - ref) <= ATOL + RTOL * np.abs(ref)


@dataclasses.dataclass
class Run:
    w: wl.Workload
    lens: np.ndarray
    bt: np.ndarray
    npages: int
    rin: dict
    R: np.ndarray
    fmt: olay.Format
    ck: np.ndarray
    kb: np.ndarray
    cv: np.ndarray
    vb: np.ndarray
    kv: object = None
    K: dict = None
    V: dict = None
    KO: dict = None   # dithered: the key offsets of each layer [batch][kv_heads][max_len]
    VO: dict = None


def setup(w: wl.Workload, layers=(0,), prepared_operands=True, compress_lens=None):
    """Builds the library cache for w and compresses `layers` on the GPU (inputs from workloads).
    compress_lens: optional per-sequence token counts to compress instead of the full
    lengths (the cache's block table still covers the full lengths)."""
    from compressed_decode_attention_tq_b200.runtime import PagedKV
    lens = wl.seq_lens(w)
    bt, npages = wl.block_table(w, lens)
    rin = wl.rotation_inputs(w)
    run = Run(w=w, lens=lens, bt=bt, npages=npages, rin=rin,
              R=orot.rotation_matrix(w.rotation, rin["signs"], rin["pi"]),
              fmt=olay.Format(key_bits=w.key_bits, key_qjl=w.key_qjl, value_bits=w.value_bits,
                              value_qjl=w.value_qjl, dither=w.dither),
              ck=None, kb=None, cv=None, vb=None)
    book = ocb.dither_codebook_f32 if w.dither else ocb.codebook_f32
    run.ck, run.kb = book(w.key_bits, 128)
    run.cv, run.vb = book(w.value_bits, 128)
    run.kv = PagedKV(batch=w.batch, kv_heads=w.kv_heads, num_pages=npages, block_table=bt,
                     key_bits=w.key_bits, key_qjl=w.key_qjl, value_bits=w.value_bits, value_qjl=w.value_qjl,
                     rotation=w.rotation, num_layers=max(layers) + 1, signs=rin["signs"],
                     pi=rin["pi"], s=rin["s"], prepared_operands=prepared_operands, dither=w.dither,
                     key_corrected_norm=w.key_corrected_norm)
    run.K, run.V, run.KO, run.VO = {}, {}, {}, {}
    dt = torch.float16 if w.in_dtype == "f16" else torch.float32
    seq = torch.as_tensor(lens if compress_lens is None else compress_lens, dtype=torch.int32, device="cuda")
    for layer in layers:
        K, V = wl.make_kv(w, layer)
        run.K[layer], run.V[layer] = K, V
        offs = {}
        if w.dither:
            # offsets uniform over one cell of each grid
            KO, VO = wl.dither_offsets(w, layer, 0.5 * float(run.ck[1] - run.ck[0]),
                                       0.5 * float(run.cv[1] - run.cv[0]))
            run.KO[layer], run.VO[layer] = KO, VO
            offs = dict(k_offsets=torch.as_tensor(KO, dtype=torch.float32, device="cuda"),
                        v_offsets=torch.as_tensor(VO, dtype=torch.float32, device="cuda"))
        run.kv.compress(layer, torch.as_tensor(K, dtype=dt, device="cuda"),
                        torch.as_tensor(V, dtype=dt, device="cuda"), seq, **offs)
    return run


def seq_dev(run):
    return torch.as_tensor(run.lens, dtype=torch.int32, device="cuda")


def q_dev(run, layer=0):
    q = wl.make_q(run.w, layer)
    dt = torch.float16 if run.w.in_dtype == "f16" else torch.float32
    return q, torch.as_tensor(q, dtype=dt, device="cuda")


@dataclasses.dataclass
class CompressReport:
    tokens: int = 0
    idx_mismatch_in_band: int = 0
    idx_mismatch_out_of_band: int = 0
    sign_mismatch_in_band: int = 0
    sign_mismatch_out_of_band: int = 0
    sign_tokens_skipped: int = 0
    norm_fail: int = 0


# Every compress comparison and decode check of the session, printed at the end of the run by
# tests/conftest.py (pytest_terminal_summary), so that the counts the tolerances allow are
# visible in the run's output even under -q.
REPORTS: list = []


def record(name: str, rep) -> None:
    """Keeps a CompressReport (or a one-line decode summary string) for the session summary."""
    REPORTS.append((name, rep))


def _check_qjl(gpu_sigma, gpu_rnorm, comp, mis, rep):
    """Residual norms and sign bits of the tokens whose indices all agree (a token whose
    index differs inside the band has a different residual, so its signs are skipped)."""
    ok_tok = ~mis
    rep.sign_tokens_skipped += int(np.sum(mis))
    rep.norm_fail += int(np.sum(~close(gpu_rnorm[ok_tok], comp.rnorm[ok_tok])))
    diff = (gpu_sigma != comp.sigma) & ok_tok[:, None]
    band = np.abs(comp.sr) <= SIGN_BAND * comp.sr_scale
    rep.sign_mismatch_in_band += int(np.sum(diff & band))
    rep.sign_mismatch_out_of_band += int(np.sum(diff & ~band))


def _compare_unpacked(fmt, u, K, V, R, ck, kb, cv, vb, S, rep, KO=None, VO=None, corrected=False):
    kx = dict(offsets=KO, corrected_norm=corrected)
    vx = dict(offsets=VO)
    kc = oq.compress_prod(K, R, ck, kb, S, **kx) if fmt.key_qjl else oq.compress_mse(K, R, ck, kb, **kx)
    vc = oq.compress_prod(V, R, cv, vb, S, **vx) if fmt.value_qjl else oq.compress_mse(V, R, cv, vb, **vx)
    rep.tokens += K.shape[0]
    if fmt.dither:
        # the stored offsets are the fp16 roundings of the given ones, exactly
        rep.norm_fail += int(np.sum(u.k_offset != kc.offset)) + int(np.sum(u.v_offset != vc.offset))
    kmis = _check_idx(u.k_idx, kc, kb, rep)
    vmis = _check_idx(u.v_idx, vc, vb, rep)
    rep.norm_fail += int(np.sum(~close(u.k_norm, kc.norm)))
    rep.norm_fail += int(np.sum(~close(u.v_norm, vc.norm)))
    if fmt.key_qjl:
        _check_qjl(u.k_sigma, u.k_rnorm, kc, kmis, rep)
    if fmt.value_qjl:
        _check_qjl(u.v_sigma, u.v_rnorm, vc, vmis, rep)
    return rep


def compare_compress_rows(fmt, u, K, V, R, ck, kb, cv, vb, S, rep: CompressReport, corrected=False):
    """Compares unpacked GPU codes u (tokens in the order of the rows) with the oracle's
    compression of the same float64 rows K, V [n][d]."""
    return _compare_unpacked(fmt, u, K, V, R, ck, kb, cv, vb, S, rep, corrected=corrected)


def compare_compress(run, pages, layer, b, h, tokens=None, rep: CompressReport = None):
    """Compares the GPU's packed (layer, b, h) against the oracle on the same inputs.
    tokens: optional index array of positions to check (default all)."""
    rep = rep or CompressReport()
    n = int(run.lens[b])
    u = olay.read_sequence(pages, run.fmt, layer, h, run.bt[b], n)
    sel = np.arange(n) if tokens is None else np.asarray(tokens)
    sub = olay.Unpacked(k_idx=u.k_idx[sel], k_norm=u.k_norm[sel], v_idx=u.v_idx[sel], v_norm=u.v_norm[sel])
    for f in ("k_rnorm", "k_sigma", "v_rnorm", "v_sigma", "k_offset", "v_offset"):
        if getattr(u, f) is not None:
            setattr(sub, f, getattr(u, f)[sel])
    KO = run.KO[layer][b, h][sel] if run.w.dither else None
    VO = run.VO[layer][b, h][sel] if run.w.dither else None
    return _compare_unpacked(run.fmt, sub, run.K[layer][b, h][sel], run.V[layer][b, h][sel], run.R,
                             run.ck, run.kb, run.cv, run.vb, run.rin["s"], rep, KO, VO,
                             run.w.key_corrected_norm)


def _check_idx(gpu_idx, comp, boundaries, rep):
    diff = gpu_idx != comp.idx
    dist = np.min(np.abs(comp.y[..., None] - boundaries.astype(np.float64)), axis=-1)
    band = dist < BOUNDARY_BAND
    rep.idx_mismatch_in_band += int(np.sum(diff & band))
    rep.idx_mismatch_out_of_band += int(np.sum(diff & ~band))
    return np.any(diff, axis=1)


def oracle_decode(run, pages, layer, q, heads=None):
    return oatt.decode(pages, run.fmt, layer, q, run.bt, run.lens, run.R, run.ck, run.cv,
                       run.rin["s"] if (run.w.key_qjl or run.w.value_qjl) else None, heads=heads)


def oracle_scores(run, pages, layer, q, b, h):
    """Scores of query head h of sequence b over its cached tokens: [seq_q, n]."""
    G = run.w.group
    u = olay.read_sequence(pages, run.fmt, layer, h // G, run.bt[b], int(run.lens[b]))
    k_mse = oq.reconstruct_mse(u.k_idx, u.k_norm, run.R, run.ck, u.k_offset)
    return oatt.scores_compressed(q[b, h], k_mse, u.k_rnorm, u.k_sigma,
                                  run.rin["s"] if run.w.key_qjl else None)
