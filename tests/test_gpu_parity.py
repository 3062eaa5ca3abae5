"""GPU parity: the library's compress, decode, score and decompress kernels against the
CPU oracle on the same seeded inputs, at sizes the oracle finishes in seconds that span
several tiles, several pages and a ragged tail (shapes and distributions of the five
workloads, shrunk)."""
import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu

from parity_util import (CompressReport, close, compare_compress, oracle_decode, oracle_scores,
                         q_dev, record, seq_dev, setup)

SMALL = {
    "c1": lambda: wl.config1(max_len=1000, n_splits=3),
    "c2": lambda: wl.config2(kv_heads=2, q_heads=8, max_len=1300, n_splits=4),
    "c3": lambda: wl.config3(batch=3, max_len=900, min_len=300, n_splits=2),
    "c4": lambda: wl.config4(batch=2, kv_heads=2, q_heads=8, max_len=2000, n_splits=8),
    "c5": lambda: wl.config5(kv_heads=2, q_heads=8, max_len=700, num_layers=2, n_splits=3),
    "k1v4": lambda: wl.config2(kv_heads=1, q_heads=2, max_len=520, key_bits=1, value_bits=4,
                               n_splits=2, name="k1v4"),
    "k4qjl_v1_dense": lambda: wl.config2(kv_heads=1, q_heads=3, max_len=300, key_bits=4,
                                         value_bits=1, rotation=wl.ROT_DENSE, rot_seed=9,
                                         n_splits=1, name="k4qjl_v1_dense"),
    # values with QJL (TurboQuant_prod on the value cache): with merged QJL keys under HD,
    # and with MSE-only keys under a dense rotation (the value sketch alone)
    "c2_vqjl": lambda: wl.config2(kv_heads=2, q_heads=8, max_len=1300, n_splits=4, value_qjl=True,
                                  name="c2_vqjl"),
    "c3_vqjl_dense": lambda: wl.config3(batch=2, max_len=700, min_len=300, n_splits=3, value_qjl=True,
                                        name="c3_vqjl_dense"),
    # 2-bit values with QJL in a two-sequence batch (the value sketch as a second tensor-core launch)
    "c4_vqjl": lambda: wl.config4(batch=2, kv_heads=2, q_heads=8, max_len=1100, n_splits=5, value_qjl=True,
                                  name="c4_vqjl"),
    # dithered HD: merged QJL keys and 3-bit values; MSE-only 2-bit keys and 4-bit values
    "c2_dither": lambda: wl.config2(kv_heads=2, q_heads=8, max_len=1300, n_splits=4, dither=True,
                                    name="c2_dither"),
    "k2v4_dither": lambda: wl.config2(kv_heads=1, q_heads=4, max_len=600, key_bits=2, key_qjl=False,
                                      value_bits=4, n_splits=2, dither=True, name="k2v4_dither"),
    # dithered on the tensor-core split decode: 2-bit QJL keys and values; 32 rows per KV head
    "c4_dither": lambda: wl.config4(batch=2, kv_heads=2, q_heads=8, max_len=1100, n_splits=5, dither=True,
                                    name="c4_dither"),
    "c5_dither": lambda: wl.config5(kv_heads=2, q_heads=8, max_len=700, num_layers=1, n_splits=3, dither=True,
                                    name="c5_dither"),
    # corrected key norms: merged QJL keys (fast decode) and dense 4-bit keys without QJL
    "c2_corrected_norm": lambda: wl.config2(kv_heads=2, q_heads=8, max_len=1300, n_splits=4,
                                            key_corrected_norm=True, name="c2_corrected_norm"),
    "c3_corrected_norm": lambda: wl.config3(batch=2, max_len=700, min_len=300, n_splits=3,
                                            key_corrected_norm=True, name="c3_corrected_norm"),
    # the fast decode's key and value formats under a dense rotation (served by the general kernels)
    "c2_dense": lambda: wl.config2(kv_heads=2, q_heads=8, max_len=900, n_splits=3, rotation=wl.ROT_DENSE,
                                   rot_seed=11, name="c2_dense"),
}


# the same kernels with the tensor-core operands (H D, S D H) formed inside every thread
# block instead of prepared once per cache; the dense rotation without prepared operands
# compresses on the CUDA cores
IN_BLOCK = {
    "c3_unprepared_dense": lambda: wl.config3(batch=3, max_len=900, min_len=300, n_splits=2,
                                              name="c3_unprepared_dense"),
    "c2_in_block_operands": lambda: wl.config2(kv_heads=2, q_heads=8, max_len=1300, n_splits=4,
                                               name="c2_in_block_operands"),
    "c4_in_block_operands": lambda: wl.config4(batch=2, kv_heads=2, q_heads=8, max_len=2000, n_splits=8,
                                               name="c4_in_block_operands"),
    "c2_vqjl_in_block_operands": lambda: wl.config2(kv_heads=2, q_heads=8, max_len=1300, n_splits=4,
                                                    value_qjl=True, name="c2_vqjl_in_block_operands"),
}


@pytest.fixture(scope="module", params=sorted(SMALL) + sorted(IN_BLOCK))
def run(request):
    w = (SMALL.get(request.param) or IN_BLOCK[request.param])()
    layers = tuple(range(w.num_layers))
    r = setup(w, layers, prepared_operands=request.param not in IN_BLOCK)
    r.kv.raise_on_error("compress")
    r.pages = r.kv.pages_numpy()
    return r


def test_compress_bit_exact(run):
    rep = CompressReport()
    for layer in range(run.w.num_layers):
        for b in range(run.w.batch):
            for h in range(run.w.kv_heads):
                compare_compress(run, run.pages, layer, b, h, rep=rep)
    print(f"\n{run.w.name}: {rep}")
    record(f"compress {run.w.name}", rep)
    assert rep.idx_mismatch_out_of_band == 0
    assert rep.sign_mismatch_out_of_band == 0
    assert rep.norm_fail == 0
    assert rep.sign_tokens_skipped <= max(1, rep.tokens // 1000)


def test_decode_matches_oracle(run):
    seq = seq_dev(run)
    for layer in range(run.w.num_layers):
        q, qd = q_dev(run, layer)
        out = run.kv.decode(layer, qd, seq, run.w.n_splits)
        run.kv.raise_on_error("decode")
        ref = oracle_decode(run, run.pages, layer, q)
        ok = close(out.cpu().numpy(), ref)
        assert ok.all(), f"max |diff| {np.max(np.abs(out.cpu().numpy() - ref))}"


@pytest.mark.parametrize("n_splits", [1, 7, 1024])
def test_decode_split_count_invariance(run, n_splits):
    # more splits than pages leaves empty splits; results must not change beyond rounding
    seq = seq_dev(run)
    q, qd = q_dev(run, 0)
    out = run.kv.decode(0, qd, seq, n_splits).cpu().numpy()
    run.kv.raise_on_error("decode")
    ref = oracle_decode(run, run.pages, 0, q)
    assert close(out, ref).all()


def test_scores_match_oracle(run):
    seq = seq_dev(run)
    q, qd = q_dev(run, 0)
    sc = run.kv.scores(0, qd, seq, run.w.max_len).cpu().numpy()
    run.kv.raise_on_error("scores")
    for b in range(run.w.batch):
        n = int(run.lens[b])
        for h in range(run.w.q_heads):
            ref = oracle_scores(run, run.pages, 0, q, b, h)
            assert close(sc[b, h, :, :n], ref).all()
            assert np.all(np.isnan(sc[b, h, :, n:]))


def test_decompress_matches_oracle(run):
    from oracle import layout as olay
    from oracle import quant as oq
    seq = seq_dev(run)
    kh, vh = run.kv.decompress(0, seq, run.w.max_len)
    run.kv.raise_on_error("decompress")
    kh, vh = kh.cpu().numpy(), vh.cpu().numpy()
    for b in range(run.w.batch):
        n = int(run.lens[b])
        for h in range(run.w.kv_heads):
            u = olay.read_sequence(run.pages, run.fmt, 0, h, run.bt[b], n)
            assert close(kh[b, h, :n], oq.reconstruct_mse(u.k_idx, u.k_norm, run.R, run.ck, u.k_offset)).all()
            assert close(vh[b, h, :n], oq.reconstruct_mse(u.v_idx, u.v_norm, run.R, run.cv, u.v_offset)).all()
            assert np.all(kh[b, h, n:] == 0)


def test_end_to_end_quality_reported(run):
    # each side on its own cache is reported, not gated: the GPU output against exact
    # softmax attention on the raw inputs (the "output" of config 1)
    from oracle import attention as oatt
    seq = seq_dev(run)
    q, qd = q_dev(run, 0)
    out = run.kv.decode(0, qd, seq, run.w.n_splits).cpu().numpy()
    G = run.w.group
    cos = []
    for b in range(run.w.batch):
        n = int(run.lens[b])
        for h in range(run.w.q_heads):
            ex = oatt.softmax_attention(q[b, h], run.K[0][b, h // G][:n], run.V[0][b, h // G][:n])
            g = out[b, h]
            cos.append(np.sum(g * ex, -1) / (np.linalg.norm(g, axis=-1) * np.linalg.norm(ex, axis=-1) + 1e-30))
    print(f"\n{run.w.name}: mean cosine(GPU decode, exact attention) = {np.mean(cos):.4f}")
    assert np.mean(cos) > 0.5
