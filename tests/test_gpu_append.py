"""GPU parity of the incremental append ("tq-kv" crate documentation, incremental cache:
append a compressed token to the cache; "TurboQuant Limits And Assumptions": packed page
update) against the oracle: tq_append_kv alone, and a decode step with its append fused in
(tq_append_attend_decode).

Each case compresses all but the last few tokens of every sequence with tq_compress_kv,
then appends the rest in steps of one or more tokens, some of which cross a page boundary.
After the steps, every cached token (old and appended) must match the oracle's compression
of the same inputs under the compress tolerances; the tokens stored before the append must
be unchanged; each fused step's attention output must match the oracle's decode of the
cache as it stands after that step's append."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import layout as olay

pytestmark = pytest.mark.gpu

from parity_util import CompressReport, close, compare_compress, oracle_decode, setup

# (workload, append steps: new tokens per step).  The final lengths are chosen so that the
# appended positions cross a page boundary (multiples of 256) in at least one sequence.
CASES = {
    # fused fast path: 3-bit keys with QJL (merged nibbles), 3-bit values
    "c2": (lambda: wl.config2(kv_heads=2, q_heads=8, max_len=1283, n_splits=4), (1, 1, 3)),
    # generic path: dense rotation, 4-bit keys without QJL, ragged batch, permuted pages
    "c3": (lambda: wl.config3(batch=3, max_len=900, min_len=300, n_splits=2), (2, 1)),
    # fused fast path: 2-bit keys with the separate sign chunk, 2-bit values
    "c4": (lambda: wl.config4(batch=2, kv_heads=2, q_heads=8, max_len=1027, n_splits=8), (1, 4)),
    # fp32 inputs, one head
    "c1": (lambda: wl.config1(max_len=514, n_splits=3), (1, 1, 1)),
    # 32 query rows per kv head (four runs of the fast kernel)
    "c5": (lambda: wl.config5(kv_heads=2, q_heads=8, max_len=770, num_layers=1, n_splits=3), (2,)),
    # 1-bit keys, 4-bit values
    "k1v4": (lambda: wl.config2(kv_heads=1, q_heads=2, max_len=520, key_bits=1, value_bits=4,
                                n_splits=2, name="k1v4"), (1, 2)),
    # 4-bit keys with QJL (sign chunk) under a dense rotation, 1-bit values
    "k4qjl_v1_dense": (lambda: wl.config2(kv_heads=1, q_heads=3, max_len=300, key_bits=4,
                                          value_bits=1, rotation=wl.ROT_DENSE, rot_seed=9,
                                          n_splits=1, name="k4qjl_v1_dense"), (3,)),
    # values with QJL
    "c2_vqjl": (lambda: wl.config2(kv_heads=2, q_heads=8, max_len=1283, n_splits=4, value_qjl=True,
                                   name="c2_vqjl"), (1, 3)),
    "c3_vqjl_dense": (lambda: wl.config3(batch=2, max_len=700, min_len=300, n_splits=2, value_qjl=True,
                                         name="c3_vqjl_dense"), (2,)),
    # corrected key norms: merged QJL keys (fused fast path) and 4-bit MSE-only keys (dense)
    "c2_corrected_norm": (lambda: wl.config2(kv_heads=2, q_heads=8, max_len=1283, n_splits=4,
                                             key_corrected_norm=True, name="c2_corrected_norm"), (1, 3)),
    "c3_corrected_norm": (lambda: wl.config3(batch=2, max_len=700, min_len=300, n_splits=2,
                                             key_corrected_norm=True, name="c3_corrected_norm"), (2,)),
    # dithered: the new tokens' offsets through the _dithered calls (MSE-only 2-bit keys too)
    "c2_dither": (lambda: wl.config2(kv_heads=2, q_heads=8, max_len=1283, n_splits=4, dither=True,
                                     name="c2_dither"), (1, 3)),
    "k2v4_dither": (lambda: wl.config2(kv_heads=1, q_heads=4, max_len=520, key_bits=2, key_qjl=False,
                                       value_bits=4, n_splits=2, dither=True, name="k2v4_dither"), (2,)),
}


def _offsets(run, layer, after, n_new):
    """Dithered workloads: the offsets of positions after[b] - n_new .. after[b] - 1, as keyword
    arguments of the append calls (none otherwise)."""
    if not run.w.dither:
        return {}
    B, H = run.w.batch, run.w.kv_heads
    ko = np.zeros((B, H, n_new))
    vo = np.zeros((B, H, n_new))
    for b in range(B):
        p0 = int(after[b]) - n_new
        ko[b] = run.KO[layer][b, :, p0:p0 + n_new]
        vo[b] = run.VO[layer][b, :, p0:p0 + n_new]
    return dict(k_offsets=torch.as_tensor(ko, dtype=torch.float32, device="cuda").contiguous(),
                v_offsets=torch.as_tensor(vo, dtype=torch.float32, device="cuda").contiguous())


def _new_tokens(run, layer, after, n_new, dt):
    """k_new, v_new [batch][kv_heads][n_new][d] on the device: positions after[b] - n_new .. after[b] - 1."""
    B, H = run.w.batch, run.w.kv_heads
    kn = np.zeros((B, H, n_new, 128))
    vn = np.zeros((B, H, n_new, 128))
    for b in range(B):
        p0 = int(after[b]) - n_new
        kn[b] = run.K[layer][b, :, p0:p0 + n_new]
        vn[b] = run.V[layer][b, :, p0:p0 + n_new]
    return (torch.as_tensor(kn, dtype=dt, device="cuda").contiguous(),
            torch.as_tensor(vn, dtype=dt, device="cuda").contiguous())


def _prepare(name):
    make, steps = CASES[name]
    w = make()
    lens = wl.seq_lens(w)
    start = lens - sum(steps)
    assert (start >= 0).all()
    run = setup(w, (0,), compress_lens=start)
    run.kv.raise_on_error("compress")
    return run, steps, start


def _check_all_tokens(run, pages):
    rep = CompressReport()
    for b in range(run.w.batch):
        for h in range(run.w.kv_heads):
            compare_compress(run, pages, 0, b, h, rep=rep)
    assert rep.idx_mismatch_out_of_band == 0, rep
    assert rep.sign_mismatch_out_of_band == 0, rep
    assert rep.norm_fail == 0, rep
    assert rep.sign_tokens_skipped <= max(1, rep.tokens // 1000), rep
    return rep


def _check_old_tokens_unchanged(run, before, after, start):
    for b in range(run.w.batch):
        for h in range(run.w.kv_heads):
            n = int(start[b])
            u0 = olay.read_sequence(before, run.fmt, 0, h, run.bt[b], n)
            u1 = olay.read_sequence(after, run.fmt, 0, h, run.bt[b], n)
            for f in ("k_idx", "v_idx", "k_norm", "v_norm", "k_rnorm", "k_sigma", "v_rnorm", "v_sigma", "k_offset",
                      "v_offset"):
                a0, a1 = getattr(u0, f), getattr(u1, f)
                if a0 is not None:
                    np.testing.assert_array_equal(a0, a1, err_msg=f"{f} of b={b} h={h} changed")


@pytest.mark.parametrize("name", sorted(CASES))
def test_append_kv_matches_oracle(name):
    run, steps, start = _prepare(name)
    before = run.kv.pages_numpy()
    dt = torch.float16 if run.w.in_dtype == "f16" else torch.float32
    cur = start.copy()
    for n_new in steps:
        cur = cur + n_new
        kn, vn = _new_tokens(run, 0, cur, n_new, dt)
        run.kv.append(0, kn, vn, torch.as_tensor(cur, dtype=torch.int32, device="cuda"), **_offsets(run, 0, cur, n_new))
    run.kv.raise_on_error("append")
    assert (cur == run.lens).all()
    pages = run.kv.pages_numpy()
    rep = _check_all_tokens(run, pages)
    print(f"\n{name}: {rep}")
    _check_old_tokens_unchanged(run, before, pages, start)


@pytest.mark.parametrize("name", sorted(CASES))
def test_fused_append_decode_matches_oracle(name):
    run, steps, start = _prepare(name)
    before = run.kv.pages_numpy()
    dt = torch.float16 if run.w.in_dtype == "f16" else torch.float32
    q = wl.make_q(run.w, 0)
    qd = torch.as_tensor(q, dtype=dt, device="cuda")
    full = run.lens
    cur = start.copy()
    for n_new in steps:
        cur = cur + n_new
        kn, vn = _new_tokens(run, 0, cur, n_new, dt)
        seq = torch.as_tensor(cur, dtype=torch.int32, device="cuda")
        out = run.kv.decode(0, qd, seq, run.w.n_splits, k_new=kn, v_new=vn, **_offsets(run, 0, cur, n_new))
        run.kv.raise_on_error("append+decode")
        pages = run.kv.pages_numpy()
        run.lens = cur  # the oracle decodes the cache as it stands after this step
        ref = oracle_decode(run, pages, 0, q)
        got = out.cpu().numpy()
        ok = close(got, ref)
        assert ok.all(), f"step n_new={n_new}: max |diff| {np.max(np.abs(got - ref))}"
        # the same step as two calls gives the same result
        out2 = run.kv.decode(0, qd, seq, run.w.n_splits)
        run.kv.raise_on_error("decode")
        np.testing.assert_allclose(out2.cpu().numpy(), got, rtol=1e-6, atol=1e-6)
    run.lens = full
    pages = run.kv.pages_numpy()
    _check_all_tokens(run, pages)
    _check_old_tokens_unchanged(run, before, pages, start)


def test_append_bounds_are_reported_and_nothing_is_written():
    run, steps, start = _prepare("c2")
    before = run.kv.pages_numpy()
    kn, vn = _new_tokens(run, 0, start + 1, 1, torch.float16)
    # a length past the block-table row: reported, the token is not written
    bad = torch.full((run.w.batch,), run.kv.max_pages * 256 + 1, dtype=torch.int32, device="cuda")
    run.kv.append(0, kn, vn, bad)
    assert run.kv.check() == 6  # TQ_ERR_BOUNDS
    # a length shorter than the number of new tokens
    kn2, vn2 = _new_tokens(run, 0, np.maximum(start, 2), 2, torch.float16)
    short = torch.ones(run.w.batch, dtype=torch.int32, device="cuda")
    run.kv.append(0, kn2, vn2, short)
    assert run.kv.check() == 6
    np.testing.assert_array_equal(run.kv.pages_numpy(), before)
