"""GPU edge cases and device-side error reporting (no test faults or hangs the GPU: every
failure is a bounds-checked condition the kernels detect and report in dev_status)."""
import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu

from parity_util import close, oracle_decode, q_dev, setup


def _run(w):
    r = setup(w)
    r.pages = r.kv.pages_numpy()
    return r


def test_empty_and_single_token_sequences():
    w = wl.config2(batch=3, kv_heads=1, q_heads=4, max_len=300, n_splits=2)
    lens = np.array([0, 1, 257], dtype=np.int32)
    import parity_util as pu
    orig = wl.seq_lens
    try:
        wl.seq_lens = lambda _w: lens
        r = setup(w)
    finally:
        wl.seq_lens = orig
    r.kv.raise_on_error("compress")
    r.pages = r.kv.pages_numpy()
    seq = torch.as_tensor(lens, device="cuda")
    q, qd = q_dev(r)
    out = r.kv.decode(0, qd, seq, 4).cpu().numpy()
    r.kv.raise_on_error("decode")
    assert np.all(out[0] == 0)
    ref = oracle_decode(r, r.pages, 0, q)
    assert close(out, ref).all()


def test_sequence_longer_than_page_table_reports_bounds():
    w = wl.config2(kv_heads=1, q_heads=4, max_len=256, n_splits=1)
    r = _run(w)
    r.kv.raise_on_error("compress")
    seq = torch.tensor([600], dtype=torch.int32, device="cuda")  # 1 page in the table
    q, qd = q_dev(r)
    r.kv.decode(0, qd, seq, 1)
    assert r.kv.check() == 6
    k = torch.zeros((1, 1, 600, 128), dtype=torch.float16, device="cuda")
    r.kv.compress(0, k, k, seq)
    assert r.kv.check() == 6


def test_page_id_out_of_range_reports_bounds():
    from compressed_decode_attention_tq_b200.runtime import PagedKV
    rin = wl.rotation_inputs(wl.config2())
    kv = PagedKV(batch=1, kv_heads=1, num_pages=1, block_table=np.array([[5]]), key_bits=3, key_qjl=True,
                 value_bits=3, signs=rin["signs"], s=rin["s"])
    k = torch.randn((1, 1, 10, 128), device="cuda").half()
    seq = torch.tensor([10], dtype=torch.int32, device="cuda")
    kv.compress(0, k, k, seq)
    assert kv.check() == 6


def test_norm_overflow_reported():
    from compressed_decode_attention_tq_b200.runtime import PagedKV
    rin = wl.rotation_inputs(wl.config2())
    kv = PagedKV(batch=1, kv_heads=1, num_pages=1, block_table=np.array([[0]]), key_bits=3, key_qjl=True,
                 value_bits=3, signs=rin["signs"], s=rin["s"])
    k = torch.full((1, 1, 4, 128), 7000.0, device="cuda")  # ||k|| = 79196 > fp16 max
    seq = torch.tensor([4], dtype=torch.int32, device="cuda")
    kv.compress(0, k, k, seq)
    assert kv.check() == 4


def test_non_fp16_sketch_matrix_rejected():
    # compress forming S D H in every thread block takes S as an fp16 MMA operand, so S must
    # be fp16-exact there; prepared operands are formed in fp32 and accept any S
    from compressed_decode_attention_tq_b200.runtime import PagedKV
    rin = wl.rotation_inputs(wl.config2())
    s = rin["s"].copy()
    s[3, 5] = 0.1  # not representable in fp16
    k = torch.randn((1, 1, 4, 128), device="cuda").half()
    for prepared, expect in ((False, 1), (True, 0)):
        kv = PagedKV(batch=1, kv_heads=1, num_pages=1, block_table=np.array([[0]]), key_bits=3, key_qjl=True,
                     value_bits=3, signs=rin["signs"], s=s, prepared_operands=prepared)
        kv.compress(0, k, k, torch.tensor([4], dtype=torch.int32, device="cuda"))
        assert kv.check() == expect


def test_zero_vector_compresses_to_zero_norm():
    from compressed_decode_attention_tq_b200.runtime import PagedKV
    from oracle import layout as olay
    rin = wl.rotation_inputs(wl.config2())
    kv = PagedKV(batch=1, kv_heads=1, num_pages=1, block_table=np.array([[0]]), key_bits=3, key_qjl=True,
                 value_bits=2, signs=rin["signs"], s=rin["s"])
    k = torch.zeros((1, 1, 3, 128), dtype=torch.float16, device="cuda")
    seq = torch.tensor([3], dtype=torch.int32, device="cuda")
    kv.compress(0, k, k, seq)
    assert kv.check() == 0
    u = olay.read_sequence(kv.pages_numpy(), olay.Format(key_bits=3, value_bits=2), 0, 0, [0], 3)
    assert np.all(u.k_norm == 0) and np.all(u.v_norm == 0) and np.all(u.k_rnorm == 0)
    # y = 0 lies on the middle boundary: index h - 1 (tie to the lower cell); sign(0) -> +1
    assert np.all(u.k_idx == 3) and np.all(u.v_idx == 1) and np.all(u.k_sigma)


def test_bounded_wait_gives_up_and_the_context_stays_usable(monkeypatch):
    # a device wait that runs out: with TQ_DEBUG_BOUNDED_WAIT_US one warp of the tensor-core
    # split kernel waits 2 ms on a barrier nothing completes; the kernel reports
    # TQ_ERR_TIMEOUT through dev_status and returns, and the next call on the same context
    # (without the knob) matches the oracle
    w = wl.config2(kv_heads=2, q_heads=8, max_len=700, n_splits=3)
    r = _run(w)
    r.kv.raise_on_error("compress")
    seq = torch.as_tensor(r.lens, dtype=torch.int32, device="cuda")
    q, qd = q_dev(r)
    monkeypatch.setenv("TQ_DEBUG_BOUNDED_WAIT_US", "2000")
    r.kv.decode(0, qd, seq, w.n_splits)
    assert r.kv.check() == 5  # TQ_ERR_TIMEOUT
    monkeypatch.delenv("TQ_DEBUG_BOUNDED_WAIT_US")
    out = r.kv.decode(0, qd, seq, w.n_splits).cpu().numpy()
    assert r.kv.check() == 0
    assert close(out, oracle_decode(r, r.pages, 0, q)).all()


@pytest.mark.parametrize("fill", [0x00, 0xFF, 0x01])
def test_decode_ignores_what_the_workspace_held(fill):
    """The workspace is scratch: whatever it holds on entry (here every byte `fill`, so that
    every ready word of the query prologue reads as set, or as clear) the decode output equals
    the oracle's.  The prologue clears each part's ready word before the split kernel may
    start, so a stale word can never let the split kernel read query terms early."""
    import compressed_decode_attention_tq_b200 as tq
    w = wl.config2(kv_heads=2, q_heads=8, max_len=1500, n_splits=5)
    r = _run(w)
    r.kv.raise_on_error("compress")
    seq = torch.as_tensor(r.lens, dtype=torch.int32, device="cuda")
    q, qd = q_dev(r)
    ws = r.kv.workspace(qd.shape[1], qd.shape[2], 5)
    ref = oracle_decode(r, r.pages, 0, q)
    for _ in range(2):
        ws.fill_(fill)
        out = torch.empty(qd.shape, dtype=torch.float32, device="cuda")
        tq.attend_decode(r.kv.cfg, r.kv.params, r.kv.cache, 0, qd, seq, 5, ws, out, r.kv.status)
        r.kv.raise_on_error("decode")
        assert close(out.cpu().numpy(), ref).all()
