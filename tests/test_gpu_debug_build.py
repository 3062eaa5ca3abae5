"""The debug build (libtq_debug.so: every kernel's index checks compiled in, a failed check
recording TQ_ERR_BOUNDS in dev_status without trapping) runs the compress, decode and
decompress paths of several formats with no check firing, and gives the release library's
results."""
import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu

from parity_util import close, oracle_decode, q_dev, setup

CASES = {
    "c1": lambda: wl.config1(max_len=1000, n_splits=3),
    "c2": lambda: wl.config2(kv_heads=2, q_heads=8, max_len=1500, n_splits=5),
    "c3": lambda: wl.config3(batch=3, max_len=900, min_len=300, n_splits=3),
    "c5": lambda: wl.config5(kv_heads=2, q_heads=8, max_len=700, n_splits=2),
    "c2_vqjl": lambda: wl.config2(kv_heads=1, q_heads=4, max_len=600, n_splits=3, value_qjl=True),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_debug_build_checks_pass_and_match_release(name, monkeypatch):
    import compressed_decode_attention_tq_b200 as tq
    dbg = tq._load(tq.DEBUG_LIB_PATH)
    w = CASES[name]()
    # the release library's cache and outputs
    rel = setup(w)
    rel.kv.raise_on_error("release compress")
    seq = torch.as_tensor(rel.lens, dtype=torch.int32, device="cuda")
    q, qd = q_dev(rel)
    out_rel = rel.kv.decode(0, qd, seq, w.n_splits).cpu().numpy()
    pages_rel = rel.kv.pages_numpy()
    # the same calls through the debug library
    monkeypatch.setattr(tq, "lib", dbg)
    run = setup(w)
    assert run.kv.check() == 0, "a debug index check fired in compress"
    out = run.kv.decode(0, qd, seq, w.n_splits).cpu().numpy()
    assert run.kv.check() == 0, "a debug index check fired in decode"
    kh, vh = run.kv.decompress(0, seq, int(max(run.lens)))
    assert run.kv.check() == 0, "a debug index check fired in decompress"
    monkeypatch.undo()
    # the packed cache is the release library's byte for byte; the outputs agree with it and
    # with the oracle
    assert np.array_equal(run.kv.pages_numpy(), pages_rel)
    assert close(out, out_rel).all()
    assert close(out, oracle_decode(run, pages_rel, 0, q)).all()
    del kh, vh
