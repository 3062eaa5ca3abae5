"""The allocation-free decode entry point, tq_attend_decode_noalloc.

It exists for callers that cannot allocate device memory - a plugin inside a runtime that
owns the whole device memory pool, or a serving loop that must not call cudaMalloc in the
middle of a step - so it keeps its scratch in a fixed device array inside the library.
These tests call it through the C ABI and check it against tq_attend_decode (which takes a
caller workspace) on the same cache and queries, twice in a row with different inputs, so
that a second call cannot pass on what the first one left in the shared array.
This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu


# the tensor-core split kernel's workload (3-bit keys with QJL, 3-bit values) and one that
# takes the general kernels (values with QJL: the sign-space partials; dense rotation, 4-bit
# keys without QJL, G = 8): both use the scratch array, for different partials
CASES = {
    "fused": lambda: wl.config2(kv_heads=2, q_heads=8, max_len=1500, n_splits=4),
    "general": lambda: wl.config3(batch=2, max_len=700, min_len=300, n_splits=3, value_qjl=True),
}


@pytest.fixture(scope="module", params=sorted(CASES))
def run(request):
    from parity_util import setup
    r = setup(CASES[request.param]())
    r.kv.raise_on_error("compress")
    return r


def _noalloc(run, q, seq, n_splits):
    import compressed_decode_attention_tq_b200 as tq
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    kv = run.kv
    st = tq.lib.tq_attend_decode_noalloc(
        ctypes.byref(kv.cfg), ctypes.byref(kv.params), ctypes.byref(kv.cache), 0, q.data_ptr(),
        tq.dtype_code(q), q.shape[1], q.shape[2], seq.data_ptr(), n_splits, out.data_ptr(),
        kv.status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == tq.TQ_OK, tq.last_error()
    return out


def test_noalloc_matches_workspace_decode_on_two_calls_in_a_row(run):
    from parity_util import close
    seq = torch.as_tensor(run.lens, dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(123)
    q1 = torch.randn((run.w.batch, run.w.q_heads, 1, 128), generator=g, device="cuda").half()
    q2 = torch.randn((run.w.batch, run.w.q_heads, 1, 128), generator=g, device="cuda").half() * 3
    got1 = _noalloc(run, q1, seq, 16)
    got2 = _noalloc(run, q2, seq, 5)
    run.kv.raise_on_error("noalloc decode")
    ref1 = run.kv.decode(0, q1, seq, 16)
    ref2 = run.kv.decode(0, q2, seq, 5)
    run.kv.raise_on_error("workspace decode")
    for got, ref in ((got1, ref1), (got2, ref2)):
        g_, r_ = got.cpu().numpy(), ref.cpu().numpy()
        assert np.isfinite(g_).all()
        assert close(g_, r_).all()
    assert not np.allclose(got1.cpu().numpy(), got2.cpu().numpy())


def test_noalloc_rejects_sizes_beyond_its_buffer(run):
    import compressed_decode_attention_tq_b200 as tq
    seq = torch.as_tensor(run.lens, dtype=torch.int32, device="cuda")
    q = torch.zeros((run.w.batch, run.w.q_heads, 4, 128), dtype=torch.float16, device="cuda")
    out = torch.zeros(q.shape, dtype=torch.float32, device="cuda")
    kv = run.kv
    # 8 heads x 4 rows x 1024 splits of (128 + 2) floats needs about 17 MB > 8 MiB
    st = tq.lib.tq_attend_decode_noalloc(
        ctypes.byref(kv.cfg), ctypes.byref(kv.params), ctypes.byref(kv.cache), 0, q.data_ptr(),
        tq.TQ_F16, q.shape[1], q.shape[2], seq.data_ptr(), 1024, out.data_ptr(), kv.status.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st == tq.TQ_ERR_UNSUPPORTED
    assert "8 MiB" in tq.last_error()
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
