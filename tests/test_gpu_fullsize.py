"""GPU parity at the full workload sizes, in the launch configuration the benchmark times.

Configuration 1 (one head, 4096 fp32 tokens) is compared whole: every token's codes and every
output coordinate.  The larger caches are too big for the oracle to recompute whole, so each
check samples: cache pages spread over every sequence (and so over every persistent CTA's tile
loop) are compared code by code with the oracle's compression of the same rows, and every
query head of one sequence is decoded by the oracle over its full length and compared with
the GPU's output.  Tolerances are the parity contract's (parity_util); the counts the
tolerances allow are kept for the session summary."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import attention as oatt
from oracle import codebook as ocb
from oracle import layout as olay
from oracle import rotation as orot
from parity_util import CompressReport, close, compare_compress_rows, record

pytestmark = pytest.mark.gpu

# the benchmark decodes with the library's default split count for the GPU, except the
# long-context configuration, which fixes 64 splits per head
BENCH_DEFAULT_SPLITS = {1, 2, 3, 5}


def _pages_of(kv, layer, phys, head):
    blocks = kv.pages.view(kv.num_layers, kv.num_pages, kv.kv_heads, kv.block_bytes)
    idx = torch.as_tensor(np.asarray(phys, dtype=np.int64), device=kv.pages.device)
    return blocks[layer].index_select(0, idx)[:, head].cpu().numpy()  # [n][block]


def _read(kv, fmt, layer, head, phys, n):
    """Unpacked tokens 0..n-1 of a pseudo-sequence made of the given physical pages."""
    mini = _pages_of(kv, layer, phys, head)[None, :, None, :]
    return olay.read_sequence(mini, fmt, 0, 0, np.arange(len(phys)), n)


@pytest.fixture(scope="module", params=[1, 2, 3, 4, 5])
def full(request):
    from compressed_decode_attention_tq_b200.runtime import PagedKV
    c = request.param
    w = wl.CONFIGS[c]()
    lens = wl.seq_lens(w)
    bt, npages = wl.block_table(w, lens)
    rin = wl.rotation_inputs(w)
    kv = PagedKV(batch=w.batch, kv_heads=w.kv_heads, num_pages=npages, block_table=bt,
                 key_bits=w.key_bits, key_qjl=w.key_qjl, value_bits=w.value_bits,
                 rotation=w.rotation, num_layers=1, signs=rin["signs"], pi=rin["pi"], s=rin["s"])
    if c == 1:
        # small enough for the host draw: the exact configuration-1 recipe (fp32, iid N(0,1)
        # with four outlier channels x8)
        Kh, Vh = wl.make_kv(w, 0)
        K = torch.as_tensor(Kh, dtype=torch.float32, device="cuda")
        V = torch.as_tensor(Vh, dtype=torch.float32, device="cuda")
        q = torch.as_tensor(wl.make_q(w, 0), dtype=torch.float32, device="cuda")
    else:
        K, V = wl.make_kv_device(w, 0, "cuda")
        q = wl.make_q_device(w, 0, "cuda")
    seq = torch.as_tensor(lens, dtype=torch.int32, device="cuda")
    kv.compress(0, K, V, seq)
    kv.raise_on_error("compress")
    from compressed_decode_attention_tq_b200.runtime import default_splits
    ns = (default_splits(w.batch, w.kv_heads, rows=w.group * w.seq_q, max_len=w.max_len)
          if c in BENCH_DEFAULT_SPLITS else w.n_splits)
    out = kv.decode(0, q, seq, ns)
    kv.raise_on_error("decode")
    ck, kb = ocb.codebook_f32(w.key_bits, 128)
    cv, vb = ocb.codebook_f32(w.value_bits, 128)
    yield dict(c=c, w=w, lens=lens, bt=bt, rin=rin, kv=kv, K=K, V=V, q=q, out=out.cpu().numpy(),
               R=orot.rotation_matrix(w.rotation, rin["signs"], rin["pi"]),
               fmt=olay.Format(key_bits=w.key_bits, key_qjl=w.key_qjl, value_bits=w.value_bits),
               ck=ck, kb=kb, cv=cv, vb=vb)
    del kv, K, V
    torch.cuda.empty_cache()


def _sample_pairs(w, rng, count):
    pairs = {(0, 0), (w.batch - 1, w.kv_heads - 1)}
    while len(pairs) < min(count, w.batch * w.kv_heads):
        pairs.add((int(rng.integers(w.batch)), int(rng.integers(w.kv_heads))))
    return sorted(pairs)


def test_fullsize_compress_sampled(full):
    w, fmt = full["w"], full["fmt"]
    P = fmt.page_tokens
    rng = np.random.default_rng(1234 + full["c"])
    rep = CompressReport()
    for b, h in _sample_pairs(w, rng, 6):
        n = int(full["lens"][b])
        npg = (n + P - 1) // P
        if full["c"] == 1:
            lps = list(range(npg))  # the whole sequence
        else:
            lps = sorted({0, npg - 1, *rng.integers(0, npg, size=3).tolist()})
        # full pages first, a partial last page (ragged lengths) at the end
        lps = [lp for lp in lps if (lp + 1) * P <= n] + [lp for lp in lps if (lp + 1) * P > n]
        tok = np.concatenate([np.arange(lp * P, min(n, (lp + 1) * P)) for lp in lps])
        u = _read(full["kv"], fmt, 0, h, full["bt"][b][lps], len(tok))
        idx = torch.as_tensor(tok, device="cuda")
        Kr = full["K"][b, h].index_select(0, idx).double().cpu().numpy()
        Vr = full["V"][b, h].index_select(0, idx).double().cpu().numpy()
        compare_compress_rows(fmt, u, Kr, Vr, full["R"], full["ck"], full["kb"], full["cv"], full["vb"],
                              full["rin"]["s"], rep)
    print(f"config {full['c']}: {rep}")
    record(f"compress full-size config {full['c']} (sampled pages)" if full["c"] != 1
           else "compress full-size config 1 (every token)", rep)
    assert rep.tokens > 0
    assert rep.idx_mismatch_out_of_band == 0, rep
    assert rep.sign_mismatch_out_of_band == 0, rep
    assert rep.norm_fail == 0, rep
    assert rep.sign_tokens_skipped <= max(2, rep.tokens // 1000), rep


def test_fullsize_decode_every_head_of_one_sequence(full):
    w, fmt = full["w"], full["fmt"]
    rng = np.random.default_rng(99 + full["c"])
    b = int(rng.integers(w.batch))
    q = full["q"].double().cpu().numpy()
    P = fmt.page_tokens
    n = int(full["lens"][b])
    npg = (n + P - 1) // P
    worst = 0.0
    for kvh in range(w.kv_heads):
        u = _read(full["kv"], fmt, 0, kvh, full["bt"][b][:npg], n)
        hs = slice(kvh * w.group, (kvh + 1) * w.group)
        # the kv head's G query heads x seq_q rows in one oracle call (one reconstruction)
        ref = oatt.decode_sequence(q[b, hs].reshape(-1, 128), u, full["R"], full["ck"], full["cv"],
                                   full["rin"]["s"] if w.key_qjl else None).reshape(q[b, hs].shape)
        got = full["out"][b, hs]
        ok = close(got, ref)
        worst = max(worst, float(np.max(np.abs(got - ref) / (1e-3 + 2e-3 * np.abs(ref)))))
        assert ok.all(), (b, kvh, np.argwhere(~ok)[:5])
    summary = (f"sequence {b} ({n} tokens), all {w.q_heads} query heads x {w.seq_q} rows: "
               f"worst |d| / allowance = {worst:.3f}")
    print(f"config {full['c']}: {summary}")
    record(f"decode full-size config {full['c']}", summary)
