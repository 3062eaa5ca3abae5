"""Benchmark of the TurboQuant compressed-KV hot path on B200.

One step = one pass of the whole path over a Llama-3-8B-shaped model cache: for each of
32 layers (8 KV heads x 32768 tokens, head_dim 128, fp16 K/V drawn with the config-2
recipe) compress K (3-bit + QJL) and V (3-bit) into the packed paged cache, then run
decode attention for 32 query heads (seq_q = 1) over every layer.  Inputs (4.3 GB of
K/V, plus the 0.99 GB packed cache) are larger than L2, so no flush is needed.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank runs its own replica (the work shards by independent
layer/head units, no data-path collective); value = all ranks' units / max-over-ranks time.
--impl reference times the CPU oracle (double precision, numpy) on a bounded sample.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode KV-tokens/s and achieved HBM GB/s (% of B200 roofline); keys compressed/s"
UNIT = "KV-tokens/s"  # token x kv-head positions compressed and then scanned by decode, per second
FALLBACK_HBM = 6650.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--layers", type=int, default=32)
    p.add_argument("--e2e-steps", type=int, default=2)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--n-splits", type=int, default=0, help="override the split count")
    p.add_argument("--no-configs", action="store_true", help="skip the per-workload one-layer timings")
    return p.parse_args()


B200_SMS = 148  # SM count of the target GPU, used where no GPU can be queried


def sm_count(device_index: int = 0) -> int:
    try:
        import torch
        if torch.cuda.is_available():
            return torch.cuda.get_device_properties(device_index).multi_processor_count
    except Exception:
        pass
    return B200_SMS


def workload(n_splits: int = 0, device_index: int = 0):
    """The benchmark layer (configuration 2) with the decode split count both arms report:
    the override if given, else the library's default for this GPU (B200's 148 SMs when
    there is none)."""
    import workloads as wl
    from compressed_decode_attention_tq_b200.runtime import splits_for
    w = wl.config2()
    w.n_splits = n_splits or splits_for(w.batch, w.kv_heads, sm_count(device_index), rows=w.group * w.seq_q,
                                        max_len=w.max_len)
    return w


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM, "fallback"


# the sources each timed kernel is built from (its traffic entry is void once any changes)
KERNEL_SOURCES = {
    "compress_tc_kernel": ("compress_tc.cu", "tq_device.cuh", "tq_kernels.h"),
    "fast_split_kernel": ("decode_fast.cu", "decode.cu", "tq_device.cuh", "tq_kernels.h"),
}


def _code_only(text: str) -> str:
    """C++ source without comments and whitespace: what the compiler sees of it (string
    literals in these sources hold no comment markers)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return re.sub(r"\s+", "", text)


def kernel_hash(kernel: str) -> str:
    h = hashlib.sha256()
    src = os.path.join(ROOT, "compressed_decode_attention_tq_b200", "csrc")
    for name in KERNEL_SOURCES.get(kernel, tuple(sorted(os.listdir(src)))):
        with open(os.path.join(src, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, or None when the
    summary is missing or was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        ent = d[kernel]
        if ent.get("source_hash") != kernel_hash(kernel):
            return None
        return float(ent["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# oracle timing (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([int(i.get("num_threads", 1)) for i in threadpool_info()] or [1])
    except Exception:
        return 1


def oracle_sample(tokens: int, heads: int, single_thread: bool = False):
    """Times the oracle on `heads` KV heads of layer 0, `tokens` tokens each: compress K (3-bit
    + QJL) and V (3-bit), pack, decode the G query heads of each KV head.  Returns
    (token*kv-heads processed, seconds, threads).  single_thread: the BLAS thread pool limited
    to one thread."""
    if single_thread:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            u, dt, _ = oracle_sample(tokens, heads)
        return u, dt, 1
    import numpy as np
    import workloads as wl
    from oracle import attention as oatt, codebook as ocb, layout as olay, quant as oq, rotation as orot
    w = workload()
    w1 = wl.config2(max_len=tokens)
    rin = wl.rotation_inputs(w)
    R = orot.rotation_matrix(w.rotation, rin["signs"], rin["pi"])
    ck, kb = ocb.codebook_f32(w.key_bits, 128)
    cv, vb = ocb.codebook_f32(w.value_bits, 128)
    K, V = wl.make_kv(w1, 0, heads=list(range(heads)))
    q = wl.make_q(w1)[:, : heads * w.group]
    fmt = olay.Format(key_bits=w.key_bits, key_qjl=w.key_qjl, value_bits=w.value_bits)
    lens = np.array([tokens], dtype=np.int32)
    npg = (tokens + 255) // 256
    bt = np.arange(npg, dtype=np.int32)[None]
    t0 = time.perf_counter()
    cache = olay.empty_cache(fmt, npg, heads)
    for h in range(heads):
        kc = oq.compress_prod(K[0, h], R, ck, kb, rin["s"])
        vc = oq.compress_mse(V[0, h], R, cv, vb)
        olay.write_sequence(cache, fmt, 0, h, bt[0], kc, vc)
    oatt.decode(cache, fmt, 0, q, bt, lens, R, ck, cv, rin["s"])
    dt = time.perf_counter() - t0
    return tokens * heads, dt, blas_threads()


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = workload(args.n_splits)
    tokens, heads = w.max_len, 1
    for _ in range(args.warmup):
        oracle_sample(tokens, heads)
    tot_units, tot_s, threads = 0, 0.0, 1
    for _ in range(args.steps):
        u, s, threads = oracle_sample(tokens, heads)
        tot_units += u
        tot_s += s
    value = tot_units / tot_s
    sample = f"layer 0, 1 of 8 KV heads, {tokens} tokens per step (compress K/V + pack + decode 4 query heads)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w, args.layers),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": os.cpu_count() or 1, "threads": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(w, layers):
    return {"workload": "llama3_8b_32k_32layers: config-2 layer (8 KV heads x 32768 tokens, 32 q heads, "
                        "fp16 K/V Gaussian x lognormal(0,0.5) channel scales + 2% outlier channels x10) "
                        "x 32 layers; compress K 3-bit+QJL / V 3-bit, then decode seq_q=1",
            "model": "Llama-3-8B KV shape", "layers": layers, "global_batch": w.batch,
            "seq_len": w.max_len, "kv_heads": w.kv_heads, "q_heads": w.q_heads, "seq_q": w.seq_q,
            "head_dim": 128, "key_bits": w.key_bits, "key_qjl": w.key_qjl, "value_bits": w.value_bits,
            "page_tokens": 256, "n_splits": w.n_splits, "rotation": "hadamard",
            "l2": "inputs larger than L2 (4.3 GB K/V read + 0.99 GB packed cache per step); no flush",
            "value_is": "token x kv-head positions compressed and then decoded per second of the whole "
                        "step (compress of 32 layers, then decode of 32 layers); the metric's separate "
                        "figures are in phases: decode kv_tokens_per_s, compress keys_per_s, each with "
                        "its HBM GB/s and roofline fraction",
            "parallelism": "replicas"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank contributes its own and receives the maximum
    (one process per GPU; with one rank the time itself)."""
    if world == 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the units all ranks processed in one step (each rank the same
    amount: weak scaling) per second of the slowest rank's step."""
    return world * units_per_rank / (ms_per_step / 1e3)


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import workloads as wl
    from compressed_decode_attention_tq_b200.runtime import PagedKV

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = workload(args.n_splits, local_rank)
    L = args.layers
    rin = wl.rotation_inputs(w)
    lens = wl.seq_lens(w)
    bt, npages = wl.block_table(w, lens)
    kv = PagedKV(batch=w.batch, kv_heads=w.kv_heads, num_pages=npages, block_table=bt,
                 key_bits=w.key_bits, key_qjl=w.key_qjl, value_bits=w.value_bits, rotation=w.rotation,
                 num_layers=L, signs=rin["signs"], pi=rin["pi"], s=rin["s"], device=str(dev))
    seq = torch.as_tensor(lens, dtype=torch.int32, device=dev)
    Ks, Vs, Qs, Outs = [], [], [], []
    for l in range(L):
        k, v = wl.make_kv_device(w, l, dev)
        Ks.append(k)
        Vs.append(v)
        Qs.append(wl.make_q_device(w, l, dev))
        Outs.append(torch.empty(Qs[-1].shape, dtype=torch.float32, device=dev))
    kv.workspace(w.q_heads, w.seq_q, w.n_splits)
    stream = torch.cuda.current_stream(dev)
    units = L * w.batch * w.kv_heads * int(lens.sum() // w.batch)  # token x kv-head per step
    tok_heads_layer = int(lens.sum()) * w.kv_heads

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        for l in range(L):
            kv.compress(l, Ks[l], Vs[l], seq, stream)
        if ev is not None:
            ev[1].record(stream)
        for l in range(L):
            kv.decode(l, Qs[l], seq, w.n_splits, out=Outs[l], stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    kv.raise_on_error("warmup")
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    phase_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        start.record(stream)
        for i in range(args.steps):
            step(phase_ev[i])
        end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    ms = max_over_ranks(start.elapsed_time(end), world, dev)
    kv.raise_on_error("timed steps")
    ms_step = ms / args.steps
    comp_ms = sum(e[0].elapsed_time(e[1]) for e in phase_ev) / args.steps
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in phase_ev) / args.steps
    value = job_value(units, world, ms_step)

    hbm, peak_kind = peaks()
    comp_bytes_launch = tok_heads_layer * (2 * 128 * 2 + kv.block_bytes / 256)
    dec_bytes_launch = tok_heads_layer * (kv.block_bytes / 256) + \
        w.batch * w.q_heads * w.seq_q * 128 * (2 + 4)
    comp_gbs = comp_bytes_launch / (comp_ms / L / 1e3) / 1e9
    dec_gbs = dec_bytes_launch / (dec_ms / L / 1e3) / 1e9
    phases = {
        "compress": {"kernel": "compress_tc_kernel", "ms_per_step": comp_ms, "launches_per_step": L,
                     "keys_per_s": L * tok_heads_layer / (comp_ms / 1e3),
                     "algorithmic_bytes_per_launch": comp_bytes_launch, "achieved_gbs": comp_gbs,
                     "frac": comp_gbs / hbm},
        "decode": {"kernel": "fast_split_kernel", "ms_per_step": dec_ms, "launches_per_step": 2 * L,
                   "kernels": "query_kernel + fast_split_kernel",
                   "kv_tokens_per_s": L * tok_heads_layer / (dec_ms / 1e3),
                   "algorithmic_bytes_per_launch": dec_bytes_launch, "achieved_gbs": dec_gbs,
                   "frac": dec_gbs / hbm},
    }
    dom = "compress" if comp_ms >= dec_ms else "decode"
    ph = phases[dom]
    roofline = {"kernel": ph["kernel"], "bound": "hbm", "achieved": ph["achieved_gbs"], "peak": hbm,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                else "fallback 6650 GB/s", "unit": "GB/s", "frac": ph["achieved_gbs"] / hbm,
                "traffic": traffic_for(ph["kernel"])}

    e2e = None
    if not args.no_e2e and args.e2e_steps > 0:
        e2e = run_e2e(args, kv, w, L, Ks, Vs, Qs, Outs, seq, stream, dev, units, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        u, s, threads = oracle_sample(w.max_len, 1)
        u1, s1, _ = oracle_sample(w.max_len // 4, 1, single_thread=True)
        cpu = {"value": u / s, "unit": UNIT, "cores": os.cpu_count() or 1, "threads": threads,
               "kind": "oracle",
               "sample": f"layer 0, 1 of 8 KV heads, {w.max_len} tokens: compress K/V + pack + "
                         f"decode 4 query heads ({s:.1f} s, BLAS pool of {threads} threads on "
                         f"{os.cpu_count()} host cores)",
               "single_thread": {"value": u1 / s1, "unit": UNIT,
                                 "sample": f"the same on {w.max_len // 4} tokens with one thread ({s1:.1f} s)"}}

    configs = None
    if rank == 0 and not args.no_configs:
        configs = config_timings(dev)
    quality = reconstruction_quality(kv, w, Ks[0], Vs[0], Qs[0], seq) if rank == 0 else None

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_dict(w, L), "phases": phases, "roofline": roofline,
            "cpu_baseline": cpu, "e2e": e2e, "configs": configs, "quality": quality,
            # per layer: compress_tc_kernel, then query_kernel + fast_split_kernel
            "gpu_launches": args.steps * L * 3,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)


def reconstruction_quality(kv, w, K, V, q, seq):
    """What the packed cache keeps of layer 0 (outside the timed region): the compression
    ratio against fp16 K/V; for keys (their MSE stage) and values, the relative squared error
    of the library's decompression and the mean cosine similarity per vector; the relative
    RMS error of the score estimator (MSE term + QJL term, from the score-only call) against
    the exact q.k / sqrt(d); and the cosine similarity of each decode output row with exact
    softmax attention over the fp16 K/V (PyTorch fp32, for this measurement only)."""
    import torch
    T = K.shape[2]

    def recon(x, xh):
        x = x.float()
        err = ((x - xh) ** 2).sum(-1)
        ref = (x ** 2).sum(-1)
        cos = (x * xh).sum(-1) / (x.norm(dim=-1) * xh.norm(dim=-1)).clamp_min(1e-30)
        return {"relative_mse": float(err.sum() / ref.sum()), "mean_cosine": float(cos.mean())}

    kh, vh = kv.decompress(0, seq, T)
    keys, values = recon(K, kh), recon(V, vh)
    del kh, vh
    G = w.q_heads // w.kv_heads
    Kr = K.float().repeat_interleave(G, dim=1)
    exact = torch.einsum("bhsd,bhtd->bhst", q.float(), Kr) / math.sqrt(128.0)
    del Kr
    est = kv.scores(0, q, seq, T)
    score_err = float(((est - exact) ** 2).mean().sqrt() / (exact ** 2).mean().sqrt())
    del est
    out = kv.decode(0, q, seq, w.n_splits)
    Vr = V.float().repeat_interleave(G, dim=1)
    ref = torch.einsum("bhst,bhtd->bhsd", torch.softmax(exact, dim=-1), Vr)
    cos = (out * ref).sum(-1) / (out.norm(dim=-1) * ref.norm(dim=-1)).clamp_min(1e-30)
    kv.raise_on_error("quality")
    del Vr, exact, ref
    torch.cuda.empty_cache()
    return {
        "layer": 0,
        "compression_ratio_vs_fp16": 2 * 128 * 2 / (kv.block_bytes / 256),
        "keys_mse_stage": keys,
        "values": values,
        "score_relative_rms_error": score_err,
        "decode_output_cosine": {"min": float(cos.min()), "mean": float(cos.mean())},
    }


def config_timings(dev, reps: int = 10):
    """One layer of every workload at full size: compress and decode each timed alone with CUDA
    events around the launch, L2 flushed before every timed launch (a 256 MB buffer written and
    read back, so that no dirty lines are left to write back during the timed launch).  Returns
    {config: {...}} with the microseconds per call, the kernel path taken and the HBM GB/s of
    the algorithmic bytes (compress: inputs read + packed bytes written; decode: packed bytes
    read + q in and out)."""
    import torch
    import workloads as wl
    from compressed_decode_attention_tq_b200.runtime import PagedKV, default_splits
    hbm, _ = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    res = {}
    # the five workloads, then the config-2 layer in the other formats of the library: values
    # with QJL, dithered HD, corrected key norms
    cases = [(str(c), c, wl.CONFIGS[c]) for c in (1, 2, 3, 4, 5)]
    cases += [("2_value_qjl", 2, lambda: wl.config2(value_qjl=True, name="c2_value_qjl")),
              ("2_dither", 2, lambda: wl.config2(dither=True, name="c2_dither")),
              ("2_corrected_norm", 2, lambda: wl.config2(key_corrected_norm=True, name="c2_corrected_norm"))]
    for key, c, make in cases:
        w = make()
        lens = wl.seq_lens(w)
        bt, npages = wl.block_table(w, lens)
        rin = wl.rotation_inputs(w)
        kv = PagedKV(batch=w.batch, kv_heads=w.kv_heads, num_pages=npages, block_table=bt,
                     key_bits=w.key_bits, key_qjl=w.key_qjl, value_bits=w.value_bits, rotation=w.rotation,
                     num_layers=1, signs=rin["signs"], pi=rin["pi"], s=rin["s"], device=str(dev),
                     value_qjl=w.value_qjl, dither=w.dither, key_corrected_norm=w.key_corrected_norm)
        offs = {}
        if w.dither:
            t = kv.tensors
            offs = dict(zip(("k_offsets", "v_offsets"), wl.dither_offsets_device(
                w, 0, 0.5 * float(t["kc"][1] - t["kc"][0]), 0.5 * float(t["vc"][1] - t["vc"][0]), dev)))
        if c == 1:
            Kh, Vh = wl.make_kv(w, 0)
            K = torch.as_tensor(Kh, dtype=torch.float32, device=dev)
            V = torch.as_tensor(Vh, dtype=torch.float32, device=dev)
            q = torch.as_tensor(wl.make_q(w, 0), dtype=torch.float32, device=dev)
        else:
            K, V = wl.make_kv_device(w, 0, dev)
            q = wl.make_q_device(w, 0, dev)
        seq = torch.as_tensor(lens, dtype=torch.int32, device=dev)
        # the library's default split count, except where the workload fixes it (64 splits
        # per head for the long-context workload)
        ns = (w.n_splits if c == 4 else
              default_splits(w.batch, w.kv_heads, dev.index or 0, rows=w.group * w.seq_q, max_len=w.max_len))
        out = torch.empty(q.shape, dtype=torch.float32, device=dev)

        def timed(fn):
            fn()
            tot = 0.0
            for _ in range(reps):
                # writing the buffer evicts the cache's lines; reading it back evicts the written
                # ones, so that the timed launch meets no write-back traffic
                flush.zero_()
                flush.sum()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                b.synchronize()
                tot += a.elapsed_time(b)
            return 1e3 * tot / reps

        comp_us = timed(lambda: kv.compress(0, K, V, seq, stream, **offs))
        dec_us = timed(lambda: kv.decode(0, q, seq, ns, out=out, stream=stream))
        kv.raise_on_error(f"config {key}")
        tokh = int(lens.sum()) * w.kv_heads
        in_b = 2 if w.in_dtype == "f16" else 4
        per_tok = kv.block_bytes / 256
        comp_bytes = tokh * (2 * 128 * in_b + per_tok)
        dec_bytes = tokh * per_tok + w.batch * w.q_heads * w.seq_q * 128 * (in_b + 4)
        res[key] = {
            "workload": w.name, "n_splits": ns, "seq_q": w.seq_q,
            "compress_us": comp_us, "compress_gbs": comp_bytes / comp_us / 1e3,
            "compress_frac": comp_bytes / comp_us / 1e3 / hbm,
            "keys_per_s": tokh / (comp_us * 1e-6),
            "decode_us": dec_us, "decode_gbs": dec_bytes / dec_us / 1e3,
            "decode_frac": dec_bytes / dec_us / 1e3 / hbm,
            "kv_tokens_per_s": tokh / (dec_us * 1e-6),
            "bytes_per_token_kv_head": per_tok,
            "l2": "flushed before every timed launch (a 256 MB buffer written, then read back)",
        }
        del kv, K, V, q, out, offs
        torch.cuda.empty_cache()
    return res


def run_e2e(args, kv, w, L, Ks, Vs, Qs, Outs, seq, stream, dev, units, world):
    """Same step through the public API starting from pinned host buffers: H2D of the step's
    K/V/q, compress + decode, D2H of the outputs, all inside the timed region."""
    import torch
    hK = [torch.empty(k.shape, dtype=k.dtype, pin_memory=True) for k in Ks]
    hV = [torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for v in Vs]
    hQ = [torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for q in Qs]
    hO = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in Outs]
    for l in range(L):
        hK[l].copy_(Ks[l])
        hV[l].copy_(Vs[l])
        hQ[l].copy_(Qs[l])
    torch.cuda.synchronize(dev)
    h2d = sum(t.numel() * t.element_size() for t in hK + hV + hQ)
    d2h = sum(t.numel() * t.element_size() for t in hO)

    def step():
        for l in range(L):
            Ks[l].copy_(hK[l], non_blocking=True)
            Vs[l].copy_(hV[l], non_blocking=True)
            Qs[l].copy_(hQ[l], non_blocking=True)
            kv.compress(l, Ks[l], Vs[l], seq, stream)
        for l in range(L):
            kv.decode(l, Qs[l], seq, w.n_splits, out=Outs[l], stream=stream)
            hO[l].copy_(Outs[l], non_blocking=True)

    step()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(args.e2e_steps):
        step()
    e.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(s.elapsed_time(e), world, dev)
    kv.raise_on_error("e2e")
    return {"value": job_value(units, world, ms / args.e2e_steps), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
