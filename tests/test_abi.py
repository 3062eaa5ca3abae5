"""CPU tests of the C ABI: the library loads, exports what include/tq.h declares, and its
host-only logic (codebook, sizes, argument checks) behaves as documented.  No kernel runs."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def tq():
    import compressed_decode_attention_tq_b200 as m
    return m


def test_every_declared_symbol_is_exported(tq):
    declared = _declared_functions()
    assert set(declared) == set(tq.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", tq.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\b(tq_[a-z_0-9]+)\b", out))
    assert set(declared) <= exported
    # nothing else leaks out of the library under the tq_ prefix
    assert exported == set(declared)


def test_debug_library_exports_the_same_symbols(tq):
    """libtq_debug.so (the kernels' index checks compiled in) is built beside libtq.so and
    exports exactly the calls tq.h declares."""
    assert os.path.exists(tq.DEBUG_LIB_PATH), "build() makes libtq_debug.so as well"
    out = subprocess.run(["nm", "-D", "--defined-only", tq.DEBUG_LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    assert set(re.findall(r"\b(tq_[a-z_0-9]+)\b", out)) == set(_declared_functions())
    dbg = tq._load(tq.DEBUG_LIB_PATH)
    assert dbg.tq_version() == tq.lib.tq_version()


def test_version_and_status_strings(tq):
    assert tq.lib.tq_version() >= 100
    assert tq.status_str(0) == "TQ_OK"
    assert tq.status_str(6) == "TQ_ERR_BOUNDS"


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("density", [0, 1])
def test_library_codebook_equals_oracle_codebook(tq, bits, density):
    from oracle import codebook as ocb
    c, b = tq.codebook(bits, 128, density)
    oc, ob = ocb.codebook_f32(bits, 128, "beta" if density == 0 else "gauss")
    np.testing.assert_array_equal(c, oc)
    np.testing.assert_array_equal(b, ob)


@pytest.mark.parametrize("d", [16, 64])
def test_library_codebook_other_d(tq, d):
    from oracle import codebook as ocb
    c, b = tq.codebook(3, d, 0)
    oc, ob = ocb.codebook_f32(3, d, "beta")
    np.testing.assert_array_equal(c, oc)
    np.testing.assert_array_equal(b, ob)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("density", [0, 1])
def test_library_dither_codebook_equals_oracle(tq, bits, density):
    from oracle import codebook as ocb
    c, b = tq.dither_codebook(bits, 128, density)
    oc, ob = ocb.dither_codebook_f32(bits, 128, "beta" if density == 0 else "gauss")
    np.testing.assert_array_equal(c, oc)
    np.testing.assert_array_equal(b, ob)


def test_dither_codebook_argument_errors(tq):
    c = np.zeros(4, np.float32)
    b = np.zeros(3, np.float32)
    assert tq.lib.tq_dither_codebook(0, 128, 0, c.ctypes.data, b.ctypes.data) == tq.TQ_ERR_INVALID_ARG
    assert tq.lib.tq_dither_codebook(2, 2, 0, c.ctypes.data, b.ctypes.data) == tq.TQ_ERR_INVALID_ARG
    assert tq.lib.tq_dither_codebook(2, 128, 9, c.ctypes.data, b.ctypes.data) == tq.TQ_ERR_INVALID_ARG
    assert tq.lib.tq_dither_codebook(2, 128, 0, c.ctypes.data, None) == tq.TQ_ERR_INVALID_ARG


def test_dither_and_corrected_norm_config(tq):
    from oracle import layout as olay
    for kb, qjl, vb in ((3, True, 3), (2, False, 4), (1, True, 1)):
        cfg = tq.make_config(key_bits=kb, key_qjl=qjl, value_bits=vb, dither=True)
        assert tq.validate_config(cfg) == 0
        fmt = olay.Format(key_bits=kb, key_qjl=qjl, value_bits=vb, dither=True)
        assert tq.page_bytes(cfg) == fmt.block_bytes
        assert tq.page_bytes(cfg) == tq.page_bytes(tq.make_config(key_bits=kb, key_qjl=qjl, value_bits=vb)) + 4 * 256
    # dithered HD only; corrected norms change no byte of the format
    assert tq.validate_config(tq.make_config(dither=True, rotation=tq.TQ_ROT_DENSE)) == tq.TQ_ERR_UNSUPPORTED
    cn = tq.make_config(key_corrected_norm=True)
    assert tq.validate_config(cn) == 0 and tq.page_bytes(cn) == tq.page_bytes(tq.make_config())
    bad = tq.make_config()
    bad.dither = 2
    assert tq.validate_config(bad) == tq.TQ_ERR_INVALID_ARG
    bad = tq.make_config()
    bad.key_corrected_norm = -1
    assert tq.validate_config(bad) == tq.TQ_ERR_INVALID_ARG


def test_dithered_compress_entry_points_check_the_mode(tq):
    by = ctypes.byref
    params, cache = tq.tq_params(), tq.tq_cache()
    dith = tq.make_config(dither=True)
    st = tq.lib.tq_compress_kv(by(dith), by(params), by(cache), 0, None, None, 0, 16, None, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "tq_compress_kv_dithered" in tq.last_error()
    plain = tq.make_config()
    st = tq.lib.tq_compress_kv_dithered(by(plain), by(params), by(cache), 0, None, None, None, None, 0, 16,
                                        None, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "dither" in tq.last_error()
    st = tq.lib.tq_compress_kv_dithered(by(dith), by(params), by(cache), 0, None, None, None, None, 0, 16,
                                        None, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "offsets" in tq.last_error()
    # appends take no offsets
    buf = ctypes.create_string_buffer(64)
    p = ctypes.addressof(buf)
    params = tq.make_params()
    params.signs = params.k_centroids = params.v_centroids = params.k_boundaries = params.v_boundaries = p
    params.s = (p + 15) & ~15
    cache = tq.tq_cache(p, p, 1, 1, 1, 1, 1)
    st = tq.lib.tq_append_kv(by(dith), by(params), by(cache), 0, p, p, 0, 1, p, None, None)
    assert st == tq.TQ_ERR_UNSUPPORTED and "offsets" in tq.last_error()
    # ... through the _dithered calls, which a plain cache and missing offsets are refused by
    st = tq.lib.tq_append_kv_dithered(by(tq.make_config()), by(params), by(cache), 0, p, p, p, p, 0, 1, p, None,
                                      None)
    assert st == tq.TQ_ERR_INVALID_ARG and "dither" in tq.last_error()
    st = tq.lib.tq_append_kv_dithered(by(dith), by(params), by(cache), 0, p, p, None, p, 0, 1, p, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "offsets" in tq.last_error()


def test_codebook_argument_errors(tq):
    c = np.zeros(4, np.float32)
    b = np.zeros(3, np.float32)
    assert tq.lib.tq_codebook(0, 128, 0, c.ctypes.data, b.ctypes.data) == tq.TQ_ERR_INVALID_ARG
    assert "bits" in tq.last_error()
    assert tq.lib.tq_codebook(2, 2, 0, c.ctypes.data, b.ctypes.data) == tq.TQ_ERR_INVALID_ARG
    assert tq.lib.tq_codebook(2, 128, 5, c.ctypes.data, b.ctypes.data) == tq.TQ_ERR_INVALID_ARG
    assert tq.lib.tq_codebook(2, 128, 0, None, b.ctypes.data) == tq.TQ_ERR_INVALID_ARG


def test_page_bytes_match_format(tq, packing_golden):
    g = packing_golden["c2_regions"]
    cfg = tq.make_config(key_bits=3, key_qjl=True, value_bits=3)
    assert tq.page_bytes(cfg) == g["total"]
    from oracle import layout as olay
    for kb in range(1, 5):
        for vb in range(1, 5):
            for qjl in (False, True):
                for vqjl in (False, True):
                    cfg = tq.make_config(key_bits=kb, key_qjl=qjl, value_bits=vb, value_qjl=vqjl)
                    fmt = olay.Format(key_bits=kb, key_qjl=qjl, value_bits=vb, value_qjl=vqjl)
                    assert tq.page_bytes(cfg) == fmt.block_bytes
    g = packing_golden["c2_value_qjl_regions"]
    assert tq.page_bytes(tq.make_config(key_bits=3, key_qjl=True, value_bits=3, value_qjl=True)) == g["total"]


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 64, 2), ("qjl_m", 64, 2), ("page_tokens", 128, 2), ("key_bits", 5, 2),
    ("value_bits", 0, 2), ("key_qjl", 2, 1), ("rotation", 7, 1), ("value_qjl", 3, 1)])
def test_validate_config_rejects(tq, field, value, code):
    cfg = tq.make_config()
    assert tq.validate_config(cfg) == 0
    setattr(cfg, field, value)
    assert tq.validate_config(cfg) == code
    assert tq.page_bytes(cfg) == 0


def test_workspace_bytes(tq):
    cfg = tq.make_config()
    nb = tq.decode_workspace_bytes(cfg, 1, 32, 1, 16)
    rows = 32
    assert nb >= rows * (128 + 128 + 16 * 130) * 4
    assert nb % 256 == 0
    assert tq.decode_workspace_bytes(cfg, 1, 32, 1, 0) == 0
    # values with QJL add the sign-space partials: m floats per query row and split
    vq = tq.make_config(value_qjl=True)
    assert tq.decode_workspace_bytes(vq, 1, 32, 1, 16) >= nb + rows * 16 * 128 * 4


def test_host_argument_errors_do_not_launch(tq):
    cfg = tq.make_config()
    params = tq.tq_params()
    cache = tq.tq_cache()
    by = ctypes.byref
    # null params / cache / tensors are rejected on the host before any CUDA call
    st = tq.lib.tq_compress_kv(by(cfg), by(params), by(cache), 0, None, None, 0, 16, None, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG
    st = tq.lib.tq_attend_decode(by(cfg), None, by(cache), 0, None, 0, 32, 1, None, 4, None, 0, None,
                                 None, None)
    assert st == tq.TQ_ERR_INVALID_ARG
    assert "params" in tq.last_error()
    bad = tq.make_config(head_dim=96)
    st = tq.lib.tq_decompress(by(bad), by(params), by(cache), 0, None, 0, None, None, None, None)
    assert st == tq.TQ_ERR_UNSUPPORTED


def test_operand_bytes_and_prepare_validation(tq):
    # host-side checks of the operand preparation entry points (no device work)
    import ctypes
    ops = 3 * 128 * 128 * 2
    cfg = tq.make_config()
    assert tq.lib.tq_operand_bytes(ctypes.byref(cfg)) == ops
    dense = tq.make_config(rotation=tq.TQ_ROT_DENSE)
    assert tq.lib.tq_operand_bytes(ctypes.byref(dense)) == 2 * 128 * 128 * 2
    bad = tq.make_config(head_dim=64)
    assert tq.lib.tq_operand_bytes(ctypes.byref(bad)) == 0
    params = tq.tq_params()
    buf = ctypes.create_string_buffer(ops + 16)
    aligned = (ctypes.addressof(buf) + 15) & ~15
    st = tq.lib.tq_prepare_operands(ctypes.byref(dense), ctypes.byref(params), aligned, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "pi" in tq.last_error()
    st = tq.lib.tq_prepare_operands(ctypes.byref(cfg), ctypes.byref(params), aligned, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "signs" in tq.last_error()
    params.signs = aligned  # any non-null pointer: the call is rejected before it is read
    st = tq.lib.tq_prepare_operands(ctypes.byref(cfg), ctypes.byref(params), aligned, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "params->s" in tq.last_error()
    params.s = aligned
    st = tq.lib.tq_prepare_operands(ctypes.byref(cfg), ctypes.byref(params), aligned + 4, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "aligned" in tq.last_error()


def test_append_argument_errors_do_not_launch(tq):
    # host-side checks of tq_append_kv and tq_append_attend_decode (no device work)
    by = ctypes.byref
    cfg = tq.make_config()
    params = tq.tq_params()
    cache = tq.tq_cache()
    st = tq.lib.tq_append_kv(by(cfg), None, by(cache), 0, None, None, 0, 1, None, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "params" in tq.last_error()
    buf = ctypes.create_string_buffer(4096)
    p = (ctypes.addressof(buf) + 255) & ~255  # any non-null pointer: nothing is dereferenced
    params = tq.tq_params(p, None, p, p, p, p, p, None)
    cache = tq.tq_cache(p, p, 4, 4, 1, 1, 1)
    st = tq.lib.tq_append_kv(by(cfg), by(params), by(cache), 0, p, p, 0, 0, p, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "n_new" in tq.last_error()
    st = tq.lib.tq_append_kv(by(cfg), by(params), by(cache), 0, None, p, 0, 1, p, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "k_new" in tq.last_error()
    st = tq.lib.tq_append_kv(by(cfg), by(params), by(cache), 0, p, p, 7, 1, p, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "in_dtype" in tq.last_error()
    st = tq.lib.tq_append_kv(by(cfg), by(params), by(cache), 0, p, p, 0, 1, None, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "seq_lens" in tq.last_error()
    st = tq.lib.tq_append_kv(by(cfg), by(params), by(cache), 1, p, p, 0, 1, p, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "layer" in tq.last_error()
    misaligned = tq.tq_params(p, None, p + 4, p, p, p, p, None)
    st = tq.lib.tq_append_kv(by(cfg), by(misaligned), by(cache), 0, p, p, 0, 1, p, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "aligned" in tq.last_error()
    nb = tq.decode_workspace_bytes(cfg, 1, 4, 1, 2)
    st = tq.lib.tq_append_attend_decode(by(cfg), by(params), by(cache), 0, p, p, 0, 0, p, 0, 4, 1, p, 2,
                                        p, nb, p, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "n_new" in tq.last_error()
    st = tq.lib.tq_append_attend_decode(by(cfg), by(params), by(cache), 0, p, None, 0, 1, p, 0, 4, 1, p, 2,
                                        p, nb, p, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "v_new" in tq.last_error()
    st = tq.lib.tq_append_attend_decode(by(cfg), by(params), by(cache), 0, p, p, 0, 1, p, 0, 4, 1, p, 2,
                                        p, nb, None, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG and "out" in tq.last_error()


def test_plain_c_caller_links_and_runs(tq, tmp_path):
    # the boundary is a C ABI: a C program that includes only tq.h and links libtq.so
    # compiles with gcc and passes its host-side checks
    exe = tmp_path / "c_abi_host"
    libdir = os.path.dirname(tq.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_host.c"), "-o", str(exe), "-L", libdir, "-ltq",
           "-Wl,-rpath," + libdir, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "FAIL" not in out.stdout and out.stdout.count("ok ") >= 12


def test_tq_check_decodes_the_status_word(tq):
    # the host copy of a dev_status word goes through tq_check: every code comes back as
    # itself, with a description of the device errors; anything else is an argument error
    for code in range(0, 7):
        assert tq.check_status(code) == code
        if code in (tq.TQ_ERR_OVERFLOW, tq.TQ_ERR_TIMEOUT, tq.TQ_ERR_BOUNDS):
            assert tq.last_error().startswith("device:")
    assert tq.check_status(0) == tq.TQ_OK and tq.last_error() == ""
    assert tq.check_status(7) == tq.TQ_ERR_INVALID_ARG and "not a status code" in tq.last_error()
    assert tq.check_status(-1) == tq.TQ_ERR_INVALID_ARG
    assert tq.lib.tq_check(None) == tq.TQ_ERR_INVALID_ARG


def test_compress_binding_rejects_mismatched_k_and_v(tq):
    # the kernel reads v with k's geometry, so the binding refuses a v that differs
    import torch
    cfg, params, cache = tq.make_config(), tq.tq_params(), tq.tq_cache()
    k = torch.zeros((1, 2, 8, 128), dtype=torch.float16)
    for v in (torch.zeros((1, 2, 9, 128), dtype=torch.float16), torch.zeros((1, 2, 8, 128), dtype=torch.float32)):
        with pytest.raises(ValueError, match="same shape and dtype"):
            tq.compress_kv(cfg, params, cache, 0, k, v, None, None, stream=0)


def test_default_split_count():
    # one wave of two thread blocks per SM over (split, kv head, sequence, run of query rows)
    from compressed_decode_attention_tq_b200.runtime import splits_for
    assert splits_for(1, 8, 148) == 37                    # 4 query rows per KV head: one run
    assert splits_for(1, 8, 148, rows=4) == 37
    assert splits_for(1, 8, 148, rows=32) == 9            # 32 rows: four runs of eight
    assert splits_for(16, 2, 148, rows=8) == 18           # eight rows: one run; twice the share for a batch
    assert splits_for(1, 1, 148, max_len=4096) == 32      # no more splits than 128-token units
    assert splits_for(64, 64, 148) == 1
    assert splits_for(1, 1, 100000) == 1024
