import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def golden():
    import json
    with open(os.path.join(ROOT, "tests", "golden", "page_values.json")) as f:
        return json.load(f)


@pytest.fixture(scope="session")
def packing_golden():
    import json
    with open(os.path.join(ROOT, "tests", "golden", "packing_example.json")) as f:
        return json.load(f)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Prints the parity counts of every GPU compress comparison of the session (tokens
    compared; index mismatches inside and outside the 1e-6 boundary band; sign-bit
    mismatches inside and outside the 1e-6 sum|S_ij r_j| band; tokens whose sign bits were
    not compared because one of their indices differed inside the band) and the decode
    checks' worst error over its allowance."""
    pu = sys.modules.get("parity_util")
    if pu is None or not getattr(pu, "REPORTS", None):
        return
    tr = terminalreporter
    tr.write_sep("-", "GPU parity counts (compress: in/out of the 1e-6 bands; decode: worst |d|/allowance)")
    for name, rep in pu.REPORTS:
        if isinstance(rep, str):
            tr.write_line(f"{name}: {rep}")
        else:
            tr.write_line(
                f"{name}: tokens {rep.tokens}, index mismatches in band {rep.idx_mismatch_in_band} / "
                f"out of band {rep.idx_mismatch_out_of_band}, sign mismatches in band "
                f"{rep.sign_mismatch_in_band} / out of band {rep.sign_mismatch_out_of_band}, "
                f"sign tokens skipped {rep.sign_tokens_skipped}, norm failures {rep.norm_fail}")
