import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# NVFP4 cases the oracle finds within one ulp of a rounding threshold, per
# workload (the parity contract exempts them from bit-exactness but asks that
# they be counted and reported); printed in the terminal summary.
_NEAR_THRESHOLD = []


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


@pytest.fixture(scope="session")
def cuda_dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture
def report_near(record_property):
    """record(workload, (near_codes, near_scales), n_codes, n_scales, bad_codes, bad_scales)."""
    def record(workload, near, n_codes, n_scales, bad_codes=0, bad_scales=0):
        row = {"workload": workload, "near_codes": int(near[0]), "near_scales": int(near[1]),
               "codes": int(n_codes), "scales": int(n_scales), "packed_bytes_differing": int(bad_codes),
               "scales_differing": int(bad_scales)}
        for key, val in row.items():
            if key != "workload":
                record_property(f"near_threshold_{key}", val)
        _NEAR_THRESHOLD.append(row)
    return record


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if not _NEAR_THRESHOLD:
        return
    terminalreporter.write_sep("-", "NVFP4 values within 1 ulp of a rounding threshold (oracle)")
    for r in _NEAR_THRESHOLD:
        terminalreporter.write_line(
            f"{r['workload']}: codes {r['near_codes']} of {r['codes']}, scales {r['near_scales']} of "
            f"{r['scales']}; GPU differs from the oracle in {r['packed_bytes_differing']} packed bytes, "
            f"{r['scales_differing']} scales")
