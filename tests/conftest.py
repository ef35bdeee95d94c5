import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    """Observed maxima of every GPU parity check against its tolerance."""
    try:
        from tests.gpu_harness import HIDDEN_RTOL, LOGITS_ATOL, REPORTS
    except Exception:
        return
    if not REPORTS:
        return
    tr = terminalreporter
    tr.section("parity margins (observed max / tolerance)")
    tr.write_line(f"{'test':<78} {'steps':>5} {'hidden rel-L2':>13} {'logits |d|':>10} "
                  f"{'K/V rel-L2':>10} {'tokens':>7}")
    for name, r in REPORTS:
        tr.write_line(f"{name[-78:]:<78} {r.steps:>5} {r.max_hidden_rel:>13.3e} "
                      f"{r.max_logit_err:>10.3e} {r.max_kv_rel:>10.3e} "
                      f"{r.token_checked - r.token_mismatch:>3}/{r.token_checked:<3}")
    tr.write_line(f"tolerances: hidden rel-L2 <= {HIDDEN_RTOL}, logits max-abs <= {LOGITS_ATOL}, "
                  f"K/V rel-L2 <= {HIDDEN_RTOL}, tokens identical where the top-2 margin > 0.1")
