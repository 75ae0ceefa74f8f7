import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(autouse=True)
def _report_rounded_comparisons(record_property):
    """Attach to each test's report the O elements its check_o calls held
    against the dtype-rounded oracle (see helpers.check_o)."""
    import helpers
    start = len(helpers.ROUNDED_COMPARISONS)
    yield
    for rec in helpers.ROUNDED_COMPARISONS[start:]:
        record_property("o_vs_rounded_oracle", rec)


def pytest_terminal_summary(terminalreporter):
    import helpers
    recs = helpers.ROUNDED_COMPARISONS
    if not recs:
        return
    terminalreporter.section("O elements compared with the dtype-rounded oracle")
    for r in recs:
        terminalreporter.write_line(f"{r['what']}: {r['elements']} element(s), raw error up to {r['raw_max']:.3e}, "
                                    f"{r['err_vs_rounded_max']:.3e} against the rounded oracle")
