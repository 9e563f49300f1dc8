import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


# Parity reports of the full-size checks (tokens checked, near-tie tokens,
# order swaps within near-ties, error ratios), printed at the end of the run
# so that they show in the output of `pytest -q` as well.
_PARITY_LOG = []


@pytest.fixture(scope="session")
def parity_log():
    return _PARITY_LOG


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if not _PARITY_LOG:
        return
    terminalreporter.write_sep("-", "parity against the fp64 oracle (near-tie tokens counted)")
    for r in _PARITY_LOG:
        parts = [f"{r['case']:<28} {r['check']:<8} tokens={r['tokens']:<6}",
                 f"boundary_ties={r['boundary_ties']}", f"order_swaps={r['order_swaps']}",
                 f"max_w_rel={r.get('max_w_rel', 0.0):.2e}"]
        if "err_ratio" in r:
            parts.append(f"max_err/max_ref={r['err_ratio']:.2e}")
        terminalreporter.write_line(" ".join(parts))
