import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    from oracle import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Both parity metrics of every GPU-vs-oracle comparison of the session: the
    tensor-scale max|x - r| / max(1, max|r|) the tests hold bf16 to, and the
    element-wise max_i |x_i - r_i| / max(1, |r_i|)."""
    try:
        from tests.parity import RECORDS
    except ImportError:
        return
    if not RECORDS:
        return
    tr = terminalreporter
    tr.section("parity metrics (tensor-scale | element-wise), worst output per case")
    for desc, main, elem in RECORDS:
        worst = max(main, key=main.get)
        worst_e = max(elem, key=elem.get)
        tr.write_line(f"{desc}: {worst} {main[worst]:.2e} | {worst_e} {elem[worst_e]:.2e}")
    allm = [v for _, m, _ in RECORDS for v in m.values()]
    alle = [v for _, _, e in RECORDS for v in e.values()]
    tr.write_line(f"cases {len(RECORDS)}: max tensor-scale {max(allm):.2e}, max element-wise {max(alle):.2e}")
