import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_addoption(parser):
    parser.addoption("--kvc-path", action="append", default=[], metavar="KNOB=CHOICE",
                     help="cross-checks: force a kernel path of libkvc for the whole session through its "
                          "diagnostic kvc_diag_set_path call (e.g. score=simt, decode=tc)")


@pytest.fixture(scope="session", autouse=True)
def _kvc_forced_paths(request):
    opts = request.config.getoption("--kvc-path")
    if not opts:
        yield
        return
    import sparse_decode_attention_window_b200 as kvc
    for o in opts:
        knob, choice = o.split("=", 1)
        kvc.kvc_diag_set_path(knob, choice)
    yield
    for o in opts:
        kvc.kvc_diag_set_path(o.split("=", 1)[0], "auto")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large CPU-side work")


def pytest_collection_modifyitems(config, items):
    # files whose name starts with test_zz_ run last (they share global device state)
    items.sort(key=lambda it: 1 if os.path.basename(str(it.fspath)).startswith("test_zz_") else 0)
