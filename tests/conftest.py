import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built libca2.so")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(autouse=True)
def _device_status_clean(request):
    """Every GPU test leaves the device status word clear: a timeout, a range error or (in the
    debug build) a failed bounds check that a test did not read and expect fails the test."""
    yield
    if "gpu" not in request.keywords:
        return
    mod = sys.modules.get("causal_kv_cache_b200.ca2")
    if mod is None or mod._lib is None:
        return
    st = mod.ca2_device_status()
    assert st == 0, "device status %d (%s) left after the test" % (st, mod.STATUS.get(st, "?"))


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Raw parity figures of every attention output checked in this session, per workload."""
    mod = sys.modules.get("tests.gpu_util")
    if mod is None:
        return
    BIG, PARITY_LOG = mod.BIG, mod.PARITY_LOG
    if not PARITY_LOG:
        return
    groups = {}
    for what, max_abs, small, n_big, n_el, rel in PARITY_LOG:
        g = groups.setdefault(what, [0, 0.0, 0.0, 0, 0, 0.0])
        g[0] += 1
        g[1] = max(g[1], max_abs)
        g[2] = max(g[2], small)
        g[3] += n_big
        g[4] += n_el
        g[5] = max(g[5], rel)
    tr = terminalreporter
    tr.section("parity against the oracle (raw figures)")
    tr.write_line("%-24s %6s %11s %13s %11s %12s %9s" % ("workload / kernel", "calls", "max-abs", "|ref|<%g" % BIG,
                                                        "|ref|>=%g" % BIG, "elements", "rel-L2"))
    for what in sorted(groups):
        c, m, sm, nb, ne, r = groups[what]
        tr.write_line("%-24s %6d %11.3e %13.3e %11d %12d %9.2e" % (what, c, m, sm, nb, ne, r))
