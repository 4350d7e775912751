import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    import torch
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture(scope="session", autouse=True)
def _built_library():
    """Builds libeta.so in-tree once per session (nvcc cross-compiles without a GPU);
    libeta_checked.so instead when ETA_CHECKED=1 selects the range-checked build."""
    from long_context_decoding_eta_b200 import build
    build.build(checked=os.environ.get("ETA_CHECKED") == "1")
    yield


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Logs the near-tie blocks (bound within 1e-5 of tau, relative) of every
    GPU-vs-oracle comparison of the session and the heads they kept out of the
    output comparison."""
    try:
        from eta_testlib import NEAR_TIE_LOG
    except Exception:
        return
    if not NEAR_TIE_LOG:
        return
    band = sum(int(e["near_ties"]) for e in NEAR_TIE_LOG)
    differ = [b for e in NEAR_TIE_LOG for b in e["blocks"]]
    skipped = [s for e in NEAR_TIE_LOG for s in e["skipped"]]
    heads = sum(int(e["heads"]) for e in NEAR_TIE_LOG)
    tr = terminalreporter
    tr.write_line(f"near-tie log: {len(NEAR_TIE_LOG)} comparisons, {band} blocks in the "
                  f"near-tie band, {len(differ)} of them with a differing admit bit, "
                  f"{len(skipped)} of {heads} heads left out of the output comparison")
    for b in differ[:20]:
        tr.write_line(f"  near-tie block (b={b[0]}, h={b[1]}, j={b[2]}): bound {b[3]:.9g}, "
                      f"tau {b[4]:.9g}")
    for s in skipped[:20]:
        tr.write_line(f"  head skipped (b={s[0]}, h={s[1]}): {s[2]}")
