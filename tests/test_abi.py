"""The C-ABI library loads and exports every entry point include/eta.h declares;
host-only entry points (calibration, status helpers, argument validation) work
without a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from long_context_decoding_eta_b200 import _lib as L
from oracle import eta_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "eta.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(eta_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = L.lib()
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.EXPORTS)


def test_header_declares_the_four_method_calls():
    names = declared_functions()
    for n in ("eta_build_block_meta", "eta_predict_tau", "eta_screen", "eta_decode"):
        assert n in names


def test_status_strings():
    assert L.eta_status_string(0) == "ok"
    assert L.eta_status_string(3).startswith("workspace")
    assert L.eta_status_from_device(0) == 0
    assert L.eta_status_from_device(L.DEVSTAT_TIMEOUT) == 5
    assert L.eta_status_from_device(L.DEVSTAT_NONFINITE_Q) == 6
    assert L.eta_status_from_device(L.DEVSTAT_BAD_BLOCK) == 1


@pytest.mark.parametrize("density", [0.16, 0.38, 0.51, 1.0])
def test_host_calibration_matches_oracle_quantile(density):
    rng = np.random.default_rng(0)
    bounds = rng.normal(size=(64, 4, 50)).astype(np.float32)
    valid = rng.random((64, 4, 50)) > 0.05
    tau = L.eta_calibrate_const_tau(torch.from_numpy(bounds), torch.from_numpy(valid), density)
    ref = O.calibrate_const_tau(bounds.astype(np.float64), valid, density)
    np.testing.assert_array_equal(tau.numpy().astype(np.float64), ref)


def test_calibration_rejects_empty_head():
    b = torch.zeros(2, 2, 3)
    v = torch.zeros(2, 2, 3, dtype=torch.bool)
    v[:, 0] = True
    with pytest.raises(L.EtaError):
        L.eta_calibrate_const_tau(b, v, 0.5)


def test_argument_validation_without_gpu():
    lib = L.lib()
    dims = L.Dims.of(2, 16, 4, 128, 64, 4096)
    # null q -> invalid argument, nothing launched
    r = lib.eta_decode(ctypes.byref(dims), None, None, None, None, None, None, None, 0.0, 0.0,
                       0, None, None, None, None, None, 0, None, None)
    assert r == 1
    bad = L.Dims.of(2, 16, 4, 96, 64, 4096)            # d = 96 unsupported
    r = lib.eta_screen(ctypes.byref(bad), None, None, 0, *([None] * 5), 0, 0.0, 0.0,
                       *([None] * 6), 0, None, None)
    assert r == 2
    odd = L.Dims.of(2, 16, 4, 128, 64, 4000)           # T_max not a multiple of blk
    assert lib.eta_build_block_meta(ctypes.byref(odd), None, None, None, 0, -1, 0,
                                    *([None] * 7)) == 2
    # unknown centroid format -> invalid argument (before any CUDA call)
    ok = L.Dims.of(2, 16, 4, 128, 64, 4096)
    import torch as _t
    buf = _t.zeros(8)
    p = ctypes.c_void_p(buf.data_ptr())
    assert lib.eta_build_block_meta(ctypes.byref(ok), p, None, p, 0, -1, 7, p, p, p, p, None,
                                    None, None) == 1
    g3 = L.Dims.of(2, 12, 4, 128, 64, 4096)            # G = 3 unsupported
    assert lib.eta_predict_tau(ctypes.byref(g3), *([None] * 7)) == 2
    assert L.eta_screen_workspace_size(dims) == 256       # 2*4 rows x 2 words, 256-aligned
    assert L.eta_screen_workspace_size(bad) == 0
    # launch-count query: invalid dims are refused; without a device the two-launch form
    assert lib.eta_screen_launches(ctypes.byref(bad), 1) == -1
    assert lib.eta_screen_launches(ctypes.byref(dims), 1) in (1, 2)
    assert lib.eta_decode_launches(ctypes.byref(bad)) == -1
    assert lib.eta_decode_launches(ctypes.byref(dims)) in (2, 3)


def test_prefill_kernel_selection_host_only():
    assert L.eta_get_prefill_kernel() == "auto"
    dims = L.Dims.of(4, 16, 4, 128, 64, 8192)
    for k in ("one_tile", "two_tile"):
        L.eta_set_prefill_kernel(k)
        assert L.eta_get_prefill_kernel() == k
        assert L.eta_prefill_kernel_for(dims, 0.0) == k
        assert L.eta_prefill_kernel_for(dims, 0.05) == k
    L.eta_set_prefill_kernel("auto")
    with pytest.raises(L.EtaError):
        L.eta_set_prefill_kernel(5)
    assert L.eta_get_prefill_kernel() == "auto"
    # shapes eta_prefill refuses are refused by the query too
    for bad in (L.Dims.of(4, 16, 4, 64, 64, 8192), L.Dims.of(4, 16, 4, 128, 64, 8256),
                L.Dims.of(4, 16, 5, 128, 64, 8192)):
        with pytest.raises(L.EtaError):
            L.eta_prefill_kernel_for(bad, 0.0)
    with pytest.raises(L.EtaError):
        L.eta_prefill_kernel_for(dims, -1.0)


def test_screen_engine_selection_host_only():
    assert L.eta_get_screen_engine() == "auto"
    for e in ("tcgen05", "fma", "auto"):
        L.eta_set_screen_engine(e)
        assert L.eta_get_screen_engine() == e
    with pytest.raises(L.EtaError):
        L.eta_set_screen_engine(9)
    # without a device the launch-count query reports the two-launch form
    dims = L.Dims.of(4, 16, 4, 128, 64, 8192)
    L.eta_set_screen_engine("tcgen05")
    assert L.eta_screen_launches(dims, "bf16") == 2
    L.eta_set_screen_engine("auto")


def test_engine_selection_host_only():
    assert L.eta_get_decode_engine() == "auto"
    L.eta_set_decode_engine("fma")
    assert L.eta_get_decode_engine() == "fma"
    L.eta_set_decode_engine("auto")
    with pytest.raises(L.EtaError):
        L.eta_set_decode_engine(7)


def test_checked_build_loads_with_the_same_entry_points():
    """The range-checked build (-DETA_CHECKED) links, exports every declared entry
    point and says it is the checked one; the release build says it is not."""
    import subprocess
    import sys
    from long_context_decoding_eta_b200 import build
    path = build.build(checked=True)
    assert path.endswith("libeta_checked.so")
    assert L.eta_build_checked() is False
    code = ("import sys; sys.path.insert(0, %r)\n"
            "from long_context_decoding_eta_b200 import _lib as L\n"
            "lib = L.lib()\n"
            "assert L.LIB_PATH.endswith('libeta_checked.so'), L.LIB_PATH\n"
            "missing = [n for n in %r if not hasattr(lib, n)]\n"
            "assert not missing, missing\n"
            "print('checked', L.eta_build_checked())\n") % (ROOT, declared_functions())
    env = dict(os.environ, ETA_CHECKED="1")
    p = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=300)
    assert p.returncode == 0, p.stderr
    assert "checked True" in p.stdout


def test_device_status_mapping_of_the_bounds_bit():
    assert L.eta_status_from_device(L.DEVSTAT_BOUNDS) == 7
    assert L.eta_status_from_device(L.DEVSTAT_BOUNDS | L.DEVSTAT_TIMEOUT) == 7
    assert "checked build" in L.eta_status_string(7)
    # argument checks run on the host: nothing is launched
    assert L.lib().eta_selftest_bounds(0, -1, ctypes.c_void_p(16), None) == 1
    assert L.lib().eta_selftest_bounds(0, 4, None, None) == 1
