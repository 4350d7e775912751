"""Host logic of bench.py that needs no GPU: the reference arm (the float64 oracle
timed on a bounded sample) prints the same workload keys as the eta arm, its
ms_per_step is the measured sampled step, and its value is that step scaled to the
whole batch; the density offset puts no bound exactly on a threshold."""
import os
import sys
import types

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _args(**kw):
    a = dict(workload="mid", B=2, ctx=2048, cpu_rows=2, warmup=1, steps=2, density=0.0,
             density_kind="", tau_mode="", bound="", cent="bf16", engine="auto", graph=False,
             fused=False, separate_prologue=False)
    a.update(kw)
    return types.SimpleNamespace(**a)


def test_reference_arm_line_on_cpu():
    args = _args()
    r = bench.run_reference(args, 0, 1, torch.device("cpu"))
    w = bench.with_overrides(bench.workload_by_name(args.workload, args.B), args)
    assert r["impl"] == "reference" and r["metric"] == bench.METRIC
    assert r["config"] == bench.workload_config(w, args)
    assert r["steps"] == 2 and r["unit"] == "steps/s" and r["higher_is_better"] is True
    # value = (sampled rows / B) / measured seconds per sampled step
    rows = r["density"]["rows"]
    assert abs(r["value"] - rows / w.B / (r["ms_per_step"] * 1e-3)) < 1e-9 * r["value"]
    assert abs(r["ms_per_full_step_extrapolated"] - r["ms_per_step"] * w.B / rows) < 1e-6
    assert r["cpu_baseline"]["value"] == r["value"] and r["cpu_baseline"]["cores"] == 1
    assert r["e2e"] == {"value": r["value"], "unit": "steps/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert r["gpu_launches"] == 0


def test_cpu_baseline_matches_reference_sample():
    """The eta arm's cpu_baseline times the same oracle sample with the same inputs."""
    args = _args()
    w = bench.with_overrides(bench.workload_by_name(args.workload, args.B), args)
    g = __import__("long_context_decoding_eta_b200.synth", fromlist=["x"]).generate(w, "cpu")
    c = bench.cpu_baseline(w, g, rows=2, warmup=1, reps=2)
    assert c["kind"] == "oracle" and c["cores"] == 1 and c["unit"] == "steps/s"
    assert c["value"] > 0


def test_density_offset_sits_between_two_margins():
    rng = np.random.default_rng(3)
    B, Hq, NB, G = 2, 8, 50, 4
    bounds = rng.normal(size=(B, Hq, NB))
    tau0 = rng.normal(size=(B, Hq))
    valid = rng.random((B, Hq, NB)) > 0.1
    for kind in ("head", "union"):
        for dens in (0.16, 0.38, 0.51):
            off = bench.density_offset(bounds, tau0, valid, dens, G, kind)
            m = np.where(valid, bounds - tau0[:, :, None], -np.inf)
            if kind == "union":
                m = m.reshape(B, Hq // G, G, NB).max(axis=2)
            v = m[np.isfinite(m)]
            assert not np.any(v == off)                   # no margin on the threshold
            frac = (v >= off).mean()
            assert dens <= frac <= dens + 1.0 / v.size + 1e-12
