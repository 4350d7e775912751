"""Full-size workloads, in the launch configuration the benchmark times (whole
batch on the GPU, default engine), checked against the float64 oracle on sampled
batch rows (the oracle computes those rows one by one), plus properties that hold
at any size for every row."""
import gc
import math

import numpy as np
import pytest
import torch

from long_context_decoding_eta_b200 import _lib as L
from long_context_decoding_eta_b200 import synth
from long_context_decoding_eta_b200.api import EtaDecoder
from oracle import eta_oracle as O

from eta_testlib import check_meta, compare_step, f64, gpu_meta, run_cuda, unpack_mask

pytestmark = pytest.mark.gpu


def rows_f64(t, rows):
    return t[rows].double().cpu().numpy()


def sampled_oracle_bias(w, g, rows, scale, cent_format="f32"):
    """Threshold offset from the oracle on the sampled rows (density target of the
    workload), so that no input of the comparison comes from the CUDA path."""
    K64 = rows_f64(g["K"], rows)
    q64 = rows_f64(g["q"], rows)
    L64 = g["lengths"][rows].cpu().numpy()
    meta = O.cache_meta(K64, L64, w.blk, cent_format=cent_format)
    W64 = g["W"].double().cpu().numpy()
    tau0 = O.predict_tau(q64, W64, np.zeros(w.Hq))
    ub = O.screen(q64, tau0, meta, scale, w.bound, w.z)["bounds"]
    valid = np.repeat(meta["cnt"] > 0, w.G, axis=1)
    return O.offset_for_density(ub, tau0, valid, w.density, w.G, w.density_kind)


def whole_batch_properties(dec, gpu, w):
    """Checks that hold for every row at any size."""
    G, NB = w.G, dec.NB
    hm = gpu["head_mask"]                                   # [B, Hq, NB]
    cnt = dec.cnt.cpu().numpy()
    assert not np.any(hm & ~np.repeat(cnt > 0, G, axis=1)), "empty block admitted"
    un = hm.reshape(w.B, w.Hkv, G, NB).any(axis=2)
    assert np.array_equal(gpu["union_cnt"], un.sum(axis=2))
    for b in range(w.B):
        for g in range(w.Hkv):
            c = gpu["union_cnt"][b, g]
            assert np.array_equal(gpu["union_idx"][b, g, :c], np.nonzero(un[b, g])[0])
    assert np.all(np.isfinite(gpu["o"]))
    return un.mean()


def run_fullsize(w, rows, tau_const=None, engine="auto", cent_format="f32", g=None,
                 keep=False):
    """The whole batch through the CUDA path; the oracle on `rows`.  With keep=True
    the decoder is returned too (the caller frees it)."""
    L.eta_set_decode_engine(engine)
    scale = 1.0 / math.sqrt(w.d)
    own = g is None
    g = synth.generate(w, "cuda") if own else g
    dec = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk, bound=w.bound, z=w.z,
                     T=w.gate_T, keep_bounds=True, cent_format=cent_format)
    dec.build_meta()
    if tau_const is None:
        bias = sampled_oracle_bias(w, g, rows, scale, cent_format)
        gpu = run_cuda(dec, g["q"], g["W"], torch.full((w.Hq,), bias, device="cuda"))
        b64 = np.full(w.Hq, bias)
    else:
        gpu = run_cuda(dec, g["q"], tau_const=torch.tensor(tau_const, dtype=torch.float32,
                                                            device="cuda"))
        b64 = None
    union_density = whole_batch_properties(dec, gpu, w)
    # oracle on the sampled rows
    K64, V64, q64 = rows_f64(g["K"], rows), rows_f64(g["V"], rows), rows_f64(g["q"], rows)
    L64 = g["lengths"][rows].cpu().numpy()
    meta = O.cache_meta(K64, L64, w.blk, cent_format=cent_format)
    if tau_const is None:
        tau = O.predict_tau(q64, g["W"].double().cpu().numpy(), b64)
    else:
        tau = O.const_tau(len(rows), np.asarray(tau_const, dtype=np.float64))
    sc = O.screen(q64, tau, meta, scale, w.bound, w.z)
    o, lse = O.decode(q64, tau, K64, V64, L64, sc["union_idx"], w.blk, scale, w.gate_T)
    check_meta(gpu_meta(dec, rows), meta)
    rep = compare_step(gpu, tau, sc, o, lse, q64, K64, V64, L64, w.blk, scale, w.gate_T, w.G,
                       rows=rows)
    L.eta_set_decode_engine("auto")
    if keep:
        return rep, union_density, dec, gpu
    del dec
    if own:
        del g
    gc.collect()
    torch.cuda.empty_cache()
    return rep, union_density


@pytest.mark.parametrize("engine,cent", [("auto", "f32"), ("fma", "f32"), ("auto", "bf16")])
def test_long_128k_b64_union16(engine, cent):
    w = synth.LONG128K
    from long_context_decoding_eta_b200 import _lib as L
    # 16 groups of 128 blocks per row: the two-launch screen (screening, compaction)
    dims = L.Dims.of(w.B, w.Hq, w.Hkv, w.d, w.blk, w.T_max)
    assert L.eta_screen_launches(dims, cent) == 2
    # the tensor-core decode lays out its shares itself: decode + combine
    L.eta_set_decode_engine(engine)
    try:
        assert L.eta_decode_launches(dims) == (2 if engine != "fma" else 3)
    finally:
        L.eta_set_decode_engine("auto")
    rep, dens = run_fullsize(w, rows=[0, 37, 63], engine=engine, cent_format=cent)
    # the density target is set on the 3 sampled rows only; across the batch it
    # varies with the rows' thresholds: require real pruning and real admission
    assert 0.01 < dens < 0.6, dens
    print(rep, dens)


@pytest.mark.parametrize("engine", ["auto", "fma"])
def test_d64_b32_ctx64k_union16(engine):
    """Head dimension 64 at a realistic size (B = 32, 16 / 4 heads, 64K context, 128
    (row, KV head) pairs): the tensor-core decode (one 64-dim box per sub-tile, P V
    over a zero upper half) with its in-kernel share plan, and the CUDA-core engine,
    against the oracle on sampled rows."""
    w = synth.LONG128K.with_(d=64, B=32, ctx=65536)
    from long_context_decoding_eta_b200 import _lib as L
    dims = L.Dims.of(w.B, w.Hq, w.Hkv, w.d, w.blk, w.T_max)
    L.eta_set_decode_engine(engine)
    try:
        assert L.eta_decode_launches(dims) == (2 if engine != "fma" else 3)
    finally:
        L.eta_set_decode_engine("auto")
    rep, dens = run_fullsize(w, rows=[0, 17, 31], engine=engine, cent_format="bf16")
    assert 0.01 < dens < 0.6, dens
    print(rep, dens)


@pytest.mark.parametrize("density,kind", [(0.38, "head"), (0.51, "union")])
def test_long_128k_b64_trained_operating_points(density, kind):
    """The 128K configuration at the pages' trained operating point: about 38% of
    blocks per head, or 51% in the union (review Summary: 51.2% union density at
    B = 64)."""
    w = synth.LONG128K.with_(density=density, density_kind=kind)
    rep, dens = run_fullsize(w, rows=[1, 50], cent_format="bf16")
    lo, hi = (0.3, 0.95) if kind == "head" else (0.35, 0.7)
    assert lo < dens < hi, dens
    print(rep, dens)


def test_extreme_512k_b64_prob_and_exact_bound_blk128():
    """512K context, block 128: the probabilistic bound (z = 3) and the exact bound,
    each with its threshold offset set for 16% union density on the sampled rows, on
    the same cache; and at the probabilistic arm's thresholds, every block the z = 3
    bound admits is one the exact bound admits too (its bound is never larger), on
    every row of the batch."""
    w = synth.EXTREME512K
    g = synth.generate(w, "cuda")
    rep, dens, dec, gpu = run_fullsize(w, rows=[5, 60], g=g, keep=True)
    assert 0.01 < dens < 0.6, dens
    ex_mask = torch.empty_like(dec.head_mask)
    ex_cnt = torch.empty_like(dec.union_cnt)
    L.eta_screen(dec.dims, g["q"], dec.tau, dec.cent, dec.rmax, dec.var, dec.cnt, "exact",
                 w.z, dec.scale, ex_mask, torch.empty_like(dec.union_idx), ex_cnt, None,
                 torch.empty_like(dec.head_cnt), dec.ws_screen, dec.dev_status)
    torch.cuda.synchronize()
    dec.check_status()
    ex = unpack_mask(ex_mask, dec.NB)
    assert not np.any(gpu["head_mask"] & ~ex), "z = 3 admitted a block the exact bound pruned"
    nonempty = int((dec.cnt > 0).sum())
    dens_exact = float(ex_cnt.sum()) / nonempty
    assert dens_exact >= dens
    print(rep, "union density z=3:", dens, "exact bound at the same tau:", dens_exact)
    del dec, gpu
    gc.collect()
    rep_ex, dens_ex = run_fullsize(w.with_(bound="exact"), rows=[5, 60], g=g)
    assert 0.01 < dens_ex < 0.6, dens_ex
    print(rep_ex, "exact-bound arm union density:", dens_ex)
    del g
    gc.collect()
    torch.cuda.empty_cache()


def calibrated_tau_const(w, g, rows, scale):
    """Per-head constants from the calibration rule on the oracle, with the
    calibration queries paired with the sampled rows (the full-batch pairing would
    need the oracle's metadata of every row)."""
    K64 = rows_f64(g["K"], rows)
    L64 = g["lengths"][rows].cpu().numpy()
    meta = O.cache_meta(K64, L64, w.blk)
    qc = synth.calibration_queries(w, g["mu"]).double().cpu().numpy()
    n = qc.shape[0]
    bounds = np.zeros((n, w.Hq, w.NB))
    valid = np.zeros((n, w.Hq, w.NB), dtype=bool)
    for i in range(n):
        r = i % len(rows)
        mrow = {k: v[r:r + 1] for k, v in meta.items()}
        bounds[i] = O.screen(qc[i:i + 1], np.zeros((1, w.Hq)), mrow, scale)["bounds"][0]
        valid[i] = np.repeat(meta["cnt"][r] > 0, w.G, axis=0)
    return O.calibrate_const_tau(bounds, valid, w.density)


def test_calibrated_256k_const_tau_and_predictor_same_inputs():
    """256K, B = 64: frozen per-head constants from the calibration rule, then the
    predictor (Eq. 1, offset for the same 38% per-head target) on the same inputs."""
    w = synth.CALIB256K
    rows = [3, 42]
    scale = 1.0 / math.sqrt(w.d)
    g = synth.generate(w, "cuda")
    tau_const = calibrated_tau_const(w, g, rows, scale)
    rep, dens = run_fullsize(w, rows=rows, tau_const=tau_const, g=g)
    print("const tau:", rep, dens)
    rep_p, dens_p = run_fullsize(w.with_(tau_mode="predictor"), rows=rows, g=g)
    print("predictor:", rep_p, dens_p)
    del g
    gc.collect()
    torch.cuda.empty_cache()


def test_calibrated_256k_b32_const_tau():
    """The calibrated configuration at B = 32 (the pages report ETA slower than
    FlashAttention-2 there on H100)."""
    w = synth.CALIB256K.with_(B=32, name="calibrated-b32-h16x4-d128-ctx256k-blk64")
    rows = [0, 31]
    scale = 1.0 / math.sqrt(w.d)
    g = synth.generate(w, "cuda")
    tau_const = calibrated_tau_const(w, g, rows, scale)
    rep, dens = run_fullsize(w, rows=rows, tau_const=tau_const, g=g)
    print(rep, dens)
    del g
    gc.collect()
    torch.cuda.empty_cache()


def test_long_128k_fused_step_equals_separate_calls():
    """The one-launch step at full size, in the launch configuration `bench.py --fused`
    times: every output equals the separate calls' bit for bit; the sampled rows
    against the oracle."""
    w = synth.LONG128K
    rows = [0, 63]
    scale = 1.0 / math.sqrt(w.d)
    g = synth.generate(w, "cuda")
    bias = sampled_oracle_bias(w, g, rows, scale, "bf16")
    bias_t = torch.full((w.Hq,), bias, device="cuda")
    kw = dict(bound=w.bound, z=w.z, T=w.gate_T, cent_format="bf16")
    sep = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk, **kw)
    fus = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk, fused=True, **kw)
    sep.build_meta()
    fus.build_meta()
    sep.step(g["q"], g["W"], bias_t)
    fus.step(g["q"], g["W"], bias_t)
    torch.cuda.synchronize()
    sep.check_status()
    fus.check_status()
    for name in ("tau", "head_mask", "union_cnt", "head_cnt", "o", "lse", "cent", "rmax", "var",
                 "cnt"):
        assert torch.equal(getattr(sep, name), getattr(fus, name)), name
    live = torch.arange(fus.NB, device="cuda") < fus.union_cnt[..., None]
    assert torch.equal(sep.union_idx[live], fus.union_idx[live])
    gpu = dict(tau=f64(fus.tau), head_mask=unpack_mask(fus.head_mask, fus.NB),
               union_idx=fus.union_idx.cpu().numpy(), union_cnt=fus.union_cnt.cpu().numpy(),
               head_cnt=fus.head_cnt.cpu().numpy(), o=f64(fus.o), lse=f64(fus.lse))
    K64, V64, q64 = rows_f64(g["K"], rows), rows_f64(g["V"], rows), rows_f64(g["q"], rows)
    L64 = g["lengths"][rows].cpu().numpy()
    meta = O.cache_meta(K64, L64, w.blk, cent_format="bf16")
    tau = O.predict_tau(q64, g["W"].double().cpu().numpy(), np.full(w.Hq, bias))
    sc = O.screen(q64, tau, meta, scale, w.bound, w.z)
    o, lse = O.decode(q64, tau, K64, V64, L64, sc["union_idx"], w.blk, scale, w.gate_T)
    check_meta(gpu_meta(fus, rows), meta)
    rep = compare_step(gpu, tau, sc, o, lse, q64, K64, V64, L64, w.blk, scale, w.gate_T, w.G,
                       rows=rows)
    print(rep)
    del sep, fus, g
    gc.collect()
    torch.cuda.empty_cache()
