"""CUDA path (through the C ABI) against the float64 oracle on the same seeded
inputs.  Masks bit-exact except logged near-ties; o within max-abs 1e-2 and
mean-abs 1e-3; lse within 1e-3."""
import math

import numpy as np
import pytest
import torch

from long_context_decoding_eta_b200 import synth
from long_context_decoding_eta_b200._lib import EtaError
from long_context_decoding_eta_b200.api import EtaDecoder
from oracle import eta_oracle as O

from eta_testlib import (check_meta, compare_step, density_bias, f64, gpu_meta, oracle_step,
                         run_cuda, unpack_mask)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True, params=["fma", "tcgen05"])
def engine(request):
    """Every parity test runs on both engines: the CUDA-core decode with the CUDA-core
    screen, and the tensor-core decode with the tensor-core screen where it applies
    (bf16 centroids, d = 128, not the per-dimension bound)."""
    from long_context_decoding_eta_b200 import _lib as L
    L.eta_set_decode_engine(request.param)
    L.eta_set_screen_engine(request.param)
    yield request.param
    L.eta_set_decode_engine("auto")
    L.eta_set_screen_engine("auto")


def make(w, lengths=None, seed=None):
    g = synth.generate(w, "cpu", seed=seed, lengths=lengths)
    return g


def to_dev(g):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in g.items()}


def full_parity(w, *, lengths=None, prune="skip", T=None, bound=None, z=None, density=None,
                kind=None, seed=None, tau_const=None, cent_format="f32"):
    T = w.gate_T if T is None else T
    bound = w.bound if bound is None else bound
    z = w.z if z is None else z
    density = w.density if density is None else density
    kind = w.density_kind if kind is None else kind
    g = make(w, lengths, seed)
    K64, V64, q64, W64 = f64(g["K"]), f64(g["V"]), f64(g["q"]), f64(g["W"])
    L = g["lengths"].numpy().astype(np.int64)
    scale = 1.0 / math.sqrt(w.d)
    bias = np.full(w.Hq, density_bias(K64, q64, L, W64, w.blk, scale, w.G, density, kind,
                                      bound, z, cent_format))
    gd = to_dev(g)
    dec = EtaDecoder(gd["K"], gd["V"], gd["lengths"], w.Hq, w.blk, bound=bound, z=z, T=T,
                     prune=prune, keep_bounds=True, cent_format=cent_format)
    dec.build_meta()
    bias_t = torch.tensor(bias, dtype=torch.float32, device=DEV)
    tc = None if tau_const is None else torch.tensor(tau_const, dtype=torch.float32, device=DEV)
    gpu = run_cuda(dec, gd["q"], gd["W"], bias_t, tc)
    meta, tau, sc, o, lse = oracle_step(K64, V64, q64, L, W64, bias, w.blk, scale, T, bound, z,
                                        prune, tau_const, cent_format)
    check_meta(gpu_meta(dec), meta)
    rep = compare_step(gpu, tau, sc, o, lse, q64, K64, V64, L, w.blk, scale, T, w.G)
    return rep, gpu, sc


def test_tiny_workload_end_to_end():
    rep, gpu, sc = full_parity(synth.TINY)
    dens = sc["admit"].mean()
    assert 0.3 < dens < 0.46, dens
    print(rep)


def test_mid_workload_needles_soft_gate():
    rep, gpu, sc = full_parity(synth.MID)
    print(rep)


@pytest.mark.parametrize("T", [0.0, 0.05])
@pytest.mark.parametrize("prune", ["skip", "floor"])
def test_sharp_variant_keys_above_tau(T, prune):
    w = synth.MID.with_(B=4, ctx=8192, q_scale=8.0, needles=16, density=0.3,
                        density_kind="head", seed=77)
    rep, gpu, sc = full_parity(w, T=T, prune=prune)
    print(rep)


def test_ragged_lengths_empty_and_single_token_rows():
    w = synth.MID.with_(B=6, ctx=4096, needles=0, seed=78)
    lengths = torch.tensor([4096, 0, 1, 4031, 65, 2000], dtype=torch.int32)
    for prune in ("skip", "floor"):
        rep, gpu, sc = full_parity(w, lengths=lengths, prune=prune, T=0.0, density=0.5)
        # the empty row: SKIP gives o = 0, lse = -inf; FLOOR too (no keys at all)
        assert np.all(gpu["o"][1] == 0) and np.all(np.isneginf(gpu["lse"][1]))


@pytest.mark.parametrize("B,Hkv", [(8, 4), (11, 3), (1, 1), (32, 4)])
def test_batch_shapes_and_repeat_determinism(B, Hkv, engine):
    """Batches of 32, 33, 1 and 128 (batch row, KV head) pairs, with empty, single-token,
    single-block and ragged rows, against the oracle; repeated steps on one decoder
    are bit-identical (the split plan and the combine order depend only on the
    admitted counts)."""
    w = synth.MID.with_(B=B, Hkv=Hkv, Hq=4 * Hkv, ctx=4096, needles=2, seed=90 + B)
    lens = ([4096, 0, 64, 4031, 1, 3000, 128, 2049, 4096, 777, 3333] * 3)[:B]
    lengths = torch.tensor(lens, dtype=torch.int32)
    from long_context_decoding_eta_b200 import _lib as L
    dims = L.Dims.of(B, w.Hq, w.Hkv, w.d, w.blk, w.T_max)
    # these small batches take the one-launch screen (screening + compaction)
    assert L.eta_screen_launches(dims, "f32") == 1
    # 128 pairs and more: the tensor-core decode plans its own shares
    if engine == "tcgen05":
        assert L.eta_decode_launches(dims) == (2 if B * Hkv >= 128 else 3)
    rep, gpu, sc = full_parity(w, lengths=lengths, density=0.4)
    if B > 1:
        assert np.all(gpu["o"][1] == 0) and np.all(np.isneginf(gpu["lse"][1]))
    gd = to_dev(make(w, lengths))
    dec = EtaDecoder(gd["K"], gd["V"], gd["lengths"], w.Hq, w.blk, T=w.gate_T)
    dec.build_meta()
    bias = torch.full((w.Hq,), 1.5, device=DEV)
    first = run_cuda(dec, gd["q"], gd["W"], bias)
    for _ in range(2):
        again = run_cuda(dec, gd["q"], gd["W"], bias)
        assert np.array_equal(again["o"], first["o"]) and np.array_equal(again["lse"], first["lse"])


@pytest.mark.parametrize("d,G,blk", [(64, 1, 64), (64, 8, 128), (128, 2, 128), (128, 8, 64),
                                     (128, 4, 128)])
def test_shapes(d, G, blk):
    w = synth.Workload("shape", B=3, Hq=2 * G, Hkv=2, d=d, ctx=3000, blk=blk, n_clusters=16,
                       seg=200, needles=2, gate_T=0.0, density=0.4, density_kind="head",
                       seed=100 + d + G + blk)
    lengths = torch.tensor([3000, 2777, 1234], dtype=torch.int32)
    rep, gpu, sc = full_parity(w, lengths=lengths)


def test_probabilistic_bound_blk128():
    w = synth.EXTREME512K.with_(B=2, ctx=16384, seed=79)
    rep, gpu, sc = full_parity(w, bound="prob", z=3.0)
    rep2, gpu2, sc2 = full_parity(w, bound="exact")
    # same inputs, same metadata: the probabilistic bound is never looser
    assert np.all(gpu["bounds"] <= gpu2["bounds"] + 1e-6)


def test_const_tau_mode():
    w = synth.MID.with_(B=2, ctx=8192, seed=80)
    rep, gpu, sc = full_parity(w, tau_const=np.linspace(1.6, 2.2, w.Hq))
    assert np.allclose(gpu["tau"], np.linspace(1.6, 2.2, w.Hq)[None, :], atol=1e-6)


def test_tau_neg_inf_is_dense_attention_and_dense_kernel():
    w = synth.MID.with_(B=3, ctx=5000, needles=0, seed=81)
    g = to_dev(make(w, lengths=torch.tensor([5000, 4097, 64], dtype=torch.int32)))
    dec = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk, T=0.0)
    dec.build_meta()
    tau = torch.full((w.B, w.Hq), -math.inf, device=DEV)
    gpu = run_cuda(dec, g["q"], tau=tau)
    o_d, lse_d = [t.clone() for t in dec.dense_decode(g["q"])]
    torch.cuda.synchronize()
    dec.check_status()
    K64, V64, q64 = f64(g["K"]), f64(g["V"]), f64(g["q"])
    L = g["lengths"].cpu().numpy()
    o_ref, lse_ref = O.dense_decode(q64, K64, V64, L, 1.0 / math.sqrt(w.d))
    for o, lse in ((gpu["o"], gpu["lse"]), (f64(o_d), f64(lse_d))):
        err = np.abs(o - o_ref)
        assert err.max() <= 1e-2 and err.mean() <= 1e-3
        assert np.abs(lse - lse_ref).max() <= 1e-3
    np.testing.assert_allclose(gpu["o"], f64(o_d), atol=1e-5)


def test_tau_above_every_score_gives_uniform_mean():
    w = synth.MID.with_(B=2, ctx=4096, needles=0, seed=82)
    g = to_dev(make(w))
    dec = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk, T=0.0, prune="floor")
    dec.build_meta()
    tau = torch.full((w.B, w.Hq), 1e3, device=DEV)   # above every bound too: all pruned
    gpu = run_cuda(dec, g["q"], tau=tau)
    assert gpu["union_cnt"].sum() == 0
    V64 = f64(g["V"])
    for b in range(w.B):
        for h in range(w.Hq):
            np.testing.assert_allclose(gpu["o"][b, h], V64[b, h // w.G, :4096].mean(0),
                                       atol=1e-5)
            assert abs(gpu["lse"][b, h] - math.log(4096)) < 1e-5


@pytest.mark.parametrize("cent_format", ["f32", "bf16"])
def test_tail_append_update_matches_rebuild(cent_format):
    w = synth.MID.with_(B=3, ctx=4096, needles=0, seed=83)
    lengths = torch.tensor([4000, 4095, 100], dtype=torch.int32)
    g = to_dev(make(w, lengths=lengths))
    dec = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk, prune="floor",
                     cent_format=cent_format)
    dec.build_meta()
    # append one token per row and update only the tail blocks
    for b in range(w.B):
        t = int(dec.lengths[b])
        dec.K[b, :, t] = torch.randn(w.Hkv, w.d, device=DEV).to(torch.bfloat16)
        dec.V[b, :, t] = torch.randn(w.Hkv, w.d, device=DEV).to(torch.bfloat16)
    dec.lengths += 1
    dec.append_update()
    inc = {k: v.copy() for k, v in gpu_meta(dec).items()}
    dec.build_meta()
    full = gpu_meta(dec)
    for k in full:
        assert np.array_equal(inc[k], full[k]), k
    o_meta = O.cache_meta(f64(dec.K), dec.lengths.cpu().numpy(), w.blk, f64(dec.V),
                          cent_format)
    check_meta(full, o_meta)


def test_status_nonfinite_query_and_bad_arguments():
    w = synth.TINY.with_(seed=84)
    g = to_dev(make(w))
    dec = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk)
    dec.build_meta()
    q = g["q"].clone()
    q[0, 1, 3] = float("nan")
    dec.predict_tau(q, g["W"], None, None)
    torch.cuda.synchronize()
    with pytest.raises(EtaError):
        dec.check_status()
    # host-side validation: workspace too small, null pointer
    from long_context_decoding_eta_b200 import _lib as L
    small = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(EtaError) as ei:
        L.eta_decode(dec.dims, g["q"], dec.tau, dec.K, dec.V, dec.lengths, dec.union_idx,
                     dec.union_cnt, 0.0, 0.0, "skip", None, None, dec.o, dec.lse, small)
    assert ei.value.code == 3
    with pytest.raises(EtaError) as ei:
        L.eta_decode(dec.dims, None, dec.tau, dec.K, dec.V, dec.lengths, dec.union_idx,
                     dec.union_cnt, 0.0, 0.0, "skip", None, None, dec.o, dec.lse, dec.ws_decode)
    assert ei.value.code == 1


def test_calibration_matches_oracle_rule():
    w = synth.MID.with_(B=4, ctx=8192, needles=0, seed=85)
    g = make(w)
    gd = to_dev(g)
    dec = EtaDecoder(gd["K"], gd["V"], gd["lengths"], w.Hq, w.blk, keep_bounds=True)
    dec.build_meta()
    qc = synth.calibration_queries(w, g["mu"], n=16)
    tau_gpu = dec.calibrate_const_tau(qc, 0.38).numpy()
    # oracle: bounds of the same calibration queries on oracle metadata
    K64 = f64(g["K"])
    L = g["lengths"].numpy()
    meta = O.cache_meta(K64, L, w.blk)
    q64 = f64(qc)
    rows = np.arange(16) % w.B
    scale = 1.0 / math.sqrt(w.d)
    bounds = np.zeros((16, w.Hq, w.NB))
    valid = np.zeros((16, w.Hq, w.NB), dtype=bool)
    for i in range(16):
        mrow = {k: v[rows[i]:rows[i] + 1] for k, v in meta.items()}
        bounds[i] = O.screen(q64[i:i + 1], np.zeros((1, w.Hq)), mrow, scale)["bounds"][0]
        valid[i] = np.repeat(meta["cnt"][rows[i]] > 0, w.G, axis=0)
    tau_ref = O.calibrate_const_tau(bounds, valid, 0.38)
    np.testing.assert_allclose(tau_gpu, tau_ref, rtol=0, atol=2e-5)


def test_bounded_wait_times_out_with_status_and_context_survives():
    from long_context_decoding_eta_b200 import _lib as L
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)     # nothing ever sets it
    L.eta_selftest_wait_timeout(1 << 12, flag, status)
    torch.cuda.synchronize()
    assert int(status.item()) & L.DEVSTAT_TIMEOUT
    assert L.eta_status_from_device(int(status.item())) == 5
    # the context is still usable: a normal decode runs and matches the oracle
    rep, gpu, sc = full_parity(synth.TINY.with_(seed=86))


@pytest.mark.parametrize("d,G,blk,ctx", [(128, 4, 64, 8192), (128, 4, 64, 3000), (64, 8, 128, 4096),
                                          (128, 2, 128, 5000)])
def test_bf16_centroids(d, G, blk, ctx):
    """Compact metadata: centroids rounded to bf16, radii measured against them
    (vector screen when NB % 8 == 0, scalar otherwise)."""
    w = synth.Workload("bf16cent", B=3, Hq=2 * G, Hkv=2, d=d, ctx=ctx, blk=blk, n_clusters=16,
                       seg=200, needles=2, gate_T=0.0, density=0.3, density_kind="head",
                       q_scale=4.0, seed=300 + d + G + blk)
    rep, gpu, sc = full_parity(w, cent_format="bf16")
    for prune in ("skip", "floor"):
        full_parity(w, cent_format="bf16", prune=prune, bound="prob", z=2.0)


def test_cuda_graph_replay_matches_eager_step():
    w = synth.MID.with_(B=4, ctx=8192, seed=87)
    g = to_dev(make(w))
    dec = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk, T=w.gate_T, cent_format="bf16")
    dec.build_meta()
    bias = torch.full((w.Hq,), 1.9, device=DEV)
    q = g["q"].clone()
    o_e, l_e = [t.clone() for t in dec.step(q, g["W"], bias)]
    dec.capture(q, g["W"], bias, split=True)
    for k in range(2):                       # new queries written in place, replayed twice
        q.copy_(g["q"] * (1.0 + 0.5 * k))
        o_g, l_g = [t.clone() for t in dec.replay()]
        o_r, l_r = [t.clone() for t in dec.step(q, g["W"], bias)]
        torch.cuda.synchronize()
        dec.check_status()
        assert torch.equal(o_g, o_r) and torch.equal(l_g, l_r)
    assert not torch.equal(o_g, o_e)


@pytest.mark.parametrize("cent_format", ["f32", "bf16"])
@pytest.mark.parametrize("ctx", [8192, 3000])
def test_per_dimension_variance_bound(cent_format, ctx):
    w = synth.MID.with_(B=3, ctx=ctx, needles=4, q_scale=4.0, density=0.3, seed=310 + ctx)
    for z in (1.0, 3.0):
        full_parity(w, bound="prob_dim", z=z, cent_format=cent_format, T=0.0)


@pytest.mark.parametrize("d,G,Hkv,bound", [(128, 4, 2, "exact"), (128, 4, 2, "prob"),
                                           (128, 8, 1, "prob_dim"), (128, 1, 4, "exact"),
                                           (64, 2, 2, "prob")])
def test_bf16_screen_of_long_rows(d, G, Hkv, bound, engine):
    """Rows longer than two rounds of the one-launch screen's group buffers take the
    two-launch screen (vector screening, then compaction) with bf16 centroids, a
    partial last group and one ragged row: masks, bounds and union lists against the
    oracle."""
    from long_context_decoding_eta_b200 import _lib as L
    # more groups per row than two rounds of the one-launch screen's buffers (5 at
    # d = 128, 8 at d = 64), and a partial last group
    ctx = (96 if d == 128 else 160) * 1024 + 512
    w = synth.Workload("bf16-long-rows", B=2, Hq=G * Hkv, Hkv=Hkv, d=d, ctx=ctx,
                       blk=64, n_clusters=32, seg=(384, 640), needles=2, gate_T=0.0,
                       density=0.3, density_kind="head", q_scale=2.0, seed=320 + d + G)
    dims = L.Dims.of(w.B, w.Hq, w.Hkv, w.d, w.blk, w.T_max)
    if engine == "fma":
        assert L.eta_screen_launches(dims, "bf16") == 2
    elif bound != "prob_dim":
        # the tensor-core screen: a CTA per pair with its compaction (13 or 21 groups
        # per row)
        assert L.eta_screen_launches(dims, "bf16") == 1
    lengths = torch.tensor([w.ctx, w.ctx - 7000], dtype=torch.int32)
    full_parity(w, lengths=lengths, bound=bound, z=2.0, cent_format="bf16")


@pytest.mark.parametrize("B,Hkv,G,ctx,bound,d", [(3, 2, 4, 9216, "exact", 128),
                                                (2, 1, 8, 40960, "prob", 128),
                                                (40, 4, 1, 8192, "exact", 128),
                                                (37, 4, 2, 4096, "prob", 128),
                                                (20, 8, 4, 6144, "exact", 128),
                                                (6, 2, 4, 9216, "prob", 64),
                                                (40, 4, 2, 8192, "exact", 64)])
def test_tensor_core_screen_against_cuda_core_screen(B, Hkv, G, ctx, bound, d, engine):
    """eta_screen on the tensor cores (one launch with a CTA per pair for small
    batches, or (row, group) items over one CTA per SM and the compaction after)
    against the CUDA-core screen on the same inputs: the bounds agree to fp32
    rounding, the admit words bit for bit except blocks whose bound lies within
    1e-5 (relative) of tau, the union lists and counts follow the words.  Ragged
    rows, a partial last group, G = 1/2/4/8, the exact and the variance bound."""
    from long_context_decoding_eta_b200 import _lib as L
    if engine == "fma":
        pytest.skip("one comparison of the two screens is enough")
    w = synth.Workload("tc-screen", B=B, Hq=G * Hkv, Hkv=Hkv, d=d, ctx=ctx, blk=64,
                       n_clusters=24, seg=(200, 500), needles=2, gate_T=0.0, density=0.35,
                       density_kind="union", q_scale=2.0, seed=600 + B + G)
    lens = [(ctx - 977 * i) if i % 3 else ctx for i in range(B)]
    lens = [max(x, 1) for x in lens]
    g = to_dev(make(w, lengths=torch.tensor(lens, dtype=torch.int32)))
    dec = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk, bound=bound, z=2.0, T=0.0,
                     cent_format="bf16")
    dims = dec.dims
    R, NB = B * Hkv, dec.NB
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    assert L.eta_screen_launches(dims, "bf16") == (1 if R <= n_sm and (NB + 127) // 128 <= 32
                                                   else 2)
    dec.build_meta()
    q = g["q"]
    bias = torch.zeros(w.Hq, device=DEV)
    dec.predict_tau(q, g["W"], bias)
    out = {}
    for eng in ("tcgen05", "fma"):
        L.eta_set_screen_engine(eng)
        bnd = torch.empty(B, w.Hq, NB, device=DEV)
        dec.screen(q, bounds=bnd)
        if eng == "tcgen05":
            # threshold offset for ~35% union, from the tensor-core bounds
            m = (bnd - dec.tau[..., None]).view(B, Hkv, G, NB).amax(2).flatten()
            off = float(torch.quantile(m.float()[::3], 0.65))
            dec.tau += off
            dec.screen(q, bounds=bnd)
        torch.cuda.synchronize()
        dec.check_status()
        out[eng] = dict(b=bnd.clone(), hm=dec.head_mask.clone(), uc=dec.union_cnt.clone(),
                        ui=dec.union_idx.clone())
    L.eta_set_screen_engine("auto")
    t, f = out["tcgen05"], out["fma"]
    valid = dec.cnt.view(B, Hkv, 1, NB).expand(B, Hkv, G, NB).reshape(B, w.Hq, NB) > 0
    db = (t["b"] - f["b"]).abs()[valid]
    assert float(db.max()) <= 1e-4 * max(1.0, float(f["b"][valid].abs().max()))
    tau = dec.tau[..., None]
    near = ((f["b"] - tau).abs() <= 1e-5 * torch.clamp(tau.abs(), min=1.0)) & valid
    mt, mf = unpack_mask(t["hm"], NB), unpack_mask(f["hm"], NB)
    diff = (mt != mf)
    assert not np.any(diff & ~near.cpu().numpy()), int(np.sum(diff & ~near.cpu().numpy()))
    # union lists follow the words
    ut = mt.reshape(B, Hkv, G, NB).any(2)
    cnt_t = t["uc"].cpu().numpy()
    assert np.array_equal(cnt_t, ut.sum(-1))
    ui = t["ui"].cpu().numpy()
    for b in range(B):
        for k in range(Hkv):
            assert np.array_equal(ui[b, k, :cnt_t[b, k]], np.nonzero(ut[b, k])[0])
    adm = float(ut.mean())
    assert 0.05 < adm < 0.95, adm
