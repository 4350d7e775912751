"""The one-launch decode step (eta_decode_step) against the four separate calls
(bit for bit) and against the float64 oracle (the stated tolerances), after a
token was appended to every row that has room."""
import math

import numpy as np
import pytest
import torch

from long_context_decoding_eta_b200 import synth
from long_context_decoding_eta_b200._lib import EtaError
from long_context_decoding_eta_b200.api import EtaDecoder

from eta_testlib import (check_meta, compare_step, density_bias, f64, gpu_meta, oracle_step,
                         unpack_mask)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _append_token(K, V, lengths, gen):
    """Appends one random key/value to every row with room (in place)."""
    T_max = K.shape[2]
    for b in range(K.shape[0]):
        t = int(lengths[b])
        if t < T_max:
            K[b, :, t] = (0.3 * torch.randn(K.shape[1], K.shape[3], generator=gen)).to(DEV).to(
                torch.bfloat16)
            V[b, :, t] = torch.randn(V.shape[1], V.shape[3], generator=gen).to(DEV).to(
                torch.bfloat16)
            lengths[b] += 1


def _outputs(dec):
    cnt = dec.union_cnt.cpu().numpy()
    uidx = dec.union_idx.cpu().numpy()
    return dict(tau=dec.tau.cpu().numpy(), head_mask=dec.head_mask.cpu().numpy(), union_cnt=cnt,
                union_lists=[[uidx[b, g, :cnt[b, g]] for g in range(cnt.shape[1])]
                             for b in range(cnt.shape[0])],
                head_cnt=dec.head_cnt.cpu().numpy(), o=dec.o.cpu().numpy(),
                lse=dec.lse.cpu().numpy(), **gpu_meta(dec))


def _assert_identical(a, b):
    for k in a:
        if k == "union_lists":
            for ra, rb in zip(a[k], b[k]):
                for la, lb in zip(ra, rb):
                    assert np.array_equal(la, lb), k
        else:
            assert np.array_equal(a[k], b[k], equal_nan=True), k


def fused_vs_separate(w, *, lengths=None, bound=None, z=None, T=None, cent_format="f32",
                      tau_const=None, density=None, check_oracle=True):
    T = w.gate_T if T is None else T
    bound = w.bound if bound is None else bound
    z = w.z if z is None else z
    density = w.density if density is None else density
    g = synth.generate(w, "cpu", lengths=lengths)
    K64, V64, q64, W64 = f64(g["K"]), f64(g["V"]), f64(g["q"]), f64(g["W"])
    Lh = g["lengths"].numpy().astype(np.int64)
    scale = 1.0 / math.sqrt(w.d)
    bias = np.full(w.Hq, density_bias(K64, q64, Lh, W64, w.blk, scale, w.G, density,
                                      w.density_kind, bound, z, cent_format))
    K, V = g["K"].to(DEV), g["V"].to(DEV)
    lens = g["lengths"].to(DEV)
    q, W = g["q"].to(DEV), g["W"].to(DEV)
    kw = dict(bound=bound, z=z, T=T, cent_format=cent_format)
    sep = EtaDecoder(K, V, lens, w.Hq, w.blk, **kw)
    fus = EtaDecoder(K, V, lens, w.Hq, w.blk, fused=True, **kw)
    assert sep.lengths.data_ptr() == fus.lengths.data_ptr()     # one cache, two metadata sets
    sep.build_meta()
    fus.build_meta()
    _append_token(K, V, sep.lengths, torch.Generator().manual_seed(w.seed + 7))
    bias_t = torch.tensor(bias, dtype=torch.float32, device=DEV)
    tc = None if tau_const is None else torch.tensor(tau_const, dtype=torch.float32, device=DEV)
    Wp = None if tc is not None else W
    sep.step(q, Wp, bias_t, tc)
    fus.step(q, Wp, bias_t, tc)
    torch.cuda.synchronize()
    sep.check_status()
    fus.check_status()
    a, b = _outputs(sep), _outputs(fus)
    _assert_identical(a, b)
    if check_oracle:
        K64, V64 = f64(K), f64(V)
        Lh = sep.lengths.cpu().numpy().astype(np.int64)
        meta, tau, sc, o, lse = oracle_step(K64, V64, q64, Lh, W64, bias, w.blk, scale, T, bound,
                                            z, "skip", tau_const, cent_format)
        check_meta(gpu_meta(fus), meta)
        gpu = dict(tau=f64(fus.tau), head_mask=unpack_mask(fus.head_mask, fus.NB),
                   union_idx=fus.union_idx.cpu().numpy(), union_cnt=fus.union_cnt.cpu().numpy(),
                   head_cnt=fus.head_cnt.cpu().numpy(), o=f64(fus.o), lse=f64(fus.lse))
        compare_step(gpu, tau, sc, o, lse, q64, K64, V64, Lh, w.blk, scale, T, w.G)
    return sep, fus, q, Wp, bias_t, tc


def test_mid_soft_gate():
    fused_vs_separate(synth.MID.with_(B=4, ctx=8192, seed=401))


def test_bf16_centroids_per_dimension_bound():
    w = synth.MID.with_(B=3, ctx=8192, needles=4, q_scale=4.0, density=0.3, seed=402)
    fused_vs_separate(w, bound="prob_dim", z=2.0, cent_format="bf16", T=0.0)


def test_probabilistic_bound_blk128():
    fused_vs_separate(synth.EXTREME512K.with_(B=2, ctx=16384, seed=403), cent_format="bf16")


@pytest.mark.parametrize("screen_engine", ["auto", "fma"])
@pytest.mark.parametrize("bound", ["exact", "prob"])
def test_bf16_screening_forms(screen_engine, bound):
    """bf16 centroids with the exact and the variance bound: the step screens on the
    tensor cores when eta_screen does (the default) and on the CUDA cores when the
    screen engine says so; either way it writes the separate calls' bits.  A
    multi-group row with a partial last group (NB = 144)."""
    from long_context_decoding_eta_b200 import _lib as L
    w = synth.MID.with_(B=5, ctx=9216, needles=3, q_scale=3.0, density=0.35, seed=420)
    L.eta_set_screen_engine(screen_engine)
    try:
        fused_vs_separate(w, bound=bound, z=2.0, cent_format="bf16")
    finally:
        L.eta_set_screen_engine("auto")


def test_const_tau():
    w = synth.MID.with_(B=2, ctx=8192, seed=404)
    fused_vs_separate(w, tau_const=np.linspace(1.6, 2.2, w.Hq))


@pytest.mark.parametrize("cent_format", ["f32", "bf16"])
@pytest.mark.parametrize("G,blk", [(1, 64), (2, 128), (8, 64), (4, 128)])
def test_shapes_ragged_lengths(G, blk, cent_format):
    """Rows that are full, empty, one token long and ragged (bf16 centroids: the
    screening on the tensor cores in both the step and the separate calls)."""
    w = synth.Workload("fused-shape", B=4, Hq=2 * G, Hkv=2, d=128, ctx=3072, blk=blk,
                       n_clusters=16, seg=200, needles=2, gate_T=0.0, density=0.4,
                       density_kind="head", seed=410 + G + blk)
    lengths = torch.tensor([3072, 0, 1, 2000], dtype=torch.int32)
    sep, fus, *_ = fused_vs_separate(w, lengths=lengths, cent_format=cent_format)
    # the empty row got its token; a row whose union is empty reads o = 0, lse = -inf
    cnt = fus.union_cnt.cpu().numpy()
    for b, g in zip(*np.nonzero(cnt == 0)):
        hs = slice(g * G, (g + 1) * G)
        assert torch.all(fus.o[b, hs] == 0) and torch.all(torch.isneginf(fus.lse[b, hs]))


def test_repeated_calls_and_graph_replay():
    """The workspace counters reset themselves: back-to-back calls and replays of a
    captured graph keep matching the separate calls."""
    w = synth.MID.with_(B=4, ctx=8192, seed=405)
    sep, fus, q, Wp, bias_t, tc = fused_vs_separate(w, check_oracle=False)
    q0 = q.clone()
    for k in range(3):
        q.copy_(q0 * (1.0 + 0.25 * k))
        sep.step(q, Wp, bias_t, tc)
        fus.step(q, Wp, bias_t, tc)
        torch.cuda.synchronize()
        fus.check_status()
        _assert_identical(_outputs(sep), _outputs(fus))
    fus.capture(q, Wp, bias_t, tc)
    for k in range(3):
        q.copy_(q0 * (0.5 + 0.5 * k))
        fus.replay()
        sep.step(q, Wp, bias_t, tc)
        torch.cuda.synchronize()
        fus.check_status()
        _assert_identical(_outputs(sep), _outputs(fus))


def test_rejects_unsupported():
    w = synth.TINY.with_(seed=406)        # d = 64: the fused step needs d = 128
    g = synth.generate(w, "cpu")
    dec = EtaDecoder(g["K"].to(DEV), g["V"].to(DEV), g["lengths"].to(DEV), w.Hq, w.blk,
                     fused=True)
    dec.build_meta()
    with pytest.raises(EtaError) as ei:
        dec.step(g["q"].to(DEV), g["W"].to(DEV), None, None)
    assert ei.value.code == 2                  # ETA_ERR_UNSUPPORTED
    with pytest.raises(ValueError):
        EtaDecoder(g["K"].to(DEV), g["V"].to(DEV), g["lengths"].to(DEV), w.Hq, w.blk,
                   fused=True, prune="floor")


@pytest.mark.parametrize("cent_format,bound,tau_mode", [("f32", "exact", "predictor"),
                                                         ("bf16", "prob_dim", "predictor"),
                                                         ("bf16", "exact", "const")])
def test_append_and_predict_tau_equals_the_two_calls(cent_format, bound, tau_mode):
    """eta_append_and_predict_tau writes the same bits as eta_build_block_meta on the tail
    block plus eta_predict_tau, after a token was appended to each row with room."""
    w = synth.MID.with_(B=4, ctx=4096, needles=0, seed=420)
    lengths = torch.tensor([4096, 0, 1, 2000], dtype=torch.int32)
    g = synth.generate(w, "cpu", lengths=lengths)
    K, V, q, W = (g[k].to(DEV) for k in ("K", "V", "q", "W"))
    lens = g["lengths"].to(DEV)
    kw = dict(bound=bound, cent_format=cent_format, prune="floor")
    a = EtaDecoder(K, V, lens, w.Hq, w.blk, merged_prologue=False, **kw)
    b = EtaDecoder(K, V, lens, w.Hq, w.blk, merged_prologue=True, **kw)
    a.build_meta()
    b.build_meta()
    _append_token(K, V, a.lengths, torch.Generator().manual_seed(421))
    bias = torch.full((w.Hq,), 0.7, device=DEV)
    tc = torch.linspace(1.0, 2.0, w.Hq, device=DEV) if tau_mode == "const" else None
    Wp = None if tc is not None else W
    a.prepare(q, Wp, bias, tc)
    b.prepare(q, Wp, bias, tc)
    torch.cuda.synchronize()
    a.check_status()
    b.check_status()
    _assert_identical(_outputs(a), _outputs(b))
