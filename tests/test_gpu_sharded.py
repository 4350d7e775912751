"""Sequence-sharded decode on one GPU: the cache split into block-aligned shards,
each shard stepped by its own EtaDecoder, the shards' (o, lse) merged by
eta_lse_merge, against the unsharded step and the float64 oracle.  (The gather
between GPUs is plain torch.distributed; its host side is covered on CPU in
test_multirank_cpu.py.)"""
import math

import numpy as np
import pytest
import torch

from long_context_decoding_eta_b200 import _lib as L
from long_context_decoding_eta_b200 import synth
from long_context_decoding_eta_b200.api import EtaDecoder
from long_context_decoding_eta_b200.sharded import ShardedEtaDecoder, shard_lengths, shard_range
from oracle import eta_oracle as O

from eta_testlib import density_bias, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("world,prune,T", [(2, "skip", 0.0), (3, "skip", 0.05), (4, "floor", 0.0)])
def test_shards_merge_to_the_whole_cache(world, prune, T):
    w = synth.MID.with_(B=3, ctx=8192, seed=500 + world)
    lengths = torch.tensor([8192, 5000, 700], dtype=torch.int32)
    g = synth.generate(w, "cpu", lengths=lengths)
    K64, V64, q64, W64 = f64(g["K"]), f64(g["V"]), f64(g["q"]), f64(g["W"])
    Lh = lengths.numpy().astype(np.int64)
    scale = 1.0 / math.sqrt(w.d)
    bias = np.full(w.Hq, density_bias(K64, q64, Lh, W64, w.blk, scale, w.G, 0.3, "head"))
    K, V, q, W = (g[k].to(DEV) for k in ("K", "V", "q", "W"))
    bias_t = torch.tensor(bias, dtype=torch.float32, device=DEV)
    whole = EtaDecoder(K, V, lengths.to(DEV), w.Hq, w.blk, T=T, prune=prune)
    whole.build_meta()
    o_w, lse_w = [t.clone() for t in whole.step(q, W, bias_t)]
    o_parts, lse_parts = [], []
    for r in range(world):
        t0, t1 = shard_range(w.ctx, w.blk, world, r)
        dec = EtaDecoder(K[:, :, t0:t1].contiguous(), V[:, :, t0:t1].contiguous(),
                         shard_lengths(lengths, t0, t1).to(DEV), w.Hq, w.blk, T=T, prune=prune)
        dec.build_meta()
        o, lse = dec.step(q, W, bias_t)
        o_parts.append(o.clone())
        lse_parts.append(lse.clone())
        # the shard admits exactly the whole cache's union blocks in its range
        nb0 = t0 // w.blk
        for b in range(w.B):
            for gg in range(w.Hkv):
                cw = int(whole.union_cnt[b, gg])
                want = whole.union_idx[b, gg, :cw].cpu().numpy()
                want = want[(want >= nb0) & (want < t1 // w.blk)] - nb0
                cs = int(dec.union_cnt[b, gg])
                assert np.array_equal(dec.union_idx[b, gg, :cs].cpu().numpy(), want)
    o_m = torch.empty_like(o_w)
    lse_m = torch.empty_like(lse_w)
    L.eta_lse_merge(torch.stack(o_parts), torch.stack(lse_parts), o_m, lse_m)
    torch.cuda.synchronize()
    # against the unsharded step: the same gated softmax, split differently
    assert torch.allclose(o_m, o_w, atol=2e-5, rtol=0)
    assert torch.allclose(lse_m, lse_w, atol=2e-5, rtol=0)
    # against the oracle (the whole cache)
    meta = O.cache_meta(K64, Lh, w.blk, V64 if prune == "floor" else None)
    tau = O.predict_tau(q64, W64, bias)
    sc = O.screen(q64, tau, meta, scale)
    o_ref, lse_ref = O.decode(q64, tau, K64, V64, Lh, sc["union_idx"], w.blk, scale, T, prune,
                              meta)
    keep = np.ones((w.B, w.Hq), dtype=bool)
    for b in range(w.B):                       # heads whose union had a near-tie are skipped
        for h in range(w.Hq):
            cw = int(whole.union_cnt[b, h // w.G])
            if sorted(sc["union_idx"][b][h // w.G]) != list(whole.union_idx[b, h // w.G, :cw].cpu().numpy()):
                keep[b, h] = False
    e = np.abs(f64(o_m) - o_ref)[keep]
    assert e.max() <= 1e-2 and e.mean() <= 1e-3
    assert np.abs(f64(lse_m) - lse_ref)[keep].max() <= 1e-3


def test_merge_edge_cases():
    d, rows = 128, 5
    o_parts = torch.randn(3, rows, d, device=DEV)
    lse_parts = torch.randn(3, rows, device=DEV)
    lse_parts[:, 0] = -math.inf                 # every part empty
    lse_parts[1, 1] = -math.inf                 # one part empty
    lse_parts[:, 2] = torch.tensor([50.0, -50.0, 0.0])   # one part dominates
    o = torch.empty(rows, d, device=DEV)
    lse = torch.empty(rows, device=DEV)
    L.eta_lse_merge(o_parts, lse_parts, o, lse)
    torch.cuda.synchronize()
    ref_o, ref_l = O.lse_merge(f64(o_parts), f64(lse_parts))
    assert torch.all(o[0] == 0) and math.isinf(lse[0].item()) and lse[0].item() < 0
    np.testing.assert_allclose(f64(o)[1:], ref_o[1:], rtol=0, atol=1e-5)
    np.testing.assert_allclose(f64(lse)[1:], ref_l[1:], rtol=0, atol=1e-5)
    # a single part is passed through (row 0 of it has no keys: o = 0, lse = -inf)
    L.eta_lse_merge(o_parts[2:], lse_parts[2:], o, lse)
    torch.cuda.synchronize()
    assert torch.equal(o[1:], o_parts[2, 1:]) and torch.equal(lse[1:], lse_parts[2, 1:])
    assert torch.all(o[0] == 0) and math.isinf(lse[0].item())


def test_sharded_decoder_without_process_group_is_the_plain_step():
    w = synth.MID.with_(B=2, ctx=4096, seed=510)
    g = synth.generate(w, "cpu")
    K, V, q, W = (g[k].to(DEV) for k in ("K", "V", "q", "W"))
    lens = g["lengths"].to(DEV)
    bias = torch.full((w.Hq,), 1.9, device=DEV)
    plain = EtaDecoder(K, V, lens, w.Hq, w.blk, T=0.05)
    plain.build_meta()
    o_p, l_p = [t.clone() for t in plain.step(q, W, bias)]
    sh = ShardedEtaDecoder(K, V, lens, 0, w.Hq, w.blk, T=0.05)
    sh.build_meta()
    o_s, l_s = sh.step(q, W, bias)
    torch.cuda.synchronize()
    assert torch.equal(o_s, o_p) and torch.equal(l_s, l_p)
