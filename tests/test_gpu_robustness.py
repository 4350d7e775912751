"""Robustness claims of the kernels, tested rather than asserted:

* cache memory at and past lengths[b] is never used: it is filled with NaN and
  +Inf here (and the prefill's queries and thresholds past the length too), and
  every output must still match the float64 oracle, which reads valid keys only;
* nothing a call reads from its workspace needs to start at any value: the decode
  workspace (and the partial-result slots of the one-launch step's workspace) is
  filled with 0xFF bytes (NaN as fp32, -1 as int32) before every call, and the
  outputs must be the same bits as with a clean workspace.
"""
import math

import numpy as np
import pytest
import torch

from long_context_decoding_eta_b200 import _lib as L
from long_context_decoding_eta_b200 import synth
from long_context_decoding_eta_b200.api import EtaDecoder
from oracle import eta_oracle as O

from eta_testlib import (check_meta, compare_step, density_bias, f64, gpu_meta, oracle_step,
                         run_cuda, unpack_mask)

pytestmark = pytest.mark.gpu


def poison_past_lengths(x: torch.Tensor, lengths: torch.Tensor):
    """x [B, H, T_max, ...]: NaN past the length of even rows, +Inf of odd rows."""
    for b in range(x.shape[0]):
        n = int(lengths[b])
        x[b, :, n:] = float("nan") if b % 2 == 0 else float("inf")


def poisoned_case(w, lengths):
    g = synth.generate(w, "cpu", lengths=lengths)
    for k in ("K", "V"):
        poison_past_lengths(g[k], g["lengths"])
    return g


@pytest.mark.parametrize("engine", ["fma", "tcgen05"])
@pytest.mark.parametrize("T,prune,cent", [(0.0, "skip", "f32"), (0.05, "floor", "f32"),
                                          (0.0, "skip", "bf16")])
def test_cache_past_lengths_poisoned(engine, T, prune, cent):
    w = synth.MID.with_(B=4, ctx=4096, seed=301)
    lengths = torch.tensor([4096, 4000, 1, 2113], dtype=torch.int32)
    g = poisoned_case(w, lengths)
    K64, V64, q64, W64 = f64(g["K"]), f64(g["V"]), f64(g["q"]), f64(g["W"])
    Lr = g["lengths"].numpy().astype(np.int64)
    scale = 1.0 / math.sqrt(w.d)
    bias = np.full(w.Hq, density_bias(K64, q64, Lr, W64, w.blk, scale, w.G, 0.4, "union",
                                      cent_format=cent))
    L.eta_set_decode_engine(engine)
    try:
        dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in g.items()}
        dec = EtaDecoder(dev["K"], dev["V"], dev["lengths"], w.Hq, w.blk, T=T, prune=prune,
                         keep_bounds=True, cent_format=cent)
        dec.build_meta()
        gpu = run_cuda(dec, dev["q"], dev["W"], torch.tensor(bias, dtype=torch.float32,
                                                             device="cuda"))
    finally:
        L.eta_set_decode_engine("auto")
    assert np.all(np.isfinite(gpu["o"])) and np.all(np.isfinite(gpu["tau"]))
    meta, tau, sc, o, lse = oracle_step(K64, V64, q64, Lr, W64, bias, w.blk, scale, T,
                                        prune=prune, cent_format=cent)
    check_meta(gpu_meta(dec), meta)
    rep = compare_step(gpu, tau, sc, o, lse, q64, K64, V64, Lr, w.blk, scale, T, w.G)
    print(rep)


def test_fused_step_cache_past_lengths_poisoned():
    """The one-launch step (tail refresh, thresholds, screening, decode) on a cache
    poisoned past every length, after a token was appended to every row."""
    w = synth.MID.with_(B=4, ctx=4096, seed=302, gate_T=0.0)
    lengths = torch.tensor([4096, 3001, 64, 2113], dtype=torch.int32)
    g = poisoned_case(w, lengths)
    K64, V64, q64, W64 = f64(g["K"]), f64(g["V"]), f64(g["q"]), f64(g["W"])
    Lr = g["lengths"].numpy().astype(np.int64)
    scale = 1.0 / math.sqrt(w.d)
    bias = np.full(w.Hq, density_bias(K64, q64, Lr, W64, w.blk, scale, w.G, 0.4, "union",
                                      cent_format="bf16"))
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in g.items()}
    # metadata built one token short, then the step's tail refresh brings it level
    short = (dev["lengths"] - 1).clamp(min=0)
    fus = EtaDecoder(dev["K"], dev["V"], short, w.Hq, w.blk, fused=True, cent_format="bf16")
    fus.build_meta()
    fus.lengths.copy_(dev["lengths"])
    fus.step(dev["q"], dev["W"], torch.tensor(bias, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    fus.check_status()
    gpu = dict(tau=f64(fus.tau), head_mask=unpack_mask(fus.head_mask, fus.NB),
               union_idx=fus.union_idx.cpu().numpy(), union_cnt=fus.union_cnt.cpu().numpy(),
               head_cnt=fus.head_cnt.cpu().numpy(), o=f64(fus.o), lse=f64(fus.lse))
    assert np.all(np.isfinite(gpu["o"]))
    meta, tau, sc, o, lse = oracle_step(K64, V64, q64, Lr, W64, bias, w.blk, scale, 0.0,
                                        cent_format="bf16")
    check_meta(gpu_meta(fus), meta)
    print(compare_step(gpu, tau, sc, o, lse, q64, K64, V64, Lr, w.blk, scale, 0.0, w.G))


@pytest.mark.parametrize("kernel", ["one_tile", "two_tile"])
@pytest.mark.parametrize("T_gate", [0.0, 0.05])
def test_prefill_past_lengths_poisoned(T_gate, kernel):
    L.eta_set_prefill_kernel(kernel)
    try:
        _prefill_past_lengths_poisoned(T_gate)
    finally:
        L.eta_set_prefill_kernel("auto")


def _prefill_past_lengths_poisoned(T_gate):
    B, Hq, Hkv, T_max, d = 2, 8, 2, 384, 128
    gen = torch.Generator().manual_seed(303)
    q = torch.randn(B, Hq, T_max, d, generator=gen).to(torch.bfloat16)
    K = torch.randn(B, Hkv, T_max, d, generator=gen).to(torch.bfloat16)
    V = torch.randn(B, Hkv, T_max, d, generator=gen).to(torch.bfloat16)
    tau = (0.5 + 0.5 * torch.randn(B, Hq, T_max, generator=gen)).float()
    lengths = torch.tensor([300, 129], dtype=torch.int32)
    for x in (q, K, V, tau):
        poison_past_lengths(x, lengths)
    dims = L.Dims.of(B, Hq, Hkv, d, 64, T_max)
    O_g = torch.zeros(B, Hq, T_max, d, device="cuda")
    lse_g = torch.zeros(B, Hq, T_max, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.eta_prefill(dims, q.cuda(), tau.cuda(), K.cuda(), V.cuda(), lengths.cuda(), T_gate, 0.0,
                  O_g, lse_g, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    scale = 1.0 / math.sqrt(d)
    q64, K64, V64, t64 = (x.double().numpy() for x in (q, K, V, tau))
    o_r, lse_r = O.prefill(q64, t64, K64, V64, lengths.numpy(), scale, T_gate)
    o_g, l_g = O_g.double().cpu().numpy(), lse_g.double().cpu().numpy()
    G = Hq // Hkv
    errs, lerrs = [], []
    for b in range(B):
        for h in range(Hq):
            for t in range(int(lengths[b])):
                if T_gate == 0.0:
                    s = scale * K64[b, h // G, :t + 1] @ q64[b, h, t]
                    if np.any(np.abs(s - t64[b, h, t]) <= 1e-5 * max(1.0, abs(t64[b, h, t]))):
                        continue
                errs.append(np.abs(o_g[b, h, t] - o_r[b, h, t]))
                lerrs.append(abs(l_g[b, h, t] - lse_r[b, h, t]))
    e = np.stack(errs)
    assert e.max() <= 1e-2 and e.mean() <= 1e-3, (e.max(), e.mean())
    assert max(lerrs) <= 1e-3, max(lerrs)
    for b in range(B):
        assert torch.all(O_g[b, :, int(lengths[b]):] == 0)


def _decoder(w, lengths, prune="skip", fused=False):
    g = synth.generate(w, "cuda", lengths=lengths)
    dec = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk, T=w.gate_T, prune=prune,
                     fused=fused, cent_format="bf16")
    dec.build_meta()
    return g, dec


@pytest.mark.parametrize("engine", ["fma", "tcgen05"])
@pytest.mark.parametrize("B,prune", [(4, "skip"), (4, "floor"), (32, "skip")])
def test_decode_workspace_poisoned_before_every_call(engine, B, prune):
    """4 x 4 = 16 pairs (separate share plan) and 32 x 4 = 128 pairs (the tensor-core
    decode plans its shares in the kernel); each decode twice, the workspace filled
    with 0xFF before each call."""
    w = synth.MID.with_(B=B, ctx=2048, seed=304 + B)
    g, dec = _decoder(w, synth.ragged_lengths(B, 2048, 64, gen_seed=5), prune)
    bias = torch.full((w.Hq,), 1.9, device="cuda")
    L.eta_set_decode_engine(engine)
    try:
        dec.predict_tau(g["q"], g["W"], bias)
        dec.screen(g["q"])
        dec.ws_decode.zero_()
        dec.decode(g["q"])
        ref_o, ref_l = dec.o.clone(), dec.lse.clone()
        for _ in range(2):
            dec.ws_decode.fill_(0xFF)
            dec.o.fill_(float("nan"))
            dec.lse.fill_(float("nan"))
            dec.decode(g["q"])
            torch.cuda.synchronize()
            dec.check_status()
            assert torch.equal(dec.o, ref_o) and torch.equal(dec.lse, ref_l)
    finally:
        L.eta_set_decode_engine("auto")
    assert bool(torch.isfinite(ref_o).all())


def _fused_partial_bytes(dec) -> int:
    """Bytes at the start of the one-launch step's workspace that hold the partial
    (m, l, o) slots: (P + R) slots of G * (2 + d) floats, each part 256-aligned
    (the rest holds the self-resetting counters, which must stay zeroed)."""
    P = torch.cuda.get_device_properties(dec.K.device).multi_processor_count
    R, G = dec.B * dec.Hkv, dec.Hq // dec.Hkv
    up = lambda x: (x + 255) // 256 * 256
    return up(up((P + R) * G * 2 * 4) + (P + R) * G * dec.d * 4)


@pytest.mark.parametrize("B", [4, 32])
def test_fused_step_partial_slots_poisoned_before_every_call(B):
    w = synth.MID.with_(B=B, ctx=2048, seed=310 + B, gate_T=0.0)
    g, dec = _decoder(w, synth.ragged_lengths(B, 2048, 64, gen_seed=6), fused=True)
    bias = torch.full((w.Hq,), 1.9, device="cuda")
    dec.step(g["q"], g["W"], bias, append=False)
    torch.cuda.synchronize()
    dec.check_status()
    ref_o, ref_l = dec.o.clone(), dec.lse.clone()
    n = _fused_partial_bytes(dec)
    assert n < dec.ws_step.numel()
    for _ in range(2):
        dec.ws_step[:n].fill_(0xFF)
        dec.o.fill_(float("nan"))
        dec.lse.fill_(float("nan"))
        dec.step(g["q"], g["W"], bias, append=False)
        torch.cuda.synchronize()
        dec.check_status()
        assert torch.equal(dec.o, ref_o) and torch.equal(dec.lse, ref_l)
    assert bool(torch.isfinite(ref_o).all())
