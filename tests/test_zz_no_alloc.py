"""eta_decode_static: the decode entry point for callers that cannot allocate
device memory (for example a serving loop whose memory is all reserved by its
own pool, or code that must not call cudaMalloc on the decode path because it
can synchronize the device).  It runs the same kernels as eta_decode with a
caller workspace, so its outputs must be the same bits, call after call,
although its scratch is a fixed array shared by all calls and left holding the
previous call's data.  This file is collected last on purpose."""
import pytest
import torch

from long_context_decoding_eta_b200 import _lib as L
from long_context_decoding_eta_b200 import synth
from long_context_decoding_eta_b200.api import EtaDecoder

pytestmark = pytest.mark.gpu


def _inputs(w, lengths, prune):
    g = synth.generate(w, "cpu", lengths=lengths)
    g = {k: (v.to("cuda") if isinstance(v, torch.Tensor) else v) for k, v in g.items()}
    dec = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk, T=w.gate_T, prune=prune)
    dec.build_meta()
    dec.predict_tau(g["q"], g["W"], torch.full((w.Hq,), 1.9, device="cuda"))
    dec.screen(g["q"])
    return g, dec


def _same_bits(g, dec, prune):
    """eta_decode with the decoder's workspace, then eta_decode_static into
    NaN-filled outputs: every output bit must agree."""
    ref_o, ref_l = torch.empty_like(dec.o), torch.empty_like(dec.lse)
    L.eta_decode(dec.dims, g["q"], dec.tau, dec.K, dec.V, dec.lengths, dec.union_idx,
                 dec.union_cnt, dec.T, 0.0, prune, dec.vsum, dec.cnt, ref_o, ref_l,
                 dec.ws_decode, dec.dev_status)
    o = torch.full_like(dec.o, float("nan"))
    lse = torch.full_like(dec.lse, float("nan"))
    L.eta_decode_static(dec.dims, g["q"], dec.tau, dec.K, dec.V, dec.lengths, dec.union_idx,
                        dec.union_cnt, dec.T, 0.0, prune, dec.vsum, dec.cnt, o, lse,
                        dec.dev_status)
    torch.cuda.synchronize()
    dec.check_status()
    assert torch.equal(o, ref_o)
    assert torch.equal(lse, ref_l)
    assert bool(torch.isfinite(o).all())


def test_static_scratch_decode_matches_workspace_decode_twice():
    w = synth.MID.with_(B=4, ctx=8192, seed=91)
    # two calls in a row, different inputs and prune modes (4 x 4 = 16 pairs: the
    # separate share-plan launch)
    for seed, lengths, prune in ((91, [8192, 5000, 77, 8000], "skip"),
                                 (92, [8192, 8191, 4096, 1], "floor")):
        g, dec = _inputs(w.with_(seed=seed), torch.tensor(lengths, dtype=torch.int32), prune)
        _same_bits(g, dec, prune)
    # a workload whose scratch would exceed the fixed array is refused, not run
    big = L.Dims.of(4096, 16, 4, 128, 64, 4096)
    assert L.eta_decode_workspace_size(big) > L.eta_decode_static_max_workspace()
    with pytest.raises(L.EtaError) as ei:
        L.eta_decode_static(big, g["q"], dec.tau, dec.K, dec.V, dec.lengths, dec.union_idx,
                            dec.union_cnt, 0.0, 0.0, "skip", None, None, dec.o, dec.lse)
    assert ei.value.code == 3


def test_static_scratch_in_kernel_plan_and_fma_engine_after_other_shapes():
    """The other two scratch layouts: 32 x 4 = 128 pairs, where the tensor-core
    decode lays out its shares itself and writes the plan into the scratch for the
    combine, and the CUDA-core engine; each right after a call of another shape,
    so the array holds stale data from a different layout."""
    small = synth.MID.with_(B=2, ctx=4096, seed=93)
    large = synth.MID.with_(B=32, ctx=2048, seed=94)
    g_s, dec_s = _inputs(small, torch.tensor([4096, 3001], dtype=torch.int32), "skip")
    g_l, dec_l = _inputs(large, synth.ragged_lengths(32, 2048, 64, gen_seed=11), "skip")
    assert L.eta_decode_launches(dec_l.dims) == 2
    _same_bits(g_s, dec_s, "skip")
    _same_bits(g_l, dec_l, "skip")
    L.eta_set_decode_engine("fma")
    try:
        assert L.eta_decode_launches(dec_l.dims) == 3
        _same_bits(g_l, dec_l, "skip")
        _same_bits(g_s, dec_s, "skip")
    finally:
        L.eta_set_decode_engine("auto")
    _same_bits(g_l, dec_l, "skip")
