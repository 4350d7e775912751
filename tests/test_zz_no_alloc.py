"""eta_decode_static: the decode entry point for callers that cannot allocate
device memory (for example a serving loop whose memory is all reserved by its
own pool, or code that must not call cudaMalloc on the decode path because it
can synchronize the device).  It must give the same result as eta_decode with
a caller workspace, call after call, although its scratch is a fixed array
shared by all calls.  This file is collected last on purpose."""
import math

import numpy as np
import pytest
import torch

from long_context_decoding_eta_b200 import _lib as L
from long_context_decoding_eta_b200 import synth
from long_context_decoding_eta_b200.api import EtaDecoder

pytestmark = pytest.mark.gpu


def _inputs(w, lengths):
    g = synth.generate(w, "cpu", lengths=lengths)
    g = {k: (v.to("cuda") if isinstance(v, torch.Tensor) else v) for k, v in g.items()}
    dec = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk, T=w.gate_T, prune="floor")
    dec.build_meta()
    dec.predict_tau(g["q"], g["W"], torch.full((w.Hq,), 1.9, device="cuda"))
    dec.screen(g["q"])
    return g, dec


def test_static_scratch_decode_matches_workspace_decode_twice():
    w = synth.MID.with_(B=4, ctx=8192, seed=91)
    runs = [(_inputs(w, torch.tensor([8192, 5000, 77, 8000], dtype=torch.int32)), "skip"),
            (_inputs(w.with_(seed=92), torch.tensor([8192, 8191, 4096, 1], dtype=torch.int32)),
             "floor")]
    for (g, dec), prune in runs:
        ref_o, ref_l = torch.empty_like(dec.o), torch.empty_like(dec.lse)
        L.eta_decode(dec.dims, g["q"], dec.tau, dec.K, dec.V, dec.lengths, dec.union_idx,
                     dec.union_cnt, dec.T, 0.0, prune, dec.vsum, dec.cnt, ref_o, ref_l,
                     dec.ws_decode, dec.dev_status)
        o = torch.full_like(dec.o, float("nan"))
        lse = torch.full_like(dec.lse, float("nan"))
        L.eta_decode_static(dec.dims, g["q"], dec.tau, dec.K, dec.V, dec.lengths,
                            dec.union_idx, dec.union_cnt, dec.T, 0.0, prune, dec.vsum,
                            dec.cnt, o, lse, dec.dev_status)
        torch.cuda.synchronize()
        dec.check_status()
        err = (o - ref_o).abs()
        assert float(err.max()) <= 1e-2 and float(err.mean()) <= 1e-3
        fin = torch.isfinite(ref_l)
        assert torch.equal(fin, torch.isfinite(lse))
        if bool(fin.any()):
            assert float((lse[fin] - ref_l[fin]).abs().max()) <= 1e-3
    # a workload whose scratch would exceed the fixed array is refused, not run
    big = L.Dims.of(4096, 16, 4, 128, 64, 4096)
    assert L.eta_decode_workspace_size(big) > L.eta_decode_static_max_workspace()
    with pytest.raises(L.EtaError) as ei:
        L.eta_decode_static(big, g["q"], dec.tau, dec.K, dec.V, dec.lengths, dec.union_idx,
                            dec.union_cnt, 0.0, 0.0, "skip", None, None, dec.o, dec.lse)
    assert ei.value.code == 3
