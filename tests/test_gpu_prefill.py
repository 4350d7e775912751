"""Dense gated causal prefill (eta_prefill, tcgen05) against the float64 oracle:
o within max-abs 1e-2 / mean-abs 1e-3, lse within 1e-3, on valid query rows;
rows whose hard gate has a key within 1e-5 of tau are logged and skipped."""
import math

import numpy as np
import pytest
import torch

from long_context_decoding_eta_b200 import _lib as L
from oracle import eta_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=["one_tile", "two_tile"])
def prefill_kernel(request):
    """Every case runs through both prefill kernels."""
    L.eta_set_prefill_kernel(request.param)
    yield request.param
    L.eta_set_prefill_kernel("auto")


def run_case(B, Hq, Hkv, T_max, lengths, T_gate, seed, q_gain=1.0, tau_mu=0.5):
    g = torch.Generator().manual_seed(seed)
    d = 128
    q = (torch.randn(B, Hq, T_max, d, generator=g) * q_gain).to(torch.bfloat16)
    K = torch.randn(B, Hkv, T_max, d, generator=g).to(torch.bfloat16)
    V = torch.randn(B, Hkv, T_max, d, generator=g).to(torch.bfloat16)
    tau = (tau_mu + 0.5 * torch.randn(B, Hq, T_max, generator=g)).float()
    lengths = torch.tensor(lengths, dtype=torch.int32)
    dims = L.Dims.of(B, Hq, Hkv, d, 64, T_max)
    dev = "cuda"
    O_g = torch.zeros(B, Hq, T_max, d, device=dev)
    lse_g = torch.zeros(B, Hq, T_max, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    L.eta_prefill(dims, q.to(dev), tau.to(dev), K.to(dev), V.to(dev), lengths.to(dev), T_gate,
                  0.0, O_g, lse_g, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    scale = 1.0 / math.sqrt(d)
    q64, K64, V64, t64 = q.double().numpy(), K.double().numpy(), V.double().numpy(), tau.double().numpy()
    o_r, lse_r = O.prefill(q64, t64, K64, V64, lengths.numpy(), scale, T_gate)
    o_g, l_g = O_g.double().cpu().numpy(), lse_g.double().cpu().numpy()
    G = Hq // Hkv
    errs, lerrs, skipped = [], [], 0
    for b in range(B):
        for h in range(Hq):
            for t in range(int(lengths[b])):
                if T_gate == 0.0:
                    s = scale * K64[b, h // G, :t + 1] @ q64[b, h, t]
                    if np.any(np.abs(s - t64[b, h, t]) <= 1e-5 * max(1.0, abs(t64[b, h, t]))):
                        skipped += 1
                        continue
                errs.append(np.abs(o_g[b, h, t] - o_r[b, h, t]))
                lerrs.append(abs(l_g[b, h, t] - lse_r[b, h, t]))
    e = np.stack(errs)
    assert e.max() <= 1e-2 and e.mean() <= 1e-3, (e.max(), e.mean())
    assert max(lerrs) <= 1e-3, max(lerrs)
    # rows at and past lengths[b] are not written
    for b in range(B):
        assert torch.all(O_g[b, :, int(lengths[b]):] == 0)
    return e.max(), e.mean(), max(lerrs), skipped


@pytest.mark.parametrize("T_gate", [0.0, 0.05])
@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 4), (8, 1)])
def test_prefill_matches_oracle(T_gate, Hq, Hkv):
    print(run_case(2, Hq, Hkv, 512, [512, 300], T_gate, seed=40 + Hq + Hkv))


def test_prefill_sharp_scores_and_rescaling():
    # large logits force the running max to grow across key tiles (O rescaled in TMEM)
    print(run_case(1, 4, 2, 1024, [1000], 0.0, seed=51, q_gain=6.0, tau_mu=2.0))


def test_prefill_tau_neg_inf_is_causal_attention():
    print(run_case(1, 4, 2, 384, [384], 0.0, seed=52, tau_mu=-1e30))


def test_prefill_rejects_unsupported_shapes():
    dims = L.Dims.of(1, 4, 2, 128, 64, 200)     # T_max not a multiple of 128
    x = torch.zeros(1, 4, 200, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.EtaError) as ei:
        L.eta_prefill(dims, x, torch.zeros(1, 4, 200, device="cuda"), x, x,
                      torch.tensor([200], dtype=torch.int32, device="cuda"), 0.0, 0.0,
                      torch.zeros(1, 4, 200, 128, device="cuda"),
                      torch.zeros(1, 4, 200, device="cuda"))
    assert ei.value.code == 2


def test_prefill_edge_lengths():
    # an empty row, a one-token row and a row one past a tile boundary
    print(run_case(3, 4, 2, 256, [0, 1, 129], 0.0, seed=53))
    print(run_case(3, 4, 2, 256, [0, 1, 129], 0.05, seed=54))


def test_prefill_fullsize_sampled_rows():
    """The benchmark's configuration (B=4, 16/4 heads, d=128, T=8192, causal): every
    output finite, and sampled query rows against the oracle's dense gated attention
    over their causal prefix.  Inputs come from torch's generator, tau included."""
    B, Hq, Hkv, d, T = 4, 16, 4, 128, 8192
    dev = "cuda"
    g = torch.Generator(device=dev).manual_seed(77)
    q = torch.randn(B, Hq, T, d, generator=g, device=dev).to(torch.bfloat16)
    K = torch.randn(B, Hkv, T, d, generator=g, device=dev).to(torch.bfloat16)
    V = torch.randn(B, Hkv, T, d, generator=g, device=dev).to(torch.bfloat16)
    tau = 0.5 + 0.5 * torch.randn(B, Hq, T, generator=g, device=dev)
    lengths = torch.full((B,), T, dtype=torch.int32, device=dev)
    O_g = torch.empty(B, Hq, T, d, device=dev)
    lse_g = torch.empty(B, Hq, T, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(d)
    rng = np.random.default_rng(5)
    rows = [(0, 0, 0), (1, 5, 127), (2, 9, 128), (3, 15, T - 1)] + [
        (int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(T))) for _ in range(28)]
    for T_gate in (0.0, 0.05):
        L.eta_prefill(L.Dims.of(B, Hq, Hkv, d, 64, T), q, tau, K, V, lengths, T_gate, 0.0, O_g,
                      lse_g, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert bool(torch.isfinite(O_g).all()) and bool(torch.isfinite(lse_g).all())
        errs, checked = [], 0
        for b, h, t in rows:
            kh = h // (Hq // Hkv)
            q64 = q[b, h, t].double().cpu().numpy()
            K64 = K[b, kh, :t + 1].double().cpu().numpy()
            V64 = V[b, kh, :t + 1].double().cpu().numpy()
            t64 = float(tau[b, h, t])
            if T_gate == 0.0:
                s = scale * (K64 @ q64)
                if np.any(np.abs(s - t64) <= 1e-5 * max(1.0, abs(t64))):
                    continue                               # a gate near-tie: logged, skipped
            o_r, l_r = O.dense_gated(q64, t64, K64, V64, t + 1, scale, T_gate)
            errs.append(np.abs(O_g[b, h, t].double().cpu().numpy() - o_r))
            assert abs(float(lse_g[b, h, t]) - l_r) <= 1e-3
            checked += 1
        e = np.stack(errs)
        assert checked >= 24 and e.max() <= 1e-2 and e.mean() <= 1e-3, (checked, e.max(), e.mean())


def test_prefill_auto_kernel_choice(prefill_kernel):
    """The automatic choice: the two-tile kernel once its tile pairs exceed half the SM
    count (hard gate) or twice the SM count (soft gate)."""
    L.eta_set_prefill_kernel("auto")
    n = torch.cuda.get_device_properties(0).multi_processor_count
    for B, Hq, T in [(1, 16, 1024), (1, 16, 2048), (1, 16, 4096), (2, 16, 4096), (4, 16, 8192)]:
        pairs = B * Hq * ((T // 128 + 1) // 2)
        dims = L.Dims.of(B, Hq, 4, 128, 64, T)
        assert L.eta_prefill_kernel_for(dims, 0.0) == ("two_tile" if pairs > n // 2 else "one_tile")
        assert L.eta_prefill_kernel_for(dims, 0.05) == ("two_tile" if pairs > 2 * n else "one_tile")
    # the prefill benchmark's configuration takes the two-tile kernel with both gates
    assert L.eta_prefill_kernel_for(L.Dims.of(4, 16, 4, 128, 64, 8192), 0.05) == "two_tile"
