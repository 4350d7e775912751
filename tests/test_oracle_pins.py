"""Pins of the float64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a library
routine (torch scaled_dot_product_attention / logsumexp in float64), a closed
form, an invariant the method guarantees, or brute force on tiny inputs.  The
set is chosen so that a plausible slip in the oracle (a dropped term, a wrong
sign, the wrong GQA group, a transposed predictor, a mis-sized block) fails at
least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from long_context_decoding_eta_b200 import synth
from oracle import eta_oracle as O


def f64(t):
    return t.detach().to("cpu").double().numpy()


def tiny(seed=0, B=2, Hq=4, Hkv=2, d=16, ctx=200, blk=16, q_scale=1.0, lengths=None,
         n_clusters=4, seg=40, needles=0):
    w = synth.Workload("tiny-test", B=B, Hq=Hq, Hkv=Hkv, d=d, ctx=ctx, blk=blk,
                       n_clusters=n_clusters, seg=seg, needles=needles, q_scale=q_scale,
                       seed=seed)
    g = synth.generate(w, "cpu", lengths=lengths)
    K, V, q = f64(g["K"]), f64(g["V"]), f64(g["q"])
    L = g["lengths"].numpy().astype(np.int64)
    return w, K, V, q, L, f64(g["W"])


def sdpa_reference(q, K, V, L, scale):
    """torch SDPA in float64 with GQA head h -> KV head h // G, per row lengths."""
    B, Hq, d = q.shape
    Hkv, Tm = K.shape[1], K.shape[2]
    G = Hq // Hkv
    Kt = torch.from_numpy(K).repeat_interleave(G, dim=1)
    Vt = torch.from_numpy(V).repeat_interleave(G, dim=1)
    qt = torch.from_numpy(q)[:, :, None, :]
    mask = torch.arange(Tm)[None, :] < torch.from_numpy(L)[:, None]       # [B, Tm]
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, Kt, Vt, attn_mask=mask[:, None, None, :], scale=scale)[:, :, 0, :]
    s = torch.einsum("bhd,bhtd->bht", torch.from_numpy(q), Kt) * scale
    s = s.masked_fill(~mask[:, None, :], -math.inf)
    return o.numpy(), torch.logsumexp(s, dim=-1).numpy()


# --------------------------------------------------------------------------
# tau = -inf reduces to standard softmax attention (library routine)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("T", [0.0, 0.05])
@pytest.mark.parametrize("prune", [O.PRUNE_SKIP, O.PRUNE_FLOOR])
def test_tau_neg_inf_is_softmax_attention(T, prune):
    w, K, V, q, L, W = tiny(seed=1, lengths=torch.tensor([200, 77]))
    scale = O.default_scale(w.d)
    meta = O.cache_meta(K, L, w.blk, V)
    tau = np.full((w.B, w.Hq), -np.inf)
    sc = O.screen(q, tau, meta, scale)
    o, lse = O.decode(q, tau, K, V, L, sc["union_idx"], w.blk, scale, T, prune, meta)
    o_ref, lse_ref = sdpa_reference(q, K, V, L, scale)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)
    # every non-empty block is admitted, empty ones never
    assert np.array_equal(sc["union"], meta["cnt"] > 0)


def test_dense_decode_matches_library():
    w, K, V, q, L, W = tiny(seed=2, lengths=torch.tensor([131, 200]))
    scale = O.default_scale(w.d)
    o, lse = O.dense_decode(q, K, V, L, scale)
    o_ref, lse_ref = sdpa_reference(q, K, V, L, scale)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


def test_gqa_group_is_h_div_G():
    # If head h used KV head h % Hkv instead of h // G, the library check fails:
    # make the two KV heads very different so the mapping matters.
    w, K, V, q, L, W = tiny(seed=3, Hq=4, Hkv=2)
    V[:, 1] += 5.0
    scale = O.default_scale(w.d)
    o, _ = O.dense_decode(q, K, V, L, scale)
    o_ref, _ = sdpa_reference(q, K, V, L, scale)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    assert o[:, 0].mean() < 2.5 < o[:, 3].mean()


# --------------------------------------------------------------------------
# tau above every score: hard gate sends every logit to 0 -> uniform mean
# --------------------------------------------------------------------------
def test_tau_above_scores_gives_uniform_mean():
    w, K, V, q, L, W = tiny(seed=4, lengths=torch.tensor([200, 93]))
    scale = O.default_scale(w.d)
    meta = O.cache_meta(K, L, w.blk, V)
    G = w.G
    tau = np.zeros((w.B, w.Hq))
    for b in range(w.B):
        for h in range(w.Hq):
            s = scale * K[b, h // G, :L[b]] @ q[b, h]
            tau[b, h] = s.max() + 0.25
            o, lse = O.dense_gated(q[b, h], tau[b, h], K[b, h // G], V[b, h // G], L[b], scale, 0.0)
            np.testing.assert_allclose(o, V[b, h // G, :L[b]].mean(axis=0), atol=1e-12)
            assert abs(lse - math.log(L[b])) < 1e-12
    # FLOOR mode with pruning gives the same uniform mean over all valid keys
    sc = O.screen(q, tau, meta, scale)
    o, lse = O.decode(q, tau, K, V, L, sc["union_idx"], w.blk, scale, 0.0, O.PRUNE_FLOOR, meta)
    for b in range(w.B):
        for h in range(w.Hq):
            np.testing.assert_allclose(o[b, h], V[b, h // G, :L[b]].mean(axis=0), atol=1e-12)
            assert abs(lse[b, h] - math.log(L[b])) < 1e-12


# --------------------------------------------------------------------------
# exact geometric bound is sound: brute force over every key
# --------------------------------------------------------------------------
@pytest.mark.parametrize("q_scale", [1.0, 8.0])
def test_exact_bound_dominates_every_key(q_scale):
    w, K, V, q, L, W = tiny(seed=5, q_scale=q_scale, lengths=torch.tensor([200, 150]),
                            needles=3)
    scale = O.default_scale(w.d)
    meta = O.cache_meta(K, L, w.blk)
    G = w.G
    for b in range(w.B):
        for h in range(w.Hq):
            ub = O.block_bounds(q[b, h], meta["cent"][b, h // G], meta["rmax"][b, h // G],
                                meta["var"][b, h // G], scale)
            for j in range(w.NB):
                n = meta["cnt"][b, h // G, j]
                if n == 0:
                    continue
                keys = K[b, h // G, j * w.blk: j * w.blk + n]
                s = scale * keys @ q[b, h]
                assert s.max() <= ub[j] * (1 + 1e-12) + 1e-12


@pytest.mark.parametrize("density", [0.1, 0.38, 0.7])
def test_no_key_above_tau_in_a_pruned_block(density):
    w, K, V, q, L, W = tiny(seed=6, q_scale=8.0, needles=4)
    scale = O.default_scale(w.d)
    meta = O.cache_meta(K, L, w.blk)
    G = w.G
    tau = O.predict_tau(q, W, np.zeros(w.Hq))
    ub = O.screen(q, tau, meta, scale)["bounds"]
    tau = tau + O.offset_for_density(ub, tau, np.repeat(meta["cnt"] > 0, G, 1), density, G)
    sc = O.screen(q, tau, meta, scale)
    for b in range(w.B):
        for h in range(w.Hq):
            s = scale * K[b, h // G, :L[b]] @ q[b, h]
            for t in np.nonzero(s >= tau[b, h])[0]:
                assert sc["admit"][b, h, t // w.blk]
                assert sc["union"][b, h // G, t // w.blk]


# --------------------------------------------------------------------------
# pruning: FLOOR mode equals dense hard gating (exact bound)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("density", [0.05, 0.38, 0.9])
def test_floor_prune_equals_dense_hard_gating(density):
    w, K, V, q, L, W = tiny(seed=7, q_scale=8.0, needles=4, lengths=torch.tensor([200, 121]))
    scale = O.default_scale(w.d)
    meta = O.cache_meta(K, L, w.blk, V)
    G = w.G
    tau = O.predict_tau(q, W, np.zeros(w.Hq))
    ub = O.screen(q, tau, meta, scale)["bounds"]
    tau = tau + O.offset_for_density(ub, tau, np.repeat(meta["cnt"] > 0, G, 1), density, G)
    sc = O.screen(q, tau, meta, scale)
    o, lse = O.decode(q, tau, K, V, L, sc["union_idx"], w.blk, scale, 0.0, O.PRUNE_FLOOR, meta)
    n_above = 0
    for b in range(w.B):
        for h in range(w.Hq):
            od, ld = O.dense_gated(q[b, h], tau[b, h], K[b, h // G], V[b, h // G], L[b], scale, 0.0)
            np.testing.assert_allclose(o[b, h], od, atol=1e-12)
            assert abs(lse[b, h] - ld) < 1e-12
            n_above += int((scale * K[b, h // G, :L[b]] @ q[b, h] >= tau[b, h]).sum())
    if density < 0.5:
        assert sc["union"].mean() < 1.0   # something really was pruned


def test_floor_invariant_over_every_admissible_block_subset():
    """Enumerate block subsets: any union that keeps every block holding a key
    with s >= tau gives the dense hard-gated answer in FLOOR mode."""
    w, K, V, q, L, W = tiny(seed=8, B=1, Hq=2, Hkv=1, d=8, ctx=64, blk=16, q_scale=6.0,
                            seg=16)
    scale = O.default_scale(w.d)
    meta = O.cache_meta(K, L, w.blk, V)
    s_all = scale * K[0, 0, :L[0]] @ q[0, 0]
    tau = float(np.sort(s_all)[-2])          # two keys at or above tau
    need = {t // w.blk for t in np.nonzero(s_all >= tau)[0]}
    od, ld = O.dense_gated(q[0, 0], tau, K[0, 0], V[0, 0], L[0], scale, 0.0)
    mr = {"cnt": meta["cnt"][0, 0], "vsum": meta["vsum"][0, 0]}
    checked = 0
    for r in range(w.NB + 1):
        for S in itertools.combinations(range(w.NB), r):
            o, lse = O.attend_blocks(q[0, 0], tau, K[0, 0], V[0, 0], L[0], list(S), w.blk,
                                     scale, 0.0, O.PRUNE_FLOOR, mr)
            if need <= set(S):
                np.testing.assert_allclose(o, od, atol=1e-12)
                assert abs(lse - ld) < 1e-12
                checked += 1
            elif len(need - set(S)):
                # dropping a block that holds a key above tau changes the answer
                assert not np.allclose(o, od, atol=1e-9) or abs(lse - ld) > 1e-9
    assert checked >= 2


def test_skip_prune_is_gated_softmax_over_union_keys():
    w, K, V, q, L, W = tiny(seed=9, q_scale=8.0, lengths=torch.tensor([200, 170]))
    scale = O.default_scale(w.d)
    meta = O.cache_meta(K, L, w.blk)
    G = w.G
    tau = O.predict_tau(q, W, np.zeros(w.Hq)) + 0.3
    sc = O.screen(q, tau, meta, scale)
    T = 0.05
    o, lse = O.decode(q, tau, K, V, L, sc["union_idx"], w.blk, scale, T, O.PRUNE_SKIP)
    for b in range(w.B):
        for h in range(w.Hq):
            g = h // G
            keys = [t for t in range(L[b]) if sc["union"][b, g, t // w.blk]]
            if not keys:
                assert np.all(o[b, h] == 0) and lse[b, h] == -math.inf
                continue
            s = np.array([scale * float(K[b, g, t] @ q[b, h]) for t in keys])
            gs = np.array([x / (1 + math.exp(-(x - tau[b, h]) / T)) for x in s])
            p = np.exp(gs - gs.max())
            ref = sum(p[i] * V[b, g, t] for i, t in enumerate(keys)) / p.sum()
            np.testing.assert_allclose(o[b, h], ref, atol=1e-12)
            assert abs(lse[b, h] - (gs.max() + math.log(p.sum()))) < 1e-12


def test_empty_union_and_empty_row():
    w, K, V, q, L, W = tiny(seed=10, lengths=torch.tensor([0, 50]))
    scale = O.default_scale(w.d)
    meta = O.cache_meta(K, L, w.blk, V)
    tau = np.full((w.B, w.Hq), np.inf)
    sc = O.screen(q, tau, meta, scale)
    assert not sc["union"].any()
    o, lse = O.decode(q, tau, K, V, L, sc["union_idx"], w.blk, scale, 0.0, O.PRUNE_SKIP)
    assert np.all(o == 0) and np.all(lse == -np.inf)
    o, lse = O.decode(q, tau, K, V, L, sc["union_idx"], w.blk, scale, 0.0, O.PRUNE_FLOOR, meta)
    assert np.all(o[0] == 0) and np.all(lse[0] == -np.inf)       # no keys at all
    for h in range(w.Hq):
        np.testing.assert_allclose(o[1, h], V[1, h // w.G, :50].mean(0), atol=1e-12)
        assert abs(lse[1, h] - math.log(50)) < 1e-12


# --------------------------------------------------------------------------
# metadata closed forms
# --------------------------------------------------------------------------
def test_meta_identical_keys():
    k = np.linspace(-1, 1, 8)
    Ks = np.tile(k, (32, 1))
    m = O.block_meta(Ks, 32, 16)
    np.testing.assert_allclose(m["cent"], np.tile(k, (2, 1)), atol=1e-15)
    assert np.all(m["rmax"] < 1e-15) and np.all(m["var"] < 1e-30)
    assert list(m["cnt"]) == [16, 16]


def test_meta_two_point_block_and_partial_tail():
    rng = np.random.default_rng(0)
    a, b = rng.normal(size=6), rng.normal(size=6)
    Ks = np.zeros((12, 6))
    Ks[0::2][:4] = a
    Ks[1::2][:4] = b
    Ks[8] = a
    Ks[9] = b
    V = rng.normal(size=(12, 6))
    m = O.block_meta(Ks, 10, 8, V)        # blocks: [0,8) full, [8,10) partial, rows 10.. invalid
    dist = np.linalg.norm(a - b)
    for j in (0, 1):
        np.testing.assert_allclose(m["cent"][j], (a + b) / 2, atol=1e-14)
        assert abs(m["rmax"][j] - dist / 2) < 1e-14
        assert abs(m["var"][j] - dist ** 2 / 4) < 1e-13
    assert list(m["cnt"]) == [8, 2]
    np.testing.assert_allclose(m["vsum"][1], V[8:10].sum(0), atol=1e-14)


def test_meta_against_bruteforce_loops():
    w, K, V, q, L, W = tiny(seed=11, lengths=torch.tensor([200, 37]))
    meta = O.cache_meta(K, L, w.blk, V)
    for b in range(w.B):
        for g in range(w.Hkv):
            for j in range(w.NB):
                rows = [t for t in range(j * w.blk, (j + 1) * w.blk) if t < L[b]]
                assert meta["cnt"][b, g, j] == len(rows)
                if not rows:
                    continue
                c = [sum(K[b, g, t, i] for t in rows) / len(rows) for i in range(w.d)]
                d2 = [sum((K[b, g, t, i] - c[i]) ** 2 for i in range(w.d)) for t in rows]
                np.testing.assert_allclose(meta["cent"][b, g, j], c, atol=1e-12)
                assert abs(meta["rmax"][b, g, j] - math.sqrt(max(d2))) < 1e-12
                assert abs(meta["var"][b, g, j] - sum(d2) / len(rows)) < 1e-12


# --------------------------------------------------------------------------
# threshold predictor (Eq. 1)
# --------------------------------------------------------------------------
def test_predictor_one_hot_selects_coordinate():
    B, Hq, d = 3, 4, 5
    rng = np.random.default_rng(1)
    q = rng.normal(size=(B, Hq, d))
    bias = rng.normal(size=Hq)
    for (h_src, k, h_dst) in [(0, 0, 0), (2, 3, 1), (3, 4, 3), (1, 2, 2)]:
        W = np.zeros((Hq * d, Hq))
        W[h_src * d + k, h_dst] = 1.0
        tau = O.predict_tau(q, W, bias)
        np.testing.assert_allclose(tau[:, h_dst], q[:, h_src, k] + bias[h_dst], atol=1e-15)
        others = [h for h in range(Hq) if h != h_dst]
        np.testing.assert_allclose(tau[:, others], np.broadcast_to(bias[others], (B, Hq - 1)))


def test_const_tau_broadcast():
    t = O.const_tau(3, np.array([0.5, -1.0]))
    assert t.shape == (3, 2) and np.all(t[:, 0] == 0.5) and np.all(t[:, 1] == -1.0)


# --------------------------------------------------------------------------
# gate (Eq. 2-3)
# --------------------------------------------------------------------------
def test_gate_closed_forms_and_hard_limit():
    tau, T = 0.7, 0.05
    assert abs(O.gate(np.array([tau]), tau, T)[0] - tau / 2) < 1e-15
    x = tau + T * math.log(3.0)           # sigmoid(ln 3) = 3/4
    assert abs(O.gate(np.array([x]), tau, T)[0] - 0.75 * x) < 1e-14
    x = tau - T * math.log(3.0)           # sigmoid(-ln 3) = 1/4
    assert abs(O.gate(np.array([x]), tau, T)[0] - 0.25 * x) < 1e-14
    s = np.linspace(-3, 3, 601)
    s = s[np.abs(s - tau) > 1e-3]
    np.testing.assert_allclose(O.gate(s, tau, 1e-6), O.gate(s, tau, 0.0), atol=1e-12)
    hard = O.gate(np.array([tau - 1e-12, tau, tau + 1e-12]), tau, 0.0)
    assert hard[0] == 0.0 and hard[1] == tau and hard[2] == tau + 1e-12
    # overflow safety far from tau
    assert np.all(np.isfinite(O.gate(np.array([-1e4, 1e4]), 0.0, 1e-3)))


# --------------------------------------------------------------------------
# screening structure
# --------------------------------------------------------------------------
def test_union_is_or_of_heads_and_G1_equals_head_mask():
    w, K, V, q, L, W = tiny(seed=12)
    scale = O.default_scale(w.d)
    meta = O.cache_meta(K, L, w.blk)
    tau = O.predict_tau(q, W, np.zeros(w.Hq)) + 0.2
    sc = O.screen(q, tau, meta, scale)
    for b in range(w.B):
        for g in range(w.Hkv):
            heads = sc["admit"][b, g * w.G:(g + 1) * w.G]
            assert np.array_equal(sc["union"][b, g], heads.any(0))
            assert np.all(sc["union"][b, g] >= heads)
            assert np.array_equal(sc["union_idx"][b][g], np.nonzero(heads.any(0))[0])
    # G = 1
    w1, K1, V1, q1, L1, W1 = tiny(seed=13, Hq=2, Hkv=2)
    meta1 = O.cache_meta(K1, L1, w1.blk)
    tau1 = O.predict_tau(q1, W1, np.zeros(2)) + 0.2
    sc1 = O.screen(q1, tau1, meta1, O.default_scale(w1.d))
    assert np.array_equal(sc1["union"], sc1["admit"])


def test_block_permutation_permutes_masks():
    w, K, V, q, L, W = tiny(seed=14, B=1, ctx=160, blk=16)
    scale = O.default_scale(w.d)
    perm = np.random.default_rng(3).permutation(w.NB)
    Kp = K.reshape(w.B, w.Hkv, w.NB, w.blk, w.d)[:, :, perm].reshape(K.shape)
    m, mp = O.cache_meta(K, L, w.blk), O.cache_meta(Kp, L, w.blk)
    tau = O.predict_tau(q, W, np.zeros(w.Hq)) + 0.2
    s, sp = O.screen(q, tau, m, scale), O.screen(q, tau, mp, scale)
    np.testing.assert_allclose(sp["bounds"], s["bounds"][:, :, perm], atol=1e-12)
    assert np.array_equal(sp["admit"], s["admit"][:, :, perm])


def test_ragged_lengths_blocks_beyond_length_never_admitted():
    w, K, V, q, L, W = tiny(seed=15, lengths=torch.tensor([200, 45]))
    meta = O.cache_meta(K, L, w.blk)
    assert meta["cnt"][1, 0, 2] == 45 - 32 and meta["cnt"][1, 0, 3] == 0
    tau = np.full((w.B, w.Hq), -np.inf)
    sc = O.screen(q, tau, meta, O.default_scale(w.d))
    assert not sc["union"][1, :, 3:].any() and sc["union"][1, :, :3].all()


def test_probabilistic_bound_properties():
    w, K, V, q, L, W = tiny(seed=16, q_scale=4.0)
    scale = O.default_scale(w.d)
    meta = O.cache_meta(K, L, w.blk)
    ex = O.screen(q, np.zeros((w.B, w.Hq)), meta, scale, O.BOUND_EXACT)["bounds"]
    for z in (0.5, 1.0, 3.0, math.sqrt(w.d)):
        pr = O.screen(q, np.zeros((w.B, w.Hq)), meta, scale, O.BOUND_PROB, z)["bounds"]
        assert np.all(pr <= ex + 1e-12)
    pr = O.screen(q, np.zeros((w.B, w.Hq)), meta, scale, O.BOUND_PROB, 1e9)["bounds"]
    np.testing.assert_allclose(pr, ex, atol=1e-12)


def _gaussian_blocks(rng, nblk, blk, sig):
    """nblk blocks of blk keys, k = c_j + sig * N(0, I) around random centres c_j."""
    d = sig.shape[0]
    centres = rng.normal(size=(nblk, d))
    return centres[:, None, :] + sig[None, None, :] * rng.normal(size=(nblk, blk, d))


def _tail_fraction(keys, bound, z, queries):
    """Fraction of (query, key) pairs whose score exceeds the oracle's bound of the
    key's block, with the exact-radius cap lifted (rmax = +inf) so that only the
    probabilistic term is measured.  Scores and bounds in unscaled units (scale 1)."""
    nblk, blk, d = keys.shape
    m = O.block_meta(keys.reshape(nblk * blk, d), nblk * blk, blk)
    no_cap = np.full(nblk, np.inf)
    above = 0
    for q in queries:
        ub = O.block_bounds(q, m["cent"], no_cap, m["var"], 1.0, bound, z, m["vardim"])
        above += int(((keys @ q) > ub[:, None]).sum())
    return above / (len(queries) * nblk * blk)


def _tail_tolerance(p, n_keys):
    # 4 binomial standard deviations counted over the keys alone (the queries
    # share keys, so they are not independent draws), plus 5% of p for the
    # sampling noise of the per-block variance estimates
    return 4.0 * math.sqrt(p * (1.0 - p) / n_keys) + 0.05 * p


@pytest.mark.parametrize("d,nblk", [(16, 2000), (128, 500)])
def test_probabilistic_bound_is_the_z_sigma_tail_for_isotropic_keys(d, nblk):
    """BOUND_PROB reads the cached variance as a z-sigma bound: for keys with
    isotropic Gaussian deviations from their block centre, q.(k - c) is normal with
    standard deviation ||q|| sqrt(var / d), so the fraction of keys scoring above
    the bound must be the one-sided normal tail 1 - Phi(z).  A bound built from
    sqrt(var) (no / d), from the key count instead of d, or from z^2 gives
    fractions of about 0, 1 - Phi(z sqrt(d / n)) and 1 - Phi(z^2): all far
    outside the tolerance."""
    from scipy.stats import norm
    rng = np.random.default_rng(41 + d)
    blk = 128
    keys = _gaussian_blocks(rng, nblk, blk, np.full(d, 0.3))
    queries = [rng.normal(size=d) for _ in range(8)]
    for z in (1.0, 2.0, 3.0):
        p = norm.sf(z)
        f = _tail_fraction(keys, O.BOUND_PROB, z, queries)
        assert abs(f - p) <= _tail_tolerance(p, nblk * blk), (z, f, p)


@pytest.mark.parametrize("d,nblk", [(16, 2000), (128, 500)])
def test_per_dimension_bound_is_the_z_sigma_tail_for_anisotropic_keys(d, nblk):
    """BOUND_PROB_DIM: with independent per-dimension spreads sigma_i and any q,
    q.(k - c) has variance sum_i q_i^2 sigma_i^2, so again 1 - Phi(z) of the keys
    score above the bound.  The scalar bound on the same keys, which assumes
    isotropy, misses that tail by far (the query leans on the wide dimensions)."""
    from scipy.stats import norm
    rng = np.random.default_rng(43 + d)
    blk = 128
    sig = np.exp(rng.uniform(math.log(0.1), math.log(2.0), size=d))
    keys = _gaussian_blocks(rng, nblk, blk, sig)
    queries = [rng.normal(size=d) * (0.2 + sig) for _ in range(8)]
    for z in (1.0, 2.0, 3.0):
        p = norm.sf(z)
        tol = _tail_tolerance(p, nblk * blk)
        f = _tail_fraction(keys, O.BOUND_PROB_DIM, z, queries)
        assert abs(f - p) <= tol, (z, f, p)
        f_iso = _tail_fraction(keys, O.BOUND_PROB, z, queries)
        assert abs(f_iso - p) > 4 * tol, (z, f_iso, p)


# --------------------------------------------------------------------------
# calibration rule
# --------------------------------------------------------------------------
def test_calibration_quantile_hits_density():
    rng = np.random.default_rng(5)
    n_q, Hq, NB = 64, 4, 97
    bounds = rng.normal(size=(n_q, Hq, NB))
    valid = rng.random((n_q, Hq, NB)) > 0.1
    for dens in (0.16, 0.38, 0.51):
        tau = O.calibrate_const_tau(bounds, valid, dens)
        for h in range(Hq):
            pool = bounds[:, h][valid[:, h]]
            frac = (pool >= tau[h]).mean()
            assert dens <= frac <= dens + 1.0 / pool.size + 1e-12


# --------------------------------------------------------------------------
# hand-derived worked example (tests/golden/hand_example_d2.json)
# --------------------------------------------------------------------------
def test_hand_derived_example():
    import json
    import os
    ex = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "hand_example_d2.json")))
    K = np.array(ex["K"])[None, None]
    V = np.array(ex["V"])[None, None]
    q = np.array(ex["q"])[None, None]
    L = [4]
    want = ex["expected"]
    meta = O.cache_meta(K, L, ex["blk"], V)
    np.testing.assert_allclose(meta["cent"][0, 0], want["cent"], atol=1e-15)
    np.testing.assert_allclose(meta["rmax"][0, 0], want["rmax"], atol=1e-15)
    np.testing.assert_allclose(meta["var"][0, 0], want["var"], atol=1e-15)
    tau = np.array([[ex["tau"]]])
    sc = O.screen(q, tau, meta, ex["scale"])
    np.testing.assert_allclose(sc["bounds"][0, 0], want["bounds"], atol=1e-15)
    assert list(sc["admit"][0, 0]) == want["admit"]
    o, lse = O.decode(q, tau, K, V, L, sc["union_idx"], ex["blk"], ex["scale"], 0.0,
                      O.PRUNE_SKIP)
    np.testing.assert_allclose(o[0, 0], want["o_skip"], atol=1e-15)
    assert abs(lse[0, 0] - want["lse_skip"]) < 1e-14
    o, lse = O.decode(q, tau, K, V, L, sc["union_idx"], ex["blk"], ex["scale"], 0.0,
                      O.PRUNE_FLOOR, meta)
    np.testing.assert_allclose(o[0, 0], want["o_floor"], atol=1e-15)
    assert abs(lse[0, 0] - want["lse_floor"]) < 1e-14


# --------------------------------------------------------------------------
# bf16 centroids (compact metadata)
# --------------------------------------------------------------------------
def test_round_to_bf16_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(21)
    x = np.concatenate([rng.normal(size=20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        np.array([1.0, -1.0, 1.00390625, 1.005859375, 3.0, 0.1])])
    x32 = x.astype(np.float32)
    want = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O.round_to_bf16(x32.astype(np.float64)), want)
    # ties go to even: 1 + 2^-8 is halfway between 1 and 1 + 2^-7
    assert O.round_to_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    assert O.round_to_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2 * 2.0 ** -7


@pytest.mark.parametrize("q_scale", [1.0, 8.0])
def test_bf16_centroid_bound_still_dominates_every_key(q_scale):
    w, K, V, q, L, W = tiny(seed=22, q_scale=q_scale, lengths=torch.tensor([200, 150]),
                            needles=3)
    scale = O.default_scale(w.d)
    meta = O.cache_meta(K, L, w.blk, cent_format="bf16")
    G = w.G
    assert np.array_equal(O.round_to_bf16(meta["cent"]), meta["cent"])
    for b in range(w.B):
        for h in range(w.Hq):
            ub = O.block_bounds(q[b, h], meta["cent"][b, h // G], meta["rmax"][b, h // G],
                                meta["var"][b, h // G], scale)
            for j in range(w.NB):
                n = meta["cnt"][b, h // G, j]
                if n == 0:
                    continue
                s = scale * K[b, h // G, j * w.blk: j * w.blk + n] @ q[b, h]
                assert s.max() <= ub[j] * (1 + 1e-12) + 1e-12
    # r is measured against the rounded centroid, not the exact mean
    m32 = O.cache_meta(K, L, w.blk)
    assert not np.allclose(meta["rmax"], m32["rmax"], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# per-dimension variance bound
# --------------------------------------------------------------------------
def test_per_dimension_variance_bound_properties():
    w, K, V, q, L, W = tiny(seed=23, q_scale=4.0)
    scale = O.default_scale(w.d)
    meta = O.cache_meta(K, L, w.blk)
    # vardim sums to the scalar variance (total variance = sum of per-dim variances)
    np.testing.assert_allclose(meta["vardim"].sum(axis=-1), meta["var"], rtol=1e-12, atol=1e-14)
    ex = O.screen(q, np.zeros((w.B, w.Hq)), meta, scale, O.BOUND_EXACT)["bounds"]
    for z in (0.5, 2.0, 3.0):
        pd = O.screen(q, np.zeros((w.B, w.Hq)), meta, scale, O.BOUND_PROB_DIM, z)["bounds"]
        assert np.all(pd <= ex + 1e-12)
    pd = O.screen(q, np.zeros((w.B, w.Hq)), meta, scale, O.BOUND_PROB_DIM, 1e9)["bounds"]
    np.testing.assert_allclose(pd, ex, atol=1e-12)
    # isotropic query: sum_i q_i^2 vardim_i = |q|^2 var / d -> equals the scalar prob bound
    qi = np.ones_like(q) * 0.3
    pr = O.screen(qi, np.zeros((w.B, w.Hq)), meta, scale, O.BOUND_PROB, 2.0)["bounds"]
    pdi = O.screen(qi, np.zeros((w.B, w.Hq)), meta, scale, O.BOUND_PROB_DIM, 2.0)["bounds"]
    np.testing.assert_allclose(pdi, pr, rtol=1e-12, atol=1e-12)


def test_per_dimension_variance_bound_brute_force_values():
    rng = np.random.default_rng(24)
    keys = rng.normal(size=(7, 5)) * np.array([0.1, 2.0, 0.5, 1.0, 0.01])
    m = O.block_meta(keys, 7, 8)
    c = keys.mean(0)
    assert np.allclose(m["vardim"][0], [np.mean((keys[:, i] - c[i]) ** 2) for i in range(5)])


# --------------------------------------------------------------------------
# dense gated causal prefill
# --------------------------------------------------------------------------
def _prefill_case(seed=30, B=2, Hq=4, Hkv=2, d=8, T=40):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(B, Hq, T, d))
    K = rng.normal(size=(B, Hkv, T, d))
    V = rng.normal(size=(B, Hkv, T, d))
    return q, K, V, np.array([T, T - 13])


@pytest.mark.parametrize("T_gate", [0.0, 0.05])
def test_prefill_tau_neg_inf_is_causal_softmax_attention(T_gate):
    q, K, V, L = _prefill_case()
    scale = O.default_scale(q.shape[-1])
    tau = np.full(q.shape[:3], -np.inf)
    o, lse = O.prefill(q, tau, K, V, L, scale, T_gate)
    G = q.shape[1] // K.shape[1]
    Kt = torch.from_numpy(K).repeat_interleave(G, 1)
    Vt = torch.from_numpy(V).repeat_interleave(G, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q), Kt, Vt,
                                                           is_causal=True, scale=scale).numpy()
    s = torch.einsum("bhtd,bhsd->bhts", torch.from_numpy(q), Kt) * scale
    s = s.masked_fill(torch.triu(torch.ones(q.shape[2], q.shape[2], dtype=torch.bool), 1),
                      -math.inf)
    ref_lse = torch.logsumexp(s, -1).numpy()
    for b in range(q.shape[0]):
        n = L[b]
        np.testing.assert_allclose(o[b, :, :n], ref[b, :, :n], atol=1e-12)
        np.testing.assert_allclose(lse[b, :, :n], ref_lse[b, :, :n], atol=1e-12)
        assert np.all(o[b, :, n:] == 0)


def test_prefill_tau_above_scores_is_cumulative_mean():
    q, K, V, L = _prefill_case(seed=31)
    tau = np.full(q.shape[:3], 1e6)
    o, lse = O.prefill(q, tau, K, V, L, 1.0, 0.0)
    G = q.shape[1] // K.shape[1]
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            cm = np.cumsum(V[b, h // G], axis=0) / np.arange(1, q.shape[2] + 1)[:, None]
            np.testing.assert_allclose(o[b, h, :L[b]], cm[:L[b]], atol=1e-12)
            np.testing.assert_allclose(lse[b, h, :L[b]], np.log(np.arange(1, L[b] + 1)), atol=1e-12)


def test_prefill_row_equals_gated_decode_over_its_prefix():
    """Query t of a prefill is the decode of query t over the cache prefix 0..t."""
    q, K, V, L = _prefill_case(seed=32)
    rng = np.random.default_rng(33)
    tau = rng.normal(size=q.shape[:3]) * 0.3
    scale = O.default_scale(q.shape[-1])
    o, lse = O.prefill(q, tau, K, V, L, scale, 0.0)
    G = q.shape[1] // K.shape[1]
    for (b, h, t) in [(0, 0, 0), (0, 3, 17), (1, 2, 26), (1, 1, 5)]:
        s = scale * K[b, h // G, :t + 1] @ q[b, h, t]
        sp = np.where(s >= tau[b, h, t], s, 0.0)
        p = np.exp(sp - sp.max())
        np.testing.assert_allclose(o[b, h, t], p @ V[b, h // G, :t + 1] / p.sum(), atol=1e-12)


# ----------------------------------------------------------------------------
# log-sum-exp merge of results over disjoint key sets (sequence-sharded decode)
# ----------------------------------------------------------------------------
def test_lse_merge_equals_softmax_over_the_union():
    rng = np.random.default_rng(11)
    n, d = 60, 8
    logits = rng.normal(0, 3, n)
    vals = rng.normal(0, 1, (n, d))
    cut = [0, 17, 17, 41, n]                      # the second part is empty
    o_parts, lse_parts = [], []
    for a, b in zip(cut[:-1], cut[1:]):
        l, v = logits[a:b], vals[a:b]
        if b > a:
            w = torch.softmax(torch.tensor(l), 0).numpy()
            o_parts.append(w @ v)
            lse_parts.append(float(torch.logsumexp(torch.tensor(l), 0)))
        else:
            o_parts.append(np.zeros(d))
            lse_parts.append(-math.inf)
    o, lse = O.lse_merge(np.stack(o_parts), np.array(lse_parts))
    w = torch.softmax(torch.tensor(logits), 0).numpy()
    np.testing.assert_allclose(o, w @ vals, rtol=0, atol=1e-12)
    assert abs(lse - float(torch.logsumexp(torch.tensor(logits), 0))) < 1e-12
    # one part: the identity; every part empty: o = 0, lse = -inf
    o1, l1 = O.lse_merge(np.stack(o_parts[:1]), np.array(lse_parts[:1]))
    np.testing.assert_array_equal(o1, o_parts[0])
    assert l1 == lse_parts[0]
    oe, le = O.lse_merge(np.zeros((3, d)), np.full(3, -math.inf))
    assert np.all(oe == 0) and np.isneginf(le)


@pytest.mark.parametrize("prune", [O.PRUNE_SKIP, O.PRUNE_FLOOR])
def test_block_aligned_sequence_shards_merge_to_the_unsharded_decode(prune):
    """Screening is per block and tau per query, so each shard of a block-aligned
    split admits exactly the unsharded union's blocks in its range; merging the
    shards' (o, lse) must give the unsharded decode."""
    w = synth.TINY.with_(ctx=1024, seed=91)
    g = synth.generate(w, "cpu", lengths=torch.tensor([1000], dtype=torch.int32))
    K, V, q = (g[k].double().numpy() for k in ("K", "V", "q"))
    L = g["lengths"].numpy().astype(np.int64)
    scale = O.default_scale(w.d)
    tau = O.predict_tau(q, g["W"].double().numpy(), np.full(w.Hq, 0.3))
    meta = O.cache_meta(K, L, w.blk, V)
    sc = O.screen(q, tau, meta, scale)
    o_ref, lse_ref = O.decode(q, tau, K, V, L, sc["union_idx"], w.blk, scale, 0.05, prune, meta)
    cuts = [0, 5 * w.blk, 9 * w.blk, w.ctx]       # three shards, the last partly empty
    o_parts, lse_parts = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        Ls = np.clip(L - a, 0, b - a)
        ms = O.cache_meta(K[:, :, a:b], Ls, w.blk, V[:, :, a:b])
        ss = O.screen(q, tau, ms, scale)
        o_s, l_s = O.decode(q, tau, K[:, :, a:b], V[:, :, a:b], Ls, ss["union_idx"], w.blk,
                            scale, 0.05, prune, ms)
        o_parts.append(o_s)
        lse_parts.append(l_s)
        # the shard admits exactly the unsharded union's blocks in its range
        for gg in range(w.Hkv):
            want = [j - a // w.blk for j in sc["union_idx"][0][gg] if a <= j * w.blk < b]
            assert list(ss["union_idx"][0][gg]) == want
    o, lse = O.lse_merge(np.stack(o_parts), np.stack(lse_parts))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-10)
