"""Plain float64 CPU oracle of the ETA block-sparse decode step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call this
module: only the test-suite, the smoke check of the package entry file and the
CPU-baseline / reference legs of the benchmark script use it.  It shares no
code with the CUDA path; the two meet only through the seeded input
generator, which holds none of the method's arithmetic.

Sources (untrusted web pages about arXiv 2609.20888, "Elastic Threshold
Attention: Learned Contextual Sparsity for Long-Context Decoding"):

* [abstract]   the paper's abstract (montaan.com listing / arXiv mirror):
               thresholds predicted from queries, multiplicative suppression of
               sub-threshold logits, hard pruning of KV blocks screened in O(1)
               "using cached geometric-probabilistic bounds", co-admitted tokens
               absorbed, frozen per-head constant thresholds after calibration.
* [review-FAQ] evolve.pub review, FAQ: "whole KV-cache blocks whose best
               possible score falls below the threshold are skipped entirely";
               sub-threshold logits go to zero, i.e. weight e^0 = 1.
* [review-sum] evolve.pub review, Summary: cached centroid / variance /
               max-norm block metadata.
* [Eq. 1-3]    evolve.pub review, Methodology Assessment: tau = qbar W + b on
               concatenated post-RoPE queries (Eq. 1); m = sigmoid(beta (S - tau))
               (Eq. 2); gated logits S * m (Eq. 3).

Where the pages leave a step open, this file takes the reading listed in the
design notes of the repository (bound formula, variance definition, scaling,
union semantics, pruned-block semantics, tie-breaks); each function says which.

Everything is float64.  bf16 inputs are passed in already widened (exactly).
Pure numpy; no blocking, fusion or reordering beyond the definitions.

The two probabilistic bounds of block_bounds (BOUND_PROB, BOUND_PROB_DIM) are
readings: the pages name a "probabilistic" bound from cached variance but print
no formula.  Each is pinned to the property that defines a z-sigma bound: on
blocks of keys with Gaussian deviations from their centre (isotropic for the
scalar form, one spread per dimension for the per-dimension form) the fraction
of keys scoring above the bound is the one-sided normal tail 1 - Phi(z), within
a binomial tolerance; besides, neither is ever looser than the exact bound, and
both equal it as z grows.  Every function is pinned by closed forms, brute
force, library routines or those statistics in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

BOUND_EXACT = "exact"
BOUND_PROB = "prob"
BOUND_PROB_DIM = "prob_dim"
PRUNE_SKIP = "skip"
PRUNE_FLOOR = "floor"


def default_scale(d: int) -> float:
    """Logit scale 1/sqrt(d).  The pages write S without a scale (Eq. 1-3);
    the standard attention convention is taken and tau is in the same units."""
    return 1.0 / math.sqrt(d)


# ----------------------------------------------------------------------------
# (1) per-block metadata  [review-sum; abstract: "cached ... bounds"]
# ----------------------------------------------------------------------------
def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (8 significant bits), ties to
    even.  Written from the definition of the format: x = m * 2**e, 0.5 <= |m| < 1,
    keep m to 8 bits.  (Normal range only, which is all the metadata needs.)"""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def block_meta(K_seq: np.ndarray, n_valid: int, blk: int,
               V_seq: Optional[np.ndarray] = None,
               cent_format: str = "f32") -> Dict[str, np.ndarray]:
    """Metadata of every block of one (batch row, KV head) key sequence.

    K_seq: [T_max, d] float64; keys t < n_valid are valid.
    Block j holds keys [j*blk, min((j+1)*blk, n_valid)).  For its n_j valid keys:
      cent_j = mean of the keys (cent_format "bf16": the mean rounded to bf16,
               the centroid the compact metadata stores)
      rmax_j = max_t ||k_t - cent_j||            (max deviation norm)
      var_j  = (1/n_j) sum_t ||k_t - cent_j||^2  (total variance, one scalar)
      cnt_j  = n_j
      vsum_j = sum_t v_t                         (only if V_seq is given)
      vardim_j[i] = (1/n_j) sum_t (k_t[i] - cent_j[i])^2   (per-dimension variance)
    Empty blocks (n_j = 0) get zeros.
    """
    T_max, d = K_seq.shape
    NB = (T_max + blk - 1) // blk
    cent = np.zeros((NB, d))
    rmax = np.zeros(NB)
    var = np.zeros(NB)
    cnt = np.zeros(NB, dtype=np.int64)
    vardim = np.zeros((NB, d))
    vsum = np.zeros((NB, d)) if V_seq is not None else None
    for j in range(NB):
        lo = j * blk
        hi = min(lo + blk, n_valid)
        n = hi - lo
        if n <= 0:
            continue
        keys = K_seq[lo:hi]
        c = keys.mean(axis=0)
        if cent_format == "bf16":
            c = round_to_bf16(c)
        dist = np.sqrt(((keys - c) ** 2).sum(axis=1))
        cent[j] = c
        rmax[j] = dist.max()
        var[j] = (dist ** 2).mean()
        vardim[j] = ((keys - c) ** 2).mean(axis=0)
        cnt[j] = n
        if vsum is not None:
            vsum[j] = V_seq[lo:hi].sum(axis=0)
    out = dict(cent=cent, rmax=rmax, var=var, cnt=cnt, vardim=vardim)
    if vsum is not None:
        out["vsum"] = vsum
    return out


def cache_meta(K: np.ndarray, lengths: Sequence[int], blk: int,
               V: Optional[np.ndarray] = None, cent_format: str = "f32") -> Dict[str, np.ndarray]:
    """block_meta over a whole cache K [B, Hkv, T_max, d] -> arrays [B, Hkv, NB, ...]."""
    B, Hkv = K.shape[:2]
    rows = [[block_meta(K[b, h], int(lengths[b]), blk,
                        None if V is None else V[b, h], cent_format) for h in range(Hkv)]
            for b in range(B)]
    keys = rows[0][0].keys()
    return {k: np.stack([np.stack([rows[b][h][k] for h in range(Hkv)]) for b in range(B)])
            for k in keys}


# ----------------------------------------------------------------------------
# (2) threshold  [Eq. 1; abstract: frozen per-head constants]
# ----------------------------------------------------------------------------
def predict_tau(q: np.ndarray, W: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """tau[b, h] = sum_i qbar[b, i] W[i, h] + bias[h], qbar[b] = concat_h q[b, h].

    q: [B, Hq, d]; W: [Hq*d, Hq]; bias: [Hq].  (Eq. 1)"""
    B, Hq, d = q.shape
    qbar = q.reshape(B, Hq * d)
    return qbar @ W + bias[None, :]


def const_tau(B: int, tau_const: np.ndarray) -> np.ndarray:
    """Calibrated mode: tau[b, h] = tau_const[h], no predictor."""
    return np.broadcast_to(np.asarray(tau_const, dtype=np.float64)[None, :],
                           (B, len(tau_const))).copy()


# ----------------------------------------------------------------------------
# (3) O(1) screening  [abstract "geometric-probabilistic bounds";
#                      review-FAQ "best possible score falls below the threshold"]
# ----------------------------------------------------------------------------
def block_bounds(q_h: np.ndarray, cent: np.ndarray, rmax: np.ndarray, var: np.ndarray,
                 scale: float, bound: str = BOUND_EXACT, z: float = 3.0,
                 vardim: Optional[np.ndarray] = None) -> np.ndarray:
    """Upper bound on scale*(q.k) over each block, in logit units, shape [NB].

    exact (Cauchy-Schwarz):  scale * (q.c + ||q|| * rmax)
    prob  (variance):        scale * (q.c + ||q|| * min(rmax, z * sqrt(var / d)))
    prob_dim (per-dimension variance, vardim [NB, d]):
                             scale * (q.c + min(||q|| * rmax, z * sqrt(sum_i q_i^2 vardim_i)))
    The two probabilistic forms are readings of a z-sigma bound (see the module
    note): for Gaussian key deviations a fraction 1 - Phi(z) of keys exceeds them.
    """
    d = q_h.shape[0]
    qc = cent @ q_h
    qn = math.sqrt(float(q_h @ q_h))
    if bound == BOUND_EXACT:
        return scale * (qc + qn * rmax)
    if bound == BOUND_PROB:
        return scale * (qc + qn * np.minimum(rmax, z * np.sqrt(var / d)))
    if bound == BOUND_PROB_DIM:
        spread = np.sqrt(vardim @ (q_h * q_h))
        return scale * (qc + np.minimum(qn * rmax, z * spread))
    raise ValueError(bound)


def screen(q: np.ndarray, tau: np.ndarray, meta: Dict[str, np.ndarray], scale: float,
           bound: str = BOUND_EXACT, z: float = 3.0) -> Dict[str, object]:
    """Bounds, per-head admit masks, per-KV-group unions and ascending lists.

    q: [B, Hq, d]; tau: [B, Hq]; meta arrays [B, Hkv, NB, ...].
    admit[b, h, j] = (UB[b, h, j] >= tau[b, h]) and cnt[b, g(h), j] > 0
    (equality admits), with g(h) = h // G the KV head of query head h.
    union[b, g, j] = OR of admit over the G query heads of group g.
    """
    B, Hq, d = q.shape
    Hkv, NB = meta["cnt"].shape[1:3]
    G = Hq // Hkv
    UB = np.zeros((B, Hq, NB))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            UB[b, h] = block_bounds(q[b, h], meta["cent"][b, g], meta["rmax"][b, g],
                                    meta["var"][b, g], scale, bound, z,
                                    meta["vardim"][b, g] if "vardim" in meta else None)
    nonempty = meta["cnt"] > 0                                   # [B, Hkv, NB]
    nonempty_h = np.repeat(nonempty, G, axis=1)                  # [B, Hq, NB]
    admit = (UB >= tau[:, :, None]) & nonempty_h
    union = admit.reshape(B, Hkv, G, NB).any(axis=2)
    union_idx = [[np.nonzero(union[b, g])[0] for g in range(Hkv)] for b in range(B)]
    return dict(bounds=UB, admit=admit, union=union, union_idx=union_idx)


# ----------------------------------------------------------------------------
# (4) gated attention over admitted blocks  [Eq. 2-3; review-FAQ e^0 = 1]
# ----------------------------------------------------------------------------
def sigmoid(x: np.ndarray) -> np.ndarray:
    """Overflow-safe logistic function."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def gate(s: np.ndarray, tau: float, T: float) -> np.ndarray:
    """Gated logit s' (Eq. 2-3 with beta = 1/T).

    T > 0:  s' = s * sigmoid((s - tau) / T)
    T = 0:  s' = s if s >= tau else 0   (hard gate; a key scoring exactly tau
            keeps its logit)
    """
    s = np.asarray(s, dtype=np.float64)
    if T == 0.0:
        return np.where(s >= tau, s, 0.0)
    return s * sigmoid((s - tau) / T)


def _softmax_out(logits: np.ndarray, values: np.ndarray, n_floor: int = 0,
                 floor_vsum: Optional[np.ndarray] = None):
    """o = sum_t e^{l_t} v_t / sum_t e^{l_t}, lse = log sum_t e^{l_t}, where the
    key set is the listed logits plus n_floor extra keys of logit 0 whose values
    sum to floor_vsum.  Max-shifted; an empty set gives o = 0, lse = -inf."""
    d = values.shape[1] if values.ndim == 2 else floor_vsum.shape[0]
    if logits.size == 0 and n_floor == 0:
        return np.zeros(d), -math.inf
    m = logits.max() if logits.size else -math.inf
    if n_floor > 0:
        m = max(m, 0.0)
    p = np.exp(logits - m)
    num = p @ values if logits.size else np.zeros(d)
    den = p.sum()
    if n_floor > 0:
        num = num + math.exp(-m) * floor_vsum
        den = den + n_floor * math.exp(-m)
    return num / den, m + math.log(den)


def block_keys(blocks: Sequence[int], n_valid: int, blk: int) -> np.ndarray:
    """Valid token indices of the listed blocks, in block order."""
    idx = [np.arange(j * blk, min((j + 1) * blk, n_valid)) for j in blocks]
    idx = [i for i in idx if i.size]
    return np.concatenate(idx) if idx else np.zeros(0, dtype=np.int64)


def attend_blocks(q_h: np.ndarray, tau_h: float, K_seq: np.ndarray, V_seq: np.ndarray,
                  n_valid: int, blocks: Sequence[int], blk: int, scale: float, T: float,
                  prune: str = PRUNE_SKIP, meta_row: Optional[Dict[str, np.ndarray]] = None):
    """One query head over the admitted blocks of its KV group.

    SKIP:  pruned keys are absent from the softmax.
    FLOOR: every valid key of a pruned block enters with logit 0 (the value the
           hard gate gives a sub-threshold key), using the block's cnt / vsum.
    """
    idx = block_keys(blocks, n_valid, blk)
    s = scale * (K_seq[idx] @ q_h)
    sp = gate(s, tau_h, T)
    vals = V_seq[idx]
    if prune == PRUNE_SKIP:
        return _softmax_out(sp, vals)
    NB = meta_row["cnt"].shape[0]
    admitted = np.zeros(NB, dtype=bool)
    admitted[np.asarray(blocks, dtype=np.int64)] = True
    pruned = (~admitted) & (meta_row["cnt"] > 0)
    n_floor = int(meta_row["cnt"][pruned].sum())
    fv = meta_row["vsum"][pruned].sum(axis=0)
    return _softmax_out(sp, vals, n_floor, fv)


def decode(q: np.ndarray, tau: np.ndarray, K: np.ndarray, V: np.ndarray,
           lengths: Sequence[int], union_idx, blk: int, scale: float, T: float,
           prune: str = PRUNE_SKIP, meta: Optional[Dict[str, np.ndarray]] = None):
    """ETA decode for every (b, h): each query head attends over ALL union
    blocks of its KV group (co-admitted tokens are absorbed by the gate,
    [abstract]) with its own tau.  Returns o [B, Hq, d], lse [B, Hq]."""
    B, Hq, d = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    o = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            mr = None
            if prune == PRUNE_FLOOR:
                mr = {k: meta[k][b, g] for k in ("cnt", "vsum")}
            o[b, h], lse[b, h] = attend_blocks(q[b, h], float(tau[b, h]), K[b, g], V[b, g],
                                               int(lengths[b]), union_idx[b][g], blk, scale,
                                               T, prune, mr)
    return o, lse


def lse_merge(o_parts: np.ndarray, lse_parts: np.ndarray):
    """Softmax attention over the union of disjoint key sets from the results over
    each set (the log-sum-exp identity behind split-KV decoding; Eq. 2-3's softmax
    is a plain softmax over the gated logits).  Part p has lse_p = log sum e^{l_t}
    and o_p = the e^{l_t}-weighted mean of its values, so over the union
    o = sum_p e^{lse_p} o_p / sum_p e^{lse_p} and lse = log sum_p e^{lse_p}
    (evaluated max-shifted).  Parts with lse = -inf (no keys) add nothing; all
    empty gives o = 0, lse = -inf.  o_parts [P, ..., d], lse_parts [P, ...]."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    finite = np.isfinite(m)
    shift = np.where(finite, m, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - shift[None]), 0.0)
    den = w.sum(axis=0)
    num = (w[..., None] * o_parts).sum(axis=0)
    safe = np.where(den > 0, den, 1.0)
    o = np.where((den > 0)[..., None], num / safe[..., None], 0.0)
    lse = np.where(den > 0, shift + np.log(safe), -np.inf)
    return o, lse


def dense_gated(q_h: np.ndarray, tau_h: float, K_seq: np.ndarray, V_seq: np.ndarray,
                n_valid: int, scale: float, T: float):
    """Gated attention over every valid key, no pruning (Eq. 2-3)."""
    s = scale * (K_seq[:n_valid] @ q_h)
    return _softmax_out(gate(s, tau_h, T), V_seq[:n_valid])


def softmax_attention(q_h: np.ndarray, K_seq: np.ndarray, V_seq: np.ndarray,
                      n_valid: int, scale: float):
    """Textbook softmax attention of one query over the valid keys."""
    s = scale * (K_seq[:n_valid] @ q_h)
    return _softmax_out(s, V_seq[:n_valid])


def prefill(q: np.ndarray, tau: np.ndarray, K: np.ndarray, V: np.ndarray,
            lengths: Sequence[int], scale: float, T: float):
    """Dense gated causal attention of a prefill chunk (Eq. 2-3 on every pair).

    q [B, Hq, T_max, d] (query at position t of row b), tau [B, Hq, T_max],
    K/V [B, Hkv, T_max, d].  Query t < lengths[b] attends keys 0..t of its KV
    head h // G with gated logits; returns O [B, Hq, T_max, d], lse [B, Hq, T_max]
    (rows t >= lengths[b] left at zero)."""
    B, Hq, Tm, d = q.shape
    G = Hq // K.shape[1]
    o = np.zeros((B, Hq, Tm, d))
    lse = np.zeros((B, Hq, Tm))
    for b in range(B):
        for h in range(Hq):
            for t in range(int(lengths[b])):
                o[b, h, t], lse[b, h, t] = dense_gated(q[b, h, t], float(tau[b, h, t]),
                                                       K[b, h // G], V[b, h // G], t + 1, scale, T)
    return o, lse


def dense_decode(q, K, V, lengths, scale):
    """Textbook decode attention for every (b, h), GQA group h // G."""
    B, Hq, d = q.shape
    G = Hq // K.shape[1]
    o = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hq):
            o[b, h], lse[b, h] = softmax_attention(q[b, h], K[b, h // G], V[b, h // G],
                                                   int(lengths[b]), scale)
    return o, lse


# ----------------------------------------------------------------------------
# offline calibration  [abstract: frozen per-head constant thresholds]
# ----------------------------------------------------------------------------
def calibrate_const_tau(bounds: np.ndarray, valid: np.ndarray, density: float) -> np.ndarray:
    """Per-head constant tau from pooled calibration bounds.

    bounds: [n_q, Hq, NB] block bounds of n_q calibration queries; valid:
    same-shape bool (non-empty blocks).  For each head the valid bounds are
    pooled and sorted ascending; tau_h is the element at index
    floor((1 - density) * N), so that admit-iff-UB>=tau admits at least the
    target fraction of the calibration (query, block) pairs."""
    n_q, Hq, NB = bounds.shape
    tau = np.zeros(Hq)
    for h in range(Hq):
        pool = np.sort(bounds[:, h, :][valid[:, h, :]])
        k = int(math.floor((1.0 - density) * pool.size))
        k = min(max(k, 0), pool.size - 1)
        tau[h] = pool[k]
    return tau


def offset_for_density(bounds: np.ndarray, tau: np.ndarray, valid: np.ndarray,
                       density: float, G: int, kind: str = "head") -> float:
    """Common offset delta such that thresholds tau + delta admit (at least) the
    target fraction of (query head, block) pairs ("head") or of (KV group,
    block) pairs in the union ("union").  Input-synthesis helper for tests.
    delta lies halfway between the k-th margin and the one below it, so that no
    bound sits exactly on a threshold (a tie the test would have to skip)."""
    B, Hq, NB = bounds.shape
    margin = np.where(valid, bounds - tau[:, :, None], -np.inf)
    if kind == "union":
        margin = margin.reshape(B, Hq // G, G, NB).max(axis=2)
    vals = np.sort(margin[np.isfinite(margin)])
    k = int(math.floor((1.0 - density) * vals.size))
    k = min(max(k, 0), vals.size - 1)
    if k == 0:
        return float(vals[0]) - 1.0
    return 0.5 * (float(vals[k - 1]) + float(vals[k]))
