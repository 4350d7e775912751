#!/usr/bin/env python
"""Benchmark of the ETA block-sparse decode step on B200.

One step = the whole hot path for one batch of decode queries of one layer:
  eta_build_block_meta (tail block of every row: the cache grew by one token)
  eta_predict_tau      (Eq. 1 threshold predictor)
  eta_screen           (O(1) block screening, per-head masks, union compaction)
  eta_decode           (gated split-KV attention over admitted blocks + LSE combine)

Default workload: batch 64, 16 query / 4 KV heads, d = 128, 512K context (68.7 GB
of K/V), KV block 128, bf16 clustered-key cache (256 clusters, segments of 384-640
tokens), threshold bias calibrated for 16% union density, probabilistic variance
bound with z = 3 (the exact bound's union density at the same thresholds and the
keys scoring above tau that z = 3 prunes are reported beside it), hard gate.
`--workload long-b64...` selects the 128K / block-64 / exact-bound configuration.

Prints ONE JSON line (rank 0).  `--impl reference` times the float64 CPU oracle
on a bounded sample of the same workload instead (rank 0 only).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl eta|reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_decoding_eta_b200 import synth  # noqa: E402

METRIC = "decode attn steps/s and HBM GB/s on admitted KV bytes (% of B200 peak)"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1000 * 1000
# where the nvidia-smi clock samples of the timed region go (--clock-log-dir)
CLOCK_LOG_DIR = tempfile.gettempdir()
NOMINAL_HBM_GBS = 8000.0
PROLOGUE_LAUNCHES = 1   # tail-block metadata + tau in one launch (2 when separate)
LAUNCHES_PER_FUSED_STEP = 1   # eta_decode_step: one persistent kernel


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def with_overrides(w: synth.Workload, args) -> synth.Workload:
    """The workload with the operating point asked for on the command line (the
    density sweep and the threshold mode of the long-context configurations)."""
    kw = {}
    if getattr(args, "density", None):
        kw["density"] = float(args.density)
    if getattr(args, "density_kind", None):
        kw["density_kind"] = args.density_kind
    if getattr(args, "tau_mode", None):
        kw["tau_mode"] = args.tau_mode
    if getattr(args, "bound", None):
        kw["bound"] = args.bound
    if getattr(args, "ctx", 0):
        kw["ctx"] = int(args.ctx)
    if not kw:
        return w
    tag = "-".join(f"{k}{v}" for k, v in sorted(kw.items()))
    return w.with_(name=f"{w.name}-{tag}", **kw)


def workload_by_name(name: str, B: int = 0) -> synth.Workload:
    for w in synth.WORKLOADS.values():
        if w.name == name or w.name.startswith(name):
            return w.with_(B=B, name=w.name.replace(f"b{w.B}-", f"b{B}-", 1)) if B else w
    raise SystemExit(f"unknown workload {name}; choose from {list(synth.WORKLOADS)}")


def density_offset(bounds: np.ndarray, tau0: np.ndarray, valid: np.ndarray, density: float,
                   G: int, kind: str) -> float:
    """Common threshold offset that admits the target fraction of (head, block)
    pairs ("head") or (KV group, block) pairs ("union"): a quantile of the
    margins bound - tau, placed halfway to the next lower margin so that no bound
    sits exactly on a threshold.  Workload calibration only (host numpy)."""
    B, Hq, NB = bounds.shape
    m = np.where(valid, bounds - tau0[:, :, None], -np.inf)
    if kind == "union":
        m = m.reshape(B, Hq // G, G, NB).max(axis=2)
    v = m[np.isfinite(m)]
    k = int(math.floor((1.0 - density) * v.size))
    k = min(max(k, 0), v.size - 1)
    part = np.partition(v, [k - 1, k] if k > 0 else [k])
    if k == 0:
        return float(part[0]) - 1.0
    return 0.5 * (float(part[k - 1]) + float(part[k]))


def decode_traffic(admitted_kv: int, engine_tc: bool, record: str = "decode_tc_traffic.json",
                   pairs: int = 0, ctas: int = 0):
    """DRAM bytes per launch from a committed ncu capture of a small case of the same
    kernel (profiles/<record>), scaled to this workload: the reads by its admitted K/V
    bytes, the writes (partial result slots, one per CTA and pair) by its slot count.
    None when the kernel source changed since the capture or the capture does not
    cover the engine that ran."""
    import hashlib
    p = os.path.join(ROOT, "profiles", record)
    if not engine_tc or not os.path.exists(p):
        return None
    rec = json.load(open(p))
    m = hashlib.sha256()
    for f in rec["source_files"]:
        fp = os.path.join(ROOT, f)
        if not os.path.exists(fp):
            return None
        m.update(open(fp, "rb").read())
    if m.hexdigest() != rec["source_sha256"]:
        return None
    reads = rec["dram_bytes_read"] / rec["admitted_kv_bytes"] * admitted_kv
    slots = (ctas + pairs) / (rec["ctas"] + rec["pairs"]) if pairs and ctas else 1.0
    return reads + rec["dram_bytes_write"] * slots


def reduce_max(x: float, device) -> float:
    """Max over ranks of a per-rank figure (the job time of the independent,
    weak-scaled replicas).  Identity when not running distributed."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, max_ms: float) -> float:
    """Whole-job steps/s: every rank runs `steps` full-batch steps of its own
    replica; the job takes the slowest rank's time."""
    return world * steps / (max_ms * 1e-3)


class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi during a region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(CLOCK_LOG_DIR, f"eta_bench_clocks_rank{index}.csv")

    def __enter__(self):
        self.fh = None
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}",
                                          f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            if self.fh is not None:
                self.fh.close()
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def setup(w: synth.Workload, device, rank: int, cent_format: str = "f32", fused: bool = False,
          merged_prologue: bool = True):
    from long_context_decoding_eta_b200.api import EtaDecoder
    g = synth.generate(w, device, seed=w.seed + 7919 * rank)
    dec = EtaDecoder(g["K"], g["V"], g["lengths"], w.Hq, w.blk, bound=w.bound, z=w.z,
                     T=w.gate_T, keep_bounds=True, cent_format=cent_format, fused=fused,
                     merged_prologue=merged_prologue)
    dec.build_meta()
    # workload calibration: bias so that tau hits the density target
    if w.tau_mode == "const":
        qc = synth.calibration_queries(w, g["mu"])
        tau_const = dec.calibrate_const_tau(qc, w.density).to(device)
        W = bias = None
    else:
        tau_const = None
        W = g["W"]
        dec.predict_tau(g["q"], W, None, None)
        tau0 = dec.tau.clone()
        dec.screen(g["q"], tau0, bounds=dec.bounds)
        valid = (dec.cnt > 0).repeat_interleave(w.G, dim=1).cpu().numpy()
        off = density_offset(dec.bounds.cpu().numpy(), tau0.cpu().numpy(), valid, w.density,
                             w.G, w.density_kind)
        bias = torch.full((w.Hq,), off, dtype=torch.float32, device=device)
    dec.bounds = None
    return g, dec, W, bias, tau_const


def workload_config(w: synth.Workload, args) -> dict:
    """The workload keys of the JSON line, identical in the eta and reference arms
    (what was measured about the run goes elsewhere in the line)."""
    dense_kv = w.B * w.Hkv * w.ctx * w.d * 2 * 2
    nb_total = w.B * w.Hkv * ((w.ctx + w.blk - 1) // w.blk)
    cb = 2 if args.cent == "bf16" else 4
    est = w.density * dense_kv + nb_total * (cb * w.d + 12)
    return {
        "workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
        "context": w.ctx, "blk": w.blk, "bound": w.bound,
        "z": w.z if w.bound != "exact" else None, "gate_T": w.gate_T,
        "tau_mode": w.tau_mode, "density_target": f"{w.density:.2f} {w.density_kind}",
        "centroids": args.cent, "engine": args.engine, "cuda_graph": bool(args.graph),
        "fused_step": bool(args.fused),
        "prologue": "separate" if args.separate_prologue else "one launch",
        "l2": (f"no flush: a step reads about {est / 1e9:.2f} GB (admitted K/V at the density "
               "target + screened metadata), more than the 126 MB L2" if est > L2_BYTES else
               f"no flush: a step's ~{est / 1e6:.1f} MB stay L2-resident (a launch-latency "
               "figure, not a bandwidth one)"),
        "parallelism": "single GPU",
    }


def unpack_admit(words: torch.Tensor, NB: int) -> torch.Tensor:
    """uint32 mask words [..., NW] (held as int32) -> bool [..., NB] on the device."""
    j = torch.arange(NB, device=words.device)
    w = words[..., j // 32].to(torch.int64) & 0xFFFFFFFF
    return ((w >> (j % 32)) & 1).bool()


def screen_diagnostics(dec, q, w) -> dict:
    """Statistics of the step's screening, taken after the timed region:
    - near_tie_blocks: (query head, block) pairs whose bound lies within 1e-5 of
      tau (relative, floored at 1), where fp32 rounding may flip the admit bit;
    - empty_unions: (row, KV head) pairs that admitted no block;
    - keys scoring s >= tau (s = scale q.k over every valid key, fp32, computed with
      torch over all rows) and how many of them sit in blocks the screening pruned
      for their head, or pruned from their group's union (the union is what the
      decode reads).  The exact bound never prunes such a key (up to fp32 ties);
      for a probabilistic bound the ratio is its measured miss rate;
    - for a probabilistic bound, the union density the exact bound admits at the
      same thresholds."""
    from long_context_decoding_eta_b200 import _lib
    B, Hq, Hkv, NB, G, blk = dec.B, dec.Hq, dec.Hkv, dec.NB, dec.Hq // dec.Hkv, dec.blk
    dev = dec.K.device
    bounds = torch.empty(B, Hq, NB, dtype=torch.float32, device=dev)
    hm = torch.empty_like(dec.head_mask)
    ui, uc, hc = (torch.empty_like(dec.union_idx), torch.empty_like(dec.union_cnt),
                  torch.empty_like(dec.head_cnt))
    _lib.eta_screen(dec.dims, q, dec.tau, dec.cent, dec.rmax, dec.var, dec.cnt, dec.bound,
                    dec.z, dec.scale, hm, ui, uc, bounds, hc, dec.ws_screen, dec.dev_status,
                    None, dec.vardim)
    valid_blk = dec.cnt > 0
    nonempty = int(valid_blk.sum())
    tau = dec.tau
    near = ((bounds - tau[..., None]).abs() <= 1e-5 * tau.abs().clamp(min=1.0)[..., None])
    near &= valid_blk.repeat_interleave(G, dim=1)
    out = {"near_tie_blocks": int(near.sum()), "screened_pairs": int(nonempty * G),
           "empty_unions": int((uc == 0).sum()),
           "union_density": float(uc.sum()) / max(1, nonempty)}
    if dec.bound != "exact":
        uc_ex = torch.empty_like(uc)
        _lib.eta_screen(dec.dims, q, dec.tau, dec.cent, dec.rmax, dec.var, dec.cnt, "exact",
                        dec.z, dec.scale, torch.empty_like(hm), torch.empty_like(ui), uc_ex,
                        None, torch.empty_like(hc), dec.ws_screen, dec.dev_status, None,
                        dec.vardim)
        out["union_density_exact_bound_same_tau"] = float(uc_ex.sum()) / max(1, nonempty)
    admit = unpack_admit(hm, NB)                                   # [B, Hq, NB]
    above = missed_head = missed_union = 0
    for b in range(B):
        n = int(dec.lengths[b])
        if n == 0:
            continue
        s = torch.einsum("gtd,ghd->ght", dec.K[b, :, :n].float(),
                         q[b].float().view(Hkv, G, dec.d)) * dec.scale    # [Hkv, G, n]
        hi = s >= tau[b].view(Hkv, G, 1)
        blk_of = torch.arange(n, device=dev) // blk
        adm = admit[b].view(Hkv, G, NB)[:, :, blk_of]                     # [Hkv, G, n]
        uni = admit[b].view(Hkv, G, NB).any(dim=1)[:, None, blk_of]
        above += int(hi.sum())
        missed_head += int((hi & ~adm).sum())
        missed_union += int((hi & ~uni).sum())
    out.update({"keys_scoring_above_tau": above, "of_which_pruned_for_their_head": missed_head,
                "of_which_outside_the_union": missed_union,
                "miss_rate_head": (missed_head / above) if above else None,
                "miss_rate_union": (missed_union / above) if above else None})
    return out


def step_bytes(dec, w):
    """Algorithmic HBM bytes of one step, from the step's own screening output."""
    lengths = dec.lengths.to(torch.int64)
    B, Hkv, NB, blk, d = dec.B, dec.Hkv, dec.NB, dec.blk, dec.d
    cnt = dec.cnt.to(torch.int64)                          # [B, Hkv, NB] valid keys per block
    idx = dec.union_idx.to(torch.int64)
    ucnt = dec.union_cnt.to(torch.int64)
    ar = torch.arange(NB, device=cnt.device)
    take = ar[None, None, :] < ucnt[:, :, None]
    keys = torch.where(take, torch.gather(cnt, 2, idx.clamp(0, NB - 1)), 0).sum()
    adm_kv = int(keys) * d * 2 * 2                          # K + V, bf16
    qbytes = B * w.Hq * d * 2
    obytes = B * w.Hq * (d + 1) * 4
    cb = 2 if dec.cent.dtype == torch.bfloat16 else 4
    meta = B * Hkv * NB * (cb * d + 12)                     # cent + rmax + var + cnt read by screen
    tail = B * Hkv * (blk * d * 2 + (cb * d + 12))          # tail block keys read + meta written
    tau_bytes = w.Hq * d * w.Hq * 4 + B * w.Hq * 4
    dens_union = float(ucnt.sum()) / max(1.0, float((cnt > 0).sum()))
    dens_head = float(dec.head_cnt.to(torch.int64).sum()) / max(
        1.0, float((cnt > 0).sum()) * (w.Hq // Hkv))
    return dict(decode=adm_kv + qbytes + obytes, step=adm_kv + qbytes + obytes + meta + tail
                + tau_bytes, admitted_kv=adm_kv, meta=meta, union_density=dens_union,
                head_density=dens_head, dense_kv=int(lengths.sum()) * Hkv * d * 4)


def run_eta(args, rank, world, device):
    from long_context_decoding_eta_b200 import _lib
    _lib.eta_set_decode_engine(args.engine)
    w = with_overrides(workload_by_name(args.workload, args.B), args)
    fused = bool(args.fused)
    g, dec, W, bias, tau_const = setup(w, device, rank, args.cent, fused,
                                       not args.separate_prologue)
    q = g["q"]
    stream = torch.cuda.current_stream()
    # one step to measure densities / bytes, then check status
    dec.step(q, W, bias, tau_const)
    torch.cuda.synchronize()
    dec.check_status()
    by = step_bytes(dec, w)

    if args.graph:
        g_pre, g_dec = dec.capture(q, W, bias, tau_const, split=not fused)

    def one_step(ev=None):
        if fused:        # the whole step is the one launch the events bracket
            if ev is not None:
                ev[0].record(stream)
            if args.graph:
                g_pre.replay()
            else:
                dec.step_fused(q, W, bias, tau_const)
            if ev is not None:
                ev[1].record(stream)
            return
        if args.graph:
            g_pre.replay()
        else:
            dec.prepare(q, W, bias, tau_const)
        if ev is not None:
            ev[0].record(stream)
        if args.graph:
            g_dec.replay()
        else:
            dec.decode(q)
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(device.index if device.index is not None else 0) as clk:
        # keep the same load running for at least ~1 s so the 100 ms clock
        # sampler sees the GPU under this step, then time exactly `steps` steps
        t_soak = time.perf_counter()
        while time.perf_counter() - t_soak < args.clock_soak_s:
            for _ in range(8):
                one_step()
            torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(args.steps):
            one_step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    dec.check_status()
    ms = reduce_max(t0.elapsed_time(t1), device)
    dec_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps

    # dense baseline on the same cache (same pipeline, every block, no gate)
    for _ in range(3):
        dec.dense_decode(q)
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nd = max(3, min(args.steps, 10))
    d0.record(stream)
    for _ in range(nd):
        dec.dense_decode(q)
    d1.record(stream)
    torch.cuda.synchronize()
    dense_ms = d0.elapsed_time(d1) / nd

    # end to end through the public API with host buffers
    q_host = q.cpu().pin_memory()
    o_host = torch.empty(dec.o.shape, dtype=torch.float32).pin_memory()
    lse_host = torch.empty(dec.lse.shape, dtype=torch.float32).pin_memory()
    q_dev = torch.empty_like(q)

    def e2e_step():
        q_dev.copy_(q_host, non_blocking=True)
        dec.step(q_dev, W, bias, tau_const)
        o_host.copy_(dec.o, non_blocking=True)
        lse_host.copy_(dec.lse, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / args.steps, device)

    diag = screen_diagnostics(dec, q, w)
    torch.cuda.synchronize()
    dec.check_status()

    peak, peak_kind = peaks()
    ms_step = ms / args.steps
    # the dominant kernel: eta_decode's three launches, or the fused step's one launch
    # (which also reads the screened metadata: its algorithmic bytes are the step's)
    achieved = (by["step"] if fused else by["decode"]) / (dec_ms * 1e-3) / 1e9
    res = {
        "metric": METRIC,
        "value": job_throughput(world, args.steps, ms),
        "unit": "steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": dict(workload_config(w, args),
                       parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
        "density": {"union": round(by["union_density"], 4),
                    "head": round(by["head_density"], 4)},
        "screening": diag,
        "hbm_gbs": by["step"] / (ms_step * 1e-3) / 1e9,
        "hbm_frac_of_nominal_8tbs": by["step"] / (ms_step * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
        "bytes_per_step": {"admitted_kv": by["admitted_kv"], "metadata": by["meta"],
                           "total": by["step"], "dense_kv": by["dense_kv"]},
        "roofline": {"kernel": ("eta_decode_step (one persistent kernel: tail metadata, tau, "
                                "screen, decode, merge)") if fused else
                               "eta_decode (split-KV decode with its share plan + combine)",
                     "bound": "hbm",
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": f"{peak_kind} copy bandwidth",
                     "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                     "decode_ms": dec_ms,
                     "traffic": decode_traffic(
                         by["admitted_kv"], w.d == 128 and (fused or args.engine in
                                                            ("auto", "tcgen05")),
                         "step_fused_traffic.json" if fused else "decode_tc_traffic.json",
                         dec.B * dec.Hkv, torch.cuda.get_device_properties(device).multi_processor_count),
                     "traffic_source": ("profiles/step_fused_traffic.json" if fused else
                                        "profiles/decode_tc_traffic.json") +
                                       " (ncu dram__bytes_read+write of one launch of a small "
                                       "case of the same kernel: reads scaled by admitted K/V "
                                       "bytes, writes by partial-slot count)"},
        "dense_baseline": {"ms": dense_ms, "steps_per_s_decode_only": 1e3 / dense_ms,
                           "gbs": by["dense_kv"] / (dense_ms * 1e-3) / 1e9,
                           "speedup_of_eta_decode": dense_ms / dec_ms},
        "e2e": {"value": job_throughput(world, 1, e2e_ms), "unit": "steps/s",
                "h2d_bytes_per_step": q_host.numel() * 2,
                "d2h_bytes_per_step": o_host.numel() * 4 + lse_host.numel() * 4},
        # all ranks' launches in the timed region (each rank runs the same steps)
        "gpu_launches": (LAUNCHES_PER_FUSED_STEP if fused else
                         PROLOGUE_LAUNCHES + (1 if args.separate_prologue else 0) +
                         _lib.eta_screen_launches(dec.dims, args.cent) +
                         _lib.eta_decode_launches(dec.dims))
                        * args.steps * world,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, g, rows=args.cpu_rows)
    return res


class OracleSample:
    """The float64 oracle's decode step over a bounded sample of batch rows (all
    heads of those rows), on the same cache bytes the GPU reads.  The widened
    cache and its block metadata (the prefill) are prepared once, untimed; each
    step() times one oracle step: the tail-block metadata of every sampled
    (row, KV head), the thresholds, the screening and the gated decode."""

    def __init__(self, w, g, rows):
        from oracle import eta_oracle as O
        self.O, self.w = O, w
        self.rows = list(rows)
        self.K64 = g["K"][self.rows].double().cpu().numpy()
        self.V64 = g["V"][self.rows].double().cpu().numpy()
        self.q64 = g["q"][self.rows].double().cpu().numpy()
        self.L = g["lengths"][self.rows].cpu().numpy()
        self.meta = O.cache_meta(self.K64, self.L, w.blk)
        self.scale = 1.0 / math.sqrt(w.d)

    def step(self, W64, b64, tc) -> float:
        O, w, K64, L, meta = self.O, self.w, self.K64, self.L, self.meta
        t = time.perf_counter()
        for i in range(len(self.rows)):
            j = (int(L[i]) - 1) // w.blk
            for h in range(w.Hkv):
                m = O.block_meta(K64[i, h, j * w.blk:(j + 1) * w.blk], int(L[i]) - j * w.blk,
                                 w.blk)
                for k in ("cent", "rmax", "var", "cnt", "vardim"):
                    meta[k][i, h, j] = m[k][0]
        tau = (O.predict_tau(self.q64, W64, b64) if tc is None
               else O.const_tau(len(self.rows), tc))
        sc = O.screen(self.q64, tau, meta, self.scale, w.bound, w.z)
        O.decode(self.q64, tau, K64, self.V64, L, sc["union_idx"], w.blk, self.scale, w.gate_T)
        return time.perf_counter() - t

    def union_density(self, W64, b64, tc) -> float:
        O = self.O
        tau = (O.predict_tau(self.q64, W64, b64) if tc is None
               else O.const_tau(len(self.rows), tc))
        sc = O.screen(self.q64, tau, self.meta, self.scale, self.w.bound, self.w.z)
        return float(sc["union"].sum()) / max(1, int((self.meta["cnt"] > 0).sum()))


def time_oracle(sample: OracleSample, W, bias, tau_const, warmup: int, reps: int):
    """Per-step seconds of `reps` oracle steps after `warmup` untimed ones, with
    numpy's BLAS held to one thread (the oracle is single-threaded Python loops
    over rows and heads; the thread count reported is the one used)."""
    from threadpoolctl import threadpool_limits
    W64 = None if W is None else W.double().cpu().numpy()
    b64 = None if bias is None else bias.double().cpu().numpy()
    tc = None if tau_const is None else tau_const.double().cpu().numpy()
    with threadpool_limits(limits=1):
        for _ in range(warmup):
            sample.step(W64, b64, tc)
        return [sample.step(W64, b64, tc) for _ in range(reps)]


def oracle_sample_inputs(w, g, rows):
    """The oracle's sample of `rows` batch rows and its threshold inputs: the
    predictor's W with a bias the oracle sets itself on those rows by the workload's
    density rule, or (calibrated workloads) per-head constants from the calibration
    rule on them.  Both arms time the oracle on exactly these inputs."""
    from oracle import eta_oracle as O
    sample = OracleSample(w, g, rows)
    meta, q64, scale = sample.meta, sample.q64, sample.scale
    W = bias = tau_const = None
    if w.tau_mode == "const":
        qc = synth.calibration_queries(w, g["mu"]).double().cpu().numpy()
        n = qc.shape[0]
        bounds = np.zeros((n, w.Hq, w.NB))
        valid = np.zeros((n, w.Hq, w.NB), dtype=bool)
        for i in range(n):
            r = i % len(rows)
            mrow = {k: v[r:r + 1] for k, v in meta.items()}
            bounds[i] = O.screen(qc[i:i + 1], np.zeros((1, w.Hq)), mrow, scale, w.bound,
                                 w.z)["bounds"][0]
            valid[i] = np.repeat(meta["cnt"][r] > 0, w.G, axis=0)
        tau_const = torch.from_numpy(O.calibrate_const_tau(bounds, valid, w.density))
    else:
        W = g["W"]
        W64 = W.double().cpu().numpy()
        tau0 = O.predict_tau(q64, W64, np.zeros(w.Hq))
        ub = O.screen(q64, tau0, meta, scale, w.bound, w.z)["bounds"]
        off = O.offset_for_density(ub, tau0, np.repeat(meta["cnt"] > 0, w.G, axis=1),
                                   w.density, w.G, w.density_kind)
        bias = torch.full((w.Hq,), off, dtype=torch.float64)
    return sample, W, bias, tau_const


def cpu_baseline(w, g, rows=2, warmup=1, reps=3):
    """The oracle timed as the reference arm times it (same sample, same threshold
    inputs, one thread), inside the eta arm's line."""
    rows = list(range(max(1, min(rows, w.B))))
    sample, W, bias, tau_const = oracle_sample_inputs(w, g, rows)
    times = time_oracle(sample, W, bias, tau_const, warmup, reps)
    per = statistics.median(times)
    n = len(rows)
    return {"value": n / w.B / per, "unit": "steps/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} of {w.B} batch rows (all {w.Hq} heads) per oracle step, float64 "
                      f"numpy oracle on one thread, threshold offset set by the oracle on "
                      f"those rows; median of {reps} steps after {warmup} warm-up ({per:.2f} s "
                      f"each), steps/s scaled by {n}/{w.B}"}


def run_reference(args, rank, world, device):
    """The float64 CPU oracle as the reference arm.  Each step is the oracle's step
    over a bounded sample of batch rows (all heads), timed on one host thread; the
    line's value is whole-batch steps/s, scaled from the sample by rows / B, and
    ms_per_step is the measured time of one sampled step (so that steps x ms_per_step
    is the run's timed work).  The threshold bias is set by the oracle itself on the
    sampled rows with the eta arm's density rule; no CUDA kernel of this package
    runs (torch only draws the seeded inputs)."""
    w = with_overrides(workload_by_name(args.workload, args.B), args)
    g = synth.generate(w, device, seed=w.seed)
    rows = list(range(max(1, min(args.cpu_rows, w.B))))
    sample, W, bias, tau_const = oracle_sample_inputs(w, g, rows)
    del g
    times = time_oracle(sample, W, bias, tau_const, args.warmup, args.steps)
    per = sum(times) / len(times)
    v = len(rows) / w.B / per
    dens = sample.union_density(None if W is None else W.double().cpu().numpy(),
                                None if bias is None else bias.double().cpu().numpy(),
                                None if tau_const is None else tau_const.double().numpy())
    return {
        "metric": METRIC, "value": v, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "value_basis": (f"each step runs the oracle on {len(rows)} of {w.B} batch rows; value = "
                        f"whole-batch steps/s = ({len(rows)}/{w.B}) / measured seconds per "
                        f"sampled step; ms_per_step = measured time of one sampled step"),
        "ms_per_full_step_extrapolated": per * 1e3 * w.B / len(rows),
        "config": workload_config(w, args),
        "density": {"union": round(dens, 4), "rows": len(rows)},
        "cpu_baseline": {"value": v, "unit": "steps/s", "cores": 1, "kind": "oracle",
                         "sample": f"{len(rows)} of {w.B} batch rows (all {w.Hq} heads) per "
                                   f"step, float64 numpy oracle on one thread, threshold "
                                   f"offset set by the oracle on those rows, steps/s scaled "
                                   f"by {len(rows)}/{w.B}"},
        "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def run_prefill(args, rank, world, device):
    """Dense gated causal prefill (eta_prefill): tensor-core roofline."""
    from long_context_decoding_eta_b200 import _lib as L
    B, Hq, Hkv, d, T = args.pf_B, 16, 4, 128, args.pf_T
    g = torch.Generator(device=device)
    g.manual_seed(2000 + rank)
    q = torch.randn(B, Hq, T, d, generator=g, device=device).to(torch.bfloat16)
    K = torch.randn(B, Hkv, T, d, generator=g, device=device).to(torch.bfloat16)
    V = torch.randn(B, Hkv, T, d, generator=g, device=device).to(torch.bfloat16)
    # thresholds from the Eq. 1 predictor applied to every token's concatenated heads
    W = torch.randn(Hq * d, Hq, generator=g, device=device) * (0.1 / math.sqrt(d))
    qt = q.permute(0, 2, 1, 3).reshape(B * T, Hq, d).contiguous()
    tdims = L.Dims.of(B * T, Hq, Hkv, d, 64, 128)
    tau_bt = torch.empty(B * T, Hq, device=device)
    L.eta_predict_tau(tdims, qt, W, torch.full((Hq,), 0.5, device=device), None, tau_bt)
    tau = tau_bt.reshape(B, T, Hq).permute(0, 2, 1).contiguous()
    lengths = torch.full((B,), T, dtype=torch.int32, device=device)
    dims = L.Dims.of(B, Hq, Hkv, d, 64, T)
    O = torch.empty(B, Hq, T, d, device=device)
    lse = torch.empty(B, Hq, T, device=device)
    st = torch.zeros(1, dtype=torch.int32, device=device)
    run = lambda: L.eta_prefill(dims, q, tau, K, V, lengths, args.pf_gate_T, 0.0, O, lse, st)
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(device.index or 0) as clk:
        e0.record()
        for _ in range(args.steps):
            run()
        e1.record()
        torch.cuda.synchronize()
    assert int(st.item()) == 0
    ms = e0.elapsed_time(e1) / args.steps
    flops = 4.0 * d * B * Hq * (T * (T + 1) / 2)       # QK^T + PV over causal pairs
    tf = flops / (ms * 1e-3) / 1e12
    pk = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"] \
        if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else 1590.0
    return {"metric": "gated causal prefill TFLOP/s", "value": tf, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": f"prefill-b{B}-h{Hq}x{Hkv}-d{d}-T{T}-causal",
                       "gate_T": args.pf_gate_T},
            "roofline": {"kernel": ("prefill_pp_kernel (two query tiles per CTA)"
                                    if L.eta_prefill_kernel_for(dims, args.pf_gate_T) == "two_tile"
                                    else "prefill_tc_kernel"),
                         "bound": "tensor", "achieved": tf,
                         "peak": pk, "unit": "TFLOP/s", "frac": tf / pk,
                         "peak_kind": "measured cuBLAS bf16 burst"},
            "gpu_launches": args.steps * world, "clocks": clk.summary()}


def main():
    global CLOCK_LOG_DIR
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=synth.EXTREME512K.name,
                    help="workload name or prefix (tiny, mid, long, extreme, calibrated)")
    ap.add_argument("--impl", default="eta", choices=["eta", "reference"])
    ap.add_argument("--mode", default="decode", choices=["decode", "prefill"],
                    help="decode: the ETA decode step (default); prefill: eta_prefill")
    ap.add_argument("--pf-B", type=int, default=4)
    ap.add_argument("--pf-T", type=int, default=8192)
    ap.add_argument("--pf-gate-T", type=float, default=0.0)
    ap.add_argument("--cpu-rows", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--density", type=float, default=0.0,
                    help="override the workload's density target (e.g. 0.38)")
    ap.add_argument("--density-kind", default="", choices=["", "head", "union"],
                    help="override what the density target counts: per head or union")
    ap.add_argument("--tau-mode", default="", choices=["", "predictor", "const"],
                    help="override the threshold mode (the calibrated workload's comparison)")
    ap.add_argument("--clock-log-dir", default="",
                    help="keep the raw clock samples (CSV per rank) in this folder")
    ap.add_argument("--clock-soak-s", type=float, default=1.0,
                    help="untimed steps run under the clock sampler before the timed region")
    ap.add_argument("--B", type=int, default=0, help="override the batch size (profiling)")
    ap.add_argument("--ctx", type=int, default=0,
                    help="override the context length (small profiling captures)")
    ap.add_argument("--bound", default="", choices=["", "exact", "prob", "prob_dim"],
                    help="override the screening bound (the extreme workload's exact arm)")
    ap.add_argument("--engine", default="auto", choices=["auto", "tcgen05", "fma"],
                    help="decode engine of libeta.so")
    ap.add_argument("--separate-prologue", action="store_true",
                    help="tail refresh and tau as two launches (default: one)")
    ap.add_argument("--fused", action="store_true",
                    help="run the step as one eta_decode_step launch (persistent kernel)")
    ap.add_argument("--graph", action="store_true",
                    help="replay the step as CUDA graphs (launch-bound small workloads)")
    ap.add_argument("--cent", default="bf16", choices=["f32", "bf16"],
                    help="storage of the block centroids the screen reads")
    args = ap.parse_args()
    if args.clock_log_dir:
        CLOCK_LOG_DIR = args.clock_log_dir
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference" and rank != 0:
        return 0
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1 and args.impl == "eta":
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=device)
    try:
        if args.impl == "reference":
            res = run_reference(args, rank, 1, device)
        elif args.mode == "prefill":
            res = run_prefill(args, rank, world, device)
        else:
            res = run_eta(args, rank, world, device)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1 and args.impl == "eta":
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
