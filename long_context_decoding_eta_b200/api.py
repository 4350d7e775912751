"""User-facing decode object over the C ABI.

`EtaDecoder` owns (through torch, which is only the allocator here) the block
metadata, the screening outputs and the workspaces for one bf16 KV cache, and
runs one ETA decode step as four C-ABI calls on the current CUDA stream:

    eta_build_block_meta(tail block)   the cache grew by one token
    eta_predict_tau                    Eq. 1 predictor, or frozen constants
    eta_screen                         O(1) block screening, union compaction
    eta_decode                         gated split-KV attention + LSE combine

With fused=True the same step is one call, eta_decode_step (one persistent
kernel), writing the same outputs bit for bit.

Every arithmetic step runs in libeta.so's kernels; this module only allocates
and marshals arguments.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import _lib as L


class EtaDecoder:
    def __init__(self, K: torch.Tensor, V: torch.Tensor, lengths: torch.Tensor, Hq: int,
                 blk: int, *, bound: str = "exact", z: float = 3.0, T: float = 0.0,
                 scale: float = 0.0, prune: str = "skip", keep_bounds: bool = False,
                 cent_format: str = "f32", fused: bool = False,
                 merged_prologue: bool = True):
        if not K.is_cuda:
            raise ValueError("K/V must be CUDA tensors")
        if K.dtype != torch.bfloat16 or V.dtype != torch.bfloat16:
            raise ValueError("K/V must be bf16")
        B, Hkv, T_max, d = K.shape
        self.K, self.V = K, V
        self.lengths = lengths.to(device=K.device, dtype=torch.int32).contiguous()
        self.dims = L.Dims.of(B, Hq, Hkv, d, blk, T_max)
        self.B, self.Hq, self.Hkv, self.d, self.blk, self.T_max = B, Hq, Hkv, d, blk, T_max
        self.NB = T_max // blk
        self.NW = (self.NB + 31) // 32
        self.bound, self.z, self.T, self.prune = bound, float(z), float(T), prune
        self.scale = float(scale) if scale else 1.0 / math.sqrt(d)
        dev = K.device
        f32, i32 = torch.float32, torch.int32
        if cent_format not in ("f32", "bf16"):
            raise ValueError(cent_format)
        self.cent = torch.zeros(B, Hkv, d, self.NB, device=dev,
                                dtype=torch.bfloat16 if cent_format == "bf16" else f32)
        self.rmax = torch.zeros(B, Hkv, self.NB, dtype=f32, device=dev)
        self.var = torch.zeros(B, Hkv, self.NB, dtype=f32, device=dev)
        self.cnt = torch.zeros(B, Hkv, self.NB, dtype=i32, device=dev)
        self.vsum = (torch.zeros(B, Hkv, self.NB, d, dtype=f32, device=dev)
                     if prune == "floor" else None)
        self.vardim = (torch.zeros(B, Hkv, d, self.NB, dtype=f32, device=dev)
                       if bound == "prob_dim" else None)
        self.tau = torch.zeros(B, Hq, dtype=f32, device=dev)
        self.head_mask = torch.zeros(B, Hq, self.NW, dtype=torch.int32, device=dev)
        self.union_idx = torch.zeros(B, Hkv, self.NB, dtype=i32, device=dev)
        self.union_cnt = torch.zeros(B, Hkv, dtype=i32, device=dev)
        self.head_cnt = torch.zeros(B, Hq, dtype=i32, device=dev)
        self.bounds = (torch.zeros(B, Hq, self.NB, dtype=f32, device=dev)
                       if keep_bounds else None)
        self.o = torch.zeros(B, Hq, d, dtype=f32, device=dev)
        self.lse = torch.zeros(B, Hq, dtype=f32, device=dev)
        self.ws_screen = torch.empty(max(L.eta_screen_workspace_size(self.dims), 256),
                                     dtype=torch.uint8, device=dev)
        self.ws_decode = torch.empty(max(L.eta_decode_workspace_size(self.dims), 256),
                                     dtype=torch.uint8, device=dev)
        self.dev_status = torch.zeros(1, dtype=i32, device=dev)
        self.fused = bool(fused)
        self.merged_prologue = bool(merged_prologue)
        if self.fused and prune != "skip":
            raise ValueError("the fused step offers SKIP pruning only")
        # the fused step's workspace holds self-resetting counters: zero it once
        self.ws_step = (torch.zeros(max(L.eta_decode_step_workspace_size(self.dims), 256),
                                    dtype=torch.uint8, device=dev) if self.fused else None)

    # -- metadata -------------------------------------------------------------
    def build_meta(self, blk_begin: int = 0, blk_end: int = -1, stream=None):
        L.eta_build_block_meta(self.dims, self.K, self.V, self.lengths, blk_begin, blk_end,
                               self.cent, self.rmax, self.var, self.cnt, self.vsum, stream,
                               self.vardim)

    def append_update(self, stream=None):
        """Recompute the tail block of every row (call after appending a token)."""
        self.build_meta(L.TAIL_BLOCK, -1, stream)

    # -- step parts -----------------------------------------------------------
    def predict_tau(self, q, W=None, bias=None, tau_const=None, stream=None):
        L.eta_predict_tau(self.dims, q, W, bias, tau_const, self.tau, self.dev_status, stream)
        return self.tau

    def screen(self, q, tau=None, stream=None, bounds: Optional[torch.Tensor] = None):
        tau = self.tau if tau is None else tau
        L.eta_screen(self.dims, q, tau, self.cent, self.rmax, self.var, self.cnt, self.bound,
                     self.z, self.scale, self.head_mask, self.union_idx, self.union_cnt,
                     self.bounds if bounds is None else bounds, self.head_cnt, self.ws_screen,
                     self.dev_status, stream, self.vardim)

    def decode(self, q, tau=None, stream=None):
        tau = self.tau if tau is None else tau
        L.eta_decode(self.dims, q, tau, self.K, self.V, self.lengths, self.union_idx,
                     self.union_cnt, self.T, self.scale, self.prune, self.vsum, self.cnt,
                     self.o, self.lse, self.ws_decode, self.dev_status, stream)
        return self.o, self.lse

    def dense_decode(self, q, stream=None):
        L.eta_dense_decode(self.dims, q, self.K, self.V, self.lengths, self.scale, self.o,
                           self.lse, self.ws_decode, self.dev_status, stream)
        return self.o, self.lse

    def step_fused(self, q, W=None, bias=None, tau_const=None, stream=None,
                   append: bool = True):
        """The same step as one eta_decode_step launch."""
        L.eta_decode_step(self.dims, q, W, bias, tau_const, self.K, self.V, self.lengths,
                          append, self.cent, self.rmax, self.var, self.vardim, self.cnt,
                          self.bound, self.z, self.T, self.scale, self.tau, self.head_mask,
                          self.union_idx, self.union_cnt, self.head_cnt, self.o, self.lse,
                          self.ws_step, self.dev_status, stream)
        return self.o, self.lse

    def prepare(self, q, W=None, bias=None, tau_const=None, stream=None,
                append: bool = True):
        """Everything of the step before the decode: the tail-block metadata (on
        append) and the thresholds (one launch, eta_append_and_predict_tau, unless
        merged_prologue is off), then the screening."""
        if append and self.merged_prologue:
            L.eta_append_and_predict_tau(self.dims, self.K, self.V, self.lengths, self.cent,
                                         self.rmax, self.var, self.cnt, self.vsum, self.vardim,
                                         q, W, bias, tau_const, self.tau, self.dev_status,
                                         stream)
        else:
            if append:
                self.append_update(stream)
            self.predict_tau(q, W, bias, tau_const, stream)
        self.screen(q, stream=stream)

    def step(self, q, W=None, bias=None, tau_const=None, stream=None, append: bool = True):
        """One decode step: tail-block metadata, tau, screening, gated decode."""
        if self.fused:
            return self.step_fused(q, W, bias, tau_const, stream, append)
        self.prepare(q, W, bias, tau_const, stream, append)
        return self.decode(q, stream=stream)

    # -- CUDA graphs ----------------------------------------------------------
    def capture(self, q: torch.Tensor, W=None, bias=None, tau_const=None, split: bool = False):
        """Captures the step into CUDA graph(s) bound to the tensors given (write new
        queries into `q` in place, then call `replay()`).  split=True captures the
        decode call as a second graph so that it can be timed on its own.  Launch
        overhead then no longer bounds small workloads."""
        stream = torch.cuda.Stream()
        stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(stream):
            for _ in range(2):                       # warm the launch paths
                self.step(q, W, bias, tau_const)
            torch.cuda.synchronize()
            g_pre = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_pre, stream=stream):
                if self.fused:
                    self.step_fused(q, W, bias, tau_const)
                    split = False
                else:
                    self.prepare(q, W, bias, tau_const)
                    if not split:
                        self.decode(q)
            g_dec = None
            if split:
                g_dec = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g_dec, stream=stream):
                    self.decode(q)
        torch.cuda.current_stream().wait_stream(stream)
        self._graphs = (g_pre, g_dec)
        return self._graphs

    def replay(self):
        g_pre, g_dec = self._graphs
        g_pre.replay()
        if g_dec is not None:
            g_dec.replay()
        return self.o, self.lse

    # -- status ---------------------------------------------------------------
    def check_status(self):
        """Synchronizes, reads the device status word, raises on any error bit."""
        word = int(self.dev_status.item())
        if word:
            code = L.eta_status_from_device(word)
            self.dev_status.zero_()
            raise L.EtaError(f"device status 0x{word:x}", code)

    def calibrate_const_tau(self, q_calib: torch.Tensor, density: float,
                            rows: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Offline calibration of frozen per-head thresholds.

        q_calib: bf16 [n_q, Hq, d] calibration queries; query i is screened
        against batch row rows[i] (default i mod B).  Returns tau fp32 [Hq] (CPU).
        Uses eta_screen's bound output and the library's host quantile rule.
        """
        n_q = q_calib.shape[0]
        rows = (torch.arange(n_q) % self.B) if rows is None else rows
        bounds = torch.empty(n_q, self.Hq, self.NB, dtype=torch.float32)
        valid = torch.empty(n_q, self.Hq, self.NB, dtype=torch.bool)
        dev = self.K.device
        tmp_b = torch.empty(self.B, self.Hq, self.NB, dtype=torch.float32, device=dev)
        inf_tau = torch.full((self.B, self.Hq), float("inf"), device=dev)
        cnt_valid = (self.cnt > 0).repeat_interleave(self.Hq // self.Hkv, dim=1).cpu()
        for start in range(0, n_q, self.B):
            idx = list(range(start, min(n_q, start + self.B)))
            qb = torch.zeros(self.B, self.Hq, self.d, dtype=torch.bfloat16, device=dev)
            for i in idx:
                qb[int(rows[i])] = q_calib[i].to(dev)
            self.screen(qb, inf_tau, bounds=tmp_b)
            hb = tmp_b.cpu()
            for i in idx:
                bounds[i] = hb[int(rows[i])]
                valid[i] = cnt_valid[int(rows[i])]
        return L.eta_calibrate_const_tau(bounds, valid, density)
