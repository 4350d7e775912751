// Threshold predictor arithmetic shared by predict_tau_group_kernel and the fused
// decode step: Eq. 1 of the evolve.pub review of arXiv 2609.20888 (Methodology
// Assessment), tau = qbar W_tau + b_tau, for the G heads of one KV group.
//
// The reduction order is fixed: 256 virtual threads, virtual thread v owning the
// elements v, v + 256, ... of qbar (one fmaf chain each), a butterfly sum over each
// virtual warp, then the 8 warp sums added in warp order.  NWARP real warps run the
// 8 virtual warps in turns, so every caller gets bit-identical thresholds.
#pragma once

#include "eta_common.cuh"

namespace eta {

constexpr int kTauVirtThreads = 256;
constexpr int kTauVirtWarps = kTauVirtThreads / 32;

// red: shared [kTauVirtWarps][G].  Writes tau[(size_t)b * Hq + h0 + k] for k < G.
// Called by NWARP warps (local warp index wid, local thread index wid * 32 + lane)
// that `sync` synchronizes; ends synchronized.  Returns whether this thread saw a
// non-finite query element.
template <int G, int NWARP, typename Sync>
ETA_DEV bool tau_group(int Hq, int D, int b, int h0, const eta_bf16_t* __restrict__ q,
                       const float* __restrict__ W, const float* __restrict__ bias,
                       float (*red)[G], float* __restrict__ tau, int wid, Sync sync) {
  const int warp = wid, lane = threadIdx.x & 31;
  const int ltid = wid * 32 + lane;
  const int n = Hq * D;
  const eta_bf16_t* qb = q + (size_t)b * n;
  bool bad = false;
  for (int vw = warp; vw < kTauVirtWarps; vw += NWARP) {
    const int vt = vw * 32 + lane;
    float acc[G];
#pragma unroll
    for (int k = 0; k < G; ++k) acc[k] = 0.f;
#pragma unroll 8
    for (int i = vt; i < n; i += kTauVirtThreads) {
      const float x = bf16_to_f(qb[i]);
      bad |= !isfinite(x);
      const float* wr = W + (size_t)i * Hq + h0;
#pragma unroll
      for (int k = 0; k < G; ++k) acc[k] = fmaf(x, __ldg(wr + k), acc[k]);
    }
#pragma unroll
    for (int k = 0; k < G; ++k) {
      const float v = warp_sum(acc[k]);
      if (lane == 0) red[vw][k] = v;
    }
  }
  sync();
  if (ltid < G) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kTauVirtWarps; ++w) s += red[w][ltid];
    const int h = h0 + ltid;
    tau[(size_t)b * Hq + h] = s + (bias ? bias[h] : 0.f);
  }
  sync();
  return bad;
}

}  // namespace eta
