// Per-KV-block metadata arithmetic shared by the metadata kernels and the fused
// decode step ("cached centroid/variance/max-norm metadata", evolve.pub review of
// arXiv 2609.20888, Summary).
#pragma once

#include <type_traits>

#include "eta_common.cuh"

namespace eta {

// 1 + 2^-20: covers the relative rounding error of the fp32 distance
// computation below (<= ~6 ulp on the sqrt), so rmax never under-states the
// true maximum distance to the stored fp32 centroid.
constexpr float kRadiusInflate = 1.00000095367431640625f;
constexpr int kMetaWarps = 8;

template <int DPL>
ETA_DEV void load_row(const eta_bf16_t* p, float (&x)[DPL]) {
  if constexpr (DPL == 4) {
    uint2 w = *reinterpret_cast<const uint2*>(p);
    x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  } else {
    uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    x[0] = bf16_lo(w); x[1] = bf16_hi(w);
  }
}

// Centroid storage: CF = 0 fp32, CF = 1 bf16.  With bf16 the key sum is accumulated
// in fp64 (exact for up to 128 bf16 keys of ordinary range), divided in fp64 and
// rounded once to bf16 (nearest even), so the stored centroid is the correctly
// rounded mean; rmax and var are then measured against that stored centroid and the
// bound stays exact for what the screen reads.
ETA_DEV float bf16_round_from_double(double m) {
  return __bfloat162float(__double2bfloat16(m));
}

template <int CF>
ETA_DEV void store_centroid(void* cent, size_t idx, float c) {
  if constexpr (CF == 1)
    reinterpret_cast<uint16_t*>(cent)[idx] = __bfloat16_as_ushort(__float2bfloat16_rn(c));
  else
    reinterpret_cast<float*>(cent)[idx] = c;
}

// Tail-block refresh of one (row, KV head) r after a token was appended: the same
// arithmetic as meta_build_kernel (sequential sums over the keys in token order,
// one division, butterfly distance sums), with the block's keys split into
// kMetaWarps chunks ("virtual warps") whose partial sums are combined in chunk
// order, the order meta_build_kernel uses, so a tail refresh and a full rebuild of
// the same block give bit-identical metadata.  NWARP real warps (local index wid)
// run the chunks in turns; `sync` synchronizes them; returns synchronized.  status:
// the checked build's range reports (may be NULL).
template <int D, int CF>
struct TailScratch {
  using Acc = typename std::conditional<CF == 1, double, float>::type;
  Acc cpart[kMetaWarps][D];
  float vpart[kMetaWarps][D];
  float vspart[kMetaWarps][D];
  float red_max[kMetaWarps], red_sum[kMetaWarps];
};

template <int D, int CF, int NWARP, typename Sync>
ETA_DEV void meta_tail_block(int r, int Hkv, int T_max, int blk, int NB,
                             const eta_bf16_t* __restrict__ K, const eta_bf16_t* __restrict__ V,
                             const int32_t* __restrict__ lengths, void* __restrict__ cent,
                             float* __restrict__ rmax, float* __restrict__ var,
                             int32_t* __restrict__ cnt, float* __restrict__ vsum,
                             float* __restrict__ vardim, int32_t* status,
                             TailScratch<D, CF>& sc, int wid, Sync sync) {
  constexpr int DPL = D / 32;
  using Acc = typename TailScratch<D, CF>::Acc;
  const int warp = wid, lane = threadIdx.x & 31;
  const int b = r / Hkv;
  const int len = min(max(lengths[b], 0), T_max);
  if (len == 0) return;                      // uniform over the callers
  const int j = (len - 1) / blk;
  const int n = min(len - j * blk, blk);
  // (checked build) the tail block's slot and tokens; uniform over the callers
  if (!ETA_IN_BOUNDS(j, NB, status) || !ETA_RANGE_IN_BOUNDS(j * blk, j * blk + n, T_max, status))
    return;
  const int per = (blk + kMetaWarps - 1) / kMetaWarps;
  const size_t rowj = (size_t)r * NB + j;
  const eta_bf16_t* kb = K + ((size_t)r * T_max + (size_t)j * blk) * D + lane * DPL;

  // pass 1: centroid (fp32 sums, or exact fp64 sums for bf16 storage)
  for (int vw = warp; vw < kMetaWarps; vw += NWARP) {
    const int t_lo = min(vw * per, n), t_hi = min(t_lo + per, n);
    Acc pc[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) pc[i] = 0;
#pragma unroll 8
    for (int t = t_lo; t < t_hi; ++t) {
      float x[DPL];
      load_row<DPL>(kb + (size_t)t * D, x);
#pragma unroll
      for (int i = 0; i < DPL; ++i) pc[i] += (Acc)x[i];
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) sc.cpart[vw][lane * DPL + i] = pc[i];
  }
  sync();
  float c[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    Acc sum = 0;
#pragma unroll
    for (int w = 0; w < kMetaWarps; ++w) sum += sc.cpart[w][lane * DPL + i];
    if constexpr (CF == 1) c[i] = bf16_round_from_double(sum / (double)n);
    else c[i] = sum / (float)n;
  }
  // pass 2: squared distances to the stored centroid
  for (int vw = warp; vw < kMetaWarps; vw += NWARP) {
    const int t_lo = min(vw * per, n), t_hi = min(t_lo + per, n);
    float r2max = 0.f, s2 = 0.f;
    float pv[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) pv[i] = 0.f;
#pragma unroll 8
    for (int t = t_lo; t < t_hi; ++t) {
      float x[DPL];
      load_row<DPL>(kb + (size_t)t * D, x);
      float pd = 0.f;
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        const float dv = x[i] - c[i];
        pd = fmaf(dv, dv, pd);
        pv[i] = fmaf(dv, dv, pv[i]);
      }
      pd = warp_sum(pd);
      r2max = fmaxf(r2max, pd);
      s2 += pd;
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) sc.vpart[vw][lane * DPL + i] = pv[i];
    if (lane == 0) {
      sc.red_max[vw] = r2max;
      sc.red_sum[vw] = s2;
    }
  }
  if (warp == 0) {
#pragma unroll
    for (int i = 0; i < DPL; ++i)
      store_centroid<CF>(cent, ((size_t)r * D + lane * DPL + i) * NB + j, c[i]);
  }
  sync();
  if (vardim && warp == 0) {
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kMetaWarps; ++w) sum += sc.vpart[w][lane * DPL + i];
      vardim[((size_t)r * D + lane * DPL + i) * NB + j] = sum / (float)n;
    }
  }
  if (warp == 0 && lane == 0) {
    float m = 0.f, sum = 0.f;
#pragma unroll
    for (int w = 0; w < kMetaWarps; ++w) {
      m = fmaxf(m, sc.red_max[w]);
      sum += sc.red_sum[w];
    }
    rmax[rowj] = __fmul_ru(__fsqrt_ru(m), kRadiusInflate);
    var[rowj] = sum / (float)n;
    cnt[rowj] = n;
  }
  if (vsum) {
    const eta_bf16_t* vb = V + ((size_t)r * T_max + (size_t)j * blk) * D + lane * DPL;
    for (int vw = warp; vw < kMetaWarps; vw += NWARP) {
      const int t_lo = min(vw * per, n), t_hi = min(t_lo + per, n);
      float a[DPL];
#pragma unroll
      for (int i = 0; i < DPL; ++i) a[i] = 0.f;
      for (int t = t_lo; t < t_hi; ++t) {
        float x[DPL];
        load_row<DPL>(vb + (size_t)t * D, x);
#pragma unroll
        for (int i = 0; i < DPL; ++i) a[i] += x[i];
      }
#pragma unroll
      for (int i = 0; i < DPL; ++i) sc.vspart[vw][lane * DPL + i] = a[i];
    }
    sync();
    if (warp == 0) {
      float* vr = vsum + rowj * D + lane * DPL;
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kMetaWarps; ++w) s += sc.vspart[w][lane * DPL + i];
        vr[i] = s;
      }
    }
  }
  sync();
}

}  // namespace eta
