// Per-KV-block metadata (centroid, max deviation radius, variance, count, V sum).
//
// "Cached centroid/variance/max-norm metadata" (evolve.pub review of arXiv
// 2609.20888, Summary); "cached geometric-probabilistic bounds" (abstract).
// Full build: one warp per block; every lane owns d/32 consecutive dimensions, so
// each key row is one coalesced 128/256-byte warp load.  Blocks live in L2 between
// the two passes over their keys (16-32 KB each).  Tail refresh (the per-token
// append): one CTA per block, keys split over its 8 warps.
#include <type_traits>

#include "eta_common.cuh"
#include "eta_host.h"
#include "meta_dev.cuh"

namespace eta {

template <int D, int CF>
__global__ void __launch_bounds__(kMetaWarps * 32)
meta_build_kernel(int Hkv, int T_max, int blk, int NB, const eta_bf16_t* __restrict__ K,
                  const eta_bf16_t* __restrict__ V, const int32_t* __restrict__ lengths,
                  int blk_begin, int nblk, void* __restrict__ cent,
                  float* __restrict__ rmax, float* __restrict__ var, int32_t* __restrict__ cnt,
                  float* __restrict__ vsum, float* __restrict__ vardim, int32_t* status) {
  ETA_PDL_ENTRY();
  constexpr int DPL = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y;                 // (row, KV head) = b * Hkv + g
  const int b = r / Hkv;
  int len = lengths[b];
  if (len < 0 || len > T_max) {
    if (lane == 0 && warp == 0 && blockIdx.x == 0) set_status(status, ETA_DEVSTAT_BAD_LENGTH);
    len = min(max(len, 0), T_max);
  }
  const int jj = blockIdx.x * kMetaWarps + warp;
  if (jj >= nblk) return;
  const int j = blk_begin + jj;
  const int n = min(max(len - j * blk, 0), blk);
  // the block's metadata slot and the tokens its keys come from
  if (!ETA_IN_BOUNDS(j, NB, status) || !ETA_RANGE_IN_BOUNDS(j * blk, j * blk + n, T_max, status))
    return;
  const size_t rowj = (size_t)r * NB + j;
  const eta_bf16_t* kb = K + ((size_t)r * T_max + (size_t)j * blk) * D + lane * DPL;

  // The keys are summed in kMetaWarps consecutive chunks of ceil(blk / kMetaWarps)
  // keys, each chunk sequentially from zero, and the chunk sums in order: exactly
  // the order of meta_tail_kernel, so a tail refresh and a full rebuild of the same
  // block give bit-identical metadata.
  const int per = (blk + kMetaWarps - 1) / kMetaWarps;
  float c[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) c[i] = 0.f;
  // pass 1: centroid (fp32 sums, or exact fp64 sums for bf16 storage)
  using Acc = typename std::conditional<CF == 1, double, float>::type;
  Acc csum[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) csum[i] = 0;
  for (int w = 0; w < kMetaWarps; ++w) {
    const int lo = min(w * per, n), hi = min(lo + per, n);
    Acc pc[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) pc[i] = 0;
#pragma unroll 4
    for (int t = lo; t < hi; ++t) {
      float x[DPL];
      load_row<DPL>(kb + (size_t)t * D, x);
#pragma unroll
      for (int i = 0; i < DPL; ++i) pc[i] += (Acc)x[i];
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) csum[i] += pc[i];
  }
  if (n > 0) {
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      if constexpr (CF == 1) c[i] = bf16_round_from_double(csum[i] / (double)n);
      else c[i] = csum[i] / (float)n;
    }
  }
  // pass 2: squared distances to the stored fp32 centroid
  float r2max = 0.f, s2 = 0.f;
  float vd[DPL];                // per-dimension squared deviations (ETA_BOUND_PROB_DIM)
#pragma unroll
  for (int i = 0; i < DPL; ++i) vd[i] = 0.f;
  for (int w = 0; w < kMetaWarps; ++w) {
    const int lo = min(w * per, n), hi = min(lo + per, n);
    float ps = 0.f;
    float pv[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) pv[i] = 0.f;
#pragma unroll 4
    for (int t = lo; t < hi; ++t) {
      float x[DPL];
      load_row<DPL>(kb + (size_t)t * D, x);
      float p = 0.f;
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        const float dv = x[i] - c[i];
        p = fmaf(dv, dv, p);
        pv[i] = fmaf(dv, dv, pv[i]);
      }
      p = warp_sum(p);          // butterfly: bit-identical in every lane
      r2max = fmaxf(r2max, p);
      ps += p;
    }
    s2 += ps;
#pragma unroll
    for (int i = 0; i < DPL; ++i) vd[i] += pv[i];
  }
  if (vardim) {
#pragma unroll
    for (int i = 0; i < DPL; ++i)
      vardim[((size_t)r * D + lane * DPL + i) * NB + j] = n > 0 ? vd[i] / (float)n : 0.f;
  }
#pragma unroll
  for (int i = 0; i < DPL; ++i)
    store_centroid<CF>(cent, ((size_t)r * D + lane * DPL + i) * NB + j, c[i]);
  if (lane == 0) {
    rmax[rowj] = n > 0 ? __fmul_ru(__fsqrt_ru(r2max), kRadiusInflate) : 0.f;
    var[rowj] = n > 0 ? s2 / (float)n : 0.f;
    cnt[rowj] = n;
  }
  if (vsum) {
    const eta_bf16_t* vb = V + ((size_t)r * T_max + (size_t)j * blk) * D + lane * DPL;
    float a[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) a[i] = 0.f;
    for (int w = 0; w < kMetaWarps; ++w) {
      const int lo = min(w * per, n), hi = min(lo + per, n);
      float pa[DPL];
#pragma unroll
      for (int i = 0; i < DPL; ++i) pa[i] = 0.f;
#pragma unroll 4
      for (int t = lo; t < hi; ++t) {
        float x[DPL];
        load_row<DPL>(vb + (size_t)t * D, x);
#pragma unroll
        for (int i = 0; i < DPL; ++i) pa[i] += x[i];
      }
#pragma unroll
      for (int i = 0; i < DPL; ++i) a[i] += pa[i];
    }
    float* vr = vsum + rowj * D + lane * DPL;
#pragma unroll
    for (int i = 0; i < DPL; ++i) vr[i] = a[i];
  }
}

// Tail-block refresh: one CTA of kMetaWarps warps per (row, KV head), so the
// latency chain is blk / kMetaWarps keys instead of blk (arithmetic in
// meta_tail_block).
template <int D, int CF>
__global__ void __launch_bounds__(kMetaWarps * 32)
meta_tail_kernel(int Hkv, int T_max, int blk, int NB, const eta_bf16_t* __restrict__ K,
                 const eta_bf16_t* __restrict__ V, const int32_t* __restrict__ lengths,
                 void* __restrict__ cent, float* __restrict__ rmax, float* __restrict__ var,
                 int32_t* __restrict__ cnt, float* __restrict__ vsum, float* __restrict__ vardim) {
  ETA_PDL_ENTRY();
  __shared__ TailScratch<D, CF> sc;
  meta_tail_block<D, CF, kMetaWarps>(blockIdx.x, Hkv, T_max, blk, NB, K, V, lengths, cent, rmax,
                                     var, cnt, vsum, vardim, nullptr, sc, threadIdx.x >> 5,
                                     [] { __syncthreads(); });
}

template <int D, int CF>
static eta_status_t launch_meta(bool tail, const eta_dims_t* dims, int NB, int R, int blk_begin,
                                int nblk, const eta_bf16_t* K, const eta_bf16_t* V,
                                const int32_t* lengths, void* cent, float* rmax, float* var,
                                int32_t* cnt, float* vsum, float* vardim, cudaStream_t s) {
  if (tail)
    return launch_k(meta_tail_kernel<D, CF>, dim3(R), dim3(kMetaWarps * 32), 0, s, dims->Hkv,
                    dims->T_max, dims->blk, NB, K, V, lengths, cent, rmax, var, cnt, vsum,
                    vardim);
  dim3 grid((nblk + kMetaWarps - 1) / kMetaWarps, R);
  return launch_k(meta_build_kernel<D, CF>, grid, dim3(kMetaWarps * 32), 0, s, dims->Hkv,
                  dims->T_max, dims->blk, NB, K, V, lengths, blk_begin, nblk, cent, rmax, var,
                  cnt, vsum, vardim, (int32_t*)nullptr);
}

}  // namespace eta

using namespace eta;

extern "C" eta_status_t eta_build_block_meta(const eta_dims_t* dims, const eta_bf16_t* K,
                                             const eta_bf16_t* V, const int32_t* lengths,
                                             int32_t blk_begin, int32_t blk_end,
                                             eta_cent_format_t cent_format, void* cent,
                                             float* rmax, float* var, int32_t* cnt, float* vsum,
                                             float* vardim, void* stream) {
  eta_status_t st = check_dims(dims);
  if (st != ETA_OK) return st;
  if (!K || !lengths || !cent || !rmax || !var || !cnt) return ETA_ERR_INVALID_ARG;
  if (cent_format != ETA_CENT_F32 && cent_format != ETA_CENT_BF16) return ETA_ERR_INVALID_ARG;
  if (vsum && !V) return ETA_ERR_INVALID_ARG;
  if (!aligned16(K) || (V && !aligned16(V))) return ETA_ERR_INVALID_ARG;
  const int NB = num_blocks(dims);
  const int R = dims->B * dims->Hkv;
  const bool tail = blk_begin == ETA_TAIL_BLOCK;
  int nblk = 0;
  if (!tail) {
    if (blk_end < 0) blk_end = NB;
    if (blk_begin < 0 || blk_begin > blk_end || blk_end > NB) return ETA_ERR_INVALID_ARG;
    nblk = blk_end - blk_begin;
    if (nblk == 0) return ETA_OK;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bf = cent_format == ETA_CENT_BF16;
  if (dims->d == 128)
    return bf ? launch_meta<128, 1>(tail, dims, NB, R, blk_begin, nblk, K, V, lengths, cent, rmax,
                                   var, cnt, vsum, vardim, s)
              : launch_meta<128, 0>(tail, dims, NB, R, blk_begin, nblk, K, V, lengths, cent, rmax,
                                   var, cnt, vsum, vardim, s);
  return bf ? launch_meta<64, 1>(tail, dims, NB, R, blk_begin, nblk, K, V, lengths, cent, rmax,
                                var, cnt, vsum, vardim, s)
            : launch_meta<64, 0>(tail, dims, NB, R, blk_begin, nblk, K, V, lengths, cent, rmax,
                                var, cnt, vsum, vardim, s);
}
