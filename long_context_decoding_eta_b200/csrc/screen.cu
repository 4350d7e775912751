// O(1)-per-block screening with hard pruning and co-admission across the query
// heads of a KV group (arXiv 2609.20888 abstract: KV blocks screened "in O(1) time
// using cached geometric-probabilistic bounds", incidental tokens "co-admitted by
// coarse GPU block selection"; evolve.pub review FAQ: blocks whose best possible
// score falls below the threshold are skipped entirely).
//
// screen_vec_kernel (the default when NB % 4 == 0 and the metadata is 16-byte
//   aligned): a warp screens 128 consecutive blocks, lane = 4 blocks, through
//   screen_group_from (screen_dev.cuh), the arithmetic the fused step shares.
// screen_kernel (otherwise): lane = block.  Centroids are stored dimension-major per
//   (row, KV head), so each of the d loads of a warp is one 128-byte line covering 32
//   consecutive blocks; the G query heads of the group sit in shared memory as
//   [d][G] fp32 and are read as broadcasts.  One ballot per head gives the
//   head's 32-bit admit word directly; the union word is their OR.
// compact_kernel: one CTA per (row, KV head) turns union words into the ascending
//   list of admitted block indices (popcount prefix over words, lane = bit).
// screen_row_kernel (small batches): screening from TMA-staged group tiles and the
//   compaction of its row in one launch.
#include <atomic>
#include <type_traits>

#include "eta_common.cuh"
#include "eta_host.h"
#include "compact_dev.cuh"
#include "decode_tc.cuh"   // tc::tma_load_2d
#include "screen_dev.cuh"
#include "screen_tc.cuh"
#include "tma_host.h"

namespace eta {

constexpr int kScreenWarps = 8;
constexpr int kCompactThreads = 256;

template <int CF>
ETA_DEV float load_cent(const void* cent, size_t i) {
  if constexpr (CF == 1) return bf16_to_f(__ldg(reinterpret_cast<const uint16_t*>(cent) + i));
  else return __ldg(reinterpret_cast<const float*>(cent) + i);
}

template <int D, int G, int CF, bool VD>
__global__ void __launch_bounds__(kScreenWarps * 32)
screen_kernel(int Hq, int Hkv, int NB, int NW, const eta_bf16_t* __restrict__ q,
              const float* __restrict__ tau, const void* __restrict__ cent,
              const float* __restrict__ rmax, const float* __restrict__ var,
              const float* __restrict__ vardim,
              const int32_t* __restrict__ cnt, int bound, float z, float scale,
              uint32_t* __restrict__ head_mask, uint32_t* __restrict__ union_words,
              float* __restrict__ bounds_out) {
  ETA_PDL_ENTRY();
  __shared__ __align__(16) float qs[D * G];
  __shared__ float qn[G], ts[G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y, b = r / Hkv, g = r % Hkv;
  const size_t qhead0 = (size_t)b * Hq + (size_t)g * G;

  for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int h = i / D, k = i % D;
    qs[k * G + h] = bf16_to_f(q[(qhead0 + h) * D + k]);
  }
  __syncthreads();
  if (warp < G) {
    float s = 0.f;
    for (int k = lane; k < D; k += 32) s = fmaf(qs[k * G + warp], qs[k * G + warp], s);
    s = warp_sum(s);
    if (lane == 0) {
      qn[warp] = sqrtf(s);
      ts[warp] = tau[qhead0 + warp];
    }
  }
  __syncthreads();

  const int w = blockIdx.x * kScreenWarps + warp;
  if (w >= NW) return;
  const int j = w * 32 + lane;
  const bool vj = j < NB;
  const size_t c0 = (size_t)r * D * NB + (vj ? j : 0);
  float acc[G], acc2[G];
#pragma unroll
  for (int h = 0; h < G; ++h) { acc[h] = 0.f; acc2[h] = 0.f; }
#pragma unroll 16
  for (int k = 0; k < D; ++k) {
    const float c = vj ? load_cent<CF>(cent, c0 + (size_t)k * NB) : 0.f;
    float vdk = 0.f;
    if constexpr (VD) vdk = vj ? __ldg(vardim + c0 + (size_t)k * NB) : 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      acc[h] = fmaf(qs[k * G + h], c, acc[h]);
      if constexpr (VD) acc2[h] = fmaf(qs[k * G + h] * qs[k * G + h], vdk, acc2[h]);
    }
  }
  const size_t rj = (size_t)r * NB + j;
  float rad = vj ? __ldg(rmax + rj) : 0.f;
  if (bound == ETA_BOUND_PROB && vj) rad = fminf(rad, z * sqrtf(__ldg(var + rj) / (float)D));
  const int n = vj ? __ldg(cnt + rj) : 0;
  uint32_t uni = 0;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float ub;
    if constexpr (VD) ub = scale * (acc[h] + fminf(qn[h] * rad, z * sqrtf(acc2[h])));
    else ub = scale * fmaf(qn[h], rad, acc[h]);
    if (bounds_out && vj) bounds_out[(qhead0 + h) * NB + j] = ub;
    const bool adm = vj && n > 0 && ub >= ts[h];
    const uint32_t m = __ballot_sync(0xffffffffu, adm);
    uni |= m;
    if (lane == 0) head_mask[(qhead0 + h) * NW + w] = m;
  }
  if (lane == 0) union_words[(size_t)r * NW + w] = uni;
}

constexpr int kScreenVecWarps = 4;

template <int D, int G, int CF, bool VD>
__global__ void __launch_bounds__(kScreenVecWarps * 32)
screen_vec_kernel(int Hq, int Hkv, int NB, int NW, const eta_bf16_t* __restrict__ q,
                  const float* __restrict__ tau, const void* __restrict__ cent,
                  const float* __restrict__ rmax, const float* __restrict__ var,
                  const float* __restrict__ vardim,
                  const int32_t* __restrict__ cnt, int bound, float z, float scale,
                  uint32_t* __restrict__ head_mask, uint32_t* __restrict__ union_words,
                  float* __restrict__ bounds_out) {
  ETA_PDL_ENTRY();
  __shared__ __align__(16) float qs[D * G];
  __shared__ float qn[G], ts[G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y, b = r / Hkv, g = r % Hkv;
  const size_t qhead0 = (size_t)b * Hq + (size_t)g * G;

  for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int h = i / D, k = i % D;
    qs[k * G + h] = bf16_to_f(q[(qhead0 + h) * D + k]);
  }
  __syncthreads();
  for (int h = warp; h < G; h += kScreenVecWarps) {
    const float s = query_norm<D, G>(qs, h);
    if (lane == 0) {
      qn[h] = s;
      ts[h] = tau[qhead0 + h];
    }
  }
  __syncthreads();

  const int grp = blockIdx.x * kScreenVecWarps + warp;
  if (grp * kScreenGroupBlocks >= NB) return;
  screen_group<D, G, CF, VD, kScreenLoadBatch, false>(
      NB, NW, grp, r, qhead0, qs, qn, ts, cent, rmax, var, vardim, cnt, bound, z, scale, NB,
      head_mask, union_words, bounds_out);
}

__global__ void __launch_bounds__(kCompactThreads)
compact_kernel(int Hq, int Hkv, int G, int NB, int NW, const uint32_t* __restrict__ union_words,
               const uint32_t* __restrict__ head_mask, int32_t* __restrict__ union_idx,
               int32_t* __restrict__ union_cnt, int32_t* __restrict__ head_cnt,
               int32_t* status) {
  ETA_PDL_ENTRY();
  __shared__ CompactScratch<kCompactThreads> cs;
  compact_row<kCompactThreads>(blockIdx.x, Hq, Hkv, G, NB, NW, union_words, head_mask, union_idx,
                               union_cnt, head_cnt, cs, status, [] { __syncthreads(); });
}

// Small batches: one CTA per (row, KV head) pair screens the whole row and compacts
// it in the same launch.  Each warp owns one shared-memory buffer and screens the
// groups warp, warp + NBUF, ...; a group's [D][128] dimension-major centroid tile
// arrives by one TMA tensor copy and its rmax / var / cnt slices by 1-D bulk copies,
// so a group costs one memory round trip instead of D / kScreenLoadBatch dependent
// ones.  The arithmetic is screen_group_from's, as in screen_vec_kernel and the
// fused step: the masks and bounds are bit-identical to theirs.
template <int D, int CF>
struct RowScreenCfg {
  static constexpr int CENT = D * kScreenGroupBlocks * (CF == 1 ? 2 : 4);
  static constexpr int OFF_RMAX = CENT;
  static constexpr int OFF_VAR = CENT + 4 * kScreenGroupBlocks;
  static constexpr int OFF_CNT = CENT + 8 * kScreenGroupBlocks;
  static constexpr int SB = (CENT + 12 * kScreenGroupBlocks + 1023) / 1024 * 1024;
  static constexpr int NBUF_FIT = (192 * 1024) / SB;
  static constexpr int NBUF = NBUF_FIT > 8 ? 8 : NBUF_FIT;   // = warps per CTA
  static constexpr int NT = NBUF * 32;
  static constexpr int SMEM = NBUF * SB + 1024;               // + alignment slack
  static_assert(NBUF >= 2, "two group buffers must fit");
};
// At most this many rounds of NBUF groups per row take the one-launch path.
constexpr int kRowScreenMaxRounds = 2;

template <int D, int G, int CF, bool VD>
__global__ void __launch_bounds__(RowScreenCfg<D, CF>::NT, 1)
screen_row_kernel(const __grid_constant__ CUtensorMap tmC, int Hq, int Hkv, int NB, int NW,
                  const eta_bf16_t* __restrict__ q, const float* __restrict__ tau,
                  const float* __restrict__ rmax, const float* __restrict__ var,
                  const float* __restrict__ vardim, const int32_t* __restrict__ cnt, int bound,
                  float z, float scale, uint32_t* head_mask, uint32_t* union_words,
                  float* __restrict__ bounds_out, int32_t* __restrict__ union_idx,
                  int32_t* __restrict__ union_cnt, int32_t* __restrict__ head_cnt,
                  int32_t* status) {
  using C = RowScreenCfg<D, CF>;
  ETA_PDL_ENTRY();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(16) float qs[D * G];
  __shared__ float qn[G], ts[G];
  __shared__ __align__(8) uint64_t full[C::NBUF];
  __shared__ CompactScratch<C::NT> cs;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x, b = r / Hkv, g = r % Hkv;
  const size_t qhead0 = (size_t)b * Hq + (size_t)g * G;
  const int ngrp = (NB + kScreenGroupBlocks - 1) / kScreenGroupBlocks;
  const bool pv = bound == ETA_BOUND_PROB;

  auto issue = [&](int buf, int grp) {
    unsigned char* st = smem + buf * C::SB;
    const int j0 = grp * kScreenGroupBlocks;
    const uint32_t nb4 = (uint32_t)min(kScreenGroupBlocks, NB - j0) * 4u;
    // (checked build) a group starts inside the row; a skipped copy ends in a timeout
    if (!ETA_RANGE_IN_BOUNDS(j0, j0 + (int)(nb4 / 4u), NB, status)) return;
    mbar_arrive_expect_tx(&full[buf], (uint32_t)C::CENT + nb4 * (pv ? 3u : 2u));
    tc::tma_load_2d(st, &tmC, j0, r * D, &full[buf]);
    const size_t rj = (size_t)r * NB + j0;
    bulk_g2s(st + C::OFF_RMAX, rmax + rj, nb4, &full[buf]);
    if (pv) bulk_g2s(st + C::OFF_VAR, var + rj, nb4, &full[buf]);
    bulk_g2s(st + C::OFF_CNT, cnt + rj, nb4, &full[buf]);
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NBUF; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
    for (int i = 0; i < C::NBUF && i < ngrp; ++i) issue(i, i);   // first round in flight
  }
  for (int i = threadIdx.x; i < G * D; i += C::NT) {
    const int h = i / D, k = i % D;
    qs[k * G + h] = bf16_to_f(q[(qhead0 + h) * D + k]);
  }
  __syncthreads();
  for (int h = warp; h < G; h += C::NBUF) {
    const float nrm = query_norm<D, G>(qs, h);
    if (lane == 0) {
      qn[h] = nrm;
      ts[h] = tau[qhead0 + h];
    }
  }
  __syncthreads();

  bool ok = true;
  int round = 0;
  for (int grp = warp; grp < ngrp && ok; grp += C::NBUF, ++round) {
    if (round > 0) {
      // the buffer's previous tile was read by this warp's generic loads
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) issue(warp, grp);
    }
    if (!mbar_wait(&full[warp], (uint32_t)round & 1u, nullptr)) {
      if (lane == 0) set_status(status, ETA_DEVSTAT_TIMEOUT);
      ok = false;
      break;
    }
    const unsigned char* st = smem + warp * C::SB;
    SmemMeta<CF, VD> src;
    src.tile = st;
    const int jl = min(grp * kScreenGroupBlocks + lane * kScreenVW, NB - kScreenVW);
    src.vdp = VD ? reinterpret_cast<const float4*>(vardim + (size_t)r * D * NB + jl) : nullptr;
    src.rowvd = (size_t)NB / 4;
    src.rmax = reinterpret_cast<const float*>(st + C::OFF_RMAX);
    src.var = reinterpret_cast<const float*>(st + C::OFF_VAR);
    src.cnt = reinterpret_cast<const int32_t*>(st + C::OFF_CNT);
    src.lane = lane;
    screen_group_from<D, G, CF, VD, kScreenLoadBatch>(src, NB, NW, grp, r, qhead0, qs, qn, ts,
                                                      bound, z, scale, NB, head_mask,
                                                      union_words, bounds_out);
    __syncwarp();
  }
  // a warp that gave up leaves its copy in flight: wait for it (bounded) before the
  // CTA's shared memory can be released
  if (!ok && lane == 0) mbar_wait(&full[warp], (uint32_t)round & 1u, nullptr);
  __syncthreads();
  compact_row<C::NT>(r, Hq, Hkv, G, NB, NW, union_words, head_mask, union_idx, union_cnt,
                     head_cnt, cs, status, [] { __syncthreads(); });
}

template <int D, int CF, bool VD>
static eta_status_t launch_screen(bool vec, int G, dim3 grid, cudaStream_t s, int Hq, int Hkv,
                                  int NB, int NW, const eta_bf16_t* q, const float* tau,
                                  const void* cent, const float* rmax, const float* var,
                                  const float* vardim, const int32_t* cnt, int bound, float z,
                                  float scale, uint32_t* head_mask, uint32_t* uw,
                                  float* bounds_out) {
  using KernT = void (*)(int, int, int, int, const eta_bf16_t*, const float*, const void*,
                         const float*, const float*, const float*, const int32_t*, int, float,
                         float, uint32_t*, uint32_t*, float*);
  KernT kern = nullptr;
  switch (G) {
    case 1: kern = vec ? screen_vec_kernel<D, 1, CF, VD> : screen_kernel<D, 1, CF, VD>; break;
    case 2: kern = vec ? screen_vec_kernel<D, 2, CF, VD> : screen_kernel<D, 2, CF, VD>; break;
    case 4: kern = vec ? screen_vec_kernel<D, 4, CF, VD> : screen_kernel<D, 4, CF, VD>; break;
    case 8: kern = vec ? screen_vec_kernel<D, 8, CF, VD> : screen_kernel<D, 8, CF, VD>; break;
    default: return ETA_ERR_UNSUPPORTED;
  }
  const dim3 block((vec ? kScreenVecWarps : kScreenWarps) * 32);
  return launch_k(kern, grid, block, 0, s, Hq, Hkv, NB, NW, q, tau, cent, rmax, var, vardim, cnt,
                  bound, z, scale, head_mask, uw, bounds_out);
}

template <int D, int CF, bool VD>
static eta_status_t launch_screen_row(int G, const CUtensorMap& mc, int R, cudaStream_t s, int Hq,
                                      int Hkv, int NB, int NW, const eta_bf16_t* q,
                                      const float* tau, const float* rmax, const float* var,
                                      const float* vardim, const int32_t* cnt, int bound, float z,
                                      float scale, uint32_t* head_mask, uint32_t* uw,
                                      float* bounds_out, int32_t* union_idx, int32_t* union_cnt,
                                      int32_t* head_cnt, int32_t* status) {
  using C = RowScreenCfg<D, CF>;
#define ETA_ROW_LAUNCH(GG)                                                                     \
  do {                                                                                         \
    if (!set_smem_once<screen_row_kernel<D, GG, CF, VD>>(C::SMEM)) return ETA_ERR_CUDA;        \
    return launch_k(screen_row_kernel<D, GG, CF, VD>, dim3(R), dim3(C::NT), C::SMEM, s, mc, Hq, \
                    Hkv, NB, NW, q, tau, rmax, var, vardim, cnt, bound, z, scale, head_mask,   \
                    uw, bounds_out, union_idx, union_cnt, head_cnt, status);                   \
  } while (0)
  switch (G) {
    case 1: ETA_ROW_LAUNCH(1);
    case 2: ETA_ROW_LAUNCH(2);
    case 4: ETA_ROW_LAUNCH(4);
    case 8: ETA_ROW_LAUNCH(8);
  }
#undef ETA_ROW_LAUNCH
  return ETA_ERR_UNSUPPORTED;
}

// Whether the one-launch screen takes this call: few pairs (at most two waves of
// CTAs), rows of at most kRowScreenMaxRounds rounds of group buffers, and the
// alignment its bulk copies need.
template <int D, int CF>
static bool row_screen_fits(int R, int NB) {
  using C = RowScreenCfg<D, CF>;
  const int ngrp = (NB + kScreenGroupBlocks - 1) / kScreenGroupBlocks;
  return R <= 2 * sm_count() && ngrp <= kRowScreenMaxRounds * C::NBUF &&
         NB % (CF == 1 ? 8 : 4) == 0;
}

// ---------------------------------------------------------------- tensor-core screen
std::atomic<int> g_screen_engine{ETA_ENGINE_AUTO};

// One launch (a CTA per row, the row's compaction included) when every row gets its
// own SM and rows are short; otherwise the (row, group) items in equal contiguous
// shares over one CTA per SM, and compact_kernel after.
constexpr int kTcRowsMaxGroups = 32;
inline bool tc_screen_rows(int R, int NB) {
  const int ngrp = (NB + stc::GB - 1) / stc::GB;
  return R <= sm_count() && ngrp <= kTcRowsMaxGroups;
}

// ETA_ENGINE_AUTO takes the tensor cores where they measured faster on one B200: the
// one-launch form at d = 128 (128K / B = 16: 21.4 vs 27.7 us for screen + compaction;
// the one-launch step at B = 8, 32K: 76.6 vs 82.4 us per step).  For larger batches
// the CUDA-core screen is a little faster (128K / B = 64: 42.1 vs 45.8 us): each
// tensor-core CTA pays a ~4 us start-up before its first group lands, where the
// CUDA-core kernel's thousands of warps start at once.  At d = 64 the CUDA-core
// one-launch screen has half the arithmetic and stays ahead (20.4 vs 16.4 us at
// 128K / B = 16).
bool tc_screen_applies(const eta_dims_t* d, int cent_format, int bound) {
  const int e = g_screen_engine.load();
  if (e == ETA_ENGINE_FMA || cent_format != ETA_CENT_BF16 || (d->d != 128 && d->d != 64) ||
      bound == ETA_BOUND_PROB_DIM || num_blocks(d) % 8 != 0)
    return false;
  return e == ETA_ENGINE_TCGEN05 ||
         (d->d == 128 && tc_screen_rows(d->B * d->Hkv, num_blocks(d)));
}

template <int D, int G>
static eta_status_t launch_screen_tc(bool rows, const CUtensorMap& mc, const CUtensorMap& mq,
                                     const stc::Params& prm, int grid, cudaStream_t s) {
  constexpr int SM = stc::Ring<D>::SMEM_BYTES;
  if (rows) {
    if (!set_smem_once<stc::screen_tc_kernel<D, G, true>>(SM)) return ETA_ERR_CUDA;
    return launch_k(stc::screen_tc_kernel<D, G, true>, dim3(grid), dim3(stc::NT), SM, s, mc, mq,
                    prm);
  }
  if (!set_smem_once<stc::screen_tc_kernel<D, G, false>>(SM)) return ETA_ERR_CUDA;
  return launch_k(stc::screen_tc_kernel<D, G, false>, dim3(grid), dim3(stc::NT), SM, s, mc, mq,
                  prm);
}

// eta_screen on the tensor cores (tc_screen_applies).  Pointers are 16-byte aligned.
static eta_status_t run_screen_tc(const eta_dims_t* dims, const eta_bf16_t* q, const float* tau,
                                  const void* cent, const float* rmax, const float* var,
                                  const int32_t* cnt, int bound, float z, float scale,
                                  uint32_t* head_mask, uint32_t* uw, int32_t* union_idx,
                                  int32_t* union_cnt, float* bounds_out, int32_t* head_cnt,
                                  int32_t* dev_status, cudaStream_t s) {
  const int NB = num_blocks(dims), NW = num_words(dims);
  const int R = dims->B * dims->Hkv, G = dims->Hq / dims->Hkv;
  CUtensorMap mc, mq;
  const int D = dims->d;
  if (!make_map_bf16_swz(&mc, cent, NB, (uint64_t)R * D, (uint64_t)NB * 2, (uint32_t)D) ||
      !make_map(&mq, q, (uint64_t)dims->B * dims->Hq, 16, (uint64_t)D))
    return ETA_ERR_CUDA;
  stc::Params prm;
  prm.Hq = dims->Hq; prm.Hkv = dims->Hkv; prm.NB = NB; prm.NW = NW;
  prm.ngrp = (NB + stc::GB - 1) / stc::GB;
  prm.items = R * prm.ngrp;
  prm.prob = bound == ETA_BOUND_PROB ? 1 : 0;
  prm.z = z; prm.scale = scale;
  prm.q = q; prm.tau = tau; prm.rmax = rmax; prm.var = var; prm.cnt = cnt;
  prm.head_mask = head_mask; prm.union_words = uw; prm.bounds_out = bounds_out;
  prm.union_idx = union_idx; prm.union_cnt = union_cnt; prm.head_cnt = head_cnt;
  prm.status = dev_status;
  const bool rows = tc_screen_rows(R, NB);
  int grid;
  if (rows) {
    prm.chunk = prm.ngrp;
    grid = R;
  } else {
    const int n = std::max(sm_count(), 1);
    prm.chunk = (prm.items + n - 1) / n;
    grid = (prm.items + prm.chunk - 1) / prm.chunk;
  }
  eta_status_t st = ETA_ERR_UNSUPPORTED;
  const bool d64 = D == 64;
  switch (G) {
    case 1: st = d64 ? launch_screen_tc<64, 1>(rows, mc, mq, prm, grid, s)
                     : launch_screen_tc<128, 1>(rows, mc, mq, prm, grid, s); break;
    case 2: st = d64 ? launch_screen_tc<64, 2>(rows, mc, mq, prm, grid, s)
                     : launch_screen_tc<128, 2>(rows, mc, mq, prm, grid, s); break;
    case 4: st = d64 ? launch_screen_tc<64, 4>(rows, mc, mq, prm, grid, s)
                     : launch_screen_tc<128, 4>(rows, mc, mq, prm, grid, s); break;
    case 8: st = d64 ? launch_screen_tc<64, 8>(rows, mc, mq, prm, grid, s)
                     : launch_screen_tc<128, 8>(rows, mc, mq, prm, grid, s); break;
  }
  if (st != ETA_OK || rows) return st;
  return launch_k(compact_kernel, dim3(R), dim3(kCompactThreads), 0, s, dims->Hq, dims->Hkv, G,
                  NB, NW, (const uint32_t*)uw, (const uint32_t*)head_mask, union_idx, union_cnt,
                  head_cnt, dev_status);
}

}  // namespace eta

using namespace eta;

extern "C" eta_status_t eta_set_screen_engine(eta_engine_t engine) {
  if (engine != ETA_ENGINE_AUTO && engine != ETA_ENGINE_TCGEN05 && engine != ETA_ENGINE_FMA)
    return ETA_ERR_INVALID_ARG;
  g_screen_engine.store((int)engine);
  return ETA_OK;
}

extern "C" eta_engine_t eta_get_screen_engine(void) {
  return static_cast<eta_engine_t>(g_screen_engine.load());
}

extern "C" size_t eta_screen_workspace_size(const eta_dims_t* dims) {
  if (check_dims(dims) != ETA_OK) return 0;
  return align_up((size_t)dims->B * dims->Hkv * num_words(dims) * sizeof(uint32_t), 256);
}

extern "C" int32_t eta_screen_launches(const eta_dims_t* dims, eta_cent_format_t cent_format) {
  if (check_dims(dims) != ETA_OK) return -1;
  const int NB = num_blocks(dims), R = dims->B * dims->Hkv;
  const bool bf = cent_format == ETA_CENT_BF16;
  if (tc_screen_applies(dims, cent_format, ETA_BOUND_EXACT)) return tc_screen_rows(R, NB) ? 1 : 2;
  if (NB % 4 != 0) return 2;
  bool row;
  if (dims->d == 128) row = bf ? row_screen_fits<128, 1>(R, NB) : row_screen_fits<128, 0>(R, NB);
  else row = bf ? row_screen_fits<64, 1>(R, NB) : row_screen_fits<64, 0>(R, NB);
  return row ? 1 : 2;
}

extern "C" eta_status_t eta_screen(const eta_dims_t* dims, const eta_bf16_t* q, const float* tau,
                                   eta_cent_format_t cent_format, const void* cent,
                                   const float* rmax, const float* var, const float* vardim,
                                   const int32_t* cnt, eta_bound_t bound, float z, float scale,
                                   uint32_t* head_mask, int32_t* union_idx, int32_t* union_cnt,
                                   float* bounds_out, int32_t* head_cnt, void* ws,
                                   size_t ws_bytes, int32_t* dev_status, void* stream) {
  eta_status_t st = check_dims(dims);
  if (st != ETA_OK) return st;
  if (!q || !tau || !cent || !rmax || !cnt || !head_mask || !union_idx || !union_cnt)
    return ETA_ERR_INVALID_ARG;
  if (bound != ETA_BOUND_EXACT && bound != ETA_BOUND_PROB && bound != ETA_BOUND_PROB_DIM)
    return ETA_ERR_INVALID_ARG;
  if (bound == ETA_BOUND_PROB_DIM && (!vardim || !(z >= 0.f))) return ETA_ERR_INVALID_ARG;
  if (cent_format != ETA_CENT_F32 && cent_format != ETA_CENT_BF16) return ETA_ERR_INVALID_ARG;
  if (bound == ETA_BOUND_PROB && (!var || !(z >= 0.f))) return ETA_ERR_INVALID_ARG;
  if (!ws || ws_bytes < eta_screen_workspace_size(dims)) return ETA_ERR_WORKSPACE;
  if (scale == 0.f) scale = 1.f / sqrtf((float)dims->d);
  const int NB = num_blocks(dims), NW = num_words(dims);
  const int R = dims->B * dims->Hkv, G = dims->Hq / dims->Hkv;
  uint32_t* uw = static_cast<uint32_t*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bf = cent_format == ETA_CENT_BF16;
  const int VW = 4;
  const bool vd = bound == ETA_BOUND_PROB_DIM;
  const bool vec = (NB % VW == 0) && aligned16(cent) && aligned16(rmax) && aligned16(cnt) &&
                   (!var || aligned16(var)) && (!vardim || aligned16(vardim)) &&
                   (!bounds_out || aligned16(bounds_out));
  if (vec && aligned16(q) && tc_screen_applies(dims, cent_format, bound))
    return run_screen_tc(dims, q, tau, cent, rmax, var, cnt, (int)bound, z, scale, head_mask, uw,
                         union_idx, union_cnt, bounds_out, head_cnt, dev_status, s);
  bool row = vec;
  if (row) {
    if (dims->d == 128) row = bf ? row_screen_fits<128, 1>(R, NB) : row_screen_fits<128, 0>(R, NB);
    else row = bf ? row_screen_fits<64, 1>(R, NB) : row_screen_fits<64, 0>(R, NB);
  }
  if (row) {
    CUtensorMap mc;
    if (!make_map_plain(&mc, cent, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                        NB, (uint64_t)R * dims->d, (uint64_t)NB * (bf ? 2 : 4),
                        kScreenGroupBlocks, dims->d))
      return ETA_ERR_CUDA;
#define ETA_ROW_ARGS G, mc, R, s, dims->Hq, dims->Hkv, NB, NW, q, tau, rmax, var, vardim, cnt, \
                     (int)bound, z, scale, head_mask, uw, bounds_out, union_idx, union_cnt,   \
                     head_cnt, dev_status
    if (dims->d == 128) {
      if (vd) return bf ? launch_screen_row<128, 1, true>(ETA_ROW_ARGS)
                        : launch_screen_row<128, 0, true>(ETA_ROW_ARGS);
      return bf ? launch_screen_row<128, 1, false>(ETA_ROW_ARGS)
                : launch_screen_row<128, 0, false>(ETA_ROW_ARGS);
    }
    if (vd) return bf ? launch_screen_row<64, 1, true>(ETA_ROW_ARGS)
                      : launch_screen_row<64, 0, true>(ETA_ROW_ARGS);
    return bf ? launch_screen_row<64, 1, false>(ETA_ROW_ARGS)
              : launch_screen_row<64, 0, false>(ETA_ROW_ARGS);
#undef ETA_ROW_ARGS
  }
  dim3 grid;
  if (vec) {
    const int ngroups = (NB + 32 * VW - 1) / (32 * VW);
    grid = dim3((ngroups + kScreenVecWarps - 1) / kScreenVecWarps, R);
  } else {
    grid = dim3((NW + kScreenWarps - 1) / kScreenWarps, R);
  }
#define ETA_SCREEN_ARGS vec, G, grid, s, dims->Hq, dims->Hkv, NB, NW, q, tau, cent, rmax, var, \
                        vardim, cnt, (int)bound, z, scale, head_mask, uw, bounds_out
  if (dims->d == 128) {
    if (vd) st = bf ? launch_screen<128, 1, true>(ETA_SCREEN_ARGS)
                    : launch_screen<128, 0, true>(ETA_SCREEN_ARGS);
    else st = bf ? launch_screen<128, 1, false>(ETA_SCREEN_ARGS)
                 : launch_screen<128, 0, false>(ETA_SCREEN_ARGS);
  } else {
    if (vd) st = bf ? launch_screen<64, 1, true>(ETA_SCREEN_ARGS)
                    : launch_screen<64, 0, true>(ETA_SCREEN_ARGS);
    else st = bf ? launch_screen<64, 1, false>(ETA_SCREEN_ARGS)
                 : launch_screen<64, 0, false>(ETA_SCREEN_ARGS);
  }
#undef ETA_SCREEN_ARGS
  if (st != ETA_OK) return st;
  return launch_k(compact_kernel, dim3(R), dim3(kCompactThreads), 0, s, dims->Hq, dims->Hkv, G,
                  NB, NW, (const uint32_t*)uw, (const uint32_t*)head_mask, union_idx, union_cnt,
                  head_cnt, dev_status);
}
