// O(1)-per-block screening with hard pruning and co-admission across the query
// heads of a KV group (arXiv 2609.20888 abstract: KV blocks screened "in O(1) time
// using cached geometric-probabilistic bounds", incidental tokens "co-admitted by
// coarse GPU block selection"; evolve.pub review FAQ: blocks whose best possible
// score falls below the threshold are skipped entirely).
//
// screen_kernel: lane = block.  Centroids are stored dimension-major per (row, KV
//   head), so each of the d loads of a warp is one 128-byte line covering 32
//   consecutive blocks; the G query heads of the group sit in shared memory as
//   [d][G] fp32 and are read as broadcasts.  One ballot per head gives the
//   head's 32-bit admit word directly; the union word is their OR.
// compact_kernel: one CTA per (row, KV head) turns union words into the ascending
//   list of admitted block indices (popcount prefix over words, lane = bit).
#include <type_traits>

#include "eta_common.cuh"
#include "eta_host.h"
#include "screen_dev.cuh"

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
               int32_t* __restrict__ union_cnt, int32_t* __restrict__ head_cnt) {
  ETA_PDL_ENTRY();
  __shared__ uint32_t wbuf[kCompactThreads];
  __shared__ int woff[kCompactThreads];
  __shared__ int wsum[kCompactThreads / 32];
  const int r = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int carry = 0;
  for (int base = 0; base < NW; base += kCompactThreads) {
    const int w = base + tid;
    const uint32_t word = w < NW ? union_words[(size_t)r * NW + w] : 0u;
    const int c = __popc(word);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int wpre = 0, total = 0;
#pragma unroll
    for (int i = 0; i < kCompactThreads / 32; ++i) {
      const int v = wsum[i];
      if (i < warp) wpre += v;
      total += v;
    }
    wbuf[tid] = word;
    woff[tid] = carry + wpre + incl - c;
    __syncthreads();
    for (int i = warp; i < kCompactThreads && base + i < NW; i += kCompactThreads / 32) {
      const uint32_t wd = wbuf[i];
      if ((wd >> lane) & 1u)
        union_idx[(size_t)r * NB + woff[i] + __popc(wd & ((1u << lane) - 1u))] =
            (base + i) * 32 + lane;
    }
    carry += total;
    __syncthreads();
  }
  if (tid == 0) union_cnt[r] = carry;
  if (head_cnt && warp < G) {
    const int b = r / Hkv, g = r % Hkv;
    const size_t hq = (size_t)b * Hq + (size_t)g * G + warp;
    int s = 0;
    for (int w = lane; w < NW; w += 32) s += __popc(head_mask[hq * NW + w]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) head_cnt[hq] = s;
  }
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

}  // namespace eta

using namespace eta;

extern "C" size_t eta_screen_workspace_size(const eta_dims_t* dims) {
  if (check_dims(dims) != ETA_OK) return 0;
  return align_up((size_t)dims->B * dims->Hkv * num_words(dims) * sizeof(uint32_t), 256);
}

extern "C" eta_status_t eta_screen(const eta_dims_t* dims, const eta_bf16_t* q, const float* tau,
                                   eta_cent_format_t cent_format, const void* cent,
                                   const float* rmax, const float* var, const float* vardim,
                                   const int32_t* cnt, eta_bound_t bound, float z, float scale,
                                   uint32_t* head_mask, int32_t* union_idx, int32_t* union_cnt,
                                   float* bounds_out, int32_t* head_cnt, void* ws,
                                   size_t ws_bytes, int32_t* dev_status, void* stream) {
  (void)dev_status;
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
                  head_cnt);
}
