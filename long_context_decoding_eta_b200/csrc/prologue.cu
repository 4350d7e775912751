// The two independent parts of a decode step that come before the screening, as one
// launch: the tail-block metadata refresh after a token was appended ("cached
// centroid/variance/max-norm metadata", evolve.pub review of arXiv 2609.20888,
// Summary) and the thresholds (Eq. 1 of the review's Methodology Assessment, or the
// frozen per-head constants of the abstract).  Both are small latency-bound passes over
// the same (batch row, KV head) grid; one CTA of 16 warps does both concurrently:
// warps 0-7 refresh the tail block, warps 8-15 compute the group's G thresholds,
// through the same device functions as eta_build_block_meta and eta_predict_tau, so
// the results are bit-identical to those two calls.
#include "eta_common.cuh"
#include "eta_host.h"
#include "meta_dev.cuh"
#include "tau_dev.cuh"

namespace eta {

constexpr int kPrologueWarps = 2 * kMetaWarps;

template <int D, int CF, int G>
__global__ void __launch_bounds__(kPrologueWarps * 32)
prologue_kernel(int Hq, int Hkv, int T_max, int blk, int NB, const eta_bf16_t* __restrict__ K,
                const eta_bf16_t* __restrict__ V, const int32_t* __restrict__ lengths,
                void* __restrict__ cent, float* __restrict__ rmax, float* __restrict__ var,
                int32_t* __restrict__ cnt, float* __restrict__ vsum, float* __restrict__ vardim,
                const eta_bf16_t* __restrict__ q, const float* __restrict__ W,
                const float* __restrict__ bias, const float* __restrict__ tau_const,
                float* __restrict__ tau, int32_t* status) {
  ETA_PDL_ENTRY();
  __shared__ TailScratch<D, CF> sc;
  __shared__ float red[kTauVirtWarps][G];
  const int warp = threadIdx.x >> 5;
  const int b = blockIdx.x, g = blockIdx.y, r = b * Hkv + g;
  if (warp < kMetaWarps) {
    meta_tail_block<D, CF, kMetaWarps>(r, Hkv, T_max, blk, NB, K, V, lengths, cent, rmax, var,
                                       cnt, vsum, vardim, status, sc, warp,
                                       [] { named_bar_sync(1, kMetaWarps * 32); });
  } else if (tau_const) {
    const int lt = threadIdx.x - kMetaWarps * 32;
    if (lt < G) tau[(size_t)b * Hq + g * G + lt] = tau_const[g * G + lt];
  } else {
    const bool bad = tau_group<G, kMetaWarps>(Hq, D, b, g * G, q, W, bias, red, tau,
                                              warp - kMetaWarps,
                                              [] { named_bar_sync(2, kMetaWarps * 32); });
    if (bad && g == 0) set_status(status, ETA_DEVSTAT_NONFINITE_Q);
  }
}

template <int D, int CF>
static eta_status_t launch_prologue(const eta_dims_t* dims, const eta_bf16_t* K,
                                    const eta_bf16_t* V, const int32_t* lengths, void* cent,
                                    float* rmax, float* var, int32_t* cnt, float* vsum,
                                    float* vardim, const eta_bf16_t* q, const float* W,
                                    const float* bias, const float* tau_const, float* tau,
                                    int32_t* dev_status, cudaStream_t s) {
  const dim3 grid(dims->B, dims->Hkv);
  const int NB = num_blocks(dims);
#define ETA_PRO_ARGS dims->Hq, dims->Hkv, dims->T_max, dims->blk, NB, K, V, lengths, cent, rmax, \
                     var, cnt, vsum, vardim, q, W, bias, tau_const, tau, dev_status
  switch (dims->Hq / dims->Hkv) {
    case 1: return launch_k(prologue_kernel<D, CF, 1>, grid, dim3(kPrologueWarps * 32), 0, s, ETA_PRO_ARGS);
    case 2: return launch_k(prologue_kernel<D, CF, 2>, grid, dim3(kPrologueWarps * 32), 0, s, ETA_PRO_ARGS);
    case 4: return launch_k(prologue_kernel<D, CF, 4>, grid, dim3(kPrologueWarps * 32), 0, s, ETA_PRO_ARGS);
    case 8: return launch_k(prologue_kernel<D, CF, 8>, grid, dim3(kPrologueWarps * 32), 0, s, ETA_PRO_ARGS);
  }
#undef ETA_PRO_ARGS
  return ETA_ERR_UNSUPPORTED;
}

}  // namespace eta

using namespace eta;

extern "C" eta_status_t eta_append_and_predict_tau(
    const eta_dims_t* dims, const eta_bf16_t* K, const eta_bf16_t* V, const int32_t* lengths,
    eta_cent_format_t cent_format, void* cent, float* rmax, float* var, int32_t* cnt,
    float* vsum, float* vardim, const eta_bf16_t* q, const float* W, const float* bias,
    const float* tau_const, float* tau, int32_t* dev_status, void* stream) {
  eta_status_t st = check_dims(dims, /*rows_in_grid_y=*/false);   // grid (B, Hkv)
  if (st != ETA_OK) return st;
  if (dims->Hkv > 65535) return ETA_ERR_UNSUPPORTED;
  if (!K || !lengths || !cent || !rmax || !var || !cnt || !tau) return ETA_ERR_INVALID_ARG;
  if (cent_format != ETA_CENT_F32 && cent_format != ETA_CENT_BF16) return ETA_ERR_INVALID_ARG;
  if (vsum && !V) return ETA_ERR_INVALID_ARG;
  if (!aligned16(K) || (V && !aligned16(V))) return ETA_ERR_INVALID_ARG;
  if (!tau_const && (!q || !W)) return ETA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bf = cent_format == ETA_CENT_BF16;
#define ETA_PRO_CALL(DD, CC)                                                                 \
  launch_prologue<DD, CC>(dims, K, V, lengths, cent, rmax, var, cnt, vsum, vardim, q, W, bias, \
                          tau_const, tau, dev_status, s)
  if (dims->d == 128) return bf ? ETA_PRO_CALL(128, 1) : ETA_PRO_CALL(128, 0);
  return bf ? ETA_PRO_CALL(64, 1) : ETA_PRO_CALL(64, 0);
#undef ETA_PRO_CALL
}
