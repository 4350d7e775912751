// Threshold per (query, head): the linear predictor on the concatenated post-RoPE
// query heads (evolve.pub review of arXiv 2609.20888, Methodology Assessment,
// Eq. 1: tau = qbar W_tau + b_tau) or a frozen per-head constant (abstract: offline
// calibration "freezes per-head constant thresholds").
//
// A GEMV per batch row, split by KV group: W (Hq*d x Hq fp32, 128 KB at Hq = 16,
// d = 128) stays L2-resident across rows; every thread owns rows of W, then a
// fixed-order block reduction, so results are deterministic.
#include "eta_common.cuh"
#include "eta_host.h"
#include "tau_dev.cuh"

namespace eta {

constexpr int kTauThreads = 256;

// One CTA per (batch row, KV group): the G outputs of the group, each thread
// owning every 256th element of qbar; W's G columns of the group are read as one
// 16/32-byte piece per row of W.  2 * Hkv * B CTAs keep the GEMV latency short.
template <int G>
__global__ void __launch_bounds__(kTauThreads)
predict_tau_group_kernel(int Hq, int D, const eta_bf16_t* __restrict__ q,
                         const float* __restrict__ W, const float* __restrict__ bias,
                         float* __restrict__ tau, int32_t* status) {
  ETA_PDL_ENTRY();
  __shared__ float red[kTauVirtWarps][G];
  const int g = blockIdx.y;
  const bool bad = tau_group<G, kTauThreads / 32>(Hq, D, blockIdx.x, g * G, q, W, bias, red, tau,
                                                  threadIdx.x >> 5, [] { __syncthreads(); });
  if (bad && g == 0) set_status(status, ETA_DEVSTAT_NONFINITE_Q);
}

__global__ void const_tau_kernel(int total, int Hq, const float* __restrict__ tau_const,
                                 float* __restrict__ tau) {
  ETA_PDL_ENTRY();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < total) tau[i] = tau_const[i % Hq];
}

}  // namespace eta

using namespace eta;

extern "C" eta_status_t eta_predict_tau(const eta_dims_t* dims, const eta_bf16_t* q,
                                        const float* W, const float* bias,
                                        const float* tau_const, float* tau, int32_t* dev_status,
                                        void* stream) {
  eta_status_t st = check_dims(dims, /*rows_in_grid_y=*/false);   // grid (B, Hkv)
  if (st != ETA_OK) return st;
  if (!tau) return ETA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (tau_const) {
    const int total = dims->B * dims->Hq;
    return launch_k(const_tau_kernel, dim3((total + 255) / 256), dim3(256), 0, s, total,
                    dims->Hq, tau_const, tau);
  }
  if (!q || !W) return ETA_ERR_INVALID_ARG;
  const dim3 grid(dims->B, dims->Hkv);
  void (*kern)(int, int, const eta_bf16_t*, const float*, const float*, float*, int32_t*) = nullptr;
  switch (dims->Hq / dims->Hkv) {
    case 1: kern = predict_tau_group_kernel<1>; break;
    case 2: kern = predict_tau_group_kernel<2>; break;
    case 4: kern = predict_tau_group_kernel<4>; break;
    case 8: kern = predict_tau_group_kernel<8>; break;
    default: return ETA_ERR_UNSUPPORTED;
  }
  return launch_k(kern, grid, dim3(kTauThreads), 0, s, dims->Hq, dims->d, q, W, bias, tau,
                  dev_status);
}
