// Log-sum-exp merge of decode results computed over disjoint key sets, e.g. the
// block-aligned sequence shards of one KV cache split across GPUs: Eq. 2-3 of the
// evolve.pub review of arXiv 2609.20888 (Methodology Assessment) make the decode a
// softmax over gated logits, so results over disjoint key sets merge exactly by
// o = sum_p e^(lse_p - M) o_p / L, L = sum_p e^(lse_p - M), lse = M + log L,
// M = max_p lse_p.
//
// One CTA per output row (a (batch row, query head) pair), thread = dimension; the
// parts are read in order.  Memory-bound and small (n_parts * n_rows * (d + 1)
// floats).
#include <math.h>

#include "eta_common.cuh"
#include "eta_host.h"

namespace eta {

__global__ void __launch_bounds__(128) lse_merge_kernel(int n_parts, int n_rows, int d,
                                                        const float* __restrict__ o_parts,
                                                        const float* __restrict__ lse_parts,
                                                        float* __restrict__ o,
                                                        float* __restrict__ lse) {
  ETA_PDL_ENTRY();
  const int row = blockIdx.x, dd = threadIdx.x;
  float M = -INFINITY;
  for (int p = 0; p < n_parts; ++p) M = fmaxf(M, lse_parts[(size_t)p * n_rows + row]);
  float L = 0.f, O = 0.f;
  if (M != -INFINITY) {
    for (int p = 0; p < n_parts; ++p) {
      const float w = expf(lse_parts[(size_t)p * n_rows + row] - M);   // 0 for an empty part
      L += w;
      O = fmaf(w, o_parts[((size_t)p * n_rows + row) * d + dd], O);
    }
  }
  if (L > 0.f) {
    o[(size_t)row * d + dd] = O / L;
    if (dd == 0) lse[row] = M + logf(L);
  } else {
    o[(size_t)row * d + dd] = 0.f;
    if (dd == 0) lse[row] = -INFINITY;
  }
}

}  // namespace eta

using namespace eta;

extern "C" eta_status_t eta_lse_merge(int32_t n_parts, int32_t n_rows, int32_t d,
                                      const float* o_parts, const float* lse_parts, float* o,
                                      float* lse, void* stream) {
  if (n_parts <= 0 || n_rows <= 0 || !(d == 64 || d == 128)) return ETA_ERR_INVALID_ARG;
  if (!o_parts || !lse_parts || !o || !lse) return ETA_ERR_INVALID_ARG;
  return launch_k(lse_merge_kernel, dim3(n_rows), dim3(d), 0,
                  static_cast<cudaStream_t>(stream), n_parts, n_rows, d, o_parts, lse_parts, o,
                  lse);
}
