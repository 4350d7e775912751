// Host-only entry points: offline calibration of frozen per-head thresholds and
// status helpers.
//
// Calibration (arXiv 2609.20888 abstract: an offline calibration algorithm
// "freezes per-head constant thresholds to eliminate predictor overhead").  The
// pages do not print the algorithm; the rule here is a per-head quantile of the
// block bounds of seeded calibration queries, which admits the target fraction
// of (query, block) pairs by construction.
#include <algorithm>
#include <cmath>
#include <vector>

#include "../../include/eta.h"

extern "C" eta_status_t eta_calibrate_const_tau(const float* bounds, const uint8_t* valid,
                                                int32_t n_q, int32_t Hq, int32_t NB,
                                                float density, float* tau_out) {
  if (!bounds || !valid || !tau_out || n_q <= 0 || Hq <= 0 || NB <= 0) return ETA_ERR_INVALID_ARG;
  if (!(density >= 0.f && density <= 1.f)) return ETA_ERR_INVALID_ARG;
  std::vector<float> pool;
  pool.reserve((size_t)n_q * NB);
  for (int h = 0; h < Hq; ++h) {
    pool.clear();
    for (int i = 0; i < n_q; ++i) {
      const size_t base = ((size_t)i * Hq + h) * NB;
      for (int j = 0; j < NB; ++j)
        if (valid[base + j]) pool.push_back(bounds[base + j]);
    }
    if (pool.empty()) return ETA_ERR_INVALID_ARG;
    const double want = std::floor((1.0 - (double)density) * (double)pool.size());
    size_t k = (size_t)std::max(0.0, want);
    if (k >= pool.size()) k = pool.size() - 1;
    std::nth_element(pool.begin(), pool.begin() + (ptrdiff_t)k, pool.end());
    tau_out[h] = pool[k];
  }
  return ETA_OK;
}

extern "C" eta_status_t eta_status_from_device(int32_t dev_status) {
  if (dev_status & ETA_DEVSTAT_BOUNDS) return ETA_ERR_DEVICE_BOUNDS;
  if (dev_status & ETA_DEVSTAT_TIMEOUT) return ETA_ERR_DEVICE_TIMEOUT;
  if (dev_status & ETA_DEVSTAT_NONFINITE_Q) return ETA_ERR_NONFINITE;
  if (dev_status & (ETA_DEVSTAT_BAD_BLOCK | ETA_DEVSTAT_BAD_LENGTH)) return ETA_ERR_INVALID_ARG;
  return ETA_OK;
}

extern "C" const char* eta_status_string(eta_status_t s) {
  switch (s) {
    case ETA_OK: return "ok";
    case ETA_ERR_INVALID_ARG: return "invalid argument";
    case ETA_ERR_UNSUPPORTED: return "unsupported shape";
    case ETA_ERR_WORKSPACE: return "workspace missing or too small";
    case ETA_ERR_CUDA: return "CUDA error";
    case ETA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case ETA_ERR_NONFINITE: return "non-finite query";
    case ETA_ERR_DEVICE_BOUNDS: return "out-of-range index (checked build)";
  }
  return "unknown status";
}
