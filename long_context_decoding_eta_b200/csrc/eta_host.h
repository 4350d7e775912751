// Host-side helpers shared by the C-ABI entry points: argument checks, device
// properties, launch-error mapping.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "../../include/eta.h"

namespace eta {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int num_blocks(const eta_dims_t* d) { return d->T_max / d->blk; }
inline int num_words(const eta_dims_t* d) { return (num_blocks(d) + 31) / 32; }

// Common shape validation.  Returns ETA_OK or the error to report.  `rows_in_grid_y`:
// the caller launches B * Hkv CTAs along grid.y (65535 at most).
inline eta_status_t check_dims(const eta_dims_t* d, bool rows_in_grid_y = true) {
  if (!d) return ETA_ERR_INVALID_ARG;
  if (d->B <= 0 || d->Hq <= 0 || d->Hkv <= 0 || d->d <= 0 || d->blk <= 0 || d->T_max <= 0)
    return ETA_ERR_INVALID_ARG;
  if (d->Hq % d->Hkv != 0) return ETA_ERR_INVALID_ARG;
  const int G = d->Hq / d->Hkv;
  if (!(G == 1 || G == 2 || G == 4 || G == 8)) return ETA_ERR_UNSUPPORTED;
  if (!(d->d == 64 || d->d == 128)) return ETA_ERR_UNSUPPORTED;
  if (!(d->blk == 64 || d->blk == 128)) return ETA_ERR_UNSUPPORTED;
  if (d->T_max % d->blk != 0) return ETA_ERR_UNSUPPORTED;
  if (rows_in_grid_y && (int64_t)d->B * d->Hkv > 65535) return ETA_ERR_UNSUPPORTED;
  if (num_blocks(d) > 65536) return ETA_ERR_UNSUPPORTED;
  if (d->Hq > 256) return ETA_ERR_UNSUPPORTED;
  return ETA_OK;
}

// Whether the block screening of these dims takes the tensor-core form
// (screen_tc.cuh): bf16 centroids, d = 128 or 64, not the per-dimension bound, NB a
// multiple of 8 (the centroid rows' TMA stride), and the process-wide screen engine
// (eta_set_screen_engine): ETA_ENGINE_TCGEN05 wherever that applies, ETA_ENGINE_AUTO
// only where it measured faster (d = 128, the one-launch form), ETA_ENGINE_FMA never.  eta_screen and
// the one-launch step decide alike, so that both write the same bits.  Defined in
// screen.cu.
bool tc_screen_applies(const eta_dims_t* d, int cent_format, int bound);

// Launches `kern` on `s` with programmatic stream serialization allowed (see
// ETA_PDL_ENTRY in eta_common.cuh).
template <typename... KArgs, typename... Args>
inline eta_status_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) == cudaSuccess
             ? ETA_OK
             : ETA_ERR_CUDA;
}

// Unique identifier of the CUDA context current on the calling thread, or 0 when
// none is current (or the driver cannot say).  Per-device caches key on it rather
// than on the device ordinal: after cudaDeviceReset, or any destruction and
// re-creation of the primary context, the library's module is loaded again, so
// symbol addresses and function attributes cached for the old context are stale.
inline unsigned long long current_context_id() {
  using GetCurrentFn = CUresult (*)(CUcontext*);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static const std::pair<GetCurrentFn, GetIdFn> fns = [] {
    void* cur = nullptr;
    void* gid = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    const bool ok =
        cudaGetDriverEntryPoint("cuCtxGetCurrent", &cur, cudaEnableDefault, &q1) ==
            cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &gid, cudaEnableDefault, &q2) == cudaSuccess &&
        q2 == cudaDriverEntryPointSuccess;
    return ok ? std::make_pair(reinterpret_cast<GetCurrentFn>(cur),
                               reinterpret_cast<GetIdFn>(gid))
              : std::make_pair(GetCurrentFn(nullptr), GetIdFn(nullptr));
  }();
  if (!fns.first || !fns.second) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (fns.first(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (fns.second(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Raises a kernel's dynamic shared-memory limit once per device context (so that
// calls made during stream capture issue no attribute change).  The context id is
// remembered per device; a new context (after a device reset) sets it again.
template <auto Kern>
inline bool set_smem_once(int bytes) {
  static std::atomic<unsigned long long> done_ctx[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  const unsigned long long ctx = current_context_id();
  if (ctx != 0 && done_ctx[dev].load() == ctx) return true;
  if (cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  // the attribute call made the primary context current if none was yet
  done_ctx[dev].store(ctx != 0 ? ctx : current_context_id());
  return true;
}

inline eta_status_t launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
}

inline int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace eta
