// The whole ETA decode step as one persistent kernel: tail-block metadata, the
// threshold, block screening with union compaction, the gated split-KV decode and
// the log-sum-exp merge, without a launch or a host round trip between them.
//
// Same arithmetic as the separate calls (eta_build_block_meta on the tail block,
// eta_predict_tau, eta_screen, eta_decode), through the same device functions:
// Eq. 1 of the evolve.pub review of arXiv 2609.20888 (Methodology Assessment) for
// the threshold, the abstract's O(1) block screening with hard pruning and GQA
// co-admission, and the gated logits s * sigmoid((s - tau) / T) of Eq. 2-3.
//
// Cooperative launch, one CTA per SM (192 threads), in three phases:
//   A  row prologue, one (row, KV head) per CTA in turn: warps 0-3 recompute the tail
//      block's metadata (after a token was appended) while warps 4-5 compute the
//      group's G thresholds; then the row is released (ready[r] = 1, gpu-scope
//      release).
//   B  screening of groups of 128 blocks, taken kGrab at a time from a global counter
//      in row order (CTAs that spent longer in phase A simply take fewer).  One thread
//      waits for a group's row to be released and stages the group with TMA into a
//      shared-memory ring: the [d x 128] centroid tile (tensor copy), the rmax / var /
//      cnt slices and the G query rows (bulk copies).  Up to five warps (no more than
//      the ring has stages) screen the staged groups (head words, union word); where
//      eta_screen takes the tensor cores (tc_screen_applies) the step does too:
//      warp 5 issues each group's q . c product (screen_tc.cuh) and warps 0-3 read
//      it from TMEM.  The screening warps also count each row's admitted blocks.
//   -  grid barrier; then warps compact the rows' union lists (and write o = 0,
//      lse = -inf for a row with nothing admitted), flagging each row as it is done;
//      every CTA lays out the CTA shares in its own shared memory (prefix sum of the
//      admitted counts over rows, as plan_kernel).
//   C  the tcgen05 decode of the CTA's share; the CTA that writes the last partial
//      slot of a (row, KV head) merges that row (decode_tc_body, fused hook).
// Flags carry tokens derived from the grid barrier's generation (distinct per
// launch), counters reset themselves (the last user sets them back to zero), and the
// admitted counts alternate between two halves by launch parity; so the workspace
// must be zero-filled once before the first call, and again after a call that
// latched ETA_DEVSTAT_TIMEOUT.
#include <cuda.h>
#include <math.h>

#include "combine_dev.cuh"
#include "decode_tc.cuh"
#include "eta_common.cuh"
#include "eta_host.h"
#include "meta_dev.cuh"
#include "screen_dev.cuh"
#include "screen_tc.cuh"
#include "tau_dev.cuh"
#include "tma_host.h"

namespace eta {
namespace fused {

constexpr int D = 128;
constexpr uint32_t kFlagWaitLimit = 1u << 20;
enum { kSyncArrive = 0, kSyncGen = 1, kSyncAbort = 2, kSyncItems = 3, kSyncWords = 4 };

struct StepParams {
  int Hq, Hkv, T_max, NB, NW, blk, ngroups, R;
  const eta_bf16_t* q;
  const float* W;
  const float* bias;
  const float* tau_const;
  const eta_bf16_t* K;
  const eta_bf16_t* V;
  const int32_t* lengths;
  int update_tail;
  void* cent;
  float* rmax;
  float* var;
  float* vardim;
  int32_t* cnt;
  int bound;
  float z, scale;
  float* tau;
  uint32_t* head_mask;
  int32_t* union_idx;
  int32_t* union_cnt;
  int32_t* head_cnt;
  float* o;
  float* lse;
  uint32_t* union_words;
  int32_t* ready;          // per row: this launch's token once released / compacted
  int32_t* pair_cnt;
  int32_t* adm_cnt;        // [2][R]: admitted blocks per row, one half per launch parity
  int32_t* sync;
  int32_t* status;
};

ETA_DEV bool aborted(const StepParams& sp) {
  return *reinterpret_cast<volatile int32_t*>(sp.sync + kSyncAbort) != 0;
}

ETA_DEV void fail(const StepParams& sp) {
  set_status(sp.status, ETA_DEVSTAT_TIMEOUT);
  atomicExch(sp.sync + kSyncAbort, 1);
}

// One warp: the ascending union list of row r from its union words.
template <int G>
ETA_DEV void compact_row(const StepParams& sp, int r) {
  const int lane = threadIdx.x & 31;
  int carry = 0;
  for (int base = 0; base < sp.NW; base += 32) {
    const int w = base + lane;
    const uint32_t word = w < sp.NW ? __ldcg(sp.union_words + (size_t)r * sp.NW + w) : 0u;
    const int c = __popc(word);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int excl = carry + incl - c;
    const int nw = min(32, sp.NW - base);
    for (int i = 0; i < nw; ++i) {
      const uint32_t wd = __shfl_sync(0xffffffffu, word, i);
      const int pos = __shfl_sync(0xffffffffu, excl, i) + __popc(wd & ((1u << lane) - 1u));
      if (((wd >> lane) & 1u) && ETA_IN_BOUNDS(pos, sp.NB, sp.status))
        sp.union_idx[(size_t)r * sp.NB + pos] = (base + i) * 32 + lane;
    }
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  const int b = r / sp.Hkv, g = r % sp.Hkv;
  const size_t qhead0 = (size_t)b * sp.Hq + (size_t)g * G;
  if (lane == 0) sp.union_cnt[r] = carry;
  if (sp.head_cnt) {
    for (int h = 0; h < G; ++h) {
      int s = 0;
      for (int w = lane; w < sp.NW; w += 32) s += __popc(__ldcg(sp.head_mask + (qhead0 + h) * sp.NW + w));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) sp.head_cnt[qhead0 + h] = s;
    }
  }
  if (carry == 0) {   // nothing admitted: the empty softmax of every head of the row
    for (int i = lane; i < G * D; i += 32) sp.o[qhead0 * D + i] = 0.f;
    if (lane < G) sp.lse[qhead0 + lane] = -INFINITY;
  }
}

// Counter + generation barrier over the grid (one thread per CTA calls it, after a
// CTA barrier).  Co-residency of all CTAs is guaranteed by the cooperative launch.
ETA_DEV bool grid_barrier(const StepParams& sp) {
  const int gen0 = ld_acquire_gpu(sp.sync + kSyncGen);
  __threadfence();
  if (atomicAdd(sp.sync + kSyncArrive, 1) == (int)gridDim.x - 1) {
    // every warp has made its last (failed) grab of a screening group
    atomicExch(sp.sync + kSyncItems, 0);
    atomicExch(sp.sync + kSyncArrive, 0);
    __threadfence();
    atomicAdd(sp.sync + kSyncGen, 1);
    return true;
  }
  for (uint32_t i = 0; i < kFlagWaitLimit; ++i) {
    if (ld_acquire_gpu(sp.sync + kSyncGen) != gen0) return true;
    if (aborted(sp)) return false;
    __nanosleep(64);
  }
  return false;
}

// Phase B shared-memory layout: one fp32 query slice per consumer warp, then a ring
// of stages, all in the decode ring (unused until phase C).  A stage holds one
// group: the [D][128] centroid tile (TMA tensor copy), the rmax / var / cnt slices
// and the G query rows (1-D bulk copies).
// Consumer c takes the items c, c + NC, ...; with NC <= NSB the producer can be at
// most one ring cycle ahead of any consumer, so every mbarrier parity a consumer
// waits for is unambiguous (with NC > NSB a consumer's first wait, for parity 1 on
// a barrier that has completed no phase yet, would return at once).
template <int G, int CF, bool VD>
struct PhaseB {
  static constexpr int CENT = 128 * 128 * (CF == 1 ? 2 : 4);
  static constexpr int OFF_RMAX = CENT;
  static constexpr int OFF_VAR = OFF_RMAX + 512;
  static constexpr int OFF_CNT = OFF_VAR + 512;
  static constexpr int OFF_Q = OFF_CNT + 512;
  static constexpr int QB = G * D * 2;
  static constexpr int SB = (OFF_Q + QB + 1023) / 1024 * 1024;
  static constexpr int NC_MAX = 5;                             // warps 0-3 and 5
  static constexpr int SLICE = (D * G + 2 * G) * 4;
  static constexpr int OFF_SLICES = 0;
  static constexpr int OFF_STAGES = (NC_MAX * SLICE + 1023) / 1024 * 1024;
  static constexpr int NSB_FIT = (tc::SM_P - OFF_STAGES) / SB;
  static constexpr int NSB = NSB_FIT < tc::kFuseStages ? NSB_FIT : tc::kFuseStages;
  static constexpr int NC = NC_MAX < NSB ? NC_MAX : NSB;
  static_assert(NSB >= 1, "one screening stage must fit");
};
constexpr int kGrab = 4;                  // screening groups taken per atomic

// One thread: bounded wait until *flag == token.
ETA_DEV bool wait_flag_thread(const int32_t* flag, int token, const StepParams& sp) {
  for (uint32_t i = 0; i < kFlagWaitLimit; ++i) {
    if (ld_acquire_gpu(flag) == token) return true;
    if (aborted(sp)) return false;
    __nanosleep(64);
  }
  return false;
}

ETA_DEV void set_abort(tc::FuseSmem* fs) { *reinterpret_cast<volatile int*>(&fs->abort) = 1; }

ETA_DEV void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Phase B on the tensor cores (bf16 centroids, not the per-dimension bound): the
// groups pass in order through a ring of screen_tc stages; warp 5 issues each group's
// q . c product into one of two TMEM accumulators and warps 0-3 turn it into the
// bound, the admit words and the row's admitted count (stc::issue_mma and
// stc::epilogue, the arithmetic of the standalone tensor-core screen).
using TcTile = stc::Tile<128>;
constexpr int kTcFit = tc::SM_P / (TcTile::BYTES + stc::META);
constexpr int kTcStages = kTcFit < tc::kFuseStages ? kTcFit : tc::kFuseStages;
constexpr int kTcMeta = kTcStages * TcTile::BYTES;     // the stages' metadata slots
static_assert(kTcStages >= 2, "two tensor-core screening stages must fit");
static_assert(kTcMeta + kTcStages * stc::META <= tc::SM_P, "screening ring in the decode ring");

template <int G>
ETA_DEV void phase_b_tc(unsigned char* smem, tc::FuseSmem* fs, const StepParams& sp,
                        const CUtensorMap* tmC, const CUtensorMap* tmQ, int32_t* adm_now,
                        int tok_released) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int items = sp.R * sp.ngroups;
  const uint32_t tmem = fs->btmem;
  if (warp == tc::NWARP_SM) {
    // ------------------------------------------------------------ TMA producer
    if (lane != 0) return;
    bool ok = true;
    int k = 0, cur_r = -1, nvalid = 0;
    float ts[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int batch = atomicAdd(sp.sync + kSyncItems, kGrab);
    while (ok && batch < items) {
      const int next = atomicAdd(sp.sync + kSyncItems, kGrab);   // in flight meanwhile
      const int end = min(batch + kGrab, items);
      for (int it = batch; it < end; ++it) {
        const int r = it / sp.ngroups, grp = it % sp.ngroups;
        const int b = r / sp.Hkv, g = r % sp.Hkv;
        const size_t qhead0 = (size_t)b * sp.Hq + (size_t)g * G;
        if (r != cur_r) {
          // the row's tail metadata and thresholds are released by its prologue
          if (!wait_flag_thread(sp.ready + r, tok_released, sp)) { ok = false; break; }
          fence_proxy_async_global();       // TMA reads what the release published
          cur_r = r;
          const int len = min(max(sp.lengths[b], 0), sp.T_max);
          nvalid = (len + sp.blk - 1) / sp.blk;
#pragma unroll
          for (int h = 0; h < G; ++h) ts[h] = __ldcg(sp.tau + qhead0 + h);
        }
        const int s = k % kTcStages;
        if (!mbar_wait(&fs->bempty[s], ((uint32_t)(k / kTcStages) & 1u) ^ 1u, &fs->abort)) {
          ok = false;
          break;
        }
        tc::FuseItem& rec = fs->item[s];
        rec.r = r; rec.grp = grp; rec.nvalid = nvalid; rec.flags = 0;
#pragma unroll
        for (int h = 0; h < G; ++h) rec.ts[h] = ts[h];
        unsigned char* st = smem + s * TcTile::BYTES;
        unsigned char* mt = smem + kTcMeta + s * stc::META;
        const int j0 = grp * stc::GB;
        const uint32_t nb4 = (uint32_t)min(stc::GB, sp.NB - j0) * 4u;
        const bool pv = sp.bound == ETA_BOUND_PROB;
        mbar_arrive_expect_tx(&fs->bfull[s], (uint32_t)TcTile::BYTES + nb4 * (pv ? 3u : 2u));
        tc::tma_load_2d(st + TcTile::OFF_C0, tmC, j0, r * D, &fs->bfull[s]);
        tc::tma_load_2d(st + TcTile::OFF_C1, tmC, j0 + 64, r * D, &fs->bfull[s]);
        const int qrow = b * sp.Hq + g * G;
        tc::tma_load_2d(st + TcTile::OFF_Q0, tmQ, 0, qrow, &fs->bfull[s]);
        tc::tma_load_2d(st + TcTile::OFF_Q1, tmQ, 64, qrow, &fs->bfull[s]);
        const size_t rj = (size_t)r * sp.NB + j0;
        bulk_g2s(mt + stc::M_RMAX, sp.rmax + rj, nb4, &fs->bfull[s]);
        if (pv) bulk_g2s(mt + stc::M_VAR, sp.var + rj, nb4, &fs->bfull[s]);
        bulk_g2s(mt + stc::M_CNT, sp.cnt + rj, nb4, &fs->bfull[s]);
        ++k;
      }
      batch = next;
    }
    if (ok) {
      // one end marker: the MMA warp and the epilogue warps read every stage in order
      const int s = k % kTcStages;
      if (mbar_wait(&fs->bempty[s], ((uint32_t)(k / kTcStages) & 1u) ^ 1u, &fs->abort)) {
        fs->item[s].flags = 1;
        mbar_arrive(&fs->bfull[s]);
      } else {
        ok = false;
      }
    }
    if (!ok) {
      fail(sp);
      set_abort(fs);
      // every copy issued lands before the ring is reused or the CTA exits
      for (int kk = max(0, k - kTcStages); kk < k; ++kk)
        mbar_wait(&fs->bfull[kk % kTcStages], (uint32_t)(kk / kTcStages) & 1u, nullptr);
    }
  } else if (warp == tc::NWARP_SM + 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane != 0) return;
    bool ok = true;
    for (int k = 0;; ++k) {
      const int s = k % kTcStages, b = k & 1;
      if (!mbar_wait(&fs->bfull[s], (uint32_t)(k / kTcStages) & 1u, &fs->abort)) {
        ok = false;
        break;
      }
      if (fs->item[s].flags) break;
      if (!mbar_wait(&fs->bacc_free[b], ((uint32_t)(k >> 1) & 1u) ^ 1u, &fs->abort)) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      stc::issue_mma<D>(tmem + b * stc::kAccCols, smem + s * TcTile::BYTES);
      tc::mma_commit(&fs->bacc_full[b]);
    }
    if (!ok) {
      fail(sp);
      set_abort(fs);
    }
    tc::mma_commit(&fs->bfin);             // every MMA issued completes before TMEM is freed
    mbar_wait(&fs->bfin, 0, nullptr);
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-3)
    const uint32_t lane_sel = (uint32_t)(warp * 32) << 16;
    int cur_r = -1;
    float qn[G], ts[G];
    for (int k = 0;; ++k) {
      const int s = k % kTcStages, b = k & 1;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&fs->bfull[s],
                                                         (uint32_t)(k / kTcStages) & 1u,
                                                         &fs->abort));
      if (!got) {
        if (lane == 0) { fail(sp); set_abort(fs); }
        break;
      }
      const tc::FuseItem rec = fs->item[s];
      __syncwarp();
      if (rec.flags) {
        if (lane == 0) mbar_arrive(&fs->bempty[s]);
        break;
      }
      const int r = rec.r, bb = r / sp.Hkv, g = r % sp.Hkv;
      const size_t qhead0 = (size_t)bb * sp.Hq + (size_t)g * G;
      if (r != cur_r) {
        stc::query_norms_staged<D, G>(smem + s * TcTile::BYTES, qn);
        cur_r = r;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&fs->bacc_full[b], (uint32_t)(k >> 1) & 1u,
                                             &fs->abort))) {
        if (lane == 0) { fail(sp); set_abort(fs); }
        break;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) ts[h] = rec.ts[h];
      tc::tc_fence_after();
      float dot[16];
      tc::tmem_ld16(tmem + b * stc::kAccCols + lane_sel, dot);
      tc::tc_fence_before();
      const stc::BlockMeta bm = stc::block_meta<D>(smem + kTcMeta + s * stc::META,
                                                sp.bound == ETA_BOUND_PROB, sp.z, sp.NB, rec.grp);
      __syncwarp();
      if (lane == 0) {                      // accumulator and stage are no longer read
        mbar_arrive(&fs->bacc_free[b]);
        mbar_arrive(&fs->bempty[s]);
      }
      const int adm = stc::epilogue<G>(dot, bm, sp.scale, sp.NB, sp.NW, rec.grp, r, qhead0, qn,
                                       ts, rec.nvalid, sp.head_mask, sp.union_words, nullptr);
      if (lane == 0 && adm) atomicAdd(adm_now + r, adm);
    }
  }
}

template <int G, int CF, bool VD, bool TCS>
__global__ void __launch_bounds__(tc::NT, 1)
step_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
            const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC,
            const StepParams sp, const tc::TcParams tp) {
  using PB = PhaseB<G, CF, VD>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  tc::FuseSmem* fs = reinterpret_cast<tc::FuseSmem*>(smem + tc::SM_FUSE);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < (TCS ? kTcStages : PB::NSB); ++s) {
      mbar_init(&fs->bfull[s], 1);
      mbar_init(&fs->bempty[s], TCS ? tc::NWARP_SM : 1);   // TCS: the epilogue warps release
    }
    if constexpr (TCS) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(&fs->bacc_full[b], 1);
        mbar_init(&fs->bacc_free[b], tc::NWARP_SM);
      }
      mbar_init(&fs->bfin, 1);
    }
    fs->abort = 0;
    // the barrier generation cannot move before every CTA has arrived, so all CTAs
    // read the same value here: it names this launch's flag tokens
    fs->gen0 = ld_acquire_gpu(sp.sync + kSyncGen);
    fence_mbar_init();
  }
  if constexpr (TCS) {
    // phase B's accumulators (freed before phase C allocates its own; no relinquish)
    if (warp == tc::NWARP_SM + 1)
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(&fs->btmem)),
                   "r"(32));
    tc::tc_fence_before();
  }
  __syncthreads();
  if constexpr (TCS) tc::tc_fence_after();
  const int gen0 = fs->gen0;
  const int tok_released = 2 * gen0 + 1, tok_compacted = 2 * gen0 + 2;
  int32_t* adm_now = sp.adm_cnt + (gen0 & 1) * sp.R;
  int32_t* adm_next = sp.adm_cnt + ((gen0 & 1) ^ 1) * sp.R;

  // ---------------------------------------------------------------- A: row prologue
  // warps 0-3 refresh the tail block while warps 4-5 compute the thresholds
  {
    auto* tail = reinterpret_cast<TailScratch<D, CF>*>(smem);
    auto* red = reinterpret_cast<float(*)[G]>(smem + sizeof(TailScratch<D, CF>));
    for (int r = blockIdx.x; r < sp.R; r += gridDim.x) {
      const int b = r / sp.Hkv, g = r % sp.Hkv;
      if (warp < 4) {
        if (sp.update_tail)
          meta_tail_block<D, CF, 4>(r, sp.Hkv, sp.T_max, sp.blk, sp.NB, sp.K, sp.V, sp.lengths,
                                    sp.cent, sp.rmax, sp.var, sp.cnt, nullptr, sp.vardim,
                                    sp.status, *tail,
                                    warp, [] { named_bar_sync(1, 128); });
      } else if (sp.tau_const) {
        const int lt = threadIdx.x - 128;
        if (lt < G) sp.tau[(size_t)b * sp.Hq + g * G + lt] = sp.tau_const[g * G + lt];
      } else {
        const bool bad = tau_group<G, 2>(sp.Hq, D, b, g * G, sp.q, sp.W, sp.bias, red, sp.tau,
                                         warp - 4, [] { named_bar_sync(2, 64); });
        if (bad && g == 0) set_status(sp.status, ETA_DEVSTAT_NONFINITE_Q);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        adm_next[r] = 0;                 // the next launch counts into the other half
        __threadfence();
        st_release_gpu(sp.ready + r, tok_released);
      }
    }
    tc::fence_async_smem();     // the scratch is overwritten by TMA next
    __syncthreads();
  }

  // ---------------------------------------------------------------- B: screening
  // warp 4 (one thread) stages groups with TMA; warps 0-3 and 5 screen them
  const int items = sp.R * sp.ngroups;
  if constexpr (TCS) {
    phase_b_tc<G>(smem, fs, sp, &tmC, &tmQ, adm_now, tok_released);
    // every accumulator has been read (the MMA warp waited for its last MMA)
    tc::tc_fence_before();
    __syncthreads();
    if (warp == tc::NWARP_SM + 1) {
      __syncwarp();
      tc::tc_fence_after();
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(fs->btmem),
                   "r"(32));
    }
  } else if (warp == tc::NWARP_SM) {
    if (lane == 0) {
      bool ok = true;
      int k = 0, cur_r = -1, nvalid = 0;
      float ts[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      int batch = atomicAdd(sp.sync + kSyncItems, kGrab);
      while (ok && batch < items) {
        const int next = atomicAdd(sp.sync + kSyncItems, kGrab);   // in flight meanwhile
        const int end = min(batch + kGrab, items);
        for (int it = batch; it < end; ++it) {
          const int r = it / sp.ngroups, grp = it % sp.ngroups;
          const int b = r / sp.Hkv, g = r % sp.Hkv;
          const size_t qhead0 = (size_t)b * sp.Hq + (size_t)g * G;
          if (r != cur_r) {
            // the row's tail metadata and thresholds are released by its prologue
            if (!wait_flag_thread(sp.ready + r, tok_released, sp)) { ok = false; break; }
            fence_proxy_async_global();       // TMA reads what the release published
            cur_r = r;
            const int len = min(max(sp.lengths[b], 0), sp.T_max);
            nvalid = (len + sp.blk - 1) / sp.blk;
#pragma unroll
            for (int h = 0; h < G; ++h) ts[h] = __ldcg(sp.tau + qhead0 + h);
          }
          const int s = k % PB::NSB;
          if (!mbar_wait(&fs->bempty[s], ((uint32_t)(k / PB::NSB) & 1u) ^ 1u, &fs->abort)) {
            ok = false;
            break;
          }
          tc::FuseItem& rec = fs->item[s];
          rec.r = r; rec.grp = grp; rec.nvalid = nvalid; rec.flags = 0;
#pragma unroll
          for (int h = 0; h < G; ++h) rec.ts[h] = ts[h];
          unsigned char* st = smem + PB::OFF_STAGES + s * PB::SB;
          const int j0 = grp * kScreenGroupBlocks;
          const uint32_t nb4 = (uint32_t)min(kScreenGroupBlocks, sp.NB - j0) * 4u;
          const bool pv = sp.bound == ETA_BOUND_PROB;
          mbar_arrive_expect_tx(&fs->bfull[s], (uint32_t)(PB::CENT + PB::QB) +
                                                   nb4 * (pv ? 3u : 2u));
          tc::tma_load_2d(st, &tmC, j0, r * D, &fs->bfull[s]);
          const size_t rj = (size_t)r * sp.NB + j0;
          bulk_g2s(st + PB::OFF_RMAX, sp.rmax + rj, nb4, &fs->bfull[s]);
          if (pv) bulk_g2s(st + PB::OFF_VAR, sp.var + rj, nb4, &fs->bfull[s]);
          bulk_g2s(st + PB::OFF_CNT, sp.cnt + rj, nb4, &fs->bfull[s]);
          bulk_g2s(st + PB::OFF_Q, sp.q + qhead0 * D, PB::QB, &fs->bfull[s]);
          ++k;
        }
        batch = next;
      }
      if (!ok) {
        fail(sp);
        set_abort(fs);
      }
      // one end marker per consumer
      for (int c = 0; c < PB::NC && ok; ++c, ++k) {
        const int s = k % PB::NSB;
        if (!mbar_wait(&fs->bempty[s], ((uint32_t)(k / PB::NSB) & 1u) ^ 1u, &fs->abort)) {
          fail(sp);
          set_abort(fs);
          break;
        }
        fs->item[s].flags = 1;
        mbar_arrive(&fs->bfull[s]);
      }
    }
  } else if ((warp < 4 ? warp : 4) < PB::NC) {
    const int c = warp < 4 ? warp : 4;                 // consumer index
    float* qs = reinterpret_cast<float*>(smem + PB::OFF_SLICES + c * PB::SLICE);
    float* qn = qs + D * G;
    float* ts = qn + G;
    int staged_r = -1;                                  // the row whose query is in qs
    for (int k = c;; k += PB::NC) {
      const int s = k % PB::NSB;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&fs->bfull[s],
                                                         (uint32_t)(k / PB::NSB) & 1u,
                                                         &fs->abort));
      if (!got) {
        if (lane == 0) { fail(sp); set_abort(fs); }
        break;
      }
      const tc::FuseItem rec = fs->item[s];
      __syncwarp();
      if (lane == 0) {
        // an end marker's stage is released too: with fewer stages than consumers the
        // producer reuses it for the next marker
        if (rec.flags) mbar_arrive(&fs->bempty[s]);
      }
      if (rec.flags) break;
      const int r = rec.r, b = r / sp.Hkv, g = r % sp.Hkv;
      const size_t qhead0 = (size_t)b * sp.Hq + (size_t)g * G;
      const unsigned char* st = smem + PB::OFF_STAGES + s * PB::SB;
      if (r != staged_r) {
        const eta_bf16_t* qst = reinterpret_cast<const eta_bf16_t*>(st + PB::OFF_Q);
        for (int i = lane; i < G * D; i += 32) qs[(i % D) * G + i / D] = bf16_to_f(qst[i]);
        __syncwarp();
        for (int h = 0; h < G; ++h) {
          const float nrm = query_norm<D, G>(qs, h);
          if (lane == 0) {
            qn[h] = nrm;
            ts[h] = rec.ts[h];
          }
        }
        __syncwarp();
        staged_r = r;
      }
      SmemMeta<CF, VD> src;
      src.tile = st;
      const int jl = min(rec.grp * kScreenGroupBlocks + lane * kScreenVW, sp.NB - kScreenVW);
      src.vdp = VD ? reinterpret_cast<const float4*>(sp.vardim + (size_t)r * D * sp.NB + jl)
                   : nullptr;
      src.rowvd = (size_t)sp.NB / 4;
      src.rmax = reinterpret_cast<const float*>(st + PB::OFF_RMAX);
      src.var = reinterpret_cast<const float*>(st + PB::OFF_VAR);
      src.cnt = reinterpret_cast<const int32_t*>(st + PB::OFF_CNT);
      src.lane = lane;
      const int adm = screen_group_from<D, G, CF, VD, kScreenLoadBatch>(
          src, sp.NB, sp.NW, rec.grp, r, qhead0, qs, qn, ts, sp.bound, sp.z, sp.scale,
          rec.nvalid, sp.head_mask, sp.union_words, nullptr);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&fs->bempty[s]);
        if (adm) atomicAdd(adm_now + r, adm);
      }
    }
  }
  tc::fence_async_smem();       // generic reads and writes of the ring before phase C's TMA

  // ---------------------------------------------------------------- grid barrier 1
  __shared__ int s_ok;
  auto grid_sync = [&]() -> bool {
    __syncthreads();
    if (threadIdx.x == 0) {
      bool ok = grid_barrier(sp);
      if (!ok) fail(sp);
      ok = ok && !aborted(sp);
      __threadfence();
      s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
  };
  if (!grid_sync()) return;

  // ---------------------------------------------------------------- B2: union lists
  // every head and union word is written: warps compact rows (row r on CTA r mod P),
  // each row flagged as it is done; the decode waits for the flags of its own rows
  for (int r = blockIdx.x + warp * gridDim.x; r < sp.R; r += (tc::NT / 32) * gridDim.x) {
    compact_row<G>(sp, r);
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release_gpu(sp.ready + r, tok_compacted);
  }

  // ---------------------------------------------------------------- the share plan
  // every CTA lays out the shares itself, from the screening's own counts
  int* row_off = reinterpret_cast<int*>(smem + tc::SM_ROWOFF);
  tc::plan_local(adm_now, sp.R, sp.NB, row_off, fs, sp.status);

  // ---------------------------------------------------------------- C: decode + merge
  tc::TcParams tpl = tp;
  tpl.row_off = row_off;
  tpl.plan = fs->plan;
  tpl.cta_row = &fs->cta_row;
  tc::FuseCtx fx;
  fx.pair_cnt = sp.pair_cnt;
  fx.o = sp.o;
  fx.lse = sp.lse;
  fx.ready = sp.ready;
  fx.token = tok_compacted;
  tc::decode_tc_body<G, false, true, true>(smem, &tmK, &tmV, &tmQ, tpl, fx);
}

struct StepWs {
  size_t part_ml, part_o, words, counters, total;
};

inline StepWs step_ws(const eta_dims_t* d, int P) {
  const size_t R = (size_t)d->B * d->Hkv, G = d->Hq / d->Hkv;
  const size_t NW = (size_t)num_words(d);
  StepWs w;
  size_t x = 0;
  w.part_ml = x;  x = align_up(x + ((size_t)P + R) * G * 2 * 4, 256);
  w.part_o = x;   x = align_up(x + ((size_t)P + R) * G * d->d * 4, 256);
  w.words = x;    x = align_up(x + R * NW * 4, 256);
  // ready[R], pair_cnt[R], adm_cnt[2][R], sync[kSyncWords]
  w.counters = x; x = align_up(x + (4 * R + kSyncWords) * 4, 256);
  w.total = x;
  return w;
}

template <int G, int CF, bool VD, bool TCS>
eta_status_t launch_step(const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mq,
                         const CUtensorMap& mc, const StepParams& sp,
                         const tc::TcParams& tp, int P, cudaStream_t s) {
  auto kern = step_kernel<G, CF, VD, TCS>;
  if (!set_smem_once<step_kernel<G, CF, VD, TCS>>(tc::FUSED_SMEM_BYTES)) return ETA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P);
  cfg.blockDim = dim3(tc::NT);
  cfg.dynamicSmemBytes = tc::FUSED_SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mk, mv, mq, mc, sp, tp) == cudaSuccess
             ? ETA_OK
             : ETA_ERR_CUDA;
}

template <int CF, bool VD, bool TCS = false>
eta_status_t dispatch_g(int G, const CUtensorMap& mk, const CUtensorMap& mv,
                        const CUtensorMap& mq, const CUtensorMap& mc, const StepParams& sp,
                        const tc::TcParams& tp, int P, cudaStream_t s) {
  switch (G) {
    case 1: return launch_step<1, CF, VD, TCS>(mk, mv, mq, mc, sp, tp, P, s);
    case 2: return launch_step<2, CF, VD, TCS>(mk, mv, mq, mc, sp, tp, P, s);
    case 4: return launch_step<4, CF, VD, TCS>(mk, mv, mq, mc, sp, tp, P, s);
    case 8: return launch_step<8, CF, VD, TCS>(mk, mv, mq, mc, sp, tp, P, s);
  }
  return ETA_ERR_UNSUPPORTED;
}

// Phase A scratch fits in the decode ring, which is unused until phase C.
static_assert(sizeof(TailScratch<128, 1>) + kTauVirtWarps * 8 * 4 <= tc::SM_P, "phase A scratch");

inline int step_grid() {
  const int n = sm_count();
  return n > 0 ? n : 1;
}

}  // namespace fused
}  // namespace eta

using namespace eta;

extern "C" size_t eta_decode_step_workspace_size(const eta_dims_t* dims) {
  if (check_dims(dims, /*rows_in_grid_y=*/false) != ETA_OK) return 0;
  return fused::step_ws(dims, fused::step_grid()).total;
}

extern "C" eta_status_t eta_decode_step(
    const eta_dims_t* dims, const eta_bf16_t* q, const float* W, const float* bias,
    const float* tau_const, const eta_bf16_t* K, const eta_bf16_t* V, const int32_t* lengths,
    int32_t update_tail, eta_cent_format_t cent_format, void* cent, float* rmax, float* var,
    float* vardim, int32_t* cnt, eta_bound_t bound, float z, float T, float scale, float* tau,
    uint32_t* head_mask, int32_t* union_idx, int32_t* union_cnt, int32_t* head_cnt, float* o,
    float* lse, void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  eta_status_t st = check_dims(dims, /*rows_in_grid_y=*/false);
  if (st != ETA_OK) return st;
  if (!q || !K || !V || !lengths || !cent || !rmax || !var || !cnt || !tau || !head_mask ||
      !union_idx || !union_cnt || !o || !lse)
    return ETA_ERR_INVALID_ARG;
  if (!tau_const && !W) return ETA_ERR_INVALID_ARG;
  if (cent_format != ETA_CENT_F32 && cent_format != ETA_CENT_BF16) return ETA_ERR_INVALID_ARG;
  if (bound != ETA_BOUND_EXACT && bound != ETA_BOUND_PROB && bound != ETA_BOUND_PROB_DIM)
    return ETA_ERR_INVALID_ARG;
  if (bound != ETA_BOUND_EXACT && !(z >= 0.f)) return ETA_ERR_INVALID_ARG;
  if (bound == ETA_BOUND_PROB_DIM && !vardim) return ETA_ERR_INVALID_ARG;
  if (!(T >= 0.f) || isinf(T)) return ETA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(cent) || !aligned16(rmax) ||
      !aligned16(var) || !aligned16(cnt) || (vardim && !aligned16(vardim)))
    return ETA_ERR_INVALID_ARG;
  // the tensor-core decode (d = 128, 32-bit TMA row coordinates) and the vector screen
  const int NB = num_blocks(dims);
  // (TMA row strides of the metadata tiles are multiples of 16 bytes: NB % 8 for bf16)
  if (dims->d != 128 || NB % (cent_format == ETA_CENT_BF16 ? 8 : 4) != 0)
    return ETA_ERR_UNSUPPORTED;
  if ((uint64_t)dims->B * dims->Hkv * dims->T_max >= (1ull << 31)) return ETA_ERR_UNSUPPORTED;
  if (dims->B * dims->Hkv > tc::kFusedMaxRows) return ETA_ERR_UNSUPPORTED;
  const int P = fused::step_grid();
  const fused::StepWs L = fused::step_ws(dims, P);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return ETA_ERR_WORKSPACE;
  if (scale == 0.f) scale = 1.f / sqrtf((float)dims->d);

  char* w = static_cast<char*>(ws);
  const int R = dims->B * dims->Hkv, G = dims->Hq / dims->Hkv;
  int32_t* counters = reinterpret_cast<int32_t*>(w + L.counters);
  fused::StepParams sp;
  sp.Hq = dims->Hq; sp.Hkv = dims->Hkv; sp.T_max = dims->T_max; sp.NB = NB;
  sp.NW = num_words(dims); sp.blk = dims->blk;
  sp.ngroups = (NB + kScreenGroupBlocks - 1) / kScreenGroupBlocks; sp.R = R;
  sp.q = q; sp.W = W; sp.bias = bias; sp.tau_const = tau_const;
  sp.K = K; sp.V = V; sp.lengths = lengths; sp.update_tail = update_tail ? 1 : 0;
  sp.cent = cent; sp.rmax = rmax; sp.var = var; sp.vardim = vardim; sp.cnt = cnt;
  sp.bound = (int)bound; sp.z = z; sp.scale = scale;
  sp.tau = tau; sp.head_mask = head_mask; sp.union_idx = union_idx; sp.union_cnt = union_cnt;
  sp.head_cnt = head_cnt; sp.o = o; sp.lse = lse;
  sp.union_words = reinterpret_cast<uint32_t*>(w + L.words);
  sp.ready = counters;
  sp.pair_cnt = counters + R;
  sp.adm_cnt = counters + 2 * R;
  sp.sync = counters + 4 * R;
  sp.status = dev_status;

  tc::TcParams tp;
  tp.Hq = dims->Hq; tp.Hkv = dims->Hkv; tp.T_max = dims->T_max; tp.NB = NB; tp.blk = dims->blk;
  tp.scale = scale;
  tp.invT = T == 0.f ? -1.f : 1.f / T;
  tp.tau = tau; tp.lengths = lengths; tp.union_idx = union_idx;
  tp.row_off = nullptr; tp.cta_row = nullptr; tp.plan = nullptr;   // per CTA, in shared memory
  tp.part_o = reinterpret_cast<float*>(w + L.part_o);
  tp.part_ml = reinterpret_cast<float*>(w + L.part_ml);
  tp.status = dev_status;
  tp.R = R;
  tp.counts = nullptr; tp.row_off_g = nullptr; tp.plan_g = nullptr;   // the plan is per CTA

  CUtensorMap mk, mv, mq, mc;
  const uint64_t kv_rows = (uint64_t)dims->B * dims->Hkv * dims->T_max;
  const bool bf = cent_format == ETA_CENT_BF16, vd = bound == ETA_BOUND_PROB_DIM;
  const uint64_t meta_rows = (uint64_t)R * dims->d;     // [R * d, NB], dimension-major
  const uint32_t box = kScreenGroupBlocks;
  // the screening takes the tensor cores exactly when eta_screen would
  const bool tcs = tc_screen_applies(dims, (int)cent_format, (int)bound);
  if (!make_map(&mk, K, kv_rows, 64) || !make_map(&mv, V, kv_rows, 64) ||
      !make_map(&mq, q, (uint64_t)dims->B * dims->Hq, 16))
    return ETA_ERR_CUDA;
  if (tcs ? !make_map_bf16_swz(&mc, cent, NB, meta_rows, (uint64_t)NB * 2, 128)
          : !make_map_plain(&mc, cent, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                          : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                            NB, meta_rows, (uint64_t)NB * (bf ? 2 : 4), box, 128))
    return ETA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (tcs) return fused::dispatch_g<1, false, true>(G, mk, mv, mq, mc, sp, tp, P, s);
  if (bf) return vd ? fused::dispatch_g<1, true>(G, mk, mv, mq, mc, sp, tp, P, s)
                    : fused::dispatch_g<1, false>(G, mk, mv, mq, mc, sp, tp, P, s);
  return vd ? fused::dispatch_g<0, true>(G, mk, mv, mq, mc, sp, tp, P, s)
            : fused::dispatch_g<0, false>(G, mk, mv, mq, mc, sp, tp, P, s);
}
