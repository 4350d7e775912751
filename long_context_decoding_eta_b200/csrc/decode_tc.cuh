// Gated block-sparse decode attention on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in TMEM), d = 128.
//
// Same method and same work split as decode_kernel (decode.cu): the admitted
// blocks of all (row, KV head) pairs are cut into equal contiguous shares, one
// per CTA; each share is streamed through a ring of shared-memory stages and every
// (row, KV head) segment of the share ends in one partial (m, l, o) slot that
// combine_kernel merges.  What changes is the per-stage math:
//
//   stage     = up to 128 keys of one (row, KV head): two 64-key sub-tiles (one
//               64-key block each, or the two halves of a 128-key block), loaded by
//               TMA tensor copies with 128-byte swizzle (box 64 dims x 64 keys), plus
//               the 16 query rows starting at the group's first head (box 64 x 16).
//   S^T = K Q^T   tcgen05.mma kind::f16, M = 128 keys, N = 16 (G heads used), K = d,
//               bf16 x bf16 -> fp32 in TMEM (exact products, fp32 sums).
//   softmax   4 warps, thread = key (= TMEM lane): gate s * sigmoid((s - tau) / T)
//               or the hard gate, running max per head shared through shared memory,
//               p = exp(s' - m); P^T written to shared memory as bf16 hi + lo
//               (hi = bf16(p), lo = bf16(p - hi)) in columns [0,G) and [G,2G), so
//               P V keeps ~16 mantissa bits.
//   O^T = V^T P^T tcgen05.mma, M = 128 dims (A = V read MN-major from the same
//               swizzled tile), N = 16, K = 128 keys, fresh accumulator per stage.
//   correction the same 4 warps, thread = dim: o = o * alpha + (O[hi] + O[lo]).
//
// Warp roles (192 threads): warps 0-3 softmax / correction, warp 4 TMA producer,
// warp 5 MMA issuer (also allocates and frees 64 TMEM columns).  S and O each
// have two TMEM buffers so QK^T of stage i+1 and PV of stage i overlap the
// softmax of stage i.  Every mbarrier wait is bounded.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "combine_dev.cuh"
#include "eta_common.cuh"

namespace eta {
namespace tc {

constexpr int D = 128;
constexpr int kTileKeys = 128;
constexpr int kSubKeys = 64;
constexpr int NSTAGE = 3;
constexpr int HALF = kTileKeys * 128;              // one 64-dim half of a 128-key tile: 16 KB
constexpr int SUB_HALF = kSubKeys * 128;            // one TMA box of 64 keys x 64 dims: 8 KB
constexpr int QHALF = 16 * 128;                     // 16 query rows x 64 dims: 2 KB
constexpr int OFF_K0 = 0, OFF_K1 = HALF, OFF_V0 = 2 * HALF, OFF_V1 = 3 * HALF;
constexpr int OFF_Q0 = 4 * HALF, OFF_Q1 = 4 * HALF + QHALF;
constexpr int STAGE_BYTES = 4 * HALF + 2 * QHALF;   // 68 KB
constexpr int PBUF = 2 * 16 * 128;                  // P^T: 2 column groups x 16 key groups x 128 B
constexpr int SM_STAGES = 0;
constexpr int SM_P = NSTAGE * STAGE_BYTES;
constexpr int SM_MISC = SM_P + 2 * PBUF;
constexpr int NWARP_SM = 4;                         // softmax / correction warps
constexpr int NT = (NWARP_SM + 2) * 32;
constexpr int kTmemCols = 64;                       // S: 2 x 16, O: 2 x 16

struct TcStage {
  int row;
  int t0[2];
  int nv[2];
  int flags;
  int pad[2];
};

struct TcMisc {
  uint64_t full[NSTAGE], empty[NSTAGE];
  uint64_t s_full[2], s_free[2], p_full[2], o_full[2], o_free[2];
  uint64_t fin;
  TcStage info[NSTAGE];
  float red[2][NWARP_SM][8];
  float lsum[NWARP_SM][8];
  uint32_t tmem_base;
  int abort_flag;
};
constexpr int SMEM_BYTES = SM_MISC + (int)sizeof(TcMisc) + 1024;   // + alignment slack

// The fused decode step's own shared state, after the decode's barriers: the
// screening ring's barriers and item records, and the merge scratch.
constexpr int kFuseStages = 6;
struct FuseItem {
  int r, grp, nvalid, flags;
  float ts[8];
};
struct FuseSmem {
  uint64_t bfull[kFuseStages], bempty[kFuseStages];
  uint64_t bacc_full[2], bacc_free[2], bfin;   // tensor-core screening's accumulators
  uint32_t btmem;                               // and their TMEM columns
  FuseItem item[kFuseStages];
  CombineScratch<8> cs;   // sized for the largest group
  int last;
  int abort;
  int gen0;               // grid-barrier generation at launch: names this launch's flags
  int plan[2];            // this CTA's copy of the share plan: total, share length
  int cta_row;            // the first (row, KV head) of this CTA's share
  int wsum[NT / 32];
};
constexpr int SM_FUSE = (SM_MISC + (int)sizeof(TcMisc) + 15) / 16 * 16;
// the fused step keeps the prefix sum of admitted blocks over rows in shared memory
constexpr int kFusedMaxRows = 2048;
constexpr int SM_ROWOFF = (SM_FUSE + (int)sizeof(FuseSmem) + 15) / 16 * 16;
constexpr int FUSED_SMEM_BYTES = SM_ROWOFF + (kFusedMaxRows + 1) * 4 + 1024;
static_assert(FUSED_SMEM_BYTES <= 227 * 1024, "fused step shared memory");

// Instruction descriptor, kind::f16: D fp32, A/B bf16, M = 128, N = 16.
constexpr uint32_t kIdescBase = (1u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) |
                                ((128u >> 4) << 24);
constexpr uint32_t kIdescQK = kIdescBase;                              // A, B K-major
constexpr uint32_t kIdescPV = kIdescBase | (1u << 15) | (1u << 16);    // A, B MN-major

// Shared-memory matrix descriptor (version 1, base offset 0).
ETA_DEV uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}
constexpr uint32_t kSwizzle128 = 2, kSwizzleNone = 0;

ETA_DEV void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

ETA_DEV void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::
                   "r"(smem_u32(bar))
               : "memory");
}

ETA_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
ETA_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
ETA_DEV void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

ETA_DEV void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

ETA_DEV void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

struct TcParams {
  int Hq, Hkv, T_max, NB, blk;
  float scale, invT;   // invT < 0: hard gate
  const float* tau;
  const int32_t* lengths;
  const int32_t* union_idx;
  const int32_t* row_off;
  const int32_t* cta_row;
  const int32_t* plan;
  float* part_o;
  float* part_ml;
  int32_t* status;
  // plan in the kernel (standalone decode): the R per-pair admitted counts it is laid
  // out from, and where CTA 0 publishes row_off[0..R] and {total, share} for the
  // combine launch that follows
  int R;
  const int32_t* counts;
  int32_t* row_off_g;
  int32_t* plan_g;
};

// In-kernel merge of the fused step: the CTA that writes the last partial slot of
// a (row, KV head) pair (counted in pair_cnt, which it resets) merges the pair.
struct FuseCtx {
  int32_t* pair_cnt;
  float* o;
  float* lse;
  const int32_t* ready;   // ready[row] == token once the row's union list is written
  int token;
};

// The fused step: every CTA lays out the CTA shares itself (prefix sum of per-row
// admitted counts, exactly as plan_kernel) into its shared memory: row_off[0..R], fs->plan = {total,
// share length}, fs->cta_row = the row holding position blockIdx * share.  Every
// thread of the CTA calls it.
ETA_DEV void plan_local(const int32_t* counts, int R, int NB, int* row_off, FuseSmem* fs,
                        int32_t* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int carry = 0;
  for (int base = 0; base < R; base += NT) {
    const int r = base + threadIdx.x;
    int c = r < R ? __ldcg(counts + r) : 0;
    if (c < 0 || c > NB) {
      set_status(status, ETA_DEVSTAT_BAD_BLOCK);
      c = min(max(c, 0), NB);
    }
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) fs->wsum[warp] = incl;
    __syncthreads();
    int wpre = 0, total = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
      const int v = fs->wsum[w];
      if (w < warp) wpre += v;
      total += v;
    }
    if (r < R) row_off[r] = carry + wpre + incl - c;
    carry += total;
    __syncthreads();
  }
  int chunk = (carry + gridDim.x - 1) / gridDim.x;
  if (chunk < kMinChunk) chunk = kMinChunk;
  if (threadIdx.x == 0) {
    row_off[R] = carry;
    fs->plan[0] = carry;
    fs->plan[1] = chunk;
    fs->cta_row = 0;
  }
  __syncthreads();
  const int a = blockIdx.x * chunk;
  for (int r = threadIdx.x; r < R; r += NT) {
    const int off = row_off[r], c = row_off[r + 1] - off;
    if (c > 0 && off <= a && a < off + c) fs->cta_row = r;
  }
  __syncthreads();
}

// The decode of one CTA share.  `smem` is the CTA's dynamic shared memory aligned
// to 1024 bytes.  Every thread of the CTA calls it.
// LOCAL (the fused step): the plan, the prefix sums and the CTA's first row are the
// CTA's own copy in shared memory (plan_local; p.cta_row points at that one entry),
// and the partial results are merged in the kernel: a pair wholly inside one share
// is written directly, otherwise the CTA writing the pair's last slot merges it (the
// partial slots other CTAs write are read with L2-only loads).  For the standalone
// decode this was measured slower than plan_kernel + decode + combine_kernel
// (merges on the slowest CTAs' critical path), so decode_tc_kernel keeps LOCAL off.
// FLAGS (the fused step): the union list and tau were written by other CTAs of the
// same grid, and a row's union list is read once its compaction flag carries this
// launch's token.  Plain (L1-cached) loads still see them, because no SM reads
// those lines earlier in the launch (the screening reads tau with L2-only loads).
// PDL_IN (the standalone kernel): the shared-memory and TMEM setup runs before the
// wait for the previous grid, so it overlaps that grid's tail; the plan is read after.
// PLAN_IN (with PDL_IN, sparse): no plan launch; every CTA lays the shares out itself
// (plan_local, from the admitted counts) and CTA 0 publishes row_off and the plan
// for the combine launch.
// DD (head dimension) 128, or 64: then one 64-dim box per K/V sub-tile and for the
// query rows, QK^T in 4 steps of 16 dims, and P V still M = 128 (the V tile's upper
// 64-dim half stays zero, so those accumulator rows are zero and not written out).
template <int G, bool DENSE, bool LOCAL, bool FLAGS, bool PDL_IN = false, bool PLAN_IN = false,
          int DD = 128>
ETA_DEV void decode_tc_body(unsigned char* smem, const CUtensorMap* tmK, const CUtensorMap* tmV,
                            const CUtensorMap* tmQ, const TcParams& p, const FuseCtx& fx) {
  static_assert(G >= 1 && G <= 8, "G");
  static_assert(DD == 128 || (DD == 64 && !LOCAL), "d = 64 in the standalone decode");
  constexpr int NHALF = DD / 64;   // 64-dim boxes per K/V sub-tile and per query tile
  static_assert(!(LOCAL && DENSE), "the in-kernel merge is for the sparse decode");
  static_assert(!FLAGS || LOCAL, "flags come with the local plan");
  static_assert(!PLAN_IN || (PDL_IN && !DENSE && !LOCAL), "plan in the standalone sparse decode");
  TcMisc* ms = reinterpret_cast<TcMisc*>(smem + SM_MISC);
  const int32_t* plan = p.plan;
  const int32_t* row_off = p.row_off;
  const int32_t* cta_row = p.cta_row;
  volatile int* abort_flag = &ms->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int a = 0, e = 0;
  if constexpr (!PDL_IN) {
    const int Ntot = plan[0], chunk = plan[1];
    a = blockIdx.x * chunk;
    if (a >= Ntot) return;  // uniform, before any barrier
    e = min(a + chunk, Ntot);
  }

  // zero the V halves and the P buffers once: every row the PV MMA reads is then
  // finite (TMA only overwrites them with cache rows, and rows past a sequence's
  // length are zeroed again by the softmax warps before use)
  for (int s = 0; s < NSTAGE; ++s) {
    uint4* v = reinterpret_cast<uint4*>(smem + s * STAGE_BYTES + OFF_V0);
    for (int i = threadIdx.x; i < 2 * HALF / 16; i += NT) v[i] = make_uint4(0, 0, 0, 0);
  }
  for (int i = threadIdx.x; i < 2 * PBUF / 16; i += NT)
    reinterpret_cast<uint4*>(smem + SM_P)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&ms->full[s], 1);
      mbar_init(&ms->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ms->s_full[b], 1);
      mbar_init(&ms->s_free[b], NWARP_SM);
      mbar_init(&ms->p_full[b], NWARP_SM);
      mbar_init(&ms->o_full[b], 1);
      mbar_init(&ms->o_free[b], NWARP_SM);
    }
    mbar_init(&ms->fin, 1);
    ms->abort_flag = 0;
    fence_mbar_init();
  }
  fence_async_smem();
  if (warp == NWARP_SM + 1) {   // MMA warp owns the TMEM allocation
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&ms->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  const uint32_t tS0 = tmem, tO0 = tmem + 32;   // column offsets; lane field added per warp
  if constexpr (PDL_IN) {
    ETA_PDL_ENTRY();
    if constexpr (PLAN_IN) {
      FuseSmem* fs = reinterpret_cast<FuseSmem*>(smem + SM_FUSE);
      int* ro = reinterpret_cast<int*>(smem + SM_ROWOFF);
      plan_local(p.counts, p.R, p.NB, ro, fs, p.status);
      if (blockIdx.x == 0) {
        for (int r = threadIdx.x; r <= p.R; r += NT) p.row_off_g[r] = ro[r];
        if (threadIdx.x == 0) {
          p.plan_g[0] = fs->plan[0];
          p.plan_g[1] = fs->plan[1];
        }
      }
      plan = fs->plan;
      row_off = ro;
      cta_row = &fs->cta_row;
    }
    const int Ntot = plan[0], chunk = plan[1];
    a = blockIdx.x * chunk;
    if (a >= Ntot) {   // uniform: no share, release TMEM (nothing was issued) and leave
      if (warp == NWARP_SM + 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols));
      return;
    }
    e = min(a + chunk, Ntot);
  }

  if (warp == NWARP_SM) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int r = (LOCAL || PLAN_IN) ? cta_row[0] : cta_row[blockIdx.x];
      bool ok = true;
      if (!ETA_IN_BOUNDS(r, p.R, p.status)) {   // checked build: give up like a lost wait
        r = 0;
        ok = false;
      }
      int roff = row_off[r], rend = row_off[r + 1];
      int it = 0;
      int pend_row = -1, pend_t0 = 0, pend_nv = 0;   // a lone sub-tile waiting for a partner
      auto emit = [&](int row, int t0a, int nva, int t0b, int nvb, int flags) -> bool {
        const int s = it % NSTAGE;
        const uint32_t ph = (uint32_t)(it / NSTAGE) & 1u;
        if (!flags && !ETA_IN_BOUNDS(row, p.R, p.status)) return false;
        if (!mbar_wait(&ms->empty[s], ph ^ 1u, abort_flag)) return false;
        ms->info[s] = TcStage{row, {t0a, t0b}, {nva, nvb}, flags, {0, 0}};
        unsigned char* st = smem + s * STAGE_BYTES;
        if (flags) {
          mbar_arrive(&ms->full[s]);
        } else {
          const int nsub = nvb > 0 ? 2 : 1;
          mbar_arrive_expect_tx(&ms->full[s],
                                (uint32_t)(NHALF * (nsub * 2 * SUB_HALF + QHALF)));
          const int b = row / p.Hkv, g = row % p.Hkv;
          const int qrow = b * p.Hq + g * G;
          tma_load_2d(st + OFF_Q0, tmQ, 0, qrow, &ms->full[s]);
          if constexpr (NHALF == 2) tma_load_2d(st + OFF_Q1, tmQ, 64, qrow, &ms->full[s]);
          for (int u = 0; u < nsub; ++u) {
            const int y = row * p.T_max + (u == 0 ? t0a : t0b);
            tma_load_2d(st + OFF_K0 + u * SUB_HALF, tmK, 0, y, &ms->full[s]);
            tma_load_2d(st + OFF_V0 + u * SUB_HALF, tmV, 0, y, &ms->full[s]);
            if constexpr (NHALF == 2) {
              tma_load_2d(st + OFF_K1 + u * SUB_HALF, tmK, 64, y, &ms->full[s]);
              tma_load_2d(st + OFF_V1 + u * SUB_HALF, tmV, 64, y, &ms->full[s]);
            }
          }
        }
        ++it;
        return true;
      };
      // fused step: a row's union list is read once its compaction flag is set
      int ready_row = -1;
      bool rows_ok = true;
      auto row_ready = [&](int rr) -> bool {
        if constexpr (FLAGS) {
          if (rr == ready_row) return true;
          for (uint32_t w = 0; w < kWaitLimit; ++w) {
            if (ld_acquire_gpu(fx.ready + rr) == fx.token) {
              ready_row = rr;
              return true;
            }
            if (*abort_flag) return false;
            __nanosleep(32);
          }
          return false;
        } else {
          return true;
        }
      };
      // The block index of position pos+1 is loaded before the stages of position pos
      // are emitted, so its L2 latency overlaps the wait for a free stage.
      auto fetch = [&](int pos, int& rr, int& ro, int& re) -> int {
        while (pos >= re) {
          if (!ETA_IN_BOUNDS(rr + 2, p.R + 1, p.status)) {
            rows_ok = false;
            return 0;
          }
          ++rr;
          ro = re;
          re = row_off[rr + 1];
        }
        if (DENSE) return pos - ro;
        if (!row_ready(rr) || !ETA_IN_BOUNDS(pos - ro, p.NB, p.status)) {
          rows_ok = false;
          return 0;
        }
        return p.union_idx[(size_t)rr * p.NB + (pos - ro)];
      };
      int nr = r, nroff = roff, nrend = rend;
      int j_next = a < e ? fetch(a, nr, nroff, nrend) : 0;
      for (int pos = a; pos < e && ok; ++pos) {
        if (!rows_ok) {
          ok = false;
          break;
        }
        const int j = j_next;
        r = nr; roff = nroff; rend = nrend;
        if (pos + 1 < e) j_next = fetch(pos + 1, nr, nroff, nrend);
        const int b = r / p.Hkv;
        const int len = min(max(p.lengths[b], 0), p.T_max);
        if (j < 0 || j >= p.NB || j * p.blk >= len) {
          set_status(p.status, ETA_DEVSTAT_BAD_BLOCK);
          continue;
        }
        for (int sub = 0; sub < p.blk / kSubKeys && ok; ++sub) {
          const int t0 = j * p.blk + sub * kSubKeys;
          const int nv = min(kSubKeys, len - t0);
          if (nv <= 0) break;
          if (pend_row < 0) {
            pend_row = r; pend_t0 = t0; pend_nv = nv;
          } else if (pend_row == r) {
            ok = emit(r, pend_t0, pend_nv, t0, nv, 0);
            pend_row = -1;
          } else {
            ok = emit(pend_row, pend_t0, pend_nv, 0, 0, 0);
            pend_row = r; pend_t0 = t0; pend_nv = nv;
          }
        }
      }
      if (ok && pend_row >= 0) ok = emit(pend_row, pend_t0, pend_nv, 0, 0, 0);
      if (ok) ok = emit(-1, 0, 0, 0, 0, 1);
      if (!ok) {
        set_status(p.status, ETA_DEVSTAT_TIMEOUT);
        *abort_flag = 1;
        for (int k = max(0, it - NSTAGE); k < it; ++k)
          mbar_wait(&ms->full[k % NSTAGE], (uint32_t)(k / NSTAGE) & 1u, nullptr);
      }
    }
  } else if (warp == NWARP_SM + 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = true;
      int i = 0;
      auto issue_pv = [&](int k) -> bool {   // PV of stage k
        const int s = k % NSTAGE, pb = k & 1;
        const uint32_t ph = (uint32_t)(k >> 1) & 1u;
        if (!mbar_wait(&ms->p_full[pb], ph, abort_flag)) return false;
        if (!mbar_wait(&ms->o_free[pb], ph ^ 1u, abort_flag)) return false;
        tc_fence_after();
        const uint32_t v0 = smem_u32(smem + s * STAGE_BYTES + OFF_V0);
        const uint32_t pbase = smem_u32(smem + SM_P + pb * PBUF);
#pragma unroll
        for (int kk = 0; kk < kTileKeys / 16; ++kk) {
          const uint64_t da = smem_desc(v0 + kk * 2048, HALF, 1024, kSwizzle128);
          const uint64_t db = smem_desc(pbase + kk * 256, 128, 16 * 128, kSwizzleNone);
          mma_f16(tO0 + pb * 16, da, db, kIdescPV, kk > 0 ? 1u : 0u);
        }
        mma_commit(&ms->o_full[pb]);
        mma_commit(&ms->empty[s]);
        return true;
      };
      for (;; ++i) {
        const int s = i % NSTAGE;
        if (!mbar_wait(&ms->full[s], (uint32_t)(i / NSTAGE) & 1u, abort_flag)) { ok = false; break; }
        if (ms->info[s].flags) break;
        const int sb = i & 1;
        if (!mbar_wait(&ms->s_free[sb], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        unsigned char* st = smem + s * STAGE_BYTES;
#pragma unroll
        for (int kk = 0; kk < DD / 16; ++kk) {
          const uint32_t koff = (uint32_t)(kk & 3) * 32;
          const uint32_t ka = smem_u32(st + (kk < 4 ? OFF_K0 : OFF_K1)) + koff;
          const uint32_t qb = smem_u32(st + (kk < 4 ? OFF_Q0 : OFF_Q1)) + koff;
          mma_f16(tS0 + sb * 16, smem_desc(ka, 16, 1024, kSwizzle128),
                  smem_desc(qb, 16, 1024, kSwizzle128), kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&ms->s_full[sb]);
        if (i > 0 && !issue_pv(i - 1)) { ok = false; break; }
      }
      if (ok && i > 0) ok = issue_pv(i - 1);
      if (!ok) {
        set_status(p.status, ETA_DEVSTAT_TIMEOUT);
        *abort_flag = 1;
      }
      // every MMA issued so far has completed before TMEM is released
      mma_commit(&ms->fin);
      mbar_wait(&ms->fin, 0, nullptr);
    }
  } else {
    // ---------------------------------------------------------------- softmax / correction
    const int t = threadIdx.x;             // key row of the stage; dim for the correction
    const uint32_t lane_sel = (uint32_t)(warp * 32) << 16;
    float m_run[G], l_part[G], o_acc[G], alpha_prev[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_run[h] = -INFINITY; l_part[h] = 0.f; o_acc[h] = 0.f; alpha_prev[h] = 0.f;
    }
    float tau_h[G];
    int cur = -1;
    bool pending = false;   // stage i-1 still has to be folded into o_acc
    bool ok = true;

    // every lane polls; the warp agrees on the outcome so collectives stay converged
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    auto correct = [&](int k) -> bool {    // fold PV of stage k into o_acc
      const int pb = k & 1;
      if (!wwait(&ms->o_full[pb], (uint32_t)(k >> 1) & 1u)) return false;
      tc_fence_after();
      float c[16];
      tmem_ld16(tO0 + pb * 16 + lane_sel, c);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->o_free[pb]);
#pragma unroll
      for (int h = 0; h < G; ++h) o_acc[h] = fmaf(o_acc[h], alpha_prev[h], c[h] + c[G + h]);
      return true;
    };
    auto flush = [&](int row) {
      // l: sum of the per-thread partials over the 128 key threads
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float v = warp_sum(l_part[h]);
        if (lane == 0) ms->lsum[warp][h] = v;
      }
      named_bar_sync(1, NWARP_SM * 32);
      int p0 = 0, ns = 0;
      if constexpr (LOCAL) {
        const int off = row_off[row], c = row_off[row + 1] - off;
        const int chunk = plan[1];
        p0 = off / chunk;
        ns = (off + c - 1) / chunk - p0 + 1;
      }
      if (LOCAL && ns == 1) {
        // the whole pair lies in this share: its partial is the merged result (the
        // one-slot merge written out: weight e^(m - m) = 1, or 0 for an empty softmax)
        const int b = row / p.Hkv, g = row % p.Hkv;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float L = 0.f;
#pragma unroll
          for (int w = 0; w < NWARP_SM; ++w) L += ms->lsum[w][h];
          const float wt = m_run[h] == -INFINITY ? 0.f : 1.f;
          combine_store<D>(fx.o, fx.lse, (size_t)b * p.Hq + (size_t)g * G + h, t, m_run[h],
                           fmaf(L, wt, 0.f), fmaf(o_acc[h], wt, 0.f));
        }
        named_bar_sync(1, NWARP_SM * 32);
      } else {
        const size_t slot = (size_t)blockIdx.x + row;
        const bool slot_ok = ETA_IN_BOUNDS(slot, (long long)gridDim.x + p.R, p.status);
#pragma unroll
        for (int h = 0; h < G && slot_ok; ++h) {
          if (t < DD) p.part_o[(slot * G + h) * DD + t] = o_acc[h];
          if (t == 0) {
            float L = 0.f;
#pragma unroll
            for (int w = 0; w < NWARP_SM; ++w) L += ms->lsum[w][h];
            p.part_ml[(slot * G + h) * 2] = m_run[h];
            p.part_ml[(slot * G + h) * 2 + 1] = L;
          }
        }
        named_bar_sync(1, NWARP_SM * 32);
        if constexpr (LOCAL) {
          // this slot of the pair is written: count it; the CTA with the pair's last
          // slot merges all of them (threadFenceReduction pattern)
          FuseSmem* fs = reinterpret_cast<FuseSmem*>(smem + SM_FUSE);
          __threadfence();
          named_bar_sync(1, NWARP_SM * 32);
          if (t == 0) {
            const int old = atomicAdd(fx.pair_cnt + row, 1);
            const int last = old == ns - 1;
            if (last) fx.pair_cnt[row] = 0;
            fs->last = last;
          }
          named_bar_sync(1, NWARP_SM * 32);
          if (fs->last) {
            __threadfence();
            CombineScratch<G>& cs = *reinterpret_cast<CombineScratch<G>*>(&fs->cs);
            float O[G];
            combine_merge<D, G, true>(p.part_ml, p.part_o, row, p0, ns, t, cs, O,
                                      [] { named_bar_sync(1, NWARP_SM * 32); },
                                      (long long)gridDim.x + p.R, p.status);
            const int b = row / p.Hkv, g = row % p.Hkv;
#pragma unroll
            for (int h = 0; h < G; ++h)
              combine_store<D>(fx.o, fx.lse, (size_t)b * p.Hq + (size_t)g * G + h, t, cs.M[h],
                               cs.L[h], O[h]);
          }
          named_bar_sync(1, NWARP_SM * 32);
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m_run[h] = -INFINITY; l_part[h] = 0.f; o_acc[h] = 0.f;
      }
    };

    int i = 0;
    for (;; ++i) {
      const int s = i % NSTAGE;
      if (!wwait(&ms->full[s], (uint32_t)(i / NSTAGE) & 1u)) { ok = false; break; }
      const TcStage inf = ms->info[s];
      if (inf.flags) break;
      if (inf.row != cur) {
        if (pending) {
          if (!correct(i - 1)) { ok = false; break; }
          pending = false;
        }
        if (cur >= 0) flush(cur);
        cur = inf.row;
        if constexpr (!DENSE) {
          const int b = cur / p.Hkv, g = cur % p.Hkv;
#pragma unroll
          for (int h = 0; h < G; ++h) tau_h[h] = p.tau[(size_t)b * p.Hq + g * G + h];
        }
      }
      // S of stage i
      const int sb = i & 1;
      if (!wwait(&ms->s_full[sb], (uint32_t)(i >> 1) & 1u)) { ok = false; break; }
      tc_fence_after();
      float sv[16];
      tmem_ld16(tS0 + sb * 16 + lane_sel, sv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->s_free[sb]);
      const int sub = t >> 6, loc = t & 63;
      const int nv = sub == 0 ? inf.nv[0] : inf.nv[1];
      const bool valid = loc < nv;
      float sp[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float sc = p.scale * sv[h];
        float x = sc;
        if constexpr (!DENSE) {
          if (p.invT < 0.f) x = sc >= tau_h[h] ? sc : 0.f;
          else x = __fdividef(sc, 1.f + __expf((tau_h[h] - sc) * p.invT));   // 0 once exp overflows
        }
        sp[h] = valid ? x : -INFINITY;
        const float wm = warp_max(sp[h]);
        if (lane == 0) ms->red[sb][warp][h] = wm;
      }
      // a partial sub-tile: zero the V rows past the sequence end (finite inputs to PV)
      if (!valid && nv > 0) {
        unsigned char* st = smem + s * STAGE_BYTES;
        uint4* r0 = reinterpret_cast<uint4*>(st + OFF_V0 + t * 128);
        uint4* r1 = reinterpret_cast<uint4*>(st + OFF_V1 + t * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) { r0[c] = make_uint4(0, 0, 0, 0); r1[c] = make_uint4(0, 0, 0, 0); }
      }
      named_bar_sync(1, NWARP_SM * 32);
      float alpha[G];
      uint32_t pk0[4] = {0, 0, 0, 0}, pk1[4] = {0, 0, 0, 0};   // P^T columns 0-7, 8-15
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float tm = ms->red[sb][0][h];
#pragma unroll
        for (int w = 1; w < NWARP_SM; ++w) tm = fmaxf(tm, ms->red[sb][w][h]);
        const float mnew = fmaxf(m_run[h], tm);
        alpha[h] = (m_run[h] == -INFINITY) ? 0.f : __expf(m_run[h] - mnew);
        const float pr = valid ? __expf(sp[h] - mnew) : 0.f;
        l_part[h] = fmaf(l_part[h], alpha[h], pr);
        m_run[h] = mnew;
        const __nv_bfloat16 hb = __float2bfloat16_rn(pr);
        const __nv_bfloat16 lb = __float2bfloat16_rn(pr - __bfloat162float(hb));
        const uint32_t hu = (uint32_t)__bfloat16_as_ushort(hb);
        const uint32_t lu = (uint32_t)__bfloat16_as_ushort(lb);
        // column c of P^T: c = h (hi) and c = G + h (lo)
        const int ch = h, cl = G + h;
        if (ch < 8) pk0[ch >> 1] |= hu << ((ch & 1) * 16); else pk1[(ch - 8) >> 1] |= hu << ((ch & 1) * 16);
        if (cl < 8) pk0[cl >> 1] |= lu << ((cl & 1) * 16); else pk1[(cl - 8) >> 1] |= lu << ((cl & 1) * 16);
      }
      // P^T, MN-major, no swizzle: column group cg (8 columns) at cg * 2048 B, key group
      // t / 8 at 128 B, key t % 8 at 16 B
      unsigned char* pbuf = smem + SM_P + sb * PBUF;
      *reinterpret_cast<uint4*>(pbuf + (t >> 3) * 128 + (t & 7) * 16) =
          make_uint4(pk0[0], pk0[1], pk0[2], pk0[3]);
      if (2 * G > 8)
        *reinterpret_cast<uint4*>(pbuf + 2048 + (t >> 3) * 128 + (t & 7) * 16) =
            make_uint4(pk1[0], pk1[1], pk1[2], pk1[3]);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->p_full[sb]);
      // fold the previous stage (same row) while PV of this stage runs
      if (pending) {
        if (!correct(i - 1)) { ok = false; break; }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) alpha_prev[h] = alpha[h];
      pending = true;
    }
    // the last stage: its PV is issued after the end marker
    if (ok && pending) ok = correct(i - 1);
    if (ok && cur >= 0) flush(cur);
    if (!ok) {
      if (t == 0) set_status(p.status, ETA_DEVSTAT_TIMEOUT);
      *abort_flag = 1;
    }
  }
  __syncthreads();
  if (warp == NWARP_SM + 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

template <int G, bool DENSE, bool PLAN_IN = false, int DD = 128>
__global__ void __launch_bounds__(NT, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmQ, const TcParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  decode_tc_body<G, DENSE, false, false, true, PLAN_IN, DD>(smem, &tmK, &tmV, &tmQ, p,
                                                             FuseCtx{});
}

}  // namespace tc
}  // namespace eta
