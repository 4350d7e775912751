// Block screening on the 5th-generation tensor cores: bf16 centroids, d = 128 or 64, the
// exact (Cauchy-Schwarz) and the variance bound (arXiv 2609.20888 abstract: blocks
// screened "in O(1) time using cached geometric-probabilistic bounds"; evolve.pub
// review FAQ: a block whose best possible score falls below the threshold is
// skipped).  Same bound and the same admit rule as screen_group_from (screen_dev.cuh):
//   UB[h, j] = scale * fma(||q_h||, R_j, q_h . c_j),  admit iff cnt_j > 0 and UB >= tau_h
// with the q . c products of a 128-block group computed as one matrix product
//   D[128 blocks][16] = C^T[128 blocks][d] x Q^T[d][16]
// (tcgen05.mma kind::f16, bf16 x bf16 products are exact in fp32, fp32 sums in TMEM),
// the group's G heads in the first G of the 16 columns.  The centroid tile arrives
// by two TMA tensor copies (d dims x 64 blocks each, 128-byte swizzle) and is read
// by the tensor core MN-major (blocks contiguous), the 16 query rows K-major, as the
// decode reads V and Q.  The fp32 accumulation order differs from the CUDA-core
// screen's, so the two agree up to fp32 rounding (near-ties), not bit for bit;
// every screening form that takes this path (eta_screen and the one-launch step)
// shares these functions and writes identical bits.
//
// Epilogue: four warps (the standalone kernel runs two such groups on alternate
// groups), thread t = block t of the group (= TMEM lane): one tcgen05.ld
// of the 16 accumulator columns and the block's rmax / var / cnt from the stage
// (after which the stage and the accumulator are released), then per head the
// bound, the admit bit and a ballot into the 32-bit admit word of the warp's 32
// blocks; the union word is their OR.
#pragma once

#include "compact_dev.cuh"
#include "decode_tc.cuh"
#include "eta_common.cuh"
#include "screen_dev.cuh"

namespace eta {
namespace stc {

constexpr int GB = kScreenGroupBlocks;             // blocks per group (128)
constexpr int Q_HALF = 16 * 64 * 2;                 // [16 heads][64 dims] bf16: 2 KB
// A ring stage is a tile (the swizzled centroid and query boxes, 1024-byte aligned)
// plus a metadata slot (the group's rmax, var and cnt slices); the slots of all
// stages sit together after the tiles, so that no stage pads its tile to 1 KB.
// D = 128: two 16 KB centroid boxes and two query boxes (36 KB); D = 64: two 8 KB
// centroid boxes and one query box (18 KB).
template <int D>
struct Tile {
  static_assert(D == 128 || D == 64, "d");
  static constexpr int CENT_HALF = D * 64 * 2;      // [d rows][64 blocks] bf16
  static constexpr int NQ = D / 64;                  // 64-dim query boxes
  static constexpr int OFF_C0 = 0, OFF_C1 = CENT_HALF;
  static constexpr int OFF_Q0 = 2 * CENT_HALF, OFF_Q1 = OFF_Q0 + Q_HALF;
  static constexpr int BYTES = 2 * CENT_HALF + NQ * Q_HALF;
  static_assert(BYTES % 1024 == 0, "swizzled tiles stay 1024-byte aligned");
};
constexpr int M_RMAX = 0, M_VAR = 4 * GB, M_CNT = 8 * GB;
constexpr int META = 12 * GB;                       // 1.5 KB
// kind::f16, D fp32, bf16 operands, M = 128, N = 16; A (centroids) MN-major, B (q) K-major
constexpr uint32_t kIdesc = tc::kIdescBase | (1u << 15);
constexpr int kAccCols = 16;

// The group's q . c products into TMEM columns [d_tmem, d_tmem + 16): K = d in
// d / 16 steps of 16 dims, in order.  `st` is a stage tile laid out as Tile<D>
// (1024-aligned).
template <int D>
ETA_DEV void issue_mma(uint32_t d_tmem, const unsigned char* st) {
  using T = Tile<D>;
  const uint32_t c0 = smem_u32(st + T::OFF_C0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    // A: 16 dims (rows of 128 B) per step; the second 64 blocks one box further on
    const uint64_t da = tc::smem_desc(c0 + kk * 2048, T::CENT_HALF, 1024, tc::kSwizzle128);
    const uint32_t qb =
        smem_u32(st + (kk < 4 ? T::OFF_Q0 : T::OFF_Q1)) + (uint32_t)(kk & 3) * 32;
    const uint64_t db = tc::smem_desc(qb, 16, 1024, tc::kSwizzle128);
    tc::mma_f16(d_tmem, da, db, kIdesc, kk > 0 ? 1u : 0u);
  }
}

// ||q_h|| of the G heads of one (row, KV head) pair from the 16 query rows a stage
// holds (TMA-staged, 128-byte swizzle: the 16-byte chunk c of row h sits at chunk
// c ^ (h % 8)), by one warp into every lane's registers, so that a row change costs
// no global-memory round trip.  The fmaf order of query_norm (lane k sums dims k,
// k + 32, ...), then a butterfly sum.
template <int D, int G>
ETA_DEV void query_norms_staged(const unsigned char* st, float (&qn)[G]) {
  using T = Tile<D>;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const int k = lane + 32 * i, kk = k & 63;
      const unsigned char* row = st + (k < 64 ? T::OFF_Q0 : T::OFF_Q1) + h * 128;
      const uint16_t bits =
          *reinterpret_cast<const uint16_t*>(row + (((kk >> 3) ^ (h & 7)) << 4) + (kk & 7) * 2);
      const float x = bf16_to_f(bits);
      s = fmaf(x, x, s);
    }
    qn[h] = sqrtf(warp_sum(s));
  }
}

// This thread's block (t = threadIdx.x in [0, 128) of group `grp`): its radius term
// R_j (rmax, or min(rmax, z sqrt(var / d)) for the variance bound) and its key count,
// read from the stage's metadata slot `ms`; blocks past NB get R = 0, n = 0.  The
// stage can be released once every thread has read them.
struct BlockMeta {
  float rad;
  int n;
};
template <int D>
ETA_DEV BlockMeta block_meta(const unsigned char* ms, bool prob, float z, int NB, int grp) {
  const int t = threadIdx.x & 127;
  BlockMeta m{0.f, 0};
  if (grp * GB + t < NB) {
    m.rad = reinterpret_cast<const float*>(ms + M_RMAX)[t];
    if (prob)
      m.rad = fminf(m.rad, z * sqrtf(reinterpret_cast<const float*>(ms + M_VAR)[t] / (float)D));
    m.n = reinterpret_cast<const int32_t*>(ms + M_CNT)[t];
  }
  return m;
}

// The bound, admit words and union word of group `grp` of row r from the
// accumulator values of this thread's block (dot[h], h < G) and its BlockMeta.
// A block is admitted for head h iff it holds keys, lies below `nvalid` and its
// bound >= ts[h].  Writes head_mask[(qhead0 + h) * NW + w], union_words[r * NW + w]
// (w = the warp's word) and, if given, bounds_out[(qhead0 + h) * NB + j].  Returns
// how many of the warp's 32 blocks the union admits (in every lane).
template <int G>
ETA_DEV int epilogue(const float (&dot)[16], BlockMeta bm, float scale, int NB, int NW, int grp,
                     int r, size_t qhead0, const float (&qn)[G], const float (&ts)[G],
                     int nvalid, uint32_t* __restrict__ head_mask,
                     uint32_t* __restrict__ union_words, float* __restrict__ bounds_out) {
  const int t = threadIdx.x & 127, warp = t >> 5, lane = t & 31;
  const int j = grp * GB + t;
  const bool vj = j < NB;
  const int w = grp * (GB / 32) + warp;
  uint32_t uni = 0;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float ub = scale * fmaf(qn[h], bm.rad, dot[h]);
    const bool adm = vj && bm.n > 0 && j < nvalid && ub >= ts[h];
    const uint32_t word = __ballot_sync(0xffffffffu, adm);
    if (lane == 0 && w < NW) head_mask[(qhead0 + h) * NW + w] = word;
    uni |= word;
    if (bounds_out && vj) bounds_out[(qhead0 + h) * NB + j] = ub;
  }
  if (lane == 0 && w < NW) union_words[(size_t)r * NW + w] = uni;
  return __popc(uni);
}

// ------------------------------------------------------------------ standalone kernel
constexpr int NSTAGE = 6;
// warps 0-7 epilogue (two groups of four taking alternate items, one TMEM accumulator
// each), warp 8 TMA producer, warp 9 MMA issuer
constexpr int NT = 10 * 32;
constexpr int kWarpTma = 8, kWarpMma = 9;

struct Params {
  int Hq, Hkv, NB, NW, ngrp, items, chunk, prob;
  float z, scale;
  const eta_bf16_t* q;
  const float* tau;
  const float* rmax;
  const float* var;
  const int32_t* cnt;
  uint32_t* head_mask;
  uint32_t* union_words;
  float* bounds_out;
  int32_t* union_idx;     // ROWS: the row's compaction in the same launch
  int32_t* union_cnt;
  int32_t* head_cnt;
  int32_t* status;
};

struct Misc {
  uint64_t full[NSTAGE], empty[NSTAGE];
  uint64_t acc_full[2], acc_free[2];
  uint64_t fin;
  float ts[NSTAGE][8];    // the staged item's thresholds, written by the producer
  uint32_t tmem_base;
  int abort_flag;
};
template <int D>
struct Ring {
  static constexpr int OFF_META = NSTAGE * Tile<D>::BYTES;
  static constexpr int OFF_MISC = OFF_META + NSTAGE * META;
  static constexpr int SMEM_BYTES = OFF_MISC + (int)sizeof(Misc) + 1024;   // + align slack
  static_assert(SMEM_BYTES <= 227 * 1024, "screen_tc shared memory");
  // ROWS: the compaction's scratch reuses the first tile once every item is screened
  static_assert(sizeof(CompactScratch<128>) <= Tile<D>::BYTES, "compaction scratch");
};

// Items are (row, group) pairs in row-major order; CTA c screens items
// [c * chunk, min((c + 1) * chunk, items)) in order, so its in-flight tiles are
// neighbouring 256-byte strips of the same dimension-major centroid rows (items dealt
// round-robin over the CTAs measured slower: 54 vs 46 us at 128K, B = 64).  ROWS
// (chunk = groups per row, one CTA per row): the CTA then compacts its row's union
// list as compact_kernel does.  A row change costs no global round trip: the norms
// come from the staged query rows, the thresholds from the stage's record.
template <int D, int G, bool ROWS>
__global__ void __launch_bounds__(NT, 1)
screen_tc_kernel(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmQ,
                 const Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using T = Tile<D>;
  using RG = Ring<D>;
  Misc* ms = reinterpret_cast<Misc*>(smem + RG::OFF_MISC);
  volatile int* abort_flag = &ms->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a = blockIdx.x * p.chunk;
  const int n_local = max(min(a + p.chunk, p.items) - a, 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&ms->full[s], 1);
      mbar_init(&ms->empty[s], 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ms->acc_full[b], 1);
      mbar_init(&ms->acc_free[b], 4);
    }
    mbar_init(&ms->fin, 1);
    ms->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&ms->tmem_base)),
                 "r"(32));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  ETA_PDL_ENTRY();

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      int i = 0, cur_r = -1;
      float tsv[G];                       // the current row's thresholds
      for (; i < n_local && ok; ++i) {
        const int it = a + i, r = it / p.ngrp, grp = it % p.ngrp;
        const int s = i % NSTAGE;
        const int j0 = grp * GB;
        const int nb = min(GB, p.NB - j0);
        const int qrow = (r / p.Hkv) * p.Hq + (r % p.Hkv) * G;
        if (r != cur_r) {                 // loaded before the wait: its latency overlaps it
#pragma unroll
          for (int h = 0; h < G; ++h) tsv[h] = p.tau[qrow + h];
          cur_r = r;
        }
        // (checked build) the group's metadata slices lie inside the row
        if (!ETA_RANGE_IN_BOUNDS(j0, j0 + nb, p.NB, p.status) ||
            !mbar_wait(&ms->empty[s], ((uint32_t)(i / NSTAGE) & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) ms->ts[s][h] = tsv[h];   // published by the arrive below
        unsigned char* st = smem + s * T::BYTES;
        unsigned char* mt = smem + RG::OFF_META + s * META;
        const uint32_t nb4 = (uint32_t)nb * 4u;
        mbar_arrive_expect_tx(&ms->full[s], (uint32_t)T::BYTES + nb4 * (p.prob ? 3u : 2u));
        tc::tma_load_2d(st + T::OFF_C0, &tmC, j0, r * D, &ms->full[s]);
        tc::tma_load_2d(st + T::OFF_C1, &tmC, j0 + 64, r * D, &ms->full[s]);
        tc::tma_load_2d(st + T::OFF_Q0, &tmQ, 0, qrow, &ms->full[s]);
        if constexpr (T::NQ == 2) tc::tma_load_2d(st + T::OFF_Q1, &tmQ, 64, qrow, &ms->full[s]);
        const size_t rj = (size_t)r * p.NB + j0;
        bulk_g2s(mt + M_RMAX, p.rmax + rj, nb4, &ms->full[s]);
        if (p.prob) bulk_g2s(mt + M_VAR, p.var + rj, nb4, &ms->full[s]);
        bulk_g2s(mt + M_CNT, p.cnt + rj, nb4, &ms->full[s]);
      }
      if (!ok) {
        set_status(p.status, ETA_DEVSTAT_TIMEOUT);
        *abort_flag = 1;
        // every copy issued lands before the CTA's shared memory is released
        for (int k = max(0, i - NSTAGE); k < i; ++k)
          mbar_wait(&ms->full[k % NSTAGE], (uint32_t)(k / NSTAGE) & 1u, nullptr);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < n_local && ok; ++i) {
        const int s = i % NSTAGE, b = i & 1;
        if (!mbar_wait(&ms->full[s], (uint32_t)(i / NSTAGE) & 1u, abort_flag) ||
            !mbar_wait(&ms->acc_free[b], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        issue_mma<D>(tmem + b * kAccCols, smem + s * T::BYTES);
        tc::mma_commit(&ms->acc_full[b]);
      }
      if (!ok) {
        set_status(p.status, ETA_DEVSTAT_TIMEOUT);
        *abort_flag = 1;
      }
      // every MMA issued has completed before TMEM is released
      tc::mma_commit(&ms->fin);
      mbar_wait(&ms->fin, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-7)
    // group eg = warp / 4 takes the items i with i % 2 == eg, i.e. accumulator eg;
    // warp w reads TMEM lanes 32 (w % 4) .. + 31
    const int eg = warp >> 2;
    const uint32_t lane_sel = (uint32_t)((warp & 3) * 32) << 16;
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    int cur_r = -1;
    bool ok = true;
    float qn[G], ts[G];                     // every warp holds the row's norms itself
    for (int i = eg; i < n_local; i += 2) {
      const int it = a + i, r = it / p.ngrp, grp = it % p.ngrp;
      const int s = i % NSTAGE, b = i & 1;
      const size_t qhead0 = (size_t)(r / p.Hkv) * p.Hq + (size_t)(r % p.Hkv) * G;
      if (!wwait(&ms->full[s], (uint32_t)(i / NSTAGE) & 1u)) {
        ok = false;
        break;
      }
      if (r != cur_r) {
        query_norms_staged<D, G>(smem + s * T::BYTES, qn);
#pragma unroll
        for (int h = 0; h < G; ++h) ts[h] = ms->ts[s][h];
        cur_r = r;
      }
      if (!wwait(&ms->acc_full[b], (uint32_t)(i >> 1) & 1u)) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      float dot[16];
      tc::tmem_ld16(tmem + b * kAccCols + lane_sel, dot);
      tc::tc_fence_before();
      const BlockMeta bm =
          block_meta<D>(smem + RG::OFF_META + s * META, p.prob != 0, p.z, p.NB, grp);
      __syncwarp();
      if (lane == 0) {                      // accumulator and stage are no longer read
        mbar_arrive(&ms->acc_free[b]);
        mbar_arrive(&ms->empty[s]);
      }
      epilogue<G>(dot, bm, p.scale, p.NB, p.NW, grp, r, qhead0, qn, ts, p.NB, p.head_mask,
                  p.union_words, p.bounds_out);
    }
    if (!ok) {
      if (lane == 0) set_status(p.status, ETA_DEVSTAT_TIMEOUT);
      *abort_flag = 1;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if constexpr (ROWS) {
    // the row's words were written by the epilogue threads: they compact it (L2 reads)
    if (warp < 4 && n_local > 0 && !*abort_flag) {
      compact_row<128>((int)blockIdx.x, p.Hq, p.Hkv, G, p.NB, p.NW, p.union_words, p.head_mask,
                       p.union_idx, p.union_cnt, p.head_cnt,
                       *reinterpret_cast<CompactScratch<128>*>(smem), p.status,
                       [] { named_bar_sync(1, 128); });
    }
  }
  if (warp == kWarpMma) {
    __syncwarp();
    tc::tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(32));
  }
}

}  // namespace stc
}  // namespace eta
