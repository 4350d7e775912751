// Dense gated causal attention for a prefill chunk on the tensor cores (tcgen05).
//
// The gate of the evolve.pub review of arXiv 2609.20888 (Methodology Assessment,
// Eq. 2-3: m = sigmoid(beta (S - tau)), gated logits S * m) applied to every
// (query, key) pair of a causal prefill, with beta = 1/T (T = 0: hard gate); the
// inference-side counterpart of the paper's dense gated training forward.
//
// One CTA per (batch row, query head, 128-query tile), 320 threads:
//   warp 8  TMA producer: the 128 x 128 query tile once, then 128-key K and V
//           tiles (two 64-dim boxes each, 128-byte swizzle) into a 2-stage ring
//   warp 9  MMA issuer: S = Q K^T (M = 128 queries, N = 128 keys, K = d) into one of
//           two TMEM buffers, then O += P V (M = 128 queries, N = d, K = 128 keys,
//           V read MN-major from its swizzled tile) into the TMEM accumulator
//   warps 0-7 softmax, two threads per query row (= TMEM lane): warps 0-3 take key
//           columns 0-63 of the S tile, warps 4-7 columns 64-127, and the two halves
//           of a row agree on the tile's row max through shared memory.  Causal mask,
//           gate, running row max; O is rescaled in TMEM only when the row max grew by
//           more than kRescale (FA-style conditional rescaling), each half rescaling its
//           own 64 columns; P is written as bf16 into a swizzled shared tile (the A
//           operand of P V), each half writing its own 64-key half.
// TMEM: S 2 x 128 columns, O 128 columns (512 allocated).  Every wait is bounded.
// The two-tile kernel further down (prefill_pp_kernel: two query tiles per CTA
// sharing every K/V tile, P kept in tensor memory) is faster wherever its tile pairs
// fill the SMs; this one-tile kernel takes the small launches (see eta_prefill).
#include <cuda.h>
#include <algorithm>
#include <atomic>
#include <cudaTypedefs.h>
#include <math.h>

#include "decode_tc.cuh"
#include "eta_common.cuh"
#include "eta_host.h"
#include "tma_host.h"

namespace eta {
namespace pf {

using tc::mma_commit;
using tc::mma_f16;
using tc::smem_desc;
using tc::tc_fence_after;
using tc::tc_fence_before;
using tc::fence_async_smem;
using tc::tma_load_2d;

constexpr int D = 128;
constexpr int TILE = 128;                       // queries per CTA, keys per KV tile
constexpr int HALF = TILE * 128;                // [128 rows x 64 dims] bf16 = 16 KB
constexpr int NKV = 2;                          // KV ring stages
constexpr int OFF_Q = 0;                        // 2 halves
constexpr int OFF_KV = 2 * HALF;                // stage s: K0 K1 V0 V1
constexpr int KV_STAGE = 4 * HALF;              // 64 KB
constexpr int OFF_P = OFF_KV + NKV * KV_STAGE;  // one P tile: 2 halves (see the softmax)
constexpr int OFF_MISC = OFF_P + 2 * HALF;
constexpr int NWARP_SM = 8;                     // two warpgroups: key columns 0-63, 64-127
constexpr int NT = (NWARP_SM + 2) * 32;
constexpr int kTmemCols = 512;
constexpr float kRescale = 8.0f;                // rescale O when the max grows by > 8 (e^8)

struct Misc {
  uint64_t q_full, kv_full[NKV], kv_empty[NKV];
  uint64_t s_full[2], s_free[2], p_full[2], o_done, o_final, fin;
  float xch[2][2][TILE];   // per tile parity, per half: the row maxima of a tile
  float2 xsum[2][TILE];    // per half: the final row sums (rounded weights, exact weights)
  uint32_t tmem_base;
  int abort_flag;
};
constexpr int SMEM_BYTES = OFF_MISC + (int)sizeof(Misc) + 1024;

// kind::f16, D fp32, A/B bf16, M = 128, N = 128
constexpr uint32_t kIdescBase = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) |
                                ((128u >> 4) << 24);
constexpr uint32_t kIdescQK = kIdescBase;                 // A, B K-major
constexpr uint32_t kIdescPV = kIdescBase | (1u << 16);    // A K-major, B (V) MN-major

ETA_DEV void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

ETA_DEV void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::
          "r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

// 2^x on the SFU (PTX ex2.approx; -inf gives 0)
ETA_DEV float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float kLog2e = 1.4426950408889634f;

// max of three values in one instruction (PTX max.f32 with three sources)
ETA_DEV float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// tanh on the SFU (PTX tanh.approx)
ETA_DEV float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

ETA_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
ETA_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

struct PrefillParams {
  int Hq, Hkv, T_max, ntiles;
  float scale, invT;      // invT < 0: hard gate
  const float* tau;       // [B, Hq, T_max]
  const int32_t* lengths;
  float* O;               // [B, Hq, T_max, d]
  float* lse;             // [B, Hq, T_max]
  int32_t* status;
};

template <int G>
__global__ void __launch_bounds__(NT, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  ETA_PDL_ENTRY();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Misc* ms = reinterpret_cast<Misc*>(smem + OFF_MISC);
  volatile int* abort_flag = &ms->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // heaviest tiles (most keys) first
  const int qt = p.ntiles - 1 - (int)(blockIdx.x % p.ntiles);
  const int bh = blockIdx.x / p.ntiles;
  const int b = bh / p.Hq, h = bh % p.Hq, g = h / G;
  const int len = min(max(p.lengths[b], 0), p.T_max);
  const int q0 = qt * TILE;
  if (q0 >= len) return;                              // uniform, before any barrier
  const int nkv = (min(q0 + TILE, len) + TILE - 1) / TILE;   // key tiles 0 .. nkv-1

  if (threadIdx.x == 0) {
    mbar_init(&ms->q_full, 1);
    for (int s = 0; s < NKV; ++s) {
      mbar_init(&ms->kv_full[s], 1);
      mbar_init(&ms->kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ms->s_full[i], 1);
      mbar_init(&ms->s_free[i], NWARP_SM);
      mbar_init(&ms->p_full[i], NWARP_SM);
    }
    mbar_init(&ms->o_done, 1);
    mbar_init(&ms->o_final, 1);
    mbar_init(&ms->fin, 1);
    ms->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == NWARP_SM + 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&ms->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  const uint32_t tS = tmem, tO = tmem + 256;

  if (warp == NWARP_SM) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      const int qrow = (b * p.Hq + h) * p.T_max + q0;
      mbar_arrive_expect_tx(&ms->q_full, 2 * HALF);
      tma_load_2d(smem + OFF_Q, &tmQ, 0, qrow, &ms->q_full);
      tma_load_2d(smem + OFF_Q + HALF, &tmQ, 64, qrow, &ms->q_full);
      int j = 0;
      for (; j < nkv && ok; ++j) {
        const int s = j % NKV;
        // (checked build) the key tile lies inside the cache row; a refused copy ends
        // the CTA like a lost wait, after the copies already issued
        if (!ETA_IN_BOUNDS((j + 1) * TILE - 1, p.T_max, p.status) ||
            !mbar_wait(&ms->kv_empty[s], ((uint32_t)(j / NKV) & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        unsigned char* st = smem + OFF_KV + s * KV_STAGE;
        const int krow = (b * p.Hkv + g) * p.T_max + j * TILE;
        mbar_arrive_expect_tx(&ms->kv_full[s], 4 * HALF);
        tma_load_2d(st, &tmK, 0, krow, &ms->kv_full[s]);
        tma_load_2d(st + HALF, &tmK, 64, krow, &ms->kv_full[s]);
        tma_load_2d(st + 2 * HALF, &tmV, 0, krow, &ms->kv_full[s]);
        tma_load_2d(st + 3 * HALF, &tmV, 64, krow, &ms->kv_full[s]);
      }
      if (!ok) {
        set_status(p.status, ETA_DEVSTAT_TIMEOUT);
        *abort_flag = 1;
        mbar_wait(&ms->q_full, 0, nullptr);
        for (int k = max(0, j - NKV); k < j; ++k)
          mbar_wait(&ms->kv_full[k % NKV], (uint32_t)(k / NKV) & 1u, nullptr);
      }
    }
  } else if (warp == NWARP_SM + 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&ms->q_full, 0, abort_flag);
      const uint32_t qa = smem_u32(smem + OFF_Q);
      auto issue_pv = [&](int k) -> bool {
        const int s = k % NKV, pb = k & 1;
        if (!mbar_wait(&ms->p_full[pb], (uint32_t)(k >> 1) & 1u, abort_flag)) return false;
        tc_fence_after();
        const uint32_t pa = smem_u32(smem + OFF_P);
        const uint32_t v0 = smem_u32(smem + OFF_KV + s * KV_STAGE + 2 * HALF);
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) {
          const uint32_t aoff = (uint32_t)(kk >> 2) * HALF + (uint32_t)(kk & 3) * 32;
          mma_f16(tO, smem_desc(pa + aoff, 16, 1024, tc::kSwizzle128),
                  smem_desc(v0 + kk * 2048, HALF, 1024, tc::kSwizzle128), kIdescPV,
                  (k > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&ms->o_done);
        mma_commit(&ms->kv_empty[s]);
        return true;
      };
      int j = 0;
      for (; j < nkv && ok; ++j) {
        const int s = j % NKV, sb = j & 1;
        if (!mbar_wait(&ms->kv_full[s], (uint32_t)(j / NKV) & 1u, abort_flag)) { ok = false; break; }
        if (!mbar_wait(&ms->s_free[sb], ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ka = smem_u32(smem + OFF_KV + s * KV_STAGE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * HALF + (uint32_t)(kk & 3) * 32;
          mma_f16(tS + sb * 128, smem_desc(qa + off, 16, 1024, tc::kSwizzle128),
                  smem_desc(ka + off, 16, 1024, tc::kSwizzle128), kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&ms->s_full[sb]);
        if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && nkv > 0) ok = issue_pv(nkv - 1);
      // one-phase barrier for "every P V done": o_done's parity can alias once two of
      // its phases complete before a waiter looks
      if (ok) mma_commit(&ms->o_final);
      if (!ok) {
        set_status(p.status, ETA_DEVSTAT_TIMEOUT);
        *abort_flag = 1;
      }
      mma_commit(&ms->fin);
      mbar_wait(&ms->fin, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------------ softmax
    const int hh = warp >> 2;                         // key-column half of the tile
    const int row = threadIdx.x & (TILE - 1);         // query row of the tile = TMEM lane
    const int tq = q0 + row;
    const uint32_t lsel = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t cb = (uint32_t)hh * 64;            // first column of this half
    const float tau = (tq < p.T_max) ? p.tau[((size_t)b * p.Hq + h) * p.T_max + tq] : 0.f;
    // Gated logits in raw units u (the gated logit is scale * u), so that the scale
    // folds into the constants: the hard gate keeps s iff scale * s >= tau, i.e.
    // s >= tau / scale (scale > 0); the soft gate is
    //   scale * s * sigmoid((scale * s - tau) / T) = scale * (hs + hs * tanh(s * ta - tb)),
    // hs = s / 2, ta = scale / 2T, tb = tau / 2T; and e^(scale * (u - m)) is
    // 2^(u * c1 - m * c1), c1 = scale * log2(e): one FFMA and one ex2 per key.
    const bool hard = p.invT < 0.f;
    const float tau_raw = tau / p.scale;
    const float ta = 0.5f * p.scale * p.invT, tb = 0.5f * tau * p.invT;
    const float c1 = p.scale * kLog2e;
    const float resc_raw = kRescale / p.scale;
    // l: row sum of the bf16-rounded weights (normalizes O, which the tensor core
    // built from those weights); lx: row sum of the exact fp32 weights (for lse);
    // both over this half's columns until the end, two columns per packed add
    float m_used = -INFINITY;                         // raw units
    float2 l2 = make_float2(0.f, 0.f), lx2 = make_float2(0.f, 0.f);
    bool ok = true;
    float sv[64];
    // every lane polls; the warp agrees on the outcome so collectives stay converged
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    // The two warps that share these TMEM lanes (warp w and w + 4: the two halves of
    // the same rows) exchange through shared memory behind their own 64-thread
    // barrier.  Both pass it in every tile, failed or not: a warp whose bounded wait
    // ran out keeps looping with its work skipped, so its partner never blocks on a
    // barrier it will not reach.  The exchange buffer alternates with the tile's
    // parity, so one barrier per tile suffices.
    const int pair_bar = 4 + (warp & 3);
    auto pair_sync = [&] { named_bar_sync(pair_bar, 64); };
    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1, s = j % NKV;
      const int k0 = j * TILE;
      if (ok && !wwait(&ms->s_full[sb], (uint32_t)(j >> 1) & 1u)) ok = false;
      float mxh = -INFINITY;
      if (ok) {
        tc_fence_after();
        tmem_ld32(tS + sb * 128 + cb + lsel, sv);
        tmem_ld32(tS + sb * 128 + cb + 32 + lsel, sv + 32);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ms->s_free[sb]);
        // 8 independent partial maxima: short dependency chains
        float pm[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) pm[u] = -INFINITY;
        auto gate = [&](float x) -> float {
          if (hard) return x >= tau_raw ? x : 0.f;
          const float hs = 0.5f * x;
          return fmaf(hs, tanh_approx(fmaf(x, ta, -tb)), hs);
        };
        if (j == nkv - 1) {
          // the diagonal tile (k0 == q0): keys past the row's query are masked
          const int lim = tq - k0 - (int)cb;           // columns c <= lim are causal
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const float y = (c <= lim) ? gate(sv[c]) : -INFINITY;
            sv[c] = y;
            pm[c & 7] = fmaxf(pm[c & 7], y);
          }
        } else if (hard) {
          // every key of an earlier tile precedes every query of this one; the hard
          // gate as a 1.0 / 0.0 flag (set.ge) and one packed multiply per two scores
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            float g0, g1;
            asm("set.ge.f32.f32 %0, %1, %2;" : "=f"(g0) : "f"(sv[c]), "f"(tau_raw));
            asm("set.ge.f32.f32 %0, %1, %2;" : "=f"(g1) : "f"(sv[c + 1]), "f"(tau_raw));
            const float2 y = __fmul2_rn(make_float2(sv[c], sv[c + 1]), make_float2(g0, g1));
            sv[c] = y.x;
            sv[c + 1] = y.y;
            pm[(c >> 1) & 7] = fmax3(pm[(c >> 1) & 7], y.x, y.y);
          }
        } else {
          // every key of an earlier tile precedes every query of this one
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const float y = gate(sv[c]);
            sv[c] = y;
            pm[c & 7] = fmaxf(pm[c & 7], y);
          }
        }
        mxh = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                    fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      }
      // the row max of the tile: this half's, then the other half's
      ms->xch[sb][hh][row] = mxh;
      pair_sync();
      const float mx = fmaxf(ms->xch[sb][0][row], ms->xch[sb][1][row]);
      if (!ok) continue;
      // running max: the first tile sets it; later tiles rescale O (in TMEM) only
      // when the max grew by more than kRescale (in logit units).  Both halves of a
      // row take the same decision from the same values.
      float alpha = 1.f;
      bool resc = false;
      if (m_used == -INFINITY) {
        m_used = mx;
      } else if (mx > m_used + resc_raw) {
        alpha = ex2_approx((m_used - mx) * c1);
        m_used = mx;
        resc = true;
      }
      // P of this tile goes into the one P buffer, and a rescale touches O: both
      // wait until P V of the previous tile is done (it was issued when the previous
      // tile's P was complete, so it has usually finished by now)
      if (j > 0 && !wwait(&ms->o_done, (uint32_t)((j - 1) & 1))) {
        ok = false;
        continue;
      }
      if (__any_sync(0xffffffffu, resc)) {
        tc_fence_after();
        float ov[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tmem_ld32(tO + cb + c * 32 + lsel, ov);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(tO + cb + c * 32 + lsel, ov);
        }
        tmem_wait_st();
        tc_fence_before();
        l2.x *= alpha; l2.y *= alpha;
        lx2.x *= alpha; lx2.y *= alpha;
      }
      // P = e^(scale * (u - m)) as bf16, row `row` of this half's swizzled 64-key A tile
      const float nm = -m_used * c1;
      unsigned char* pbuf = smem + OFF_P + hh * HALF;
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 a = __ffma2_rn(make_float2(sv[c16 * 8 + 2 * e], sv[c16 * 8 + 2 * e + 1]),
                                      make_float2(c1, c1), make_float2(nm, nm));
          const float p0 = ex2_approx(a.x), p1 = ex2_approx(a.y);
          const __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
          // the row sum uses the rounded weights the tensor core multiplies, so
          // O / l is an exact convex combination of them (a dominant weight's
          // rounding cancels between numerator and denominator)
          l2 = __fadd2_rn(l2, __bfloat1622float2(pr));
          lx2 = __fadd2_rn(lx2, make_float2(p0, p1));
          w[e] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        *reinterpret_cast<uint4*>(pbuf + row * 128 + ((c16 ^ (row & 7)) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      // the last key tile: V rows past the sequence end must be finite for P V
      if (k0 + TILE > len && k0 + row >= len) {
        unsigned char* vt = smem + OFF_KV + s * KV_STAGE + 2 * HALF + hh * HALF;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(vt + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->p_full[sb]);
    }
    // every P V done (a single-phase barrier: no parity aliasing)
    if (ok && !wwait(&ms->o_final, 0u)) ok = false;
    // the halves' row sums (every warp reaches this point, failed or not)
    ms->xsum[hh][row] = make_float2(l2.x + l2.y, lx2.x + lx2.y);
    pair_sync();
    const float2 s0 = ms->xsum[0][row], s1 = ms->xsum[1][row];
    const float l_row = s0.x + s1.x, lx_row = s0.y + s1.y;
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / l_row;
      const bool store = tq < len;
      float* orow = p.O + (((size_t)b * p.Hq + h) * p.T_max + (store ? tq : 0)) * D + cb;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float ov[32];
        tmem_ld32(tO + cb + c * 32 + lsel, ov);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(orow + c * 32 + i) =
                make_float4(ov[i] * inv, ov[i + 1] * inv, ov[i + 2] * inv, ov[i + 3] * inv);
        }
      }
      if (store && hh == 0)
        p.lse[((size_t)b * p.Hq + h) * p.T_max + tq] = p.scale * m_used + logf(lx_row);
    } else {
      if (threadIdx.x == 0) set_status(p.status, ETA_DEVSTAT_TIMEOUT);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == NWARP_SM + 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

// ---------------------------------------------------------------------------------
// Two query tiles per CTA ("ping-pong").  One CTA per (batch row, query head, pair of
// 128-query tiles A = [q0, q0 + 128) and B = [q0 + 128, q0 + 256)), 576 threads:
//   warps 0-7   softmax of tile A, warps 8-15 softmax of tile B (two threads per
//               query row, 64 key columns each, as in prefill_tc_kernel)
//   warp 16     TMA producer: both query tiles, then 128-key K and V tiles into a
//               2-stage ring; each K/V tile serves both query tiles
//   warp 17     MMA issuer: S_X = Q_X K^T and O_X += P_X V for X = A, B
// TMEM (512 columns): S_A, S_B, O_A, O_B (128 each).  P_X is written by its softmax
// threads into the S_X columns they have already read (half h of a row into columns
// 64 h .. 64 h + 31 of S_X, two bf16 per column) and read from there by P V as the
// A operand (tcgen05.mma with A in tensor memory).  While one tile's softmax runs,
// the tensor core works on the other tile, so neither waits for the other's chain.
// Tile X's chain per key tile: QK_X -> softmax_X -> P V_X -> QK_X of the next tile
// (issued once P V_X has read P_X out of the S_X columns).  Every wait is bounded.
namespace pp {

constexpr int NWG = 8;                          // softmax warps per query tile
constexpr int NT = (2 * NWG + 2) * 32;
constexpr int OFF_QA = 0, OFF_QB = 2 * HALF;    // two halves each
constexpr int OFF_KV = 4 * HALF;
constexpr int OFF_MISC = OFF_KV + NKV * KV_STAGE;

struct Misc {
  uint64_t q_full, kv_full[NKV], kv_empty[NKV];
  uint64_t s_full[2], p_full[2], pv_done[2], o_final[2], fin;
  float xch[2][2][2][TILE];   // [tile][parity][half][row]: the row maxima of a key tile
  float2 xsum[2][2][TILE];    // [tile][half][row]: the final row sums
  uint32_t tmem_base;
  int abort_flag;
};
constexpr int SMEM_BYTES = OFF_MISC + (int)sizeof(Misc) + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "prefill ping-pong shared memory");

ETA_DEV void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                        uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

ETA_DEV void tmem_st16u(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

template <int G, bool HARD>
__global__ void __launch_bounds__(NT, 1)
prefill_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  ETA_PDL_ENTRY();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Misc* ms = reinterpret_cast<Misc*>(smem + OFF_MISC);
  volatile int* abort_flag = &ms->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // heaviest tile pairs (most keys) first
  const int qp = p.ntiles - 1 - (int)(blockIdx.x % p.ntiles);   // ntiles: tile pairs here
  const int bh = blockIdx.x / p.ntiles;
  const int b = bh / p.Hq, h = bh % p.Hq, g = h / G;
  const int len = min(max(p.lengths[b], 0), p.T_max);
  const int q0 = qp * 2 * TILE;
  if (q0 >= len) return;                              // uniform, before any barrier
  // key tiles of A: 0 .. q0 / 128 (its diagonal last); of B: one more, if B holds a
  // valid query
  const int nA = q0 / TILE + 1;
  const int nB = (q0 + TILE < len) ? nA + 1 : 0;
  const int nkv = nB > 0 ? nB : nA;

  if (threadIdx.x == 0) {
    mbar_init(&ms->q_full, 1);
    for (int s = 0; s < NKV; ++s) {
      mbar_init(&ms->kv_full[s], 1);
      mbar_init(&ms->kv_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&ms->s_full[x], 1);
      mbar_init(&ms->p_full[x], NWG);
      mbar_init(&ms->pv_done[x], 1);
      mbar_init(&ms->o_final[x], 1);
    }
    mbar_init(&ms->fin, 1);
    ms->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2 * NWG + 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&ms->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  const uint32_t tS[2] = {tmem, tmem + 128}, tO[2] = {tmem + 256, tmem + 384};

  if (warp == 2 * NWG) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      const int qrow = (b * p.Hq + h) * p.T_max + q0;
      mbar_arrive_expect_tx(&ms->q_full, (nB > 0 ? 4 : 2) * HALF);
      tma_load_2d(smem + OFF_QA, &tmQ, 0, qrow, &ms->q_full);
      tma_load_2d(smem + OFF_QA + HALF, &tmQ, 64, qrow, &ms->q_full);
      if (nB > 0) {
        tma_load_2d(smem + OFF_QB, &tmQ, 0, qrow + TILE, &ms->q_full);
        tma_load_2d(smem + OFF_QB + HALF, &tmQ, 64, qrow + TILE, &ms->q_full);
      }
      int j = 0;
      for (; j < nkv && ok; ++j) {
        const int s = j % NKV;
        // (checked build) the key tile lies inside the cache row; a refused copy ends
        // the CTA like a lost wait, after the copies already issued
        if (!ETA_IN_BOUNDS((j + 1) * TILE - 1, p.T_max, p.status) ||
            !mbar_wait(&ms->kv_empty[s], ((uint32_t)(j / NKV) & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        unsigned char* st = smem + OFF_KV + s * KV_STAGE;
        const int krow = (b * p.Hkv + g) * p.T_max + j * TILE;
        mbar_arrive_expect_tx(&ms->kv_full[s], 4 * HALF);
        tma_load_2d(st, &tmK, 0, krow, &ms->kv_full[s]);
        tma_load_2d(st + HALF, &tmK, 64, krow, &ms->kv_full[s]);
        tma_load_2d(st + 2 * HALF, &tmV, 0, krow, &ms->kv_full[s]);
        tma_load_2d(st + 3 * HALF, &tmV, 64, krow, &ms->kv_full[s]);
      }
      if (!ok) {
        // wait (bounded) for every copy this thread issued before the CTA exits
        set_status(p.status, ETA_DEVSTAT_TIMEOUT);
        *abort_flag = 1;
        mbar_wait(&ms->q_full, 0, nullptr);
        for (int k = max(0, j - NKV); k < j; ++k)
          mbar_wait(&ms->kv_full[k % NKV], (uint32_t)(k / NKV) & 1u, nullptr);
      }
    }
  } else if (warp == 2 * NWG + 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&ms->q_full, 0, abort_flag);
      const int nX[2] = {nA, nB};
      const uint32_t qa[2] = {smem_u32(smem + OFF_QA), smem_u32(smem + OFF_QB)};
      auto issue_qk = [&](int x, int j) -> bool {     // S_X = Q_X K_j^T
        const int s = j % NKV;
        if (!mbar_wait(&ms->kv_full[s], (uint32_t)(j / NKV) & 1u, abort_flag)) return false;
        // S_X's columns hold P_X of the previous key tile until P V has read them
        if (j > 0 && !mbar_wait(&ms->pv_done[x], (uint32_t)((j - 1) & 1), abort_flag))
          return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(smem + OFF_KV + s * KV_STAGE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * HALF + (uint32_t)(kk & 3) * 32;
          mma_f16(tS[x], smem_desc(qa[x] + off, 16, 1024, tc::kSwizzle128),
                  smem_desc(ka + off, 16, 1024, tc::kSwizzle128), kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&ms->s_full[x]);
        return true;
      };
      auto issue_pv = [&](int x, int j) -> bool {     // O_X += P_X V_j
        const int s = j % NKV;
        if (!mbar_wait(&ms->p_full[x], (uint32_t)(j & 1), abort_flag)) return false;
        tc_fence_after();
        const uint32_t v0 = smem_u32(smem + OFF_KV + s * KV_STAGE + 2 * HALF);
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) {
          // keys 16 kk .. 16 kk + 15: half kk / 4 of the row, 8 columns per 16 keys
          const uint32_t pa = tS[x] + (uint32_t)(kk >> 2) * 64 + (uint32_t)(kk & 3) * 8;
          mma_f16_ts(tO[x], pa, smem_desc(v0 + kk * 2048, HALF, 1024, tc::kSwizzle128),
                     kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&ms->pv_done[x]);
        if (j == nX[x] - 1) mma_commit(&ms->o_final[x]);
        return true;
      };
      // QK of both tiles' first key tile, then per key tile: P V of A, the next QK
      // of A, P V of B, the next QK of B; a K/V slot is released after its last P V
      if (ok) ok = issue_qk(0, 0);
      if (ok && nB > 0) ok = issue_qk(1, 0);
      for (int j = 0; j < nkv && ok; ++j) {
        if (j < nA) {
          ok = issue_pv(0, j);
          if (ok && j + 1 < nA) ok = issue_qk(0, j + 1);
        }
        if (ok && j < nB) ok = issue_pv(1, j);
        if (ok) mma_commit(&ms->kv_empty[j % NKV]);   // after the last P V of key tile j
        if (ok && j + 1 < nB) ok = issue_qk(1, j + 1);
      }
      if (!ok) {
        set_status(p.status, ETA_DEVSTAT_TIMEOUT);
        *abort_flag = 1;
      }
      mma_commit(&ms->fin);
      mbar_wait(&ms->fin, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------------ softmax
    const int x = warp >= NWG ? 1 : 0;                // query tile of this warp
    const int wl = warp - x * NWG;                    // warp within the tile's group
    const int hh = wl >> 2;                           // key-column half of the tile
    const int row = threadIdx.x & (TILE - 1);         // query row of the tile = TMEM lane
    const int nkx = x == 0 ? nA : nB;
    const int qx = q0 + x * TILE;
    const int tq = qx + row;
    const uint32_t lsel = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t cb = (uint32_t)hh * 64;            // first column of this half
    const float tau = (tq < p.T_max) ? p.tau[((size_t)b * p.Hq + h) * p.T_max + tq] : 0.f;
    // raw-unit gate and exponent constants, as in prefill_tc_kernel
    const float tau_raw = tau / p.scale;
    const float ta = 0.5f * p.scale * p.invT, tb = 0.5f * tau * p.invT;
    const float c1 = p.scale * kLog2e;
    const float resc_raw = kRescale / p.scale;
    float m_used = -INFINITY;
    float2 l2 = make_float2(0.f, 0.f), lx2 = make_float2(0.f, 0.f);
    bool ok = true;
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    // the two warps holding the halves of the same rows meet at their own barrier
    const int pair_bar = 4 + x * 4 + (warp & 3);
    auto pair_sync = [&] { named_bar_sync(pair_bar, 64); };
    for (int j = 0; j < nkx; ++j) {
      const int sb = j & 1, s = j % NKV;
      const int k0 = j * TILE;
      if (ok && !wwait(&ms->s_full[x], (uint32_t)(j & 1))) ok = false;
      float mxh = -INFINITY;
      if (ok) {
        // the gated logits go back into the same S_X columns (32 at a time), so that
        // no thread holds all 64 of them across the row-max exchange
        tc_fence_after();
        float pm[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) pm[u] = -INFINITY;
        auto gate = [&](float v) -> float {
          if constexpr (HARD) return v >= tau_raw ? v : 0.f;
          const float hs = 0.5f * v;
          return fmaf(hs, tanh_approx(fmaf(v, ta, -tb)), hs);
        };
        if (j == nkx - 1) {
          // the diagonal tile (k0 == qx): keys past the row's query are masked
          const int lim = tq - k0 - (int)cb;           // columns c <= lim are causal
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            float sv[32];
            tmem_ld32(tS[x] + cb + ch * 32 + lsel, sv);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const float y0 = (ch * 32 + c <= lim) ? gate(sv[c]) : -INFINITY;
              const float y1 = (ch * 32 + c + 1 <= lim) ? gate(sv[c + 1]) : -INFINITY;
              sv[c] = y0;
              sv[c + 1] = y1;
              pm[(c >> 1) & 7] = fmax3(pm[(c >> 1) & 7], y0, y1);
            }
            tmem_st32(tS[x] + cb + ch * 32 + lsel, sv);
          }
        } else {
          // every key of an earlier tile precedes every query of this one
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            float sv[32];
            tmem_ld32(tS[x] + cb + ch * 32 + lsel, sv);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              float y0, y1;
              if constexpr (HARD) {
                // s * [s >= tau / scale]: a 1.0 / 0.0 flag per score (set.ge) and one
                // packed multiply for two scores (S is finite)
                float g0, g1;
                asm("set.ge.f32.f32 %0, %1, %2;" : "=f"(g0) : "f"(sv[c]), "f"(tau_raw));
                asm("set.ge.f32.f32 %0, %1, %2;" : "=f"(g1) : "f"(sv[c + 1]), "f"(tau_raw));
                const float2 y = __fmul2_rn(make_float2(sv[c], sv[c + 1]), make_float2(g0, g1));
                y0 = y.x;
                y1 = y.y;
              } else {
                y0 = gate(sv[c]);
                y1 = gate(sv[c + 1]);
              }
              sv[c] = y0;
              sv[c + 1] = y1;
              pm[(c >> 1) & 7] = fmax3(pm[(c >> 1) & 7], y0, y1);
            }
            tmem_st32(tS[x] + cb + ch * 32 + lsel, sv);
          }
        }
        mxh = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                    fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
      }
      ms->xch[x][sb][hh][row] = mxh;
      pair_sync();
      const float mx = fmaxf(ms->xch[x][sb][0][row], ms->xch[x][sb][1][row]);
      if (!ok) continue;
      float alpha = 1.f;
      bool resc = false;
      if (m_used == -INFINITY) {
        m_used = mx;
      } else if (mx > m_used + resc_raw) {
        alpha = ex2_approx((m_used - mx) * c1);
        m_used = mx;
        resc = true;
      }
      if (__any_sync(0xffffffffu, resc)) {
        // P V of the previous key tile is complete: QK of this one waited for it
        float ov[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tmem_ld32(tO[x] + cb + c * 32 + lsel, ov);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(tO[x] + cb + c * 32 + lsel, ov);
        }
        l2.x *= alpha; l2.y *= alpha;
        lx2.x *= alpha; lx2.y *= alpha;
      }
      // P = e^(scale * (u - m)) as bf16 pairs into the 32 S_X columns this half read,
      // 16 columns (32 keys) at a time
      const float nm = -m_used * c1;
      tmem_wait_st();                                  // the gated logits are in TMEM
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        float sv[32];
        tmem_ld32(tS[x] + cb + ch * 32 + lsel, sv);
        tmem_wait_ld();
        uint32_t pw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c = 2 * e;
          const float2 a = __ffma2_rn(make_float2(sv[c], sv[c + 1]), make_float2(c1, c1),
                                      make_float2(nm, nm));
          const float p0 = ex2_approx(a.x), p1 = ex2_approx(a.y);
          const __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
          // the row sum uses the rounded weights the tensor core multiplies
          l2 = __fadd2_rn(l2, __bfloat1622float2(pr));
          lx2 = __fadd2_rn(lx2, make_float2(p0, p1));
          pw[e] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        tmem_st16u(tS[x] + cb + ch * 16 + lsel, pw);
      }
      // the query tile holding position len - 1 zeroes the V rows past it (its
      // diagonal key tile is the only one that reaches past the sequence end)
      if (k0 + TILE > len && k0 + row >= len) {
        unsigned char* vt = smem + OFF_KV + s * KV_STAGE + 2 * HALF + hh * HALF;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(vt + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        fence_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->p_full[x]);
    }
    if (ok && nkx > 0 && !wwait(&ms->o_final[x], 0u)) ok = false;
    ms->xsum[x][hh][row] = make_float2(l2.x + l2.y, lx2.x + lx2.y);
    pair_sync();
    const float2 s0 = ms->xsum[x][0][row], s1 = ms->xsum[x][1][row];
    const float l_row = s0.x + s1.x, lx_row = s0.y + s1.y;
    if (ok && nkx > 0) {
      tc_fence_after();
      const float inv = 1.f / l_row;
      const bool store = tq < len;
      float* orow = p.O + (((size_t)b * p.Hq + h) * p.T_max + (store ? tq : 0)) * D + cb;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float ov[32];
        tmem_ld32(tO[x] + cb + c * 32 + lsel, ov);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(orow + c * 32 + i) =
                make_float4(ov[i] * inv, ov[i + 1] * inv, ov[i + 2] * inv, ov[i + 3] * inv);
        }
      }
      if (store && hh == 0)
        p.lse[((size_t)b * p.Hq + h) * p.T_max + tq] = p.scale * m_used + logf(lx_row);
    } else if (!ok) {
      if (threadIdx.x == 0) set_status(p.status, ETA_DEVSTAT_TIMEOUT);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2 * NWG + 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

}  // namespace pp

}  // namespace pf

template <int G>
static eta_status_t launch_prefill(const CUtensorMap& mq, const CUtensorMap& mk,
                                   const CUtensorMap& mv, const pf::PrefillParams& prm,
                                   int ctas, cudaStream_t s) {
  if (!set_smem_once<pf::prefill_tc_kernel<G>>(pf::SMEM_BYTES)) return ETA_ERR_CUDA;
  return launch_k(pf::prefill_tc_kernel<G>, dim3(ctas), dim3(pf::NT), pf::SMEM_BYTES, s, mq, mk,
                  mv, prm);
}

template <int G, bool HARD>
static eta_status_t launch_prefill_pp(const CUtensorMap& mq, const CUtensorMap& mk,
                                      const CUtensorMap& mv, pf::PrefillParams prm,
                                      int B, cudaStream_t s) {
  using namespace pf;
  prm.ntiles = (prm.T_max + 2 * TILE - 1) / (2 * TILE);   // query tile pairs
  const int64_t ctas = (int64_t)B * prm.Hq * prm.ntiles;
  if (!set_smem_once<pp::prefill_pp_kernel<G, HARD>>(pp::SMEM_BYTES)) return ETA_ERR_CUDA;
  return launch_k(pp::prefill_pp_kernel<G, HARD>, dim3((unsigned)ctas), dim3(pp::NT),
                  pp::SMEM_BYTES, s, mq, mk, mv, prm);
}

std::atomic<int> g_prefill_kernel{ETA_PREFILL_AUTO};

// Which kernel eta_prefill launches.  Measured on one B200 (16 / 4 heads, d = 128):
// the two-tile kernel is faster once its tile pairs fill the SMs (B = 4, T = 8192:
// 742 vs 580 TFLOP/s hard gate, 626 vs 559 soft), but it has half as many CTAs, each
// twice as long, so on small launches idle SMs and the longest pair decide: at 64
// pairs (B = 1, T = 1024) it takes 32 vs 22 us; at 256 pairs (B = 1, T = 4096) it still
// wins with the hard gate (158 vs 164 us) and loses with the soft gate (186 vs 170 us).
inline bool prefill_two_tile(const eta_dims_t* d, bool hard) {
  const int k = g_prefill_kernel.load();
  if (k != ETA_PREFILL_AUTO) return k == ETA_PREFILL_TWO_TILE;
  const int64_t pairs = (int64_t)d->B * d->Hq * ((d->T_max / pf::TILE + 1) / 2);
  const int64_t n = std::max(sm_count(), 1);
  return hard ? pairs > n / 2 : pairs > 2 * n;
}

}  // namespace eta

using namespace eta;

extern "C" eta_status_t eta_prefill(const eta_dims_t* dims, const eta_bf16_t* Q, const float* tau,
                                    const eta_bf16_t* K, const eta_bf16_t* V,
                                    const int32_t* lengths, float T, float scale, float* O,
                                    float* lse, int32_t* dev_status, void* stream) {
  eta_status_t st = check_dims(dims, /*rows_in_grid_y=*/false);   // 1-D grid
  if (st != ETA_OK) return st;
  if (!Q || !tau || !K || !V || !lengths || !O || !lse) return ETA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return ETA_ERR_INVALID_ARG;
  if (!(T >= 0.f) || isinf(T)) return ETA_ERR_INVALID_ARG;
  if (dims->d != 128 || dims->T_max % pf::TILE != 0) return ETA_ERR_UNSUPPORTED;
  const uint64_t kv_rows = (uint64_t)dims->B * dims->Hkv * dims->T_max;
  const uint64_t q_rows = (uint64_t)dims->B * dims->Hq * dims->T_max;
  if (q_rows >= (1ull << 31)) return ETA_ERR_UNSUPPORTED;
  const int ntiles = dims->T_max / pf::TILE;
  const int64_t ctas = (int64_t)dims->B * dims->Hq * ntiles;
  if (ctas > 0x7fffffff) return ETA_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, q_rows, pf::TILE) || !make_map(&mk, K, kv_rows, pf::TILE) ||
      !make_map(&mv, V, kv_rows, pf::TILE))
    return ETA_ERR_CUDA;
  pf::PrefillParams prm;
  prm.Hq = dims->Hq; prm.Hkv = dims->Hkv; prm.T_max = dims->T_max; prm.ntiles = ntiles;
  prm.scale = scale == 0.f ? 1.f / sqrtf((float)dims->d) : scale;
  prm.invT = T == 0.f ? -1.f : 1.f / T;
  prm.tau = tau; prm.lengths = lengths; prm.O = O; prm.lse = lse; prm.status = dev_status;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool hard = prm.invT < 0.f;
  if (prefill_two_tile(dims, hard)) {
    switch ((dims->Hq / dims->Hkv) * (hard ? 1 : -1)) {
      case 1: return launch_prefill_pp<1, true>(mq, mk, mv, prm, dims->B, s);
      case 2: return launch_prefill_pp<2, true>(mq, mk, mv, prm, dims->B, s);
      case 4: return launch_prefill_pp<4, true>(mq, mk, mv, prm, dims->B, s);
      case 8: return launch_prefill_pp<8, true>(mq, mk, mv, prm, dims->B, s);
      case -1: return launch_prefill_pp<1, false>(mq, mk, mv, prm, dims->B, s);
      case -2: return launch_prefill_pp<2, false>(mq, mk, mv, prm, dims->B, s);
      case -4: return launch_prefill_pp<4, false>(mq, mk, mv, prm, dims->B, s);
      case -8: return launch_prefill_pp<8, false>(mq, mk, mv, prm, dims->B, s);
    }
    return ETA_ERR_UNSUPPORTED;
  }
  switch (dims->Hq / dims->Hkv) {
    case 1: return launch_prefill<1>(mq, mk, mv, prm, (int)ctas, s);
    case 2: return launch_prefill<2>(mq, mk, mv, prm, (int)ctas, s);
    case 4: return launch_prefill<4>(mq, mk, mv, prm, (int)ctas, s);
    case 8: return launch_prefill<8>(mq, mk, mv, prm, (int)ctas, s);
  }
  return ETA_ERR_UNSUPPORTED;
}

extern "C" eta_status_t eta_set_prefill_kernel(eta_prefill_kernel_t kernel) {
  if (kernel != ETA_PREFILL_AUTO && kernel != ETA_PREFILL_ONE_TILE &&
      kernel != ETA_PREFILL_TWO_TILE)
    return ETA_ERR_INVALID_ARG;
  g_prefill_kernel.store((int)kernel);
  return ETA_OK;
}

extern "C" eta_prefill_kernel_t eta_get_prefill_kernel(void) {
  return static_cast<eta_prefill_kernel_t>(g_prefill_kernel.load());
}

extern "C" int32_t eta_prefill_kernel_for(const eta_dims_t* dims, float T) {
  if (check_dims(dims, /*rows_in_grid_y=*/false) != ETA_OK) return -1;
  if (!(T >= 0.f) || isinf(T) || dims->d != 128 || dims->T_max % pf::TILE != 0) return -1;
  return prefill_two_tile(dims, T == 0.f) ? ETA_PREFILL_TWO_TILE : ETA_PREFILL_ONE_TILE;
}
