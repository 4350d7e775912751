// Gated block-sparse decode attention over the admitted-union blocks
// (arXiv 2609.20888 abstract: hard-pruned KV blocks, co-admitted tokens absorbed;
// evolve.pub review, Methodology Assessment Eq. 2-3: m = sigmoid(beta (S - tau)),
// gated logits S * m; review FAQ: a sub-threshold logit goes to 0, weight e^0 = 1).
//
// Pipeline per step (three launches on one stream; two when the tensor-core decode
// plans its own shares, at 128 to 2048 pairs):
//   plan_kernel    prefix sum of admitted blocks over (row, KV head) pairs, and the
//                  first pair of every CTA's share.  The admitted blocks of all pairs,
//                  laid end to end, are cut into equal contiguous shares, one per CTA
//                  (persistent grid = SM count), so every SM streams the same bytes
//                  whatever the per-pair density.
//   decode         decode_tc_kernel (tcgen05 engine, d = 128: decode_tc.cuh) or
//   decode_kernel  (this file, the CUDA-core engine): one producer warp issues 1-D TMA bulk copies (cp.async.bulk) of
//                  64-key K and V tiles into a ring of shared-memory stages guarded by
//                  mbarriers; NCW consumer warps compute, for the G query heads of the
//                  group, q.k on CUDA cores (lane = d/32 dims, transposed butterfly
//                  reduction), the gate, an fp32 online softmax and o += p v.  When the
//                  share crosses a (row, KV head) boundary the warps merge their states
//                  and write one partial (m, l, o) slot.
//   combine_kernel log-sum-exp merge of the partial slots of each (row, head), plus the
//                  floor term of pruned blocks in FLOOR mode.
#include <cudaTypedefs.h>
#include <math.h>

#include <atomic>
#include <mutex>

#include "combine_dev.cuh"
#include "decode_tc.cuh"
#include "eta_common.cuh"
#include "eta_host.h"
#include "tma_host.h"

namespace eta {

constexpr int kStageKeys = 64;   // keys per pipeline stage (a 64- or 128-key block = 1 or 2)
constexpr int kPlanThreads = 1024;
constexpr int kStageEnd = 1;

struct StageInfo {
  int row;     // (batch row, KV head) pair
  int tok0;    // token index of the stage's first key
  int nvalid;  // valid keys in the stage (1..64)
  int flags;
};

struct DecodeParams {
  int Hq, Hkv, T_max, NB, blk;
  int R;               // (row, KV head) pairs

  float scale, invT;   // invT < 0 selects the hard gate
  const eta_bf16_t* q;
  const float* tau;
  const eta_bf16_t* K;
  const eta_bf16_t* V;
  const int32_t* lengths;
  const int32_t* union_idx;
  const int32_t* row_off;
  const int32_t* cta_row;
  const int32_t* plan;
  float* part_o;
  float* part_ml;
  int32_t* status;
};

template <int D, int G, int NCW, int NSTAGES>
struct DecodeCfg {
  static constexpr int KG = 32 / G;                 // keys per warp group (KG * G = 32)
  static constexpr int NGROUPS = kStageKeys / KG;
  static constexpr int DPL = D / 32;                // dims per lane
  static constexpr int TILE = kStageKeys * D * 2;   // bytes of K (or V) per stage
  static constexpr int NT = (NCW + 1) * 32;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = NSTAGES * TILE;
  static constexpr int OFF_MO = 2 * NSTAGES * TILE;
  static constexpr int OFF_MML = OFF_MO + NCW * G * D * 4;
  static constexpr int OFF_PW = OFF_MML + NCW * G * 2 * 4;
  static constexpr int OFF_INFO = OFF_PW + NCW * 32 * 4;
  static constexpr int OFF_BAR = OFF_INFO + NSTAGES * (int)sizeof(StageInfo);
  static constexpr int OFF_FLAG = OFF_BAR + 2 * NSTAGES * 8;
  static constexpr int SMEM = OFF_FLAG + 16;
};

template <int DPL>
ETA_DEV void lds_row(const eta_bf16_t* p, float (&x)[DPL]) {
  if constexpr (DPL == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    x[0] = bf16_lo(w); x[1] = bf16_hi(w);
  }
}

// Lane l ends with the warp-wide sum of v[l] (32 values, 31 shuffles).
ETA_DEV float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = up ? v[i] : v[i + w];
      const float keep = up ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
}

template <int D, int G, bool DENSE, int NCW, int NSTAGES>
__global__ void __launch_bounds__((NCW + 1) * 32, 1) decode_kernel(const DecodeParams p) {
  ETA_PDL_ENTRY();
  using C = DecodeCfg<D, G, NCW, NSTAGES>;
  constexpr int DPL = C::DPL, KG = C::KG;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + NSTAGES;
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + C::OFF_INFO);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAG);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int Ntot = p.plan[0], chunk = p.plan[1];
  const int a = blockIdx.x * chunk;
  if (a >= Ntot) return;  // uniform over the CTA, before any barrier
  const int e = min(a + chunk, Ntot);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // ------------------------------------------------------------------ producer
  if (warp == NCW) {
    if (lane != 0) return;
    int r = p.cta_row[blockIdx.x];
    bool ok = true;
    if (!ETA_IN_BOUNDS(r, p.R, p.status)) {   // checked build: give up like a lost wait
      r = 0;
      ok = false;
    }
    int roff = p.row_off[r], rend = p.row_off[r + 1];
    int it = 0;
    for (int pos = a; pos < e && ok; ++pos) {
      while (pos >= rend) {
        if (!ETA_IN_BOUNDS(r + 2, p.R + 1, p.status)) {
          ok = false;
          break;
        }
        ++r;
        roff = rend;
        rend = p.row_off[r + 1];
      }
      if (!ok || (!DENSE && !ETA_IN_BOUNDS(pos - roff, p.NB, p.status))) {
        ok = false;
        break;
      }
      const int b = r / p.Hkv;
      const int len = min(max(p.lengths[b], 0), p.T_max);
      const int j = DENSE ? pos - roff : p.union_idx[(size_t)r * p.NB + (pos - roff)];
      if (j < 0 || j >= p.NB || j * p.blk >= len) {
        set_status(p.status, ETA_DEVSTAT_BAD_BLOCK);
        continue;
      }
      for (int sub = 0; sub < p.blk / kStageKeys; ++sub) {
        const int t0 = j * p.blk + sub * kStageKeys;
        const int nv = min(kStageKeys, len - t0);
        if (nv <= 0) break;
        const int s = it % NSTAGES;
        const uint32_t ph = (uint32_t)(it / NSTAGES) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        info[s] = StageInfo{r, t0, nv, 0};
        const uint32_t bytes = (uint32_t)nv * D * 2;
        mbar_arrive_expect_tx(&full[s], 2 * bytes);
        const size_t goff = ((size_t)r * p.T_max + t0) * D;
        bulk_g2s(smem + C::OFF_K + s * C::TILE, p.K + goff, bytes, &full[s]);
        bulk_g2s(smem + C::OFF_V + s * C::TILE, p.V + goff, bytes, &full[s]);
        ++it;
      }
    }
    if (ok) {
      const int s = it % NSTAGES;
      const uint32_t ph = (uint32_t)(it / NSTAGES) & 1u;
      if (mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
        info[s] = StageInfo{-1, 0, 0, kStageEnd};
        mbar_arrive(&full[s]);
      } else {
        ok = false;
      }
    }
    if (!ok) {
      set_status(p.status, ETA_DEVSTAT_TIMEOUT);
      *abort_flag = 1;
      // let every copy already issued land before the CTA's shared memory goes away
      for (int k = max(0, it - NSTAGES); k < it; ++k)
        mbar_wait(&full[k % NSTAGES], (uint32_t)(k / NSTAGES) & 1u, nullptr);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  float* mo = reinterpret_cast<float*>(smem + C::OFF_MO);
  float* mml = reinterpret_cast<float*>(smem + C::OFF_MML);
  float* pw = reinterpret_cast<float*>(smem + C::OFF_PW) + warp * 32;
  const int hl = lane % G;  // head of this lane's softmax slot
  float qr[G][DPL], o[G][DPL];
  float m_run = -INFINITY, l_run = 0.f, tau_l = 0.f;
  int cur = -1;

  auto flush = [&](int row) {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < DPL; ++i) mo[(warp * G + h) * D + lane * DPL + i] = o[h][i];
    if (lane < G) {
      mml[(warp * G + lane) * 2] = m_run;
      mml[(warp * G + lane) * 2 + 1] = l_run;
    }
    named_bar_sync(1, NCW * 32);
    const size_t slot = (size_t)blockIdx.x + row;
    const bool slot_ok = ETA_IN_BOUNDS(slot, (long long)gridDim.x + p.R, p.status);
    for (int idx = threadIdx.x; idx < G * D && slot_ok; idx += NCW * 32) {
      const int h = idx / D, dd = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, mml[(w * G + h) * 2]);
      float O = 0.f, L = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < NCW; ++w) {
          const float sc = __expf(mml[(w * G + h) * 2] - M);
          O = fmaf(mo[(w * G + h) * D + dd], sc, O);
          L = fmaf(mml[(w * G + h) * 2 + 1], sc, L);
        }
      }
      p.part_o[(slot * G + h) * D + dd] = O;
      if (dd == 0) {
        p.part_ml[(slot * G + h) * 2] = M;
        p.part_ml[(slot * G + h) * 2 + 1] = L;
      }
    }
    named_bar_sync(1, NCW * 32);
  };

  auto start_row = [&](int row) {
    const int b = row / p.Hkv, g = row % p.Hkv;
    const size_t qh0 = (size_t)b * p.Hq + (size_t)g * G;
    bool bad = false;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      lds_row<DPL>(p.q + (qh0 + h) * D + lane * DPL, qr[h]);
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        bad |= !isfinite(qr[h][i]);
        o[h][i] = 0.f;
      }
    }
    if (bad) set_status(p.status, ETA_DEVSTAT_NONFINITE_Q);
    if constexpr (!DENSE) tau_l = p.tau[qh0 + hl];
    m_run = -INFINITY;
    l_run = 0.f;
  };

  int it = 0;
  while (true) {
    const int s = it % NSTAGES;
    const uint32_t ph = (uint32_t)(it / NSTAGES) & 1u;
    if (!mbar_wait(&full[s], ph, abort_flag)) {
      if (lane == 0) set_status(p.status, ETA_DEVSTAT_TIMEOUT);
      *abort_flag = 1;
      return;
    }
    const StageInfo inf = info[s];
    if (inf.flags & kStageEnd) break;
    if (inf.row != cur) {
      if (cur >= 0) flush(cur);
      cur = inf.row;
      start_row(cur);
    }
    const eta_bf16_t* sK = reinterpret_cast<const eta_bf16_t*>(smem + C::OFF_K + s * C::TILE);
    const eta_bf16_t* sV = reinterpret_cast<const eta_bf16_t*>(smem + C::OFF_V + s * C::TILE);
    for (int grp = warp; grp < C::NGROUPS; grp += NCW) {
      const int k0 = grp * KG;
      if (k0 >= inf.nvalid) break;
      // q.k partials for KG keys x G heads, then one transposed reduction
      float part[32];
#pragma unroll
      for (int kk = 0; kk < KG; ++kk) {
        float kv[DPL];
        lds_row<DPL>(sK + (k0 + kk) * D + lane * DPL, kv);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < DPL; ++i) acc = fmaf(qr[h][i], kv[i], acc);
          part[kk * G + h] = acc;
        }
      }
      const float sraw = transpose_reduce32(part, lane);
      const int kk = lane / G;
      const bool valid = (k0 + kk) < inf.nvalid;
      const float sc = p.scale * sraw;
      float sp = sc;
      if constexpr (!DENSE) {
        if (p.invT < 0.f) {
          sp = sc >= tau_l ? sc : 0.f;
        } else {
          sp = sc * __frcp_rn(1.f + __expf((tau_l - sc) * p.invT));
        }
      }
      sp = valid ? sp : -INFINITY;
      float gm = sp;
#pragma unroll
      for (int off = G; off < 32; off <<= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, off));
      const float mnew = fmaxf(m_run, gm);
      const float alpha = (mnew == -INFINITY) ? 1.f : __expf(m_run - mnew);
      const float pr = valid ? __expf(sp - mnew) : 0.f;
      float ps = pr;
#pragma unroll
      for (int off = G; off < 32; off <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l_run = fmaf(l_run, alpha, ps);
      m_run = mnew;
      pw[lane] = pr;
      __syncwarp();
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float ah = __shfl_sync(0xffffffffu, alpha, h);
#pragma unroll
        for (int i = 0; i < DPL; ++i) o[h][i] *= ah;
      }
      const int nv = min(KG, inf.nvalid - k0);
#pragma unroll
      for (int k2 = 0; k2 < KG; ++k2) {
        if (k2 < nv) {
          float vv[DPL];
          lds_row<DPL>(sV + (k0 + k2) * D + lane * DPL, vv);
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float ph2 = pw[k2 * G + h];
#pragma unroll
            for (int i = 0; i < DPL; ++i) o[h][i] = fmaf(ph2, vv[i], o[h][i]);
          }
        }
      }
      __syncwarp();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    ++it;
  }
  if (cur >= 0) flush(cur);
}

// Prefix sum of admitted blocks per (row, KV head) pair and the CTA shares.
template <bool DENSE>
__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(int R, int Hkv, int NB, int blk, int T_max, const int32_t* __restrict__ union_cnt,
            const int32_t* __restrict__ lengths, int P, int32_t* __restrict__ row_off,
            int32_t* __restrict__ cta_row, int32_t* __restrict__ plan, int32_t* status) {
  ETA_PDL_ENTRY();
  __shared__ int wsum[kPlanThreads / 32];
  __shared__ int s_chunk;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int carry = 0;
  for (int base = 0; base < R; base += kPlanThreads) {
    const int r = base + tid;
    int c = 0;
    if (r < R) {
      if (DENSE) {
        int len = lengths[r / Hkv];
        if (len < 0 || len > T_max) {
          set_status(status, ETA_DEVSTAT_BAD_LENGTH);
          len = min(max(len, 0), T_max);
        }
        c = (len + blk - 1) / blk;
      } else {
        c = union_cnt[r];
        if (c < 0 || c > NB) {
          set_status(status, ETA_DEVSTAT_BAD_BLOCK);
          c = min(max(c, 0), NB);
        }
      }
    }
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int wpre = 0, total = 0;
    for (int i = 0; i < kPlanThreads / 32; ++i) {
      const int v = wsum[i];
      if (i < warp) wpre += v;
      total += v;
    }
    if (r < R) row_off[r] = carry + wpre + incl - c;
    carry += total;
    __syncthreads();
  }
  if (tid == 0) {
    row_off[R] = carry;
    int chunk = (carry + P - 1) / P;
    if (chunk < kMinChunk) chunk = kMinChunk;
    plan[0] = carry;
    plan[1] = chunk;
    s_chunk = chunk;
  }
  __syncthreads();
  const int chunk = s_chunk;
  for (int r = tid; r < R; r += kPlanThreads) {
    const int off = row_off[r], c = row_off[r + 1] - off;
    if (c <= 0) continue;
    const int p0 = (off + chunk - 1) / chunk;
    const int p1 = (off + c + chunk - 1) / chunk;
    for (int pp = p0; pp < p1 && pp < P; ++pp) cta_row[pp] = r;
  }
}

// One CTA per (row, KV head), thread = dim: merges the row's partial slots
// (combine_merge), then in FLOOR mode adds the pruned blocks' keys with logit 0.
template <int D, int G>
__global__ void __launch_bounds__(D) combine_kernel(const CombineParams p) {
  ETA_PDL_ENTRY();
  extern __shared__ uint32_t adm[];     // FLOOR mode: admitted-block bitmap of the row
  __shared__ CombineScratch<G> sc;
  __shared__ int s_nfloor;
  const int r = blockIdx.x, b = r / p.Hkv, g = r % p.Hkv;
  const int dd = threadIdx.x;
  const int off = p.row_off[r];
  int c = p.row_off[r + 1] - off;
  if (!ETA_IN_BOUNDS(c, p.NB + 1, p.status)) c = 0;   // checked build: a pair's list fits its row
  const int chunk = p.plan[1];
  float fv = 0.f;
  int nfloor = 0;
  if (p.floor_mode) {
    const int NW = (p.NB + 31) / 32;
    for (int w = dd; w < NW; w += D) adm[w] = 0u;
    if (dd == 0) s_nfloor = 0;
    __syncthreads();
    for (int i = dd; i < c; i += D) {
      const int j = p.union_idx[(size_t)r * p.NB + i];
      if (j >= 0 && j < p.NB) atomicOr(&adm[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    int myn = 0;
    for (int j = 0; j < p.NB; ++j) {
      if ((adm[j >> 5] >> (j & 31)) & 1u) continue;
      const int n = p.cnt[(size_t)r * p.NB + j];
      if (n <= 0) continue;
      fv += p.vsum[((size_t)r * p.NB + j) * D + dd];
      if (dd == 0) myn += n;
    }
    if (dd == 0) s_nfloor = myn;
    __syncthreads();
    nfloor = s_nfloor;
  }
  const int p0 = c > 0 ? off / chunk : 0;
  const int ns = c > 0 ? (off + c - 1) / chunk - p0 + 1 : 0;
  float O[G];
  combine_merge<D, G, false>(p.part_ml, p.part_o, r, p0, ns, dd, sc, O, [] { __syncthreads(); },
                             (long long)p.P + gridDim.x, p.status);
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float M = sc.M[h], L = sc.L[h], Oh = O[h];
    if (nfloor > 0) {
      const float Mf = fmaxf(M, 0.f);
      const float a = (M == -INFINITY) ? 0.f : expf(M - Mf);
      const float e0 = expf(-Mf);
      Oh = Oh * a + fv * e0;
      L = L * a + (float)nfloor * e0;
      M = Mf;
    }
    combine_store<D>(p.o, p.lse, (size_t)b * p.Hq + (size_t)g * G + h, dd, M, L, Oh);
  }
}

// ---------------------------------------------------------------- host side
constexpr int kNCW = 8;
template <int D> struct StagesFor;
template <> struct StagesFor<128> { static constexpr int value = 5; };
template <> struct StagesFor<64> { static constexpr int value = 8; };

struct WsLayout {
  size_t plan, row_off, cta_row, part_ml, part_o, total;
};

inline WsLayout ws_layout(const eta_dims_t* d, int P) {
  const size_t R = (size_t)d->B * d->Hkv, G = d->Hq / d->Hkv;
  WsLayout w;
  size_t x = 0;
  w.plan = x;    x += 256;
  w.row_off = x; x = align_up(x + (R + 1) * 4, 256);
  w.cta_row = x; x = align_up(x + (size_t)P * 4, 256);
  w.part_ml = x; x = align_up(x + ((size_t)P + R) * G * 2 * 4, 256);
  w.part_o = x;  x = align_up(x + ((size_t)P + R) * G * d->d * 4, 256);
  w.total = x;
  return w;
}

inline int decode_grid() {
  const int n = sm_count();
  return n > 0 ? n : 1;
}

template <int D, int G, bool DENSE>
eta_status_t launch_decode_t(const eta_dims_t* dims, const DecodeParams& prm, int P,
                             cudaStream_t s) {
  constexpr int NS = StagesFor<D>::value;
  using C = DecodeCfg<D, G, kNCW, NS>;
  auto kern = decode_kernel<D, G, DENSE, kNCW, NS>;
  if (!set_smem_once<decode_kernel<D, G, DENSE, kNCW, NS>>(C::SMEM)) return ETA_ERR_CUDA;
  return launch_k(kern, dim3(P), dim3(C::NT), C::SMEM, s, prm);
}

template <bool DENSE>
eta_status_t launch_decode(const eta_dims_t* dims, const DecodeParams& prm, int P,
                           cudaStream_t s) {
  const int G = dims->Hq / dims->Hkv;
#define ETA_DEC_CASE(DD, GG) \
  if (dims->d == DD && G == GG) return launch_decode_t<DD, GG, DENSE>(dims, prm, P, s);
  ETA_DEC_CASE(128, 1) ETA_DEC_CASE(128, 2) ETA_DEC_CASE(128, 4) ETA_DEC_CASE(128, 8)
  ETA_DEC_CASE(64, 1) ETA_DEC_CASE(64, 2) ETA_DEC_CASE(64, 4) ETA_DEC_CASE(64, 8)
#undef ETA_DEC_CASE
  return ETA_ERR_UNSUPPORTED;
}

inline eta_status_t launch_combine(const eta_dims_t* dims, const CombineParams& cp,
                                   cudaStream_t s) {
  const int G = dims->Hq / dims->Hkv, R = dims->B * dims->Hkv;
  const size_t smem = cp.floor_mode ? (size_t)((num_blocks(dims) + 31) / 32) * 4 : 0;
#define ETA_CMB_CASE(DD, GG)                                              \
  if (dims->d == DD && G == GG)                                           \
    return launch_k(combine_kernel<DD, GG>, dim3(R), dim3(DD), smem, s, cp);
  ETA_CMB_CASE(128, 1) ETA_CMB_CASE(128, 2) ETA_CMB_CASE(128, 4) ETA_CMB_CASE(128, 8)
  ETA_CMB_CASE(64, 1) ETA_CMB_CASE(64, 2) ETA_CMB_CASE(64, 4) ETA_CMB_CASE(64, 8)
#undef ETA_CMB_CASE
  return ETA_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------- tcgen05 engine host side
std::atomic<int> g_engine{ETA_ENGINE_AUTO};

inline bool use_tc(const eta_dims_t* d) {
  const int e = g_engine.load();
  if (e == ETA_ENGINE_FMA) return false;
  // TMA row coordinates are 32-bit
  const bool fits = (uint64_t)d->B * d->Hkv * d->T_max < (1ull << 31);
  // AUTO and TCGEN05: the tensor-core engine wherever it applies (measured ~1.6x the
  // FMA engine's bandwidth on the 128K / B = 64 workload)
  return (d->d == 128 || d->d == 64) && fits;
}

// Whether the tensor-core sparse decode plans its shares in the kernel.  Measured on
// one box: 0.4% faster per step with 256 (row, KV head) pairs, 0.7% slower with 32
// (the separate plan launch then overlaps the small screening launch's tail).
constexpr int kPlanInMinRows = 128;
inline bool plan_in_kernel(const eta_dims_t* d) {
  const int R = d->B * d->Hkv;
  return use_tc(d) && R >= kPlanInMinRows && R <= tc::kFusedMaxRows;
}

template <int G, bool DENSE, int DD>
eta_status_t launch_tc_t(const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mq,
                         const tc::TcParams& prm, int P, bool plan_in, cudaStream_t s) {
  if constexpr (!DENSE) {
    if (plan_in) {
      auto kern = tc::decode_tc_kernel<G, false, true, DD>;
      if (!set_smem_once<tc::decode_tc_kernel<G, false, true, DD>>(tc::FUSED_SMEM_BYTES))
        return ETA_ERR_CUDA;
      return launch_k(kern, dim3(P), dim3(tc::NT), tc::FUSED_SMEM_BYTES, s, mk, mv, mq, prm);
    }
  }
  auto kern = tc::decode_tc_kernel<G, DENSE, false, DD>;
  if (!set_smem_once<tc::decode_tc_kernel<G, DENSE, false, DD>>(tc::SMEM_BYTES))
    return ETA_ERR_CUDA;
  return launch_k(kern, dim3(P), dim3(tc::NT), tc::SMEM_BYTES, s, mk, mv, mq, prm);
}

// plan_in: the sparse decode lays out the shares itself from `counts` (no plan_kernel)
// and publishes row_off / plan (d.row_off, d.plan) for the combine.
template <bool DENSE>
eta_status_t launch_tc(const eta_dims_t* dims, const DecodeParams& d, const eta_bf16_t* q,
                       const eta_bf16_t* K, const eta_bf16_t* V, int P, bool plan_in,
                       const int32_t* counts, cudaStream_t s) {
  CUtensorMap mk, mv, mq;
  const uint64_t kv_rows = (uint64_t)dims->B * dims->Hkv * dims->T_max;
  const uint64_t dcols = (uint64_t)dims->d;
  if (!make_map(&mk, K, kv_rows, 64, dcols) || !make_map(&mv, V, kv_rows, 64, dcols) ||
      !make_map(&mq, q, (uint64_t)dims->B * dims->Hq, 16, dcols))
    return ETA_ERR_CUDA;
  tc::TcParams prm;
  prm.Hq = d.Hq; prm.Hkv = d.Hkv; prm.T_max = d.T_max; prm.NB = d.NB; prm.blk = d.blk;
  prm.scale = d.scale; prm.invT = d.invT; prm.tau = d.tau; prm.lengths = d.lengths;
  prm.union_idx = d.union_idx; prm.row_off = d.row_off; prm.cta_row = d.cta_row;
  prm.plan = d.plan; prm.part_o = d.part_o; prm.part_ml = d.part_ml; prm.status = d.status;
  prm.R = dims->B * dims->Hkv;
  prm.counts = counts;
  prm.row_off_g = const_cast<int32_t*>(d.row_off);   // the workspace
  prm.plan_g = const_cast<int32_t*>(d.plan);
  const bool d64 = dims->d == 64;
  switch (dims->Hq / dims->Hkv) {
    case 1: return d64 ? launch_tc_t<1, DENSE, 64>(mk, mv, mq, prm, P, plan_in, s)
                       : launch_tc_t<1, DENSE, 128>(mk, mv, mq, prm, P, plan_in, s);
    case 2: return d64 ? launch_tc_t<2, DENSE, 64>(mk, mv, mq, prm, P, plan_in, s)
                       : launch_tc_t<2, DENSE, 128>(mk, mv, mq, prm, P, plan_in, s);
    case 4: return d64 ? launch_tc_t<4, DENSE, 64>(mk, mv, mq, prm, P, plan_in, s)
                       : launch_tc_t<4, DENSE, 128>(mk, mv, mq, prm, P, plan_in, s);
    case 8: return d64 ? launch_tc_t<8, DENSE, 64>(mk, mv, mq, prm, P, plan_in, s)
                       : launch_tc_t<8, DENSE, 128>(mk, mv, mq, prm, P, plan_in, s);
  }
  return ETA_ERR_UNSUPPORTED;
}

template <bool DENSE>
eta_status_t run_decode(const eta_dims_t* dims, const eta_bf16_t* q, const float* tau,
                        const eta_bf16_t* K, const eta_bf16_t* V, const int32_t* lengths,
                        const int32_t* union_idx, const int32_t* union_cnt, float T, float scale,
                        eta_prune_t prune, const float* vsum, const int32_t* cnt, float* o,
                        float* lse, void* ws, size_t ws_bytes, int32_t* dev_status,
                        void* stream) {
  eta_status_t st = check_dims(dims);
  if (st != ETA_OK) return st;
  if (!q || !K || !V || !lengths || !o || !lse) return ETA_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(q)) return ETA_ERR_INVALID_ARG;
  if (!DENSE) {
    if (!tau || !union_idx || !union_cnt) return ETA_ERR_INVALID_ARG;
    if (prune != ETA_PRUNE_SKIP && prune != ETA_PRUNE_FLOOR) return ETA_ERR_INVALID_ARG;
    if (prune == ETA_PRUNE_FLOOR && (!vsum || !cnt)) return ETA_ERR_INVALID_ARG;
    if (!(T >= 0.f) || isinf(T)) return ETA_ERR_INVALID_ARG;
  }
  const int P = decode_grid();
  const WsLayout L = ws_layout(dims, P);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return ETA_ERR_WORKSPACE;
  if (scale == 0.f) scale = 1.f / sqrtf((float)dims->d);
  char* w = static_cast<char*>(ws);
  int32_t* plan = reinterpret_cast<int32_t*>(w + L.plan);
  int32_t* row_off = reinterpret_cast<int32_t*>(w + L.row_off);
  int32_t* cta_row = reinterpret_cast<int32_t*>(w + L.cta_row);
  float* part_ml = reinterpret_cast<float*>(w + L.part_ml);
  float* part_o = reinterpret_cast<float*>(w + L.part_o);
  const int R = dims->B * dims->Hkv, NB = num_blocks(dims);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // the tensor-core sparse decode lays out its shares itself (one launch fewer)
  const bool plan_in = !DENSE && plan_in_kernel(dims);
  if (!plan_in) {
    st = launch_k(plan_kernel<DENSE>, dim3(1), dim3(kPlanThreads), 0, s, R, dims->Hkv, NB,
                  dims->blk, dims->T_max, union_cnt, lengths, P, row_off, cta_row, plan,
                  dev_status);
    if (st != ETA_OK) return st;
  }

  DecodeParams prm;
  prm.Hq = dims->Hq; prm.Hkv = dims->Hkv; prm.T_max = dims->T_max; prm.NB = NB;
  prm.blk = dims->blk;
  prm.scale = scale;
  prm.invT = (DENSE || T == 0.f) ? -1.f : 1.f / T;
  prm.q = q; prm.tau = tau; prm.K = K; prm.V = V; prm.lengths = lengths;
  prm.union_idx = union_idx; prm.row_off = row_off; prm.cta_row = cta_row; prm.plan = plan;
  prm.part_o = part_o; prm.part_ml = part_ml; prm.status = dev_status;
  prm.R = R;
  st = use_tc(dims) ? launch_tc<DENSE>(dims, prm, q, K, V, P, plan_in, union_cnt, s)
                    : launch_decode<DENSE>(dims, prm, P, s);
  if (st != ETA_OK) return st;

  CombineParams cp;
  cp.Hq = dims->Hq; cp.Hkv = dims->Hkv; cp.NB = NB; cp.blk = dims->blk; cp.T_max = dims->T_max;
  cp.P = P; cp.floor_mode = (!DENSE && prune == ETA_PRUNE_FLOOR) ? 1 : 0;
  cp.row_off = row_off; cp.plan = plan; cp.union_idx = union_idx; cp.lengths = lengths;
  cp.cnt = cnt; cp.vsum = vsum; cp.part_o = part_o; cp.part_ml = part_ml; cp.o = o; cp.lse = lse;
  cp.status = dev_status;
  return launch_combine(dims, cp, s);
}

}  // namespace eta

using namespace eta;

extern "C" eta_status_t eta_set_decode_engine(eta_engine_t engine) {
  if (engine != ETA_ENGINE_AUTO && engine != ETA_ENGINE_TCGEN05 && engine != ETA_ENGINE_FMA)
    return ETA_ERR_INVALID_ARG;
  g_engine.store((int)engine);
  return ETA_OK;
}

extern "C" eta_engine_t eta_get_decode_engine(void) {
  return static_cast<eta_engine_t>(g_engine.load());
}

extern "C" int32_t eta_decode_launches(const eta_dims_t* dims) {
  if (check_dims(dims) != ETA_OK) return -1;
  return plan_in_kernel(dims) ? 2 : 3;
}

extern "C" size_t eta_decode_workspace_size(const eta_dims_t* dims) {
  if (check_dims(dims) != ETA_OK) return 0;
  return ws_layout(dims, decode_grid()).total;
}

extern "C" eta_status_t eta_decode(const eta_dims_t* dims, const eta_bf16_t* q, const float* tau,
                                   const eta_bf16_t* K, const eta_bf16_t* V,
                                   const int32_t* lengths, const int32_t* union_idx,
                                   const int32_t* union_cnt, float T, float scale,
                                   eta_prune_t prune, const float* vsum, const int32_t* cnt,
                                   float* o, float* lse, void* ws, size_t ws_bytes,
                                   int32_t* dev_status, void* stream) {
  return run_decode<false>(dims, q, tau, K, V, lengths, union_idx, union_cnt, T, scale, prune,
                           vsum, cnt, o, lse, ws, ws_bytes, dev_status, stream);
}

extern "C" eta_status_t eta_dense_decode(const eta_dims_t* dims, const eta_bf16_t* q,
                                         const eta_bf16_t* K, const eta_bf16_t* V,
                                         const int32_t* lengths, float scale, float* o,
                                         float* lse, void* ws, size_t ws_bytes,
                                         int32_t* dev_status, void* stream) {
  return run_decode<true>(dims, q, nullptr, K, V, lengths, nullptr, nullptr, 0.f, scale,
                          ETA_PRUNE_SKIP, nullptr, nullptr, o, lse, ws, ws_bytes, dev_status,
                          stream);
}

// ---------------------------------------------------------------- decode without a workspace
//
// Some callers cannot hand the library any device memory for scratch: a serving
// loop whose device memory is entirely owned by its own pool once it has started,
// or code that must not call cudaMalloc on the decode path because cudaMalloc can
// synchronize the device and stall every other stream.  eta_decode_static serves
// them: it runs exactly the eta_decode pipeline, but its scratch (the plan, the
// prefix sums and the per-CTA partial results) lives in the fixed array below,
// which every GPU that loads this library holds until the process exits.
namespace eta {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;   // 4 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch, looked up with cudaGetSymbolAddress (the
// array's name is only a host-side stand-in in host code) on the first call made in
// a device's context, with that device current, and cached per device together with
// the id of the context it belongs to.  A call in a new context (after a device
// reset) looks the address up again: the module, and the array with it, may then sit
// elsewhere.
constexpr int kMaxDevices = 64;
struct StaticScratchSlot {
  unsigned long long ctx = 0;
  void* ptr = nullptr;
};
static StaticScratchSlot g_static_scratch_slot[kMaxDevices];
static std::mutex g_static_scratch_mu;

inline eta_status_t static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ETA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  StaticScratchSlot& slot = g_static_scratch_slot[dev];
  const unsigned long long ctx = current_context_id();
  if (ctx == 0 || slot.ctx != ctx || !slot.ptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) return ETA_ERR_CUDA;
    slot.ptr = ptr;
    slot.ctx = ctx != 0 ? ctx : current_context_id();
  }
  *out = slot.ptr;
  return ETA_OK;
}

}  // namespace eta

extern "C" size_t eta_decode_static_max_workspace(void) { return eta::kStaticScratchBytes; }

extern "C" eta_status_t eta_decode_static(const eta_dims_t* dims, const eta_bf16_t* q,
                                          const float* tau, const eta_bf16_t* K,
                                          const eta_bf16_t* V, const int32_t* lengths,
                                          const int32_t* union_idx, const int32_t* union_cnt,
                                          float T, float scale, eta_prune_t prune,
                                          const float* vsum, const int32_t* cnt, float* o,
                                          float* lse, int32_t* dev_status, void* stream) {
  eta_status_t st = check_dims(dims);
  if (st != ETA_OK) return st;
  const size_t need = ws_layout(dims, decode_grid()).total;
  if (need > kStaticScratchBytes) return ETA_ERR_WORKSPACE;
  void* ws = nullptr;
  if ((st = static_scratch(&ws)) != ETA_OK) return st;
  // Nothing in the scratch has to start at zero: every call's plan kernel rewrites
  // all the bookkeeping the later kernels of the same call read.
  return run_decode<false>(dims, q, tau, K, V, lengths, union_idx, union_cnt, T, scale, prune,
                           vsum, cnt, o, lse, ws, kStaticScratchBytes, dev_status, stream);
}
