// Log-sum-exp merge of split-KV partial results, shared by combine_kernel and the
// fused decode step.  A (row, KV head) pair whose admitted blocks were spread over
// ns consecutive CTA shares has ns partial slots (m, l, o) per query head; the
// merged result is o = sum_s e^(m_s - M) o_s / L, L = sum_s e^(m_s - M) l_s,
// lse = M + log L (M = max_s m_s), in slot order.
#pragma once

#include "eta_common.cuh"

namespace eta {

// Minimum admitted blocks per CTA share of the split-KV decode (the share length is
// max(ceil(total / CTAs), kMinChunk)); it fixes which slots a pair's partials use.
constexpr int kMinChunk = 2;

struct CombineParams {
  int Hq, Hkv, NB, blk, T_max, P, floor_mode;
  const int32_t* row_off;
  const int32_t* plan;
  const int32_t* union_idx;
  const int32_t* lengths;
  const int32_t* cnt;
  const float* vsum;
  const float* part_o;
  const float* part_ml;
  float* o;
  float* lse;
  int32_t* status;   // the checked build's range reports (may be NULL)
};

constexpr int kCombineMaxPairs = 256;   // (head, slot) pairs staged in shared memory
constexpr int kMergeBatch = 16;         // partial-o loads in flight per thread

template <int G>
struct CombineScratch {
  float m[kCombineMaxPairs], w[kCombineMaxPairs];
  float M[G], L[G];
};

template <bool CG>
ETA_DEV float ld_part(const float* p) {
  if constexpr (CG) return __ldcg(p);
  else return *p;
}

// Called by D threads (thread = dim dd) that `sync` synchronizes.  Slot s of pair r
// and head h lives at ((p0 + s) + r) * G + h, of n_slots slots.  On return O[h] holds
// this dim's un-normalized merged output, sc.M[h] / sc.L[h] the merged max and sum
// (-inf / 0 when ns = 0).  CG: the partials were written by other CTAs of the
// same grid (L2-coherent loads).
template <int D, int G, bool CG, typename Sync>
ETA_DEV void combine_merge(const float* part_ml, const float* part_o, int r, int p0, int ns,
                           int dd, CombineScratch<G>& sc, float (&O)[G], Sync sync,
                           long long n_slots, int32_t* status) {
#pragma unroll
  for (int h = 0; h < G; ++h) O[h] = 0.f;
  // (checked build) the pair's slots lie inside the workspace; uniform over the callers
  if (!ETA_RANGE_IN_BOUNDS((long long)p0 + r, (long long)p0 + r + ns, n_slots, status)) ns = 0;
  if (ns > 0) {
    const int np = G * ns;                 // pair k = slot * G + h
    if (np <= kCombineMaxPairs) {
      // the first batch of partial outputs is loaded with the (m, l) pairs: it does not
      // depend on them, so their latencies overlap
      float v0[kMergeBatch];
#pragma unroll
      for (int u = 0; u < kMergeBatch; ++u) {
        const size_t sl = ((size_t)(p0 + u / G) + r) * G + (u % G);
        v0[u] = u < np ? ld_part<CG>(part_o + sl * D + dd) : 0.f;
      }
      for (int k = dd; k < np; k += D) {
        const size_t sl = ((size_t)(p0 + k / G) + r) * G + (k % G);
        sc.m[k] = ld_part<CG>(part_ml + sl * 2);
        sc.w[k] = ld_part<CG>(part_ml + sl * 2 + 1);
      }
      sync();
      if (dd < G) {
        float M = -INFINITY;
        for (int k = dd; k < np; k += G) M = fmaxf(M, sc.m[k]);
        float L = 0.f;
        for (int k = dd; k < np; k += G) {
          const float w = (M == -INFINITY) ? 0.f : expf(sc.m[k] - M);
          L = fmaf(sc.w[k], w, L);
          sc.m[k] = w;                       // now the slot weight
        }
        sc.M[dd] = M;
        sc.L[dd] = L;
      }
      sync();
      // loads in batches of kMergeBatch (independent, in flight together), then the
      // accumulation in slot order
      for (int k0 = 0; k0 < np; k0 += kMergeBatch) {
        float v[kMergeBatch];
#pragma unroll
        for (int u = 0; u < kMergeBatch; ++u) {
          const int k = k0 + u;
          const size_t sl = ((size_t)(p0 + k / G) + r) * G + (k % G);
          v[u] = k0 == 0 ? v0[u] : k < np ? ld_part<CG>(part_o + sl * D + dd) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kMergeBatch; ++u) {
          const int k = k0 + u;
          if (k < np) {
#pragma unroll
            for (int h = 0; h < G; ++h)
              if (k % G == h) O[h] = fmaf(v[u], sc.m[k], O[h]);
          }
        }
      }
    } else {
      // very long rows spread over many CTAs: plain two-pass merge per head
      if (dd < G) { sc.M[dd] = -INFINITY; sc.L[dd] = 0.f; }
      sync();
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float M = -INFINITY;
        for (int k = 0; k < ns; ++k)
          M = fmaxf(M, ld_part<CG>(part_ml + (((size_t)(p0 + k) + r) * G + h) * 2));
        float L = 0.f;
        for (int k = 0; k < ns; ++k) {
          const size_t sl = ((size_t)(p0 + k) + r) * G + h;
          const float w = (M == -INFINITY) ? 0.f : expf(ld_part<CG>(part_ml + sl * 2) - M);
          L = fmaf(ld_part<CG>(part_ml + sl * 2 + 1), w, L);
          O[h] = fmaf(ld_part<CG>(part_o + sl * D + dd), w, O[h]);
        }
        if (dd == 0) { sc.M[h] = M; sc.L[h] = L; }
      }
      sync();
    }
  } else {
    if (dd < G) { sc.M[dd] = -INFINITY; sc.L[dd] = 0.f; }
    sync();
  }
}

// o[oh] = O / L and lse[oh] = M + log L; an empty softmax (L = 0) gives o = 0,
// lse = -inf.
template <int D>
ETA_DEV void combine_store(float* o, float* lse, size_t oh, int dd, float M, float L, float Oh) {
  if (L > 0.f) {
    o[oh * D + dd] = Oh / L;
    if (dd == 0) lse[oh] = M + logf(L);
  } else {
    o[oh * D + dd] = 0.f;
    if (dd == 0) lse[oh] = -INFINITY;
  }
}

}  // namespace eta
