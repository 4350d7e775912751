// Block-screening arithmetic shared by screen_vec_kernel and the fused decode step:
// the O(1) score bound of every KV block against the G query heads of its group,
// the per-head admit words and their union (arXiv 2609.20888 abstract: blocks
// screened "in O(1) time using cached geometric-probabilistic bounds", tokens
// "co-admitted by coarse GPU block selection"; evolve.pub review FAQ: blocks whose
// best possible score falls below the threshold are skipped entirely).
//
// One warp screens a group of 128 consecutive blocks: lane l owns the VW = 4 blocks
// 4l .. 4l+3 of the group, so each of its d centroid loads (dimension-major
// storage) is one 16-byte (fp32) or 8-byte (bf16) load; LB loads per lane are in
// flight at a time.  The lanes' 4-bit admit chunks are assembled into 32-bit words
// with an OR butterfly over the 8 lanes of each word.  Needs NB % 4 == 0 and
// 16-byte aligned metadata.
#pragma once

#include <type_traits>

#include "eta_common.cuh"

namespace eta {

constexpr int kScreenVW = 4;                              // blocks per lane
constexpr int kScreenGroupBlocks = 32 * kScreenVW;        // blocks per warp group
constexpr int kScreenLoadBatch = 16;

// L2-coherent loads (CG = true) for metadata another CTA of the same grid may
// have written; read-only-cache loads otherwise.
template <bool CG, typename T>
ETA_DEV T ld_meta(const T* p) {
  if constexpr (CG) return __ldcg(p);
  else return __ldg(p);
}

// ||q_h|| from the staged query [D][G] (fp32); the same value in every lane.
template <int D, int G>
ETA_DEV float query_norm(const float* qs, int h) {
  const int lane = threadIdx.x & 31;
  float s = 0.f;
  for (int k = lane; k < D; k += 32) s = fmaf(qs[k * G + h], qs[k * G + h], s);
  return sqrtf(warp_sum(s));
}

// Where one lane's metadata comes from.  GlobalMeta: straight from the metadata
// arrays (read-only-cache loads, or L2-only loads when CG: another CTA of the same
// grid may have written them).  SmemMeta: a shared-memory copy of one group
// (dimension-major centroid tile of 128 blocks x D rows, then the rmax, var and cnt
// slices), as the fused step stages it with TMA; per-dimension variances stay in
// global memory.
template <int CF, bool VD, bool CG>
struct GlobalMeta {
  using LdT = typename std::conditional<CF == 1, uint2, uint4>::type;
  const LdT* cp;          // this lane's 4 centroids of dimension 0
  size_t rowv;            // LdT units per dimension
  const float4* vdp;      // this lane's 4 per-dimension variances of dimension 0
  size_t rowvd;           // float4 units per dimension
  const float* rmax;      // this lane's first block
  const float* var;
  const int32_t* cnt;
  ETA_DEV LdT cent(int k) const { return ld_meta<CG>(cp + (size_t)k * rowv); }
  ETA_DEV float4 vd(int k) const { return ld_meta<CG>(vdp + (size_t)k * rowvd); }
  ETA_DEV float4 rad() const { return ld_meta<CG>(reinterpret_cast<const float4*>(rmax)); }
  ETA_DEV float4 variance() const { return ld_meta<CG>(reinterpret_cast<const float4*>(var)); }
  ETA_DEV int4 count() const { return ld_meta<CG>(reinterpret_cast<const int4*>(cnt)); }
};

template <int CF, bool VD>
struct SmemMeta {
  using LdT = typename std::conditional<CF == 1, uint2, uint4>::type;
  const unsigned char* tile;   // [D][128] centroids (bf16 or fp32)
  const float4* vdp;           // VD: this lane's per-dimension variances of dimension 0,
  size_t rowvd;                //     read from L2 (float4 units per dimension)
  const float* rmax;           // [128]
  const float* var;
  const int32_t* cnt;
  int lane;
  ETA_DEV LdT cent(int k) const {
    return reinterpret_cast<const LdT*>(tile + (size_t)k * 128 * (CF == 1 ? 2 : 4))[lane];
  }
  ETA_DEV float4 vd(int k) const { return __ldcg(vdp + (size_t)k * rowvd); }
  ETA_DEV float4 rad() const { return reinterpret_cast<const float4*>(rmax)[lane]; }
  ETA_DEV float4 variance() const { return reinterpret_cast<const float4*>(var)[lane]; }
  ETA_DEV int4 count() const { return reinterpret_cast<const int4*>(cnt)[lane]; }
};

// Screens group `grp` of (row, KV head) r from metadata source `src`.  qs: the
// group's G query heads staged as [D][G] fp32; qn, ts: their norms and thresholds.
// A block is admitted for head h iff it holds keys (cnt > 0), lies below `nvalid`
// and its bound >= ts[h].  Writes head_mask[(qhead0 + h) * NW + w],
// union_words[r * NW + w] and, if given, bounds_out[(qhead0 + h) * NB + j].
// Returns (in every lane) how many blocks of the group the union admits.
template <int D, int G, int CF, bool VD, int LB, class Src>
ETA_DEV int screen_group_from(const Src& src, int NB, int NW, int grp, int r, size_t qhead0,
                               const float* qs, const float* qn, const float* ts, int bound,
                               float z, float scale, int nvalid,
                               uint32_t* __restrict__ head_mask,
                               uint32_t* __restrict__ union_words,
                               float* __restrict__ bounds_out) {
  constexpr int VW = kScreenVW;
  constexpr int LPW = 32 / VW;                  // lanes per 32-bit word
  using LdT = typename Src::LdT;
  const int lane = threadIdx.x & 31;
  const int j0 = grp * kScreenGroupBlocks + lane * VW;
  const bool vj = j0 < NB;                      // NB % VW == 0: all VW valid or none
  // accumulators of blocks (2p, 2p+1) side by side: one packed fp32x2 FMA per pair,
  // each component an ordinary round-to-nearest fp32 FMA
  static_assert(VW % 2 == 0, "VW");
  float2 acc[VW / 2][G], acc2[VW / 2][VD ? G : 1];
#pragma unroll
  for (int k = 0; k < VW / 2; ++k) {
#pragma unroll
    for (int h = 0; h < G; ++h) acc[k][h] = make_float2(0.f, 0.f);
#pragma unroll
    for (int h = 0; h < (VD ? G : 1); ++h) acc2[k][h] = make_float2(0.f, 0.f);
  }
#pragma unroll 1
  for (int d0 = 0; d0 < D; d0 += LB) {
    LdT cb[LB];
#pragma unroll
    for (int u = 0; u < LB; ++u) cb[u] = vj ? src.cent(d0 + u) : LdT{};
#pragma unroll
    for (int u = 0; u < LB; ++u) {
      float cv[VW];
      if constexpr (CF == 1) {
        cv[0] = bf16_lo(cb[u].x); cv[1] = bf16_hi(cb[u].x); cv[2] = bf16_lo(cb[u].y);
        cv[3] = bf16_hi(cb[u].y);
      } else {
        cv[0] = __uint_as_float(cb[u].x); cv[1] = __uint_as_float(cb[u].y);
        cv[2] = __uint_as_float(cb[u].z); cv[3] = __uint_as_float(cb[u].w);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float qv = qs[(d0 + u) * G + h];
#pragma unroll
        for (int k = 0; k < VW / 2; ++k)
          acc[k][h] = __ffma2_rn(make_float2(qv, qv), make_float2(cv[2 * k], cv[2 * k + 1]),
                                 acc[k][h]);
      }
      if constexpr (VD) {
        const float4 vv = vj ? src.vd(d0 + u) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float vk[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float q2 = qs[(d0 + u) * G + h] * qs[(d0 + u) * G + h];
#pragma unroll
          for (int k = 0; k < VW / 2; ++k)
            acc2[k][h] = __ffma2_rn(make_float2(q2, q2), make_float2(vk[2 * k], vk[2 * k + 1]),
                                    acc2[k][h]);
        }
      }
    }
  }
  float rad[VW];
  int n[VW];
#pragma unroll
  for (int k = 0; k < VW; ++k) { rad[k] = 0.f; n[k] = 0; }
  if (vj) {
    const float4 rr = src.rad();
    const int4 cc = src.count();
    rad[0] = rr.x; rad[1] = rr.y; rad[2] = rr.z; rad[3] = rr.w;
    n[0] = cc.x; n[1] = cc.y; n[2] = cc.z; n[3] = cc.w;
    if (bound == ETA_BOUND_PROB) {
      const float4 vv = src.variance();
      rad[0] = fminf(rad[0], z * sqrtf(vv.x / (float)D));
      rad[1] = fminf(rad[1], z * sqrtf(vv.y / (float)D));
      rad[2] = fminf(rad[2], z * sqrtf(vv.z / (float)D));
      rad[3] = fminf(rad[3], z * sqrtf(vv.w / (float)D));
    }
  }
  uint32_t uni = 0;
  const int wsel = grp * VW + lane / LPW;        // word index of this lane's chunk
#pragma unroll
  for (int h = 0; h < G; ++h) {
    uint32_t bits = 0;
    float ubv[VW];
#pragma unroll
    for (int k = 0; k < VW; ++k) {
      const float dot = (k & 1) ? acc[k >> 1][h].y : acc[k >> 1][h].x;
      if constexpr (VD) {
        const float qv2 = (k & 1) ? acc2[k >> 1][h].y : acc2[k >> 1][h].x;
        ubv[k] = scale * (dot + fminf(qn[h] * rad[k], z * sqrtf(qv2)));
      } else {
        ubv[k] = scale * fmaf(qn[h], rad[k], dot);
      }
      if (vj && n[k] > 0 && j0 + k < nvalid && ubv[k] >= ts[h]) bits |= 1u << k;
    }
    if (bounds_out && vj)
      *reinterpret_cast<float4*>(bounds_out + (qhead0 + h) * NB + j0) =
          make_float4(ubv[0], ubv[1], ubv[2], ubv[3]);
    uint32_t word = bits << (VW * (lane % LPW));
#pragma unroll
    for (int o = 1; o < LPW; o <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, o);
    if (lane % LPW == 0 && wsel < NW) head_mask[(qhead0 + h) * NW + wsel] = word;
    uni |= word;
  }
  if (lane % LPW == 0 && wsel < NW) union_words[(size_t)r * NW + wsel] = uni;
  int adm = (lane % LPW == 0 && wsel < NW) ? __popc(uni) : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) adm += __shfl_xor_sync(0xffffffffu, adm, o);
  return adm;
}

// Screens group `grp` of row r straight from the metadata arrays.
template <int D, int G, int CF, bool VD, int LB, bool CG>
ETA_DEV void screen_group(int NB, int NW, int grp, int r, size_t qhead0, const float* qs,
                          const float* qn, const float* ts, const void* __restrict__ cent,
                          const float* __restrict__ rmax, const float* __restrict__ var,
                          const float* __restrict__ vardim, const int32_t* __restrict__ cnt,
                          int bound, float z, float scale, int nvalid,
                          uint32_t* __restrict__ head_mask, uint32_t* __restrict__ union_words,
                          float* __restrict__ bounds_out) {
  using Src = GlobalMeta<CF, VD, CG>;
  const int lane = threadIdx.x & 31;
  const int j0 = grp * kScreenGroupBlocks + lane * kScreenVW;
  const size_t off = (size_t)r * D * NB + (j0 < NB ? j0 : 0);
  const size_t rj = (size_t)r * NB + (j0 < NB ? j0 : 0);
  Src src;
  src.cp = reinterpret_cast<const typename Src::LdT*>(
      reinterpret_cast<const unsigned char*>(cent) + off * (CF == 1 ? 2 : 4));
  src.rowv = (size_t)NB / 4;
  src.vdp = VD ? reinterpret_cast<const float4*>(vardim + off) : nullptr;
  src.rowvd = (size_t)NB / 4;
  src.rmax = rmax + rj;
  src.var = var + rj;
  src.cnt = cnt + rj;
  screen_group_from<D, G, CF, VD, LB>(src, NB, NW, grp, r, qhead0, qs, qn, ts, bound, z, scale,
                                      nvalid, head_mask, union_words, bounds_out);
}

}  // namespace eta
