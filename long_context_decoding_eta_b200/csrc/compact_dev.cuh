// Compaction of one (batch row, KV head) pair's union admit words into the
// ascending list of admitted block indices, its count, and the per-head admitted
// counts (the "coarse GPU block selection" of arXiv 2609.20888, abstract: the blocks
// any head of the group admits are the ones the decode streams).  Shared by
// compact_kernel (a CTA per pair after the screening launch) and the one-launch
// small-batch screen, which compacts the words its own CTA has just written: every
// read goes through L2 (__ldcg), never the non-coherent read-only path.
#pragma once

#include "eta_common.cuh"

namespace eta {

template <int NT>
struct CompactScratch {
  uint32_t wbuf[NT];
  int woff[NT];
  int wsum[NT / 32];
};

// Threads 0 .. NT-1 of the CTA call this; `sync` synchronises exactly them.
// union_words and head_mask: [R][NW] and [B * Hq][NW]; writes union_idx[r * NB ...],
// union_cnt[r] and, if given, head_cnt of the pair's G query heads.  status: the
// checked build's range reports (may be NULL).
template <int NT, typename Sync>
ETA_DEV void compact_row(int r, int Hq, int Hkv, int G, int NB, int NW,
                         const uint32_t* union_words, const uint32_t* head_mask,
                         int32_t* union_idx, int32_t* union_cnt, int32_t* head_cnt,
                         CompactScratch<NT>& cs, int32_t* status, Sync sync) {
  static_assert(NT % 32 == 0 && NT <= 1024, "NT");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int carry = 0;
  for (int base = 0; base < NW; base += NT) {
    const int w = base + tid;
    const uint32_t word = w < NW ? __ldcg(union_words + (size_t)r * NW + w) : 0u;
    const int c = __popc(word);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) cs.wsum[warp] = incl;
    sync();
    int wpre = 0, total = 0;
#pragma unroll
    for (int i = 0; i < NT / 32; ++i) {
      const int v = cs.wsum[i];
      if (i < warp) wpre += v;
      total += v;
    }
    cs.wbuf[tid] = word;
    cs.woff[tid] = carry + wpre + incl - c;
    sync();
    for (int i = warp; i < NT && base + i < NW; i += NT / 32) {
      const uint32_t wd = cs.wbuf[i];
      const int pos = cs.woff[i] + __popc(wd & ((1u << lane) - 1u));
      if (((wd >> lane) & 1u) && ETA_IN_BOUNDS(pos, NB, status))
        union_idx[(size_t)r * NB + pos] = (base + i) * 32 + lane;
    }
    carry += total;
    sync();
  }
  if (tid == 0) union_cnt[r] = carry;
  if (head_cnt) {
    const int b = r / Hkv, g = r % Hkv;
    for (int h = warp; h < G; h += NT / 32) {
      const size_t hq = (size_t)b * Hq + (size_t)g * G + h;
      int s = 0;
      for (int w = lane; w < NW; w += 32) s += __popc(__ldcg(head_mask + hq * NW + w));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) head_cnt[hq] = s;
    }
  }
}

}  // namespace eta
