/*
 * eta.h -- C ABI of the Elastic Threshold Attention (ETA) block-sparse decode step
 * for NVIDIA B200 (sm_100a).
 *
 * The method (arXiv 2609.20888, "Elastic Threshold Attention: Learned Contextual
 * Sparsity for Long-Context Decoding"; abstract, and the evolve.pub review's FAQ,
 * Summary and Methodology Assessment, Eq. 1-3): for each decode query, a threshold
 * tau is predicted per query head (or frozen to a calibrated per-head constant);
 * every KV block is screened in O(1) from cached per-block metadata against a
 * score bound; blocks whose bound falls below tau are never loaded; the query
 * heads of one KV group attend over the union of their admitted blocks with
 * multiplicatively gated logits s' = s * sigmoid((s - tau) / T) (T -> 0: hard gate,
 * a sub-threshold key keeps weight e^0 = 1).
 *
 * Conventions (all entry points):
 *  - Every tensor argument is a caller-owned DEVICE pointer unless said otherwise.
 *    The library never allocates, frees or retains memory.  Scratch comes from a
 *    caller-provided workspace whose size the *_workspace_size query returns (the
 *    one exception, eta_decode_static, uses a fixed array reserved at load time).
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the
 *    legacy default stream) and never synchronize the host.
 *  - Host-side argument errors are returned immediately as ETA_ERR_* and nothing is
 *    launched.  A launch failure returns ETA_ERR_CUDA.
 *  - Errors found on the device (bounded waits that ran out, non-finite queries,
 *    malformed block lists) are OR-ed into the caller's int32 word `dev_status`
 *    (device memory, may be NULL to ignore them) as ETA_DEVSTAT_* bits; read it
 *    after synchronizing the stream.  The caller zeroes it.
 *  - bf16 tensors are passed as eta_bf16_t (the raw 16-bit pattern).
 *  - Shapes: d in {64, 128}; blk in {64, 128}; G = Hq / Hkv in {1, 2, 4, 8};
 *    T_max a multiple of blk; NB = T_max / blk blocks per (row, KV head);
 *    NW = ceil(NB / 32) mask words.  Other shapes return ETA_ERR_UNSUPPORTED.
 *  - Logit units: s = scale * (q . k), scale = 1/sqrt(d) when the scale argument is
 *    0.  tau and every block bound are in these units.
 */
#ifndef ETA_H_
#define ETA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t eta_bf16_t;

typedef enum {
  ETA_OK = 0,
  ETA_ERR_INVALID_ARG = 1,     /* null pointer, negative size, misaligned pointer */
  ETA_ERR_UNSUPPORTED = 2,     /* shape outside the supported set above */
  ETA_ERR_WORKSPACE = 3,       /* workspace NULL or smaller than the query says */
  ETA_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed */
  ETA_ERR_DEVICE_TIMEOUT = 5,  /* returned by eta_status_from_device() */
  ETA_ERR_NONFINITE = 6,       /* returned by eta_status_from_device() */
  ETA_ERR_DEVICE_BOUNDS = 7    /* returned by eta_status_from_device(): checked build */
} eta_status_t;

/* Bits OR-ed into *dev_status by the kernels. */
#define ETA_DEVSTAT_TIMEOUT 0x1      /* a bounded pipeline wait gave up; outputs invalid */
#define ETA_DEVSTAT_NONFINITE_Q 0x2  /* a query element was NaN or Inf */
#define ETA_DEVSTAT_BAD_BLOCK 0x4    /* a block index out of range or an empty block */
#define ETA_DEVSTAT_BAD_LENGTH 0x8   /* lengths[b] < 0 or > T_max (clamped) */
/* Checked build only (libeta_checked.so, compiled with -DETA_CHECKED): an index that
   a kernel computed for a global load or store fell outside its buffer; that access
   was skipped, the outputs are invalid, and the first such event of each source file
   is printed (device printf) with its file and line.  A library defect, never an
   input error: the host-side checks refuse every input that could cause one. */
#define ETA_DEVSTAT_BOUNDS 0x10

typedef struct {
  int32_t B;      /* batch rows (decode queries) */
  int32_t Hq;     /* query heads */
  int32_t Hkv;    /* KV heads; query head h reads KV head h / (Hq / Hkv) */
  int32_t d;      /* head dimension */
  int32_t blk;    /* KV block size in tokens */
  int32_t T_max;  /* token capacity (stride) of the cache per (row, KV head) */
} eta_dims_t;

typedef enum { ETA_BOUND_EXACT = 0, ETA_BOUND_PROB = 1, ETA_BOUND_PROB_DIM = 2 } eta_bound_t;
/* Compute engine of the decode and of the screen (eta_set_decode_engine,
   eta_set_screen_engine). */
typedef enum { ETA_ENGINE_AUTO = 0, ETA_ENGINE_TCGEN05 = 1, ETA_ENGINE_FMA = 2 } eta_engine_t;
/* Storage of the block centroids.  ETA_CENT_BF16 halves the bytes the screen reads;
   the centroid is then rounded to bf16 (nearest even) before rmax and var are
   measured against it, so the geometric bound stays exact for what is stored. */
typedef enum { ETA_CENT_F32 = 0, ETA_CENT_BF16 = 1 } eta_cent_format_t;
typedef enum { ETA_PRUNE_SKIP = 0, ETA_PRUNE_FLOOR = 1 } eta_prune_t;

/* blk_begin value selecting the tail block (the one holding token lengths[b]-1)
   of every row: the per-token append update. */
#define ETA_TAIL_BLOCK (-1)

/*
 * eta_build_block_meta -- per-block key metadata (review Summary: "cached
 * centroid/variance/max-norm metadata"; abstract: "cached geometric-probabilistic
 * bounds").  For block j of (row b, KV head g) with n_j = clamp(lengths[b] - j*blk,
 * 0, blk) valid keys k_t:
 *   cent_j = (1/n_j) sum_t k_t   (fp32, or rounded to bf16 with ETA_CENT_BF16)
 *   rmax_j >= max_t ||k_t - cent_j||, measured against the stored cent_j and
 *            rounded up so that the Cauchy-Schwarz bound stays sound in fp32
 *   var_j  = (1/n_j) sum_t ||k_t - cent_j||^2
 *   cnt_j  = n_j;  vsum_j = sum_t v_t (only when vsum != NULL)
 *   vardim_j[i] = (1/n_j) sum_t (k_t[i] - cent_j[i])^2 (only when vardim != NULL)
 * Empty blocks get zeros.
 *
 * K, V     bf16 [B, Hkv, T_max, d].  V may be NULL when vsum is NULL.
 * lengths  int32 [B], valid tokens per row (keys t < lengths[b]).
 * blk_begin, blk_end: recompute blocks [blk_begin, blk_end) of every row
 *          (blk_end = -1: up to NB); blk_begin = ETA_TAIL_BLOCK: only the tail
 *          block of each row (rows with lengths[b] = 0 are left untouched).
 * cent_format, cent: fp32 or bf16 [B, Hkv, d, NB] (dimension-major per row, for
 *          coalesced screening)
 * rmax,var fp32 [B, Hkv, NB];  cnt int32 [B, Hkv, NB]
 * vsum     fp32 [B, Hkv, NB, d] or NULL (needed only by ETA_PRUNE_FLOOR)
 * vardim   fp32 [B, Hkv, d, NB] or NULL (dimension-major; needed only by
 *          ETA_BOUND_PROB_DIM)
 */
eta_status_t eta_build_block_meta(const eta_dims_t* dims, const eta_bf16_t* K,
                                  const eta_bf16_t* V, const int32_t* lengths,
                                  int32_t blk_begin, int32_t blk_end,
                                  eta_cent_format_t cent_format, void* cent, float* rmax,
                                  float* var, int32_t* cnt, float* vsum, float* vardim,
                                  void* stream);

/*
 * eta_predict_tau -- per-query, per-head threshold (review Methodology Assessment,
 * Eq. 1: tau = qbar W_tau + b_tau on the concatenated post-RoPE queries; abstract:
 * frozen per-head constants after calibration).
 *   predictor mode (tau_const == NULL):
 *     tau[b, h] = sum_{i < Hq*d} qbar[b, i] * W[i, h] + bias[h],  qbar[b] = concat_h q[b, h]
 *   constant mode (tau_const != NULL): tau[b, h] = tau_const[h]; W and bias ignored.
 * q     bf16 [B, Hq, d];  W fp32 [Hq*d, Hq] row-major;  bias fp32 [Hq] or NULL (= 0)
 * tau_const fp32 [Hq] or NULL;  tau (out) fp32 [B, Hq]
 * dev_status: ETA_DEVSTAT_NONFINITE_Q if q holds NaN/Inf (predictor mode).
 */
eta_status_t eta_predict_tau(const eta_dims_t* dims, const eta_bf16_t* q, const float* W,
                             const float* bias, const float* tau_const, float* tau,
                             int32_t* dev_status, void* stream);

/*
 * eta_screen -- O(1)-per-block screening with hard pruning (review FAQ: blocks whose
 * best possible score falls below the threshold are skipped; abstract: screening
 * "in O(1) time using cached geometric-probabilistic bounds"; co-admission across
 * the query heads of a KV group).
 *   UB[b,h,j] = scale * (q.cent_j + ||q|| * R_j),  q = q[b,h], g = h / G
 *   (cent in the format eta_build_block_meta stored it)
 *     ETA_BOUND_EXACT: R_j = rmax_j                      (Cauchy-Schwarz, sound)
 *     ETA_BOUND_PROB:  R_j = min(rmax_j, z * sqrt(var_j / d))
 *     ETA_BOUND_PROB_DIM: ||q|| * R_j is replaced by
 *                      min(||q|| rmax_j, z * sqrt(sum_i q_i^2 vardim_j[i]))
 *                      (per-dimension variance; needs vardim, never looser than exact)
 *   admit[b,h,j] = cnt_j > 0 && UB[b,h,j] >= tau[b,h]
 *   union[b,g,j] = OR over the G query heads of group g
 * Outputs:
 *   head_mask  uint32 [B, Hq, NW]: bit (j % 32) of word j / 32 = admit[b,h,j]
 *   union_idx  int32  [B, Hkv, NB]: admitted-union block indices, ascending; the
 *              first union_cnt[b,g] entries are valid, the rest untouched
 *   union_cnt  int32  [B, Hkv]
 *   bounds_out fp32   [B, Hq, NB] or NULL (calibration, near-tie logging)
 *   head_cnt   int32  [B, Hq] or NULL: popcount of the head's admit mask
 * ws/ws_bytes: scratch of at least eta_screen_workspace_size(dims) bytes.
 * Two forms compute the q . cent products (both tested against the float64 oracle;
 * their fp32 sums differ in order, so they agree up to rounding, i.e. near-ties):
 *   tensor cores (bf16 centroids, d = 128 or 64, ETA_BOUND_EXACT or _PROB,
 *     NB % 8 == 0, every pointer 16-byte aligned): a 128-block group's products as
 *     one tcgen05.mma (M = 128 blocks, N = 16, K = d) from TMA-staged tiles;
 *   CUDA cores: fp32 FMA chains.
 * eta_set_screen_engine (process-wide) chooses: ETA_ENGINE_TCGEN05 the tensor cores
 * wherever they apply, ETA_ENGINE_FMA the CUDA cores always, ETA_ENGINE_AUTO (the
 * default) the tensor cores where this library measures them faster: d = 128 when
 * the (row, KV head) pairs fit one per SM and rows have at most 32 groups of 128
 * blocks.  The one-launch step follows the same choice.
 * Kernel launches: one (screening and compaction together, one CTA per (row, KV
 * head) pair: the tensor-core form when the pairs fit one per SM and rows have at
 * most 32 groups of 128 blocks; the CUDA-core form for batches of at most two CTAs
 * per SM whose rows fit two rounds of the CTA's group buffers, NB a multiple of 8
 * for bf16 centroids or 4 for fp32) or two (screening, then compaction);
 * eta_screen_launches says which.
 * dev_status (may be NULL): ETA_DEVSTAT_TIMEOUT if a one-launch or tensor-core
 * form's bounded wait for a staged group tile ran out (the outputs are then
 * incomplete).
 */
/*
 * eta_append_and_predict_tau -- eta_build_block_meta(..., ETA_TAIL_BLOCK, ...) and
 * eta_predict_tau in one launch (the two parts of a step that precede the screening
 * and do not depend on each other): one CTA per (batch row, KV head) refreshes the
 * tail block's metadata with half its warps while the other half computes the
 * group's thresholds.  Arguments and layouts as those two calls (vsum, vardim
 * nullable as there; W / bias as eta_predict_tau, or tau_const non-NULL for the
 * frozen constants).  Writes the same bits as the two calls.  dev_status:
 * ETA_DEVSTAT_NONFINITE_Q.
 */
eta_status_t eta_append_and_predict_tau(const eta_dims_t* dims, const eta_bf16_t* K,
                                        const eta_bf16_t* V, const int32_t* lengths,
                                        eta_cent_format_t cent_format, void* cent, float* rmax,
                                        float* var, int32_t* cnt, float* vsum, float* vardim,
                                        const eta_bf16_t* q, const float* W, const float* bias,
                                        const float* tau_const, float* tau,
                                        int32_t* dev_status, void* stream);

size_t eta_screen_workspace_size(const eta_dims_t* dims);
/* Kernel launches eta_screen makes on the current device for these dims and centroid
 * format with the exact or variance bound, under the current screen engine, when
 * every pointer argument is 16-byte aligned (1 or 2; 2 without a device), or -1 for
 * invalid dims.  A packaging query with no counterpart in the pages; host only,
 * launches nothing. */
int32_t eta_screen_launches(const eta_dims_t* dims, eta_cent_format_t cent_format);
/* Screen engine (process-wide; see eta_screen): ETA_ENGINE_TCGEN05 takes the tensor
 * cores wherever they apply, ETA_ENGINE_AUTO where they measured faster,
 * ETA_ENGINE_FMA always the CUDA cores.  ETA_ERR_INVALID_ARG for an unknown value. */
eta_status_t eta_set_screen_engine(eta_engine_t engine);
eta_engine_t eta_get_screen_engine(void);
eta_status_t eta_screen(const eta_dims_t* dims, const eta_bf16_t* q, const float* tau,
                        eta_cent_format_t cent_format, const void* cent, const float* rmax,
                        const float* var, const float* vardim,
                        const int32_t* cnt, eta_bound_t bound, float z, float scale,
                        uint32_t* head_mask, int32_t* union_idx, int32_t* union_cnt,
                        float* bounds_out, int32_t* head_cnt, void* ws, size_t ws_bytes,
                        int32_t* dev_status, void* stream);

/*
 * eta_decode -- gated attention over the admitted-union blocks only (review
 * Methodology Assessment, Eq. 2-3 with beta = 1/T; review FAQ: a sub-threshold
 * logit goes to zero, weight e^0 = 1; abstract: co-admitted tokens are absorbed).
 * Each query head h of group g attends over every valid key t of the blocks
 * union_idx[b,g,0..union_cnt[b,g]) with its own tau[b,h]:
 *   s_t  = scale * q[b,h] . k_t
 *   s'_t = s_t * sigmoid((s_t - tau) / T)      (T > 0)
 *   s'_t = s_t if s_t >= tau else 0            (T == 0, hard gate)
 *   o[b,h] = sum_t e^{s'_t} v_t / sum_t e^{s'_t},   lse[b,h] = log sum_t e^{s'_t}
 * ETA_PRUNE_SKIP: pruned blocks are absent from the softmax; an empty union gives
 *   o = 0, lse = -inf.
 * ETA_PRUNE_FLOOR: every valid key of a pruned block enters with logit 0 (its
 *   hard-gated value), using cnt and vsum from eta_build_block_meta (both required).
 * Split-KV over the admitted list (every CTA streams an equal share of admitted
 * blocks, TMA bulk copies into shared memory), fp32 online softmax, LSE combine.
 * K, V bf16 [B, Hkv, T_max, d], 16-byte aligned.  o fp32 [B, Hq, d], lse fp32 [B, Hq].
 * ws/ws_bytes: scratch of at least eta_decode_workspace_size(dims) bytes (for the
 * current device).  dev_status bits: TIMEOUT, NONFINITE_Q, BAD_BLOCK, BAD_LENGTH.
 */
size_t eta_decode_workspace_size(const eta_dims_t* dims);
/* Kernel launches eta_decode makes for these dims with the current engine: 2 (the
 * tensor-core decode lays out its CTA shares itself, then the combine: 128 to 2048
 * (row, KV head) pairs) or 3 (plan, decode, combine); -1 for invalid dims.  A
 * packaging query with no counterpart in the pages; host only, launches nothing. */
int32_t eta_decode_launches(const eta_dims_t* dims);
eta_status_t eta_decode(const eta_dims_t* dims, const eta_bf16_t* q, const float* tau,
                        const eta_bf16_t* K, const eta_bf16_t* V, const int32_t* lengths,
                        const int32_t* union_idx, const int32_t* union_cnt, float T,
                        float scale, eta_prune_t prune, const float* vsum,
                        const int32_t* cnt, float* o, float* lse, void* ws,
                        size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * eta_decode_static -- eta_decode for callers that cannot allocate device memory.
 * (No counterpart in the paper: this is a packaging choice of this library.)
 * Some callers cannot give the library any scratch memory -- for instance a
 * serving loop whose device memory is entirely taken by its own pool once it has
 * started, or code that must not call cudaMalloc on the decode path because
 * cudaMalloc can synchronize the device and stall other streams.  This entry
 * point computes exactly what eta_decode computes, with the same arguments minus
 * the workspace: its scratch is a fixed 4 MiB array in device memory that the
 * library defines statically, so every GPU that loads the library holds those
 * 4 MiB until the process exits.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *  - Limit: returns ETA_ERR_WORKSPACE when eta_decode_workspace_size(dims) would
 *    exceed eta_decode_static_max_workspace() (4 MiB).  On a 148-SM GPU with
 *    d = 128 that admits B * Hkv up to 1864 (row, KV head) pairs at G = 4 and 859
 *    at G = 8 (the per-CTA and per-pair partial results dominate the scratch).
 *  - Set-up: the first call made in a device's context looks up the array's device
 *    address (cudaGetSymbolAddress, with that device current).  Make that first
 *    call before any stream capture.  A device reset (or any re-creation of the
 *    context) makes the next call look the address up again, so that first call
 *    after a reset should also come before any capture.
 *  - All calls share the one array and it keeps the last call's contents; nothing
 *    in it needs to start at zero.  Calls that overlap on the GPU (other streams,
 *    other host threads) race on it: serialize them.
 */
eta_status_t eta_decode_static(const eta_dims_t* dims, const eta_bf16_t* q, const float* tau,
                               const eta_bf16_t* K, const eta_bf16_t* V,
                               const int32_t* lengths, const int32_t* union_idx,
                               const int32_t* union_cnt, float T, float scale,
                               eta_prune_t prune, const float* vsum, const int32_t* cnt,
                               float* o, float* lse, int32_t* dev_status, void* stream);
size_t eta_decode_static_max_workspace(void);

/*
 * eta_decode_step -- the whole decode step in one launch: on append (update_tail != 0)
 * the tail block's metadata as eta_build_block_meta(ETA_TAIL_BLOCK), then the
 * thresholds as eta_predict_tau (W/bias, or the frozen tau_const when non-NULL),
 * the screening as eta_screen and the decode as eta_decode with ETA_PRUNE_SKIP.
 * (Arithmetic of those four calls: abstract of arXiv 2609.20888 for the cached
 * bounds, O(1) screening and co-admission; evolve.pub review, Methodology
 * Assessment, Eq. 1 for tau and Eq. 2-3 for the gate.)  Every output equals, bit for
 * bit, what the four separate calls write with the same arguments: tau, head_mask,
 * union_idx, union_cnt, head_cnt (nullable), o, lse, and the refreshed metadata.
 * One difference: a block at or past lengths[b] is never admitted, whatever its
 * cnt says (the separate calls rely on cnt alone).
 * Layouts: as the four calls.  cent_format / cent / rmax / var / vardim / cnt as
 * eta_screen (vardim nullable unless bound == ETA_BOUND_PROB_DIM; when given it is
 * refreshed with the tail block too); z for the probabilistic bounds; T: 0 = hard
 * gate; scale 0 = 1/sqrt(d).
 * One persistent cooperative kernel, one CTA per SM (no other kernel may hold SMs
 * the launch needs; else ETA_ERR_CUDA).  Requires d = 128, NB % 4 == 0, 16-byte
 * aligned q, K, V and metadata (else ETA_ERR_UNSUPPORTED / ETA_ERR_INVALID_ARG).
 * FLOOR pruning is not offered here (use the separate calls).
 * Workspace: eta_decode_step_workspace_size(dims) bytes, 16-byte aligned, zero-filled
 * once before the first call (it holds self-resetting counters) and again after any
 * call whose dev_status came back with ETA_DEVSTAT_TIMEOUT.  Calls sharing one
 * workspace must not overlap on the GPU.
 * dev_status: ETA_DEVSTAT_TIMEOUT (a bounded wait ran out), _NONFINITE_Q, _BAD_BLOCK.
 */
size_t eta_decode_step_workspace_size(const eta_dims_t* dims);
eta_status_t eta_decode_step(const eta_dims_t* dims, const eta_bf16_t* q, const float* W,
                             const float* bias, const float* tau_const, const eta_bf16_t* K,
                             const eta_bf16_t* V, const int32_t* lengths, int32_t update_tail,
                             eta_cent_format_t cent_format, void* cent, float* rmax,
                             float* var, float* vardim, int32_t* cnt, eta_bound_t bound,
                             float z, float T, float scale, float* tau, uint32_t* head_mask,
                             int32_t* union_idx, int32_t* union_cnt, int32_t* head_cnt,
                             float* o, float* lse, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream);

/*
 * eta_lse_merge -- merges decode results computed over disjoint key sets into the
 * result over their union: the log-sum-exp identity of a softmax split over key sets
 * (Eq. 2-3 of the review make the decode a softmax over gated logits).  With a KV
 * cache split into block-aligned sequence shards (one per GPU), eta_decode on each
 * shard with the same thresholds followed by this merge of the gathered results is
 * the decode of the whole cache: screening is per block, so each shard admits exactly
 * the blocks of the whole cache's union that lie in its range.
 *   M = max_p lse_p;  L = sum_p e^(lse_p - M);  o = sum_p e^(lse_p - M) o_p / L;
 *   lse = M + log L;  parts with lse_p = -inf add nothing; all empty: o = 0, lse = -inf.
 * o_parts fp32 [n_parts, n_rows, d], lse_parts fp32 [n_parts, n_rows] (device);
 * o fp32 [n_rows, d], lse fp32 [n_rows] (device, may not alias the parts).
 * n_rows = B * Hq; d in {64, 128}; n_parts >= 1 (else ETA_ERR_INVALID_ARG).
 * No workspace, no device status.
 */
eta_status_t eta_lse_merge(int32_t n_parts, int32_t n_rows, int32_t d, const float* o_parts,
                           const float* lse_parts, float* o, float* lse, void* stream);

/*
 * eta_dense_decode -- the dense baseline the speedups are measured against (the
 * pages compare with FlashAttention-2 decode): standard softmax decode attention
 * over every valid key, no threshold, no gate, same split-KV pipeline as eta_decode.
 * Workspace: eta_decode_workspace_size(dims).
 */
eta_status_t eta_dense_decode(const eta_dims_t* dims, const eta_bf16_t* q,
                              const eta_bf16_t* K, const eta_bf16_t* V,
                              const int32_t* lengths, float scale, float* o, float* lse,
                              void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * Decode engine (process-wide; both compute the same function, both are tested
 * against the float64 oracle):
 *   ETA_ENGINE_TCGEN05 -- q.k and p.v on the tensor cores (tcgen05.mma, TMEM
 *                         accumulators, TMA tensor copies with 128-byte swizzle);
 *                         d = 128 and d = 64
 *   ETA_ENGINE_FMA     -- q.k and p.v on the CUDA cores in fp32 (1-D TMA bulk copies)
 *   ETA_ENGINE_AUTO    -- the default: the engine this library measures fastest
 * eta_set_decode_engine returns ETA_ERR_INVALID_ARG for an unknown value.
 */
eta_status_t eta_set_decode_engine(eta_engine_t engine);
eta_engine_t eta_get_decode_engine(void);

/*
 * eta_prefill -- dense gated causal attention of a prefill chunk (the gate of the
 * review's Methodology Assessment, Eq. 2-3, on every (query, key) pair; the
 * inference-side counterpart of the paper's dense gated training forward).  For
 * query position t < lengths[b] of head h (KV head h / G):
 *   s_t' = scale * q_t . k_t',  t' <= t (causal)
 *   gated s'' = s' * sigmoid((s' - tau_t) / T)   (T > 0)  or  s' >= tau_t ? s' : 0 (T == 0)
 *   O[b,h,t] = sum_t' e^{s''} v_t' / sum_t' e^{s''},  lse[b,h,t] = log sum_t' e^{s''}
 * Q    bf16 [B, Hq, T_max, d] (head-major, like the cache), 16-byte aligned
 * K, V bf16 [B, Hkv, T_max, d];  tau fp32 [B, Hq, T_max] (per query token and head)
 * O    fp32 [B, Hq, T_max, d];  lse fp32 [B, Hq, T_max]; rows t >= lengths[b] untouched.
 * Tensor cores (tcgen05): S = Q K^T and O += P V on 128 x 128 tiles, fp32 TMEM
 * accumulators, P in bf16.  d = 128 and T_max % 128 == 0 only (else
 * ETA_ERR_UNSUPPORTED).  No workspace.  dev_status: ETA_DEVSTAT_TIMEOUT.
 */
eta_status_t eta_prefill(const eta_dims_t* dims, const eta_bf16_t* Q, const float* tau,
                         const eta_bf16_t* K, const eta_bf16_t* V, const int32_t* lengths,
                         float T, float scale, float* O, float* lse, int32_t* dev_status,
                         void* stream);

/*
 * Prefill kernel (process-wide; both compute the same function, both are tested
 * against the float64 oracle):
 *   ETA_PREFILL_ONE_TILE -- one CTA per (row, query head, 128-query tile)
 *   ETA_PREFILL_TWO_TILE -- one CTA per (row, query head, pair of 128-query tiles);
 *                           every K/V tile serves both, P stays in tensor memory
 *   ETA_PREFILL_AUTO     -- the default: the two-tile kernel once its tile pairs
 *                           (B * Hq * ceil(T_max / 256)) exceed half the SM count with
 *                           the hard gate, twice the SM count with the soft gate (the
 *                           sizes from which this library measures it faster)
 * eta_set_prefill_kernel returns ETA_ERR_INVALID_ARG for an unknown value.
 * eta_prefill_kernel_for returns the kernel (ETA_PREFILL_ONE_TILE or _TWO_TILE) that
 * eta_prefill would launch for these dims and gate temperature T under the current
 * setting (host only, no device work; -1 for dims or T that eta_prefill refuses).
 */
typedef enum {
  ETA_PREFILL_AUTO = 0,
  ETA_PREFILL_ONE_TILE = 1,
  ETA_PREFILL_TWO_TILE = 2
} eta_prefill_kernel_t;
eta_status_t eta_set_prefill_kernel(eta_prefill_kernel_t kernel);
eta_prefill_kernel_t eta_get_prefill_kernel(void);
int32_t eta_prefill_kernel_for(const eta_dims_t* dims, float T);

/*
 * eta_calibrate_const_tau -- offline calibration of frozen per-head thresholds
 * (abstract: "an offline calibration algorithm ... that freezes per-head constant
 * thresholds").  HOST pointers.  The pages do not print the algorithm; the rule
 * implemented: for each head h, pool bounds[i, h, j] over the n_q calibration
 * queries and the blocks with valid[i, h, j] != 0, sort ascending, and return the
 * element at index floor((1 - density) * N), so that admit-iff-bound>=tau admits
 * at least the target fraction of the pooled (query, block) pairs.
 * bounds fp32 [n_q, Hq, NB] (eta_screen's bounds_out), valid uint8 [n_q, Hq, NB],
 * tau_out fp32 [Hq].  Returns ETA_ERR_INVALID_ARG if a head has no valid entry.
 */
eta_status_t eta_calibrate_const_tau(const float* bounds, const uint8_t* valid,
                                     int32_t n_q, int32_t Hq, int32_t NB, float density,
                                     float* tau_out);

/*
 * eta_selftest_wait_timeout -- diagnostic of the failure detection (no counterpart
 * in the paper).  Launches one small kernel that waits, with the same bounded wait
 * the decode kernels use, on an mbarrier that nothing arrives on and on the int32
 * flag *never_set (device memory, may be NULL; the caller keeps it 0).  After
 * wait_limit polls each wait gives up and ETA_DEVSTAT_TIMEOUT is OR-ed into
 * *dev_status (device memory); the context stays usable.
 * wait_limit in [1, 2^24], else ETA_ERR_INVALID_ARG.
 */
eta_status_t eta_selftest_wait_timeout(uint32_t wait_limit, const int32_t* never_set,
                                       int32_t* dev_status, void* stream);

/*
 * eta_build_checked -- 1 in the checked build (libeta_checked.so: every global access
 * whose index a kernel computes is range-checked first, see ETA_DEVSTAT_BOUNDS), 0 in
 * the release build (libeta.so).  Both builds export the same entry points and
 * compute the same outputs; the checked one is a debugging aid (compute-sanitizer's
 * memcheck is not assumed to be available).
 *
 * eta_selftest_bounds -- diagnostic of the checked build: launches one thread that
 * runs the range check on (index, extent) without any memory access.  The checked
 * build ORs ETA_DEVSTAT_BOUNDS into *dev_status (device memory) when index lies
 * outside [0, extent); the release build compiles the check away and writes nothing.
 * extent < 0 or dev_status NULL: ETA_ERR_INVALID_ARG.
 */
int32_t eta_build_checked(void);
eta_status_t eta_selftest_bounds(int64_t index, int64_t extent, int32_t* dev_status,
                                 void* stream);

/* Maps a device status word (read back by the caller) to a status code. */
eta_status_t eta_status_from_device(int32_t dev_status);

/* Human-readable name of a status code (static storage). */
const char* eta_status_string(eta_status_t s);

#ifdef __cplusplus
}
#endif
#endif /* ETA_H_ */
