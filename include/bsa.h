/*
 * bsa.h -- C ABI of libbsa: top-p block-sparse self-attention for video
 * diffusion transformers on NVIDIA B200 (sm_100a).
 *
 * The method (sources named per call below):
 *   1. reorder the latent tokens along a 3-D Hilbert curve (optional),
 *   2. score key blocks per query block from block means and select, per
 *      query block, the smallest set of key blocks whose softmax mass reaches
 *      the head's top-p threshold,
 *   3. run exact softmax attention over the kept blocks only (O and LSE),
 *   4. correct the sparse output with a cached dense-minus-sparse refinement
 *      scaled per head: O + alpha_h * R.
 *
 * Conventions shared by every call
 *   - Tensors are dense, contiguous, row-major.  Q, K, V, O, R are bf16
 *     [B, H, L, D] (bsa_bf16 = raw bfloat16 bits).  NB = ceil(L / blk) blocks
 *     per sequence; the last block holds L - (NB-1)*blk tokens.
 *   - Every pointer argument is a DEVICE pointer unless its comment says
 *     "host".  Device pointers must be 16-byte aligned, except the optional
 *     device `status` word and the per-head `alpha` array, which need 4-byte
 *     alignment.  The caller owns and
 *     allocates every buffer (inputs, outputs, workspaces); the library never
 *     allocates, frees or synchronises.
 *   - Every call is asynchronous on `stream` (NULL = legacy default stream)
 *     and returns a bsa_status.  Arguments are validated on the host before
 *     anything is launched: a call that returns an error launched nothing.
 *     BSA_ECUDA means a launch failed; the CUDA error is not cleared.
 *   - Device-side faults of the input data (a kept index out of range, a
 *     timed-out internal wait) are reported through the optional device
 *     `status` word of bsa_sparse_attn_fwd, never by trapping.
 *   - Supported: D in {64, 128}; blk in {64, 128}; 1 <= NB <= 4096;
 *     B*H*L*D < 2^40; H <= 512 for bsa_select_topp_mask.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BSA_API __attribute__((visibility("default")))
#else
#define BSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t bsa_bf16;             /* bfloat16 bit pattern */
typedef struct CUstream_st* bsa_stream; /* same type as cudaStream_t */

typedef enum {
  BSA_OK = 0,
  BSA_EINVAL = 1,     /* null required pointer, misaligned pointer, p or alpha out of range */
  BSA_ESHAPE = 2,     /* unsupported or inconsistent sizes */
  BSA_ENODEV = 3,     /* no sm_100 device current */
  BSA_ECUDA = 4,      /* a kernel launch or a driver call failed */
  BSA_EWORKSPACE = 5  /* workspace missing or too small */
} bsa_status;

/* Bits a kernel may OR into a device status word. */
#define BSA_DEV_TIMEOUT 1   /* an internal pipeline wait exceeded its time limit */
#define BSA_DEV_BAD_INDEX 2 /* a kept index or count was out of range and was skipped */
#define BSA_DEV_SCHED_CONFLICT 4 /* an attention launch found its work counter in use (see below) */

typedef struct {
  int B;   /* batch */
  int H;   /* heads */
  int L;   /* tokens per sequence */
  int D;   /* head dimension */
  int blk; /* tokens per query / key block */
} bsa_shape;

/* Human-readable name of a status code (static storage). */
BSA_API const char* bsa_strerror(int status);

/* Library version, major*10000 + minor*100 + patch. */
BSA_API int bsa_version(void);

/*
 * bsa_score_blocks -- block importance scores.
 * Defines: block means as coarse attention estimates (RECAP, section 3.2),
 * block scoring for block importance (DFSAttn abstract), a per-query-block
 * distribution over key blocks for top-p selection (head-wise top-p and GSRS
 * abstracts).
 *   q_pool[b,h,i,:] = mean of Q[b,h,t,:] over the tokens t of block i
 *   k_pool[b,h,j,:] = same for K   (partial last block: its own count)
 *   probs[b,h,i,:]  = softmax_j( q_pool_i . k_pool_j / sqrt(D) )
 * Arguments: q, k bf16 [B,H,L,D]; outputs q_pool, k_pool float32 [B,H,NB,D]
 * and probs float32 [B,H,NB,NB].  Accumulation is float32.
 * Errors: BSA_EINVAL on a null or misaligned pointer; BSA_ESHAPE on an
 * unsupported shape.
 */
BSA_API int bsa_score_blocks(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, float* q_pool, float* k_pool,
                     float* probs, bsa_stream stream);

/*
 * bsa_select_topp_mask -- cumulative top-p block selection.
 * Defines: online top-p sparse attention with per-head thresholds (head-wise
 * top-p abstract); top-p selection for adaptive sparsity (GSRS abstract);
 * thresholding the top key blocks per query block (CalibAtt, Fig. 5).
 * Per row (b,h,i): clamp P to [0,1] (NaN -> 0); order key blocks by
 * (P desc, index asc); u_j = floor(P_j * 2^40) (exact integers);
 * T = ceil(p_h * sum_j u_j) in IEEE double; keep the shortest ordered prefix
 * whose u-sum is >= T (at least one block); p_h == 1 keeps every block.
 * The result is a pure function of the float32 probs: bit-identical on any
 * thread count or summation order.
 * Arguments: probs float32 [B,H,NB,NB]; p_host: HOST array of H floats,
 * each in (0, 1] (read before the call returns); outputs mask uint8
 * [B,H,NB,NB] (1 = kept), kept_idx int32 [B,H,NB,NB] (first kept_cnt entries
 * of each row: kept key-block indices ascending; the rest unspecified),
 * kept_cnt int32 [B,H,NB].
 * Errors: BSA_EINVAL on a null pointer or a p outside (0,1]; BSA_ESHAPE.
 */
BSA_API int bsa_select_topp_mask(bsa_shape s, const float* probs, const float* p_host, uint8_t* mask,
                         int32_t* kept_idx, int32_t* kept_cnt, bsa_stream stream);

/*
 * bsa_reorder_workspace_bytes -- device scratch needed by bsa_reorder_tokens
 * for a (T, Hh, W) grid (0 on an unsupported grid).
 */
BSA_API size_t bsa_reorder_workspace_bytes(int T, int Hh, int W);

/*
 * bsa_reorder_tokens -- 3-D Hilbert-curve token order of a latent grid.
 * Defines: Hilbert curve-based token reordering that makes spatially close
 * tokens contiguous (DFSAttn abstract).  Curve: Skilling's n-dimensional
 * Hilbert curve on the smallest 2^k cube holding the grid, axis order
 * (t, y, x) with t most significant; grid tokens are row-major
 * n = (t*Hh + y)*W + x; cube points outside the grid are skipped.
 * Outputs int32 perm[L] (perm[i] = grid token at Hilbert rank i) and
 * inv[L] (inv[perm[i]] = i).  Computed once per grid shape.
 * ws: device scratch of bsa_reorder_workspace_bytes(T,Hh,W) bytes, contents
 * ignored on entry and clobbered.
 * Errors: BSA_EINVAL on null pointers; BSA_ESHAPE if any extent is < 1 or
 * > 256; BSA_EWORKSPACE if ws is NULL or ws_bytes too small.
 */
BSA_API int bsa_reorder_tokens(int T, int Hh, int W, int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes,
                       bsa_stream stream);

/*
 * bsa_reorder_tokens_noalloc -- bsa_reorder_tokens for callers that cannot
 * allocate device memory.  The paper has no counterpart: this is a library
 * convenience.  Same result as bsa_reorder_tokens; the scratch it needs lives
 * in a 16 KB array inside the library (every GPU that loads the library holds
 * it until exit), which covers every grid the call accepts (extents <= 256).
 * For callers whose device memory is owned by a host framework's allocator
 * that passes only input/output buffers, whose HBM is already reserved, or
 * that cannot take cudaMalloc's implicit synchronisation.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * All calls share the array: calls that overlap on the GPU race, so
 * serialise them.  Allocates nothing, frees nothing.
 * Errors: as bsa_reorder_tokens, with BSA_ESHAPE for a grid beyond the limit.
 */
BSA_API int bsa_reorder_tokens_noalloc(int T, int Hh, int W, int32_t* perm, int32_t* inv, bsa_stream stream);

/*
 * bsa_permute_tokens -- apply a token permutation to [B,H,L,D] bf16 rows.
 *   inverse == 0:  y[b,h,i,:]       = x[b,h,perm[i],:]   (into curve order)
 *   inverse != 0:  y[b,h,perm[i],:] = x[b,h,i,:]         (back to grid order)
 * s.blk is ignored; D must be a multiple of 8.  x and y must not overlap.
 * perm must be a permutation of [0, L) (not checked on the device).
 */
BSA_API int bsa_permute_tokens(bsa_shape s, const bsa_bf16* x, const int32_t* perm, bsa_bf16* y, int inverse,
                       bsa_stream stream);

/*
 * bsa_score_blocks_gather -- the token reorder of q and k fused with scoring.
 * Same as bsa_permute_tokens(q -> q_out), bsa_permute_tokens(k -> k_out)
 * (inverse = 0, q_out[b,h,t,:] = q[b,h,perm[t],:]) followed by
 * bsa_score_blocks(q_out, k_out), in one pass that reads q and k once.
 * perm: device int32 [L], a permutation of [0, L) (e.g. from
 * bsa_reorder_tokens; not checked on the device).  q_out, k_out: bf16
 * [B,H,L,D], not overlapping q, k or each other; or both NULL to score the
 * reordered tokens without writing them (for bsa_sparse_attn_fwd_gather).
 * Outputs and errors as bsa_score_blocks and bsa_permute_tokens.
 */
BSA_API int bsa_score_blocks_gather(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const int32_t* perm,
                            bsa_bf16* q_out, bsa_bf16* k_out, float* q_pool, float* k_pool, float* probs,
                            bsa_stream stream);

/*
 * bsa_block_drift -- query-key drift of each head since a reference step.
 * Defines: Temporal Mask Reuse skips mask prediction based on query-key drift
 * (head-wise adaptive top-p abstract).  From the block means that
 * bsa_score_blocks writes (float32 [B,H,NB,D]) at the step that predicted the
 * mask (q_pool_ref, k_pool_ref) and at the current step (q_pool, k_pool):
 *   drift[b*H + h] = max( ||q_pool - q_pool_ref||_F / ||q_pool_ref||_F ,
 *                         ||k_pool - k_pool_ref||_F / ||k_pool_ref||_F )
 * over the head's [NB, D] means (0/0 -> 0; a change from an all-zero
 * reference -> +inf).  Output drift: device float32 [B*H].  The caller keeps
 * a head's mask while its drift stays at or below its threshold.
 * Errors: BSA_EINVAL on null/misaligned pointers; BSA_ESHAPE; BSA_ENODEV.
 */
BSA_API int bsa_block_drift(bsa_shape s, const float* q_pool_ref, const float* k_pool_ref, const float* q_pool,
                    const float* k_pool, float* drift, bsa_stream stream);

/*
 * bsa_score_blocks_restricted -- bsa_score_blocks with each query block's
 * softmax taken over its candidate key blocks only.
 * Defines: later top-p searches restricted to an early candidate set (GSRS
 * abstract).  candidates: device uint8 [B,H,NB,NB], nonzero = candidate (for
 * instance an earlier mask, possibly widened).  probs[b,h,i,j] = softmax over
 * the candidates j of row i of the block logits, 0 for non-candidates; a row
 * without candidates is all zeros.  Pooled means as bsa_score_blocks.
 * Errors: as bsa_score_blocks, BSA_EINVAL for a null candidates pointer.
 */
BSA_API int bsa_score_blocks_restricted(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const uint8_t* candidates,
                                float* q_pool, float* k_pool, float* probs, bsa_stream stream);

/*
 * bsa_select_topp_mask_restricted -- top-p selection over the candidate key
 * blocks of each row.
 * Defines: GSRS abstract (search restricted to an early candidate set) with
 * the top-p rule of bsa_select_topp_mask: candidates ordered by (P desc,
 * index asc), target T = ceil(p_h * sum of the candidates' fixed-point
 * masses), the shortest prefix reaching T is kept (at least one block when a
 * candidate exists); p_h == 1 keeps every candidate; non-candidates are never
 * kept; a row without candidates keeps nothing (count 0).
 * Arguments and errors as bsa_select_topp_mask, plus candidates (device uint8
 * [B,H,NB,NB], required).
 */
BSA_API int bsa_select_topp_mask_restricted(bsa_shape s, const float* probs, const float* p_host,
                                    const uint8_t* candidates, uint8_t* mask, int32_t* kept_idx,
                                    int32_t* kept_cnt, bsa_stream stream);

/*
 * Interval (skip-list) form of the kept key blocks.
 * Defines: skip lists that store, per query-block row, interval pairs of key
 * blocks; the number of intervals per row (CalibAtt appendix, Fig. S9); per-
 * layer trimming of the rows to the widest one and merging of outlier rows so
 * that the width falls further (Fig. S10 (b), (c)); the width chosen by a
 * merge percentage (Table S3, "Merge %": 100 = no merge, 99, 95).
 * A row's runs are the maximal runs of consecutive indices of its ascending
 * kept list, each stored as an int32 pair (start, end), end exclusive.  A row
 * of NB blocks has at most ceil(NB/2) runs.  Merging a row to width W fills
 * the gaps between its neighbouring runs smallest first (the leftmost of
 * equal gaps first) until W intervals remain: the merged row keeps a superset
 * of its blocks, with the fewest blocks added.
 * Rows are (b,h,i) of [B,H,NB]; kept_idx/kept_cnt as bsa_select_topp_mask
 * writes them.  A row whose count lies outside [0, NB] or whose first
 * kept_cnt entries are not strictly ascending within [0, NB) is malformed:
 * it is flagged (BSA_DEV_BAD_INDEX in the optional device status word, OR-ed;
 * the caller zeroes it) and treated as empty, as the calls below state.
 */

/*
 * bsa_interval_runs -- runs per row and their histogram.
 * Outputs n_runs: device int32 [B,H,NB] (0 for a malformed row); hist:
 * device int32 [ceil(NB/2) + 1] or NULL, hist[r] += the number of well-formed
 * rows with r runs.  hist is accumulated, not cleared: zero it once, then
 * accumulate over the heads, layers and steps that will share one width.
 * Errors: BSA_EINVAL on null required or misaligned pointers; BSA_ESHAPE;
 * BSA_ENODEV; BSA_ECUDA.
 */
BSA_API int bsa_interval_runs(bsa_shape s, const int32_t* kept_idx, const int32_t* kept_cnt, int32_t* n_runs,
                              int32_t* hist, int32_t* status, bsa_stream stream);

/*
 * bsa_interval_width_for_merge -- HOST function, no device work: the interval
 * width for a merge percentage q in (0, 1].  W is the smallest width >= 1
 * such that at least ceil(q * rows) rows (IEEE double product) have at most W
 * runs, rows being the sum of the histogram.  q = 1 gives the widest row (no
 * merge); q = 0.95 merges the 5% widest rows.
 * Arguments: hist_host: HOST int32 [nbins] (the bsa_interval_runs histogram
 * copied back, nbins = ceil(NB/2) + 1 >= 2); W_out: HOST int.
 * Errors: BSA_EINVAL on a null pointer, nbins < 2, a negative count or q
 * outside (0, 1].
 */
BSA_API int bsa_interval_width_for_merge(const int32_t* hist_host, int nbins, double q, int* W_out);

/*
 * bsa_kept_to_intervals -- encode the kept lists as interval pairs of width W.
 * Outputs intervals: device int32 [B,H,NB,W,2], each row's pairs ascending,
 * pairs past its count set to (-1, -1); n_int: device int32 [B,H,NB] =
 * min(runs, W); n_runs: device int32 [B,H,NB] (runs before merging) or NULL.
 * A row with more than W runs is merged to exactly W intervals.  A malformed
 * row gets n_int = 0 and all pairs (-1, -1).  1 <= W <= NB.
 * Errors: BSA_EINVAL on null required or misaligned pointers or W out of
 * range; BSA_ESHAPE; BSA_ENODEV; BSA_ECUDA.
 */
BSA_API int bsa_kept_to_intervals(bsa_shape s, const int32_t* kept_idx, const int32_t* kept_cnt, int W,
                                  int32_t* intervals, int32_t* n_int, int32_t* n_runs, int32_t* status,
                                  bsa_stream stream);

/*
 * bsa_intervals_to_kept -- decode interval pairs into the mask and kept lists
 * that bsa_sparse_attn_fwd takes.
 * Inputs intervals int32 [B,H,NB,W,2] and n_int int32 [B,H,NB] as
 * bsa_kept_to_intervals writes them.  A row is well formed when
 * 0 <= n_int <= W and its first n_int pairs satisfy 0 <= start < end <= NB
 * and start >= the previous pair's end; a malformed row decodes as empty.
 * Outputs mask uint8 [B,H,NB,NB] or NULL (1 = kept, whole row written),
 * kept_idx int32 [B,H,NB,NB] (first kept_cnt entries ascending; the rest
 * unspecified), kept_cnt int32 [B,H,NB].  1 <= W <= NB.
 * Errors: as bsa_kept_to_intervals.
 */
BSA_API int bsa_intervals_to_kept(bsa_shape s, const int32_t* intervals, const int32_t* n_int, int W, uint8_t* mask,
                                  int32_t* kept_idx, int32_t* kept_cnt, int32_t* status, bsa_stream stream);

/*
 * Coarse tail of the omitted blocks and its reconstruction (RECAP, section
 * 3.2).  Per head, with a = q / sqrt(D) and T(i) the blocks query block i does
 * NOT keep:
 *   block log-mass  log n_j + a . kbar_j + 1/2 sum_d a_d^2 s2_j[d]
 *   lbar  = log sum_{j in T(i)} exp(block log-mass)          (-inf if T(i) is empty)
 *   obar  = sum_{j in T(i)} w_j vbar_j + C a                   (0 if T(i) is empty)
 * kbar_j, s2_j, vbar_j: the block's key mean, per-dimension key variance
 * (population) and value mean; w_j the normalised block masses; C[e][d] =
 * (1/L) sum over all tokens of (v - vbar_block)[e] (k - kbar_block)[d], the
 * pooled within-block value-key covariance.  At a dense refresh the cached
 * refinement is d = (l_T - lbar, o_T - obar) with (l_T, o_T) the exact
 * attention over T(i); a later sparse step returns
 *   LSE = logaddexp(l_S, lbar + d_l),  O = w_S O_S + w_T (obar + d_o).
 * D must be 128 for the statistics and the tail.
 */

/* Workspace bytes that bsa_tail_stats and bsa_coarse_tail share (0 for an
 * unsupported shape). */
BSA_API size_t bsa_tail_workspace_bytes(bsa_shape s);

/*
 * bsa_tail_stats -- block moments and the pooled covariance of K and V.
 * Outputs kbar, s2, vbar float32 [B,H,NB,D], C float32 [B,H,D,D]; ws (device,
 * bsa_tail_workspace_bytes) receives the operand tables bsa_coarse_tail reads.
 * Errors: BSA_EINVAL, BSA_ESHAPE (D != 128), BSA_EWORKSPACE, BSA_ENODEV,
 * BSA_ECUDA.
 */
BSA_API int bsa_tail_stats(bsa_shape s, const bsa_bf16* k, const bsa_bf16* v, float* kbar, float* s2, float* vbar,
                           float* C, void* ws, size_t ws_bytes, int32_t* status, bsa_stream stream);

/*
 * bsa_coarse_tail -- lbar float32 [B,H,L] and obar bf16 [B,H,L,D] over the
 * blocks each query block omits.  mask: uint8 [B,H,NB,NB] (1 = kept), as
 * bsa_select_topp_mask writes it; ws as written by bsa_tail_stats for the same
 * K and V.  s.blk must be 128 and s.D 128.
 */
BSA_API int bsa_coarse_tail(bsa_shape s, const bsa_bf16* q, const uint8_t* mask, const void* ws, size_t ws_bytes,
                            float* lbar, bsa_bf16* obar, int32_t* status, bsa_stream stream);

/* bsa_tail_refinement -- d_l = l_T - lbar, d_o = bf16(o_T - obar) (both 0
 * where the tail is empty); l_T, o_T: the exact attention over the omitted
 * blocks (bsa_sparse_attn_fwd with bsa_complement_lists). */
BSA_API int bsa_tail_refinement(bsa_shape s, const float* l_T, const bsa_bf16* o_T, const float* lbar,
                                const bsa_bf16* obar, float* d_l, bsa_bf16* d_o, bsa_stream stream);

/* bsa_tail_reconstruct -- the sparse part (l_S, o_S) merged with the
 * reconstructed tail (lbar + d_l, obar + d_o): o bf16 [B,H,L,D], lse float32. */
BSA_API int bsa_tail_reconstruct(bsa_shape s, const float* l_S, const bsa_bf16* o_S, const float* lbar,
                                 const bsa_bf16* obar, const float* d_l, const bsa_bf16* d_o, bsa_bf16* o,
                                 float* lse, bsa_stream stream);

/* bsa_complement_lists -- the blocks each row does not keep (mask 0), as
 * ascending lists in the layout of bsa_select_topp_mask. */
BSA_API int bsa_complement_lists(bsa_shape s, const uint8_t* mask, int32_t* idx, int32_t* cnt, bsa_stream stream);

/*
 * bsa_wait_selftest -- exercises the bounded wait that every pipeline wait of
 * the library uses: one thread waits on an mbarrier that nothing arrives at,
 * gives up after limit_ns (1 ns .. 2 s) of the GPU's global timer, ORs
 * BSA_DEV_TIMEOUT into *status (device int32, 4-byte aligned) and returns;
 * the context stays usable.
 */
BSA_API int bsa_wait_selftest(int32_t* status, unsigned long long limit_ns, bsa_stream stream);

/*
 * bsa_sparse_attn_fwd -- block-sparse attention forward with an optional
 * fused correction epilogue.
 * Defines: computing the selected connections densely and skipping the
 * unselected blocks (CalibAtt abstract, Fig. 5(b)); block-sparse attention
 * for selected interactions and dense attention for refreshes (RECAP,
 * section 4.1); cached dense refinement correcting the sparse estimate
 * (RECAP, section 1 and abstract).
 * For every query token r of query block i with kept key blocks K(i):
 *   LSE[r] = log sum_{c in K(i), c < L} exp(q_r . k_c / sqrt(D))
 *   O[r]   = sum_c exp(q_r . k_c / sqrt(D) - LSE[r]) v_c       (+ alpha_h R[r])
 * Arguments: q, k, v bf16 [B,H,L,D]; kept_idx/kept_cnt as produced by
 * bsa_select_topp_mask, or both NULL for dense attention (every block kept);
 * R bf16 [B,H,L,D] and alpha float32 [H] (device), both NULL for no
 * correction; with R the epilogue writes bf16(O_fp32 + alpha_h * R) and LSE
 * stays the sparse LSE.  Outputs o bf16 [B,H,L,D], lse float32 [B,H,L]
 * (natural log; -inf and O = 0 for a row with no kept key).
 * status: optional device int32 that receives BSA_DEV_* bits (OR-ed; the
 * caller zeroes it); NULL to skip.  Kept indices outside [0, NB) and counts
 * outside [0, NB] are skipped/clamped and flagged, never dereferenced.
 * Work distribution (blk = 128): the launch's CTAs draw query blocks from a
 * work counter in a ring of 256 counters inside the library, one per launch,
 * assigned round robin and released by the launch's last CTA, so no scratch
 * is needed.  A launch that finds its counter still owned by another launch
 * -- more than 256 attention launches (of this call, the scatter form and
 * bsa_sparse_attn_refresh) executing at the same time, or one captured CUDA
 * graph holding an attention call replayed on two streams at once -- leaves
 * (part of) its output unwritten and sets BSA_DEV_SCHED_CONFLICT; do not
 * replay such a graph concurrently with itself.
 * Errors: BSA_EINVAL on null/misaligned pointers or exactly one of
 * kept_idx/kept_cnt (or R/alpha) NULL; BSA_ESHAPE; BSA_ENODEV; BSA_ECUDA.
 */
BSA_API int bsa_sparse_attn_fwd(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const bsa_bf16* v,
                        const int32_t* kept_idx, const int32_t* kept_cnt, const bsa_bf16* R,
                        const float* alpha, bsa_bf16* o, float* lse, int32_t* status, bsa_stream stream);

/*
 * bsa_sparse_attn_fwd_scatter -- bsa_sparse_attn_fwd that writes each output
 * row through a row map, so that attention on Hilbert-ordered tokens returns
 * O and LSE in grid order without a separate scatter (DFSAttn abstract: the
 * tokens are reordered along a Hilbert curve for the attention only).
 * Same computation and arguments as bsa_sparse_attn_fwd, plus out_rows: device
 * int32 [L]; output row r of every (b, h) goes to row out_rows[r] of o and lse
 * (the `perm` of bsa_reorder_tokens undoes the curve order).  R is read in the
 * order of q/k/v.  out_rows must be a permutation of [0, L); a row whose
 * target is out of range is skipped and flagged (BSA_DEV_BAD_INDEX).
 * s.blk must be 128 (BSA_ESHAPE otherwise).
 */
BSA_API int bsa_sparse_attn_fwd_scatter(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const bsa_bf16* v,
                                const int32_t* kept_idx, const int32_t* kept_cnt, const bsa_bf16* R,
                                const float* alpha, const int32_t* out_rows, bsa_bf16* o, float* lse,
                                int32_t* status, bsa_stream stream);

/*
 * bsa_sparse_attn_fwd_gather -- the block-sparse attention of tokens taken in
 * the order `rows` gives, with every tensor in the caller's (grid) order: the
 * Hilbert reorder of the DFSAttn abstract without reordered copies of q, k, v.
 * Token t of the attention's order is row rows[t] of every (b, h) of q, k and
 * v (the `perm` of bsa_reorder_tokens); query and key blocks are the 128
 * consecutive tokens of that order, and kept_idx/kept_cnt index those blocks
 * (as bsa_select_topp_mask gives them after bsa_score_blocks_gather).  The
 * output of token t goes to row rows[t] of o and lse, and R (with alpha) is
 * read at that row too: o = bsa_permute_tokens(inverse) of what
 * bsa_sparse_attn_fwd gives on the reordered q, k, v and reordered R.
 * The kernel loads its Q, K and V tiles with 4-row TMA gathers.
 * rows: device int32 [L], 16-byte aligned, a permutation of [0, L); a row
 * outside [0, L) reads zeros, its output is skipped, and BSA_DEV_BAD_INDEX is
 * set.  Other arguments and errors as bsa_sparse_attn_fwd; s.blk and s.D must
 * be 128 and B*H*L below 2^31 (BSA_ESHAPE otherwise).
 */
BSA_API int bsa_sparse_attn_fwd_gather(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const bsa_bf16* v,
                                       const int32_t* rows, const int32_t* kept_idx, const int32_t* kept_cnt,
                                       const bsa_bf16* R, const float* alpha, bsa_bf16* o, float* lse,
                                       int32_t* status, bsa_stream stream);

/*
 * bsa_sparse_attn_fwd_intervals -- bsa_sparse_attn_fwd with the kept blocks
 * given as interval pairs, walked by the attention kernel itself (CalibAtt
 * appendix, Fig. S10: the skip lists are what the kernel reads); no decode to
 * padded lists.  intervals: device int32 [B,H,NB,W,2] and n_int: device int32
 * [B,H,NB], as bsa_kept_to_intervals writes them (a row's first n_int pairs
 * (start, end), end exclusive, ascending).  The result equals
 * bsa_sparse_attn_fwd on the lists bsa_intervals_to_kept decodes from the
 * same pairs, bit for bit.  A malformed row (n_int outside [0, W], or a pair
 * with start < the previous end, start >= end or end > NB) is attended as
 * empty (O = 0, LSE = -inf) and sets BSA_DEV_BAD_INDEX.
 * Other arguments and errors as bsa_sparse_attn_fwd; 1 <= W <= NB (BSA_EINVAL
 * otherwise); s.blk must be 128 (BSA_ESHAPE otherwise).
 */
BSA_API int bsa_sparse_attn_fwd_intervals(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const bsa_bf16* v,
                                          const int32_t* intervals, const int32_t* n_int, int W,
                                          const bsa_bf16* R, const float* alpha, bsa_bf16* o, float* lse,
                                          int32_t* status, bsa_stream stream);

/*
 * FP8 Q.K^T.  Defines: the sparse attention of a distilled pipeline run in
 * FP8 with fused kernels (abstract on the page titled RECAP).  The page gives
 * no format or scaling rule; here Q and K are quantized to OCP E4M3 (max 448,
 * round to nearest even, saturating) with one scale per (b, h, token block),
 * the logits are (s_q * s_k) * (q8 . k8) accumulated in fp32 by the tensor
 * cores, and the softmax, P.V (bf16 V) and the epilogue are those of
 * bsa_sparse_attn_fwd.  The result is the block-sparse attention of the
 * dequantized Q and K.
 */

/*
 * bsa_quantize_fp8 -- E4M3 codes and per-block scales of a bf16 tensor.
 *   per (b, h, block j of s.blk tokens): amax = max |x|,
 *   scale[b,h,j] = amax / 448 (1 for an all-zero block),
 *   codes = E4M3_rn_satfinite(x * (448 / amax))  (float32 reciprocal and product)
 * x: bf16 [B,H,L,D]; codes: uint8 [B,H,L,D]; scales: float32 [B,H,NB].
 * Errors: BSA_EINVAL on null or misaligned pointers; BSA_ESHAPE; BSA_ENODEV;
 * BSA_ECUDA.
 */
BSA_API int bsa_quantize_fp8(bsa_shape s, const bsa_bf16* x, uint8_t* codes, float* scales, bsa_stream stream);

/*
 * bsa_sparse_attn_fwd_fp8 -- bsa_sparse_attn_fwd with S = Q.K^T from E4M3
 * codes (kind::f8f6f4 tensor-core MMAs).  q8/q_scale and k8/k_scale as
 * bsa_quantize_fp8 writes them (blocks of 128 tokens); v, kept lists, R/alpha,
 * o, lse and status as bsa_sparse_attn_fwd.  s.blk and s.D must be 128.
 * Errors: as bsa_sparse_attn_fwd; BSA_ESHAPE for another blk or D.
 */
BSA_API int bsa_sparse_attn_fwd_fp8(bsa_shape s, const uint8_t* q8, const float* q_scale, const uint8_t* k8,
                                    const float* k_scale, const bsa_bf16* v, const int32_t* kept_idx,
                                    const int32_t* kept_cnt, const bsa_bf16* R, const float* alpha, bsa_bf16* o,
                                    float* lse, int32_t* status, bsa_stream stream);

/*
 * bsa_refresh_refinement -- renew the cached refinement at a dense refresh.
 * Defines: the refinement cached at a dense refresh and renewed only there
 * (RECAP, sections 1, 3.4 and 4.3).
 *   R = bf16( float(o_dense) - float(o_sparse) )   elementwise, [B,H,L,D]
 * s.blk is ignored; D must be a multiple of 8.
 */
BSA_API int bsa_refresh_refinement(bsa_shape s, const bsa_bf16* o_dense, const bsa_bf16* o_sparse, bsa_bf16* R,
                           bsa_stream stream);

/*
 * bsa_sparse_attn_refresh -- a dense refresh in one pass over every key block.
 * Defines: the dense refresh that renews the cached refinement (RECAP,
 * section 1 and section 3.4 with Fig. 3) and the exact share of the attention
 * weight carried by the kept blocks, evaluated inside the attention
 * computation (GSRS abstract).  With K(i) the kept blocks of query block i and
 * s_c = q_r . k_c / sqrt(D) over keys c < L:
 *   lse_dense[r]  = log sum_{all c} exp(s_c),  o_dense[r]  = sum_c exp(s_c - lse_dense[r]) v_c
 *   lse_sparse[r] = log sum_{c in K(i)} exp(s_c),  o_sparse[r] likewise over K(i)
 *   R[r]          = bf16( bf16(o_dense[r]) - bf16(o_sparse[r]) )   (as bsa_refresh_refinement)
 *   kept_mass[r]  = exp(lse_sparse[r] - lse_dense[r])             (0 for an empty K(i))
 * One pass: every key block is read once; a kept block's P.V goes to one
 * accumulator and any other block's to a second, under one running max.
 * Arguments: q, k, v bf16 [B,H,L,D]; kept_idx/kept_cnt (required) as produced
 * by bsa_select_topp_mask -- each row's list must be ascending; entries out of
 * range or out of order are skipped and flagged in status.  Outputs o_dense,
 * o_sparse bf16 [B,H,L,D]; lse_dense, lse_sparse float32 [B,H,L] (natural
 * log); R bf16 [B,H,L,D] or NULL; kept_mass float32 [B,H,L] or NULL.
 * s.blk must be 128 and s.D 64 or 128.
 * status: optional device int32 as for bsa_sparse_attn_fwd.
 * Errors: BSA_EINVAL on null required or misaligned pointers; BSA_ESHAPE;
 * BSA_ENODEV; BSA_ECUDA.
 */
BSA_API int bsa_sparse_attn_refresh(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const bsa_bf16* v,
                            const int32_t* kept_idx, const int32_t* kept_cnt, bsa_bf16* o_dense,
                            float* lse_dense, bsa_bf16* o_sparse, float* lse_sparse, bsa_bf16* R,
                            float* kept_mass, int32_t* status, bsa_stream stream);

/*
 * bsa_apply_correction -- standalone form of the fused correction.
 * Defines: fresh sparse statistics regulating how strongly the aging cached
 * refinement is applied (RECAP, section 1 and abstract), here as a
 * caller-supplied per-head strength alpha_h.
 *   o[b,h,:,:] = bf16( float(o_sparse[b,h,:,:]) + alpha[h] * float(R[b,h,:,:]) )
 * alpha: device float32 [H].  o may alias o_sparse.  D multiple of 8.
 */
BSA_API int bsa_apply_correction(bsa_shape s, const bsa_bf16* o_sparse, const bsa_bf16* R, const float* alpha,
                         bsa_bf16* o, bsa_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H_ */
