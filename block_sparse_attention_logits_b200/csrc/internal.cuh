// Private declarations shared by the libbsa translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/bsa.h"

namespace bsa {

constexpr int kMaxNB = 4096;     // key/query blocks per sequence
constexpr int kMaxHeadsP = 512;  // heads whose top-p threshold travels as a kernel argument

struct TopP {
  float p[kMaxHeadsP];
};

inline int n_blocks(int L, int blk) { return (L + blk - 1) / blk; }

// Per-device host state (host_state.cu), valid for the context it was made in:
// raise a kernel's dynamic shared-memory limit to `bytes` on the current device
// (no-op up to 48 KB, once per kernel and context); the current device's SM
// count; the current device's address of one of the library's __device__
// arrays (BSA_OK, BSA_ENODEV or BSA_ECUDA).
cudaError_t smem_opt_in(const void* func, size_t bytes);
int sm_count();
int symbol_address(const void* symbol, void** out);

// launchers (return cudaSuccess or the launch error)
// perm (nullable): gather form -- token t is input row perm[t]; the gathered
// rows are also written to q_out / k_out
cudaError_t launch_pool(const bsa_shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k, float* qp, float* kp,
                        cudaStream_t st, const int32_t* perm = nullptr, __nv_bfloat16* q_out = nullptr,
                        __nv_bfloat16* k_out = nullptr);
// cand: optional uint8 [B,H,NB,NB]; non-null restricts each row's softmax and
// top-p search to its candidate blocks (the others get P = 0 / are never kept)
cudaError_t launch_block_softmax(const bsa_shape& s, const float* qp, const float* kp, float* probs,
                                 const uint8_t* cand, cudaStream_t st);
cudaError_t launch_select(const bsa_shape& s, const float* probs, const TopP& p, const uint8_t* cand, uint8_t* mask,
                          int32_t* idx, int32_t* cnt, cudaStream_t st);
// drift[b*H + h] of the block means against reference means, [B,H,NB,D] each
cudaError_t launch_drift(const bsa_shape& s, const float* qp_ref, const float* kp_ref, const float* qp,
                         const float* kp, float* drift, cudaStream_t st);
// interval form of the kept lists: W == 0 counts runs per row (n_runs
// required, hist nullable, accumulated); W >= 1 encodes intervals of width W
int max_intervals(int NB);
cudaError_t launch_interval_encode(const bsa_shape& s, const int32_t* kept_idx, const int32_t* kept_cnt, int W,
                                   int32_t* intervals, int32_t* n_int, int32_t* n_runs, int32_t* hist,
                                   int32_t* status, cudaStream_t st);
cudaError_t launch_interval_decode(const bsa_shape& s, const int32_t* intervals, const int32_t* n_int, int W,
                                   uint8_t* mask, int32_t* kept_idx, int32_t* kept_cnt, int32_t* status,
                                   cudaStream_t st);
// one thread waits on an mbarrier nothing arrives at, for limit_ns
cudaError_t launch_wait_selftest(int32_t* status, unsigned long long limit_ns, cudaStream_t st);
// coarse tail (D = 128): moments and pooled covariance, then the tail itself;
// `ws` holds the centred transposed K/V and the operand tables between them
size_t tail_workspace_bytes(const bsa_shape& s);
int launch_tail_stats(const bsa_shape& s, const __nv_bfloat16* k, const __nv_bfloat16* v, float* kbar, float* s2,
                      float* vbar, float* C, void* ws, int32_t* status, cudaStream_t st);
int launch_coarse_tail(const bsa_shape& s, const __nv_bfloat16* q, const uint8_t* mask, const void* ws,
                       float* lbar, __nv_bfloat16* obar, int32_t* status, cudaStream_t st);
int launch_tail_refine(const bsa_shape& s, const float* l_T, const __nv_bfloat16* o_T, const float* lbar,
                       const __nv_bfloat16* obar, float* d_l, __nv_bfloat16* d_o, cudaStream_t st);
int launch_tail_merge(const bsa_shape& s, const float* l_S, const __nv_bfloat16* o_S, const float* lbar,
                      const __nv_bfloat16* obar, const float* d_l, const __nv_bfloat16* d_o, __nv_bfloat16* o,
                      float* lse, cudaStream_t st);
int launch_complement(const bsa_shape& s, const uint8_t* mask, int32_t* idx, int32_t* cnt, cudaStream_t st);
// E4M3 codes and per-block scales of a bf16 [B,H,L,D] tensor (blocks of s.blk tokens)
cudaError_t launch_quantize_fp8(const bsa_shape& s, const __nv_bfloat16* x, uint8_t* codes, float* scales,
                                cudaStream_t st);
size_t hilbert_workspace_bytes(int T, int Hh, int W);
cudaError_t launch_hilbert(int T, int Hh, int W, int32_t* perm, int32_t* inv, void* ws, cudaStream_t st);
cudaError_t launch_permute(const bsa_shape& s, const __nv_bfloat16* x, const int32_t* perm, __nv_bfloat16* y,
                           int inverse, cudaStream_t st);
cudaError_t launch_refresh(size_t n, const __nv_bfloat16* od, const __nv_bfloat16* os, __nv_bfloat16* R,
                           cudaStream_t st);
cudaError_t launch_correct(const bsa_shape& s, const __nv_bfloat16* os, const __nv_bfloat16* R, const float* alpha,
                           __nv_bfloat16* o, cudaStream_t st);

struct AttnArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* kept_idx;
  const int32_t* kept_cnt;
  const __nv_bfloat16* R;
  const float* alpha;
  __nv_bfloat16* o;
  float* lse;
  int32_t* status;
  // fused refresh (blk = 128 only): non-null o2 selects it; o/lse receive the
  // dense output, o2/lse2 the sparse output over the kept blocks
  __nv_bfloat16* o2 = nullptr;
  float* lse2 = nullptr;
  __nv_bfloat16* r_out = nullptr;  // nullable
  float* mass = nullptr;           // nullable
  // blk = 128, not the fused refresh: output row r of (b, h) goes to row
  // out_rows[r] of o and lse (nullable = identity)
  const int32_t* out_rows = nullptr;
  // blk = 128, bf16, not the fused refresh: token t of the attention's order
  // is row in_rows[t] of q, k and v (loaded by row gathers), and R is read in
  // the order of o (nullable = q, k, v already in the attention's order)
  const int32_t* in_rows = nullptr;
  // blk = 128, bf16, not the fused refresh: the kept blocks as interval pairs
  // (intervals [B,H,NB,W,2], n_int [B,H,NB]) instead of kept_idx / kept_cnt
  const int32_t* intervals = nullptr;
  const int32_t* n_int = nullptr;
  int W = 0;
  // FP8 Q.K^T (blk = 128, D = 128): E4M3 codes of Q and K ([B,H,L,D] bytes) and
  // their dequantization scales per (b, h, 128-token block); non-null q8
  // selects it (q and k are then unused)
  const uint8_t* q8 = nullptr;
  const uint8_t* k8 = nullptr;
  const float* q_scale = nullptr;
  const float* k_scale = nullptr;
};
// Returns BSA_OK / BSA_ECUDA (tensor-map encoding or launch failure).
// blk = 128: persistent one-tile-per-step kernel (attention_tile.cu);
// blk = 64: paired-tile kernel over the union of kept lists (attention.cu).
int launch_sparse_attn(const bsa_shape& s, const AttnArgs& a, cudaStream_t st);
int launch_sparse_attn_pair(const bsa_shape& s, const AttnArgs& a, cudaStream_t st);
int launch_sparse_attn_tile(const bsa_shape& s, const AttnArgs& a, cudaStream_t st);

}  // namespace bsa
