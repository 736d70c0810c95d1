// extern "C" entry points of libbsa (declared in include/bsa.h): host-side
// argument validation, then one or two kernel launches on the caller's
// stream.  Nothing here allocates, frees or synchronises.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "internal.cuh"

namespace {

using bsa::n_blocks;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// A 32-bit word the device reads or updates atomically (status, alpha):
// null is allowed here, the callers decide whether it is required.
bool word_ok(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int check_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ENODEV;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return BSA_ENODEV;
  return major == 10 ? BSA_OK : BSA_ENODEV;
}

// Shape rules shared by the block-level calls.
int check_block_shape(const bsa_shape& s) {
  if (s.B < 1 || s.H < 1 || s.L < 1) return BSA_ESHAPE;
  if (s.D != 64 && s.D != 128) return BSA_ESHAPE;
  if (s.blk != 64 && s.blk != 128) return BSA_ESHAPE;
  if (n_blocks(s.L, s.blk) > bsa::kMaxNB) return BSA_ESHAPE;
  if (static_cast<long long>(s.B) * s.H > 65535) return BSA_ESHAPE;
  const double elems = static_cast<double>(s.B) * s.H * s.L * s.D;
  if (elems >= 1099511627776.0) return BSA_ESHAPE;  // 2^40
  return BSA_OK;
}

// Shape rules of the elementwise calls (any D that is a multiple of 8).
int check_rows_shape(const bsa_shape& s) {
  if (s.B < 1 || s.H < 1 || s.L < 1 || s.D < 8 || (s.D % 8) != 0) return BSA_ESHAPE;
  const double elems = static_cast<double>(s.B) * s.H * s.L * s.D;
  if (elems >= 1099511627776.0) return BSA_ESHAPE;
  return BSA_OK;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ECUDA; }

}  // namespace

extern "C" {

const char* bsa_strerror(int status) {
  switch (status) {
    case BSA_OK: return "ok";
    case BSA_EINVAL: return "invalid argument (null or misaligned pointer, or value out of range)";
    case BSA_ESHAPE: return "unsupported or inconsistent shape";
    case BSA_ENODEV: return "no sm_100 CUDA device is current";
    case BSA_ECUDA: return "CUDA launch or driver call failed";
    case BSA_EWORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int bsa_version(void) { return 10000; }

int bsa_score_blocks(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, float* q_pool, float* k_pool, float* probs,
                     bsa_stream stream) {
  if (!q || !k || !q_pool || !k_pool || !probs) return BSA_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_pool) || !aligned16(k_pool) || !aligned16(probs))
    return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (int r = check_device()) return r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const auto* qb = reinterpret_cast<const __nv_bfloat16*>(q);
  const auto* kb = reinterpret_cast<const __nv_bfloat16*>(k);
  if (cudaError_t e = bsa::launch_pool(s, qb, kb, q_pool, k_pool, st)) return from_cuda(e);
  return from_cuda(bsa::launch_block_softmax(s, q_pool, k_pool, probs, nullptr, st));
}

int bsa_score_blocks_restricted(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const uint8_t* candidates,
                                float* q_pool, float* k_pool, float* probs, bsa_stream stream) {
  if (!q || !k || !candidates || !q_pool || !k_pool || !probs) return BSA_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(candidates) || !aligned16(q_pool) || !aligned16(k_pool) ||
      !aligned16(probs))
    return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (int r = check_device()) return r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const auto* qb = reinterpret_cast<const __nv_bfloat16*>(q);
  const auto* kb = reinterpret_cast<const __nv_bfloat16*>(k);
  if (cudaError_t e = bsa::launch_pool(s, qb, kb, q_pool, k_pool, st)) return from_cuda(e);
  return from_cuda(bsa::launch_block_softmax(s, q_pool, k_pool, probs, candidates, st));
}

int bsa_score_blocks_gather(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const int32_t* perm, bsa_bf16* q_out,
                            bsa_bf16* k_out, float* q_pool, float* k_pool, float* probs, bsa_stream stream) {
  if (!q || !k || !perm || !q_pool || !k_pool || !probs) return BSA_EINVAL;
  if ((q_out == nullptr) != (k_out == nullptr)) return BSA_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(perm) || (q_out && !aligned16(q_out)) ||
      (k_out && !aligned16(k_out)) || !aligned16(q_pool) || !aligned16(k_pool) || !aligned16(probs))
    return BSA_EINVAL;
  if (q_out && (q_out == q || q_out == k || k_out == q || k_out == k || q_out == k_out)) return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (int r = check_device()) return r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaError_t e = bsa::launch_pool(s, reinterpret_cast<const __nv_bfloat16*>(q),
                                       reinterpret_cast<const __nv_bfloat16*>(k), q_pool, k_pool, st, perm,
                                       reinterpret_cast<__nv_bfloat16*>(q_out), reinterpret_cast<__nv_bfloat16*>(k_out)))
    return from_cuda(e);
  return from_cuda(bsa::launch_block_softmax(s, q_pool, k_pool, probs, nullptr, st));
}

int bsa_block_drift(bsa_shape s, const float* q_pool_ref, const float* k_pool_ref, const float* q_pool,
                    const float* k_pool, float* drift, bsa_stream stream) {
  if (!q_pool_ref || !k_pool_ref || !q_pool || !k_pool || !drift) return BSA_EINVAL;
  if (!aligned16(q_pool_ref) || !aligned16(k_pool_ref) || !aligned16(q_pool) || !aligned16(k_pool) ||
      !aligned16(drift))
    return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (int r = check_device()) return r;
  return from_cuda(bsa::launch_drift(s, q_pool_ref, k_pool_ref, q_pool, k_pool, drift,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

namespace {
int select_common(bsa_shape s, const float* probs, const float* p_host, const uint8_t* cand, uint8_t* mask,
                  int32_t* kept_idx, int32_t* kept_cnt, bsa_stream stream) {
  if (!probs || !p_host || !mask || !kept_idx || !kept_cnt) return BSA_EINVAL;
  if (!aligned16(probs) || !aligned16(mask) || !aligned16(kept_idx) || !aligned16(kept_cnt)) return BSA_EINVAL;
  if (cand && !aligned16(cand)) return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (s.H > bsa::kMaxHeadsP) return BSA_ESHAPE;
  bsa::TopP tp;
  for (int h = 0; h < bsa::kMaxHeadsP; ++h) tp.p[h] = 1.0f;
  for (int h = 0; h < s.H; ++h) {
    const float p = p_host[h];
    if (!(p > 0.0f) || !(p <= 1.0f)) return BSA_EINVAL;  // rejects NaN too
    tp.p[h] = p;
  }
  if (int r = check_device()) return r;
  return from_cuda(
      bsa::launch_select(s, probs, tp, cand, mask, kept_idx, kept_cnt, reinterpret_cast<cudaStream_t>(stream)));
}
}  // namespace

int bsa_select_topp_mask(bsa_shape s, const float* probs, const float* p_host, uint8_t* mask, int32_t* kept_idx,
                         int32_t* kept_cnt, bsa_stream stream) {
  return select_common(s, probs, p_host, nullptr, mask, kept_idx, kept_cnt, stream);
}

int bsa_select_topp_mask_restricted(bsa_shape s, const float* probs, const float* p_host, const uint8_t* candidates,
                                    uint8_t* mask, int32_t* kept_idx, int32_t* kept_cnt, bsa_stream stream) {
  if (!candidates) return BSA_EINVAL;
  return select_common(s, probs, p_host, candidates, mask, kept_idx, kept_cnt, stream);
}

int bsa_interval_runs(bsa_shape s, const int32_t* kept_idx, const int32_t* kept_cnt, int32_t* n_runs, int32_t* hist,
                      int32_t* status, bsa_stream stream) {
  if (!kept_idx || !kept_cnt || !n_runs) return BSA_EINVAL;
  if (!aligned16(kept_idx) || !aligned16(kept_cnt) || !aligned16(n_runs) || (hist && !aligned16(hist)))
    return BSA_EINVAL;
  if (!word_ok(status)) return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (int r = check_device()) return r;
  return from_cuda(bsa::launch_interval_encode(s, kept_idx, kept_cnt, 0, nullptr, nullptr, n_runs, hist, status,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

int bsa_interval_width_for_merge(const int32_t* hist_host, int nbins, double q, int* W_out) {
  if (!hist_host || !W_out || nbins < 2) return BSA_EINVAL;
  if (!(q > 0.0) || !(q <= 1.0)) return BSA_EINVAL;  // rejects NaN too
  long long rows = 0;
  for (int r = 0; r < nbins; ++r) {
    if (hist_host[r] < 0) return BSA_EINVAL;
    rows += hist_host[r];
  }
  const double need = std::ceil(q * static_cast<double>(rows));
  long long covered = hist_host[0];
  int W = nbins - 1;
  for (int w = 1; w < nbins; ++w) {
    covered += hist_host[w];
    if (static_cast<double>(covered) >= need) {
      W = w;
      break;
    }
  }
  *W_out = W;
  return BSA_OK;
}

int bsa_kept_to_intervals(bsa_shape s, const int32_t* kept_idx, const int32_t* kept_cnt, int W, int32_t* intervals,
                          int32_t* n_int, int32_t* n_runs, int32_t* status, bsa_stream stream) {
  if (!kept_idx || !kept_cnt || !intervals || !n_int) return BSA_EINVAL;
  if (!aligned16(kept_idx) || !aligned16(kept_cnt) || !aligned16(intervals) || !aligned16(n_int) ||
      (n_runs && !aligned16(n_runs)) || !word_ok(status))
    return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (W < 1 || W > n_blocks(s.L, s.blk)) return BSA_EINVAL;
  if (int r = check_device()) return r;
  return from_cuda(bsa::launch_interval_encode(s, kept_idx, kept_cnt, W, intervals, n_int, n_runs, nullptr, status,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

int bsa_intervals_to_kept(bsa_shape s, const int32_t* intervals, const int32_t* n_int, int W, uint8_t* mask,
                          int32_t* kept_idx, int32_t* kept_cnt, int32_t* status, bsa_stream stream) {
  if (!intervals || !n_int || !kept_idx || !kept_cnt) return BSA_EINVAL;
  if (!aligned16(intervals) || !aligned16(n_int) || !aligned16(kept_idx) || !aligned16(kept_cnt) ||
      (mask && !aligned16(mask)) || !word_ok(status))
    return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (W < 1 || W > n_blocks(s.L, s.blk)) return BSA_EINVAL;
  if (int r = check_device()) return r;
  return from_cuda(bsa::launch_interval_decode(s, intervals, n_int, W, mask, kept_idx, kept_cnt, status,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

size_t bsa_tail_workspace_bytes(bsa_shape s) {
  if (check_block_shape(s) != BSA_OK || s.D != 128) return 0;
  return bsa::tail_workspace_bytes(s);
}

int bsa_tail_stats(bsa_shape s, const bsa_bf16* k, const bsa_bf16* v, float* kbar, float* s2, float* vbar, float* C,
                   void* ws, size_t ws_bytes, int32_t* status, bsa_stream stream) {
  if (!k || !v || !kbar || !s2 || !vbar || !C) return BSA_EINVAL;
  if (!aligned16(k) || !aligned16(v) || !aligned16(kbar) || !aligned16(s2) || !aligned16(vbar) || !aligned16(C) ||
      !word_ok(status))
    return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (s.D != 128) return BSA_ESHAPE;
  if (!ws || ws_bytes < bsa::tail_workspace_bytes(s)) return BSA_EWORKSPACE;
  if (!aligned16(ws)) return BSA_EINVAL;
  if (int r = check_device()) return r;
  return bsa::launch_tail_stats(s, reinterpret_cast<const __nv_bfloat16*>(k), reinterpret_cast<const __nv_bfloat16*>(v),
                                kbar, s2, vbar, C, ws, status, reinterpret_cast<cudaStream_t>(stream));
}

int bsa_coarse_tail(bsa_shape s, const bsa_bf16* q, const uint8_t* mask, const void* ws, size_t ws_bytes, float* lbar,
                    bsa_bf16* obar, int32_t* status, bsa_stream stream) {
  if (!q || !mask || !lbar || !obar) return BSA_EINVAL;
  if (!aligned16(q) || !aligned16(mask) || !aligned16(lbar) || !aligned16(obar) || !word_ok(status))
    return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (s.D != 128 || s.blk != 128) return BSA_ESHAPE;
  if (!ws || ws_bytes < bsa::tail_workspace_bytes(s)) return BSA_EWORKSPACE;
  if (!aligned16(ws)) return BSA_EINVAL;
  if (int r = check_device()) return r;
  return bsa::launch_coarse_tail(s, reinterpret_cast<const __nv_bfloat16*>(q), mask, ws, lbar,
                                 reinterpret_cast<__nv_bfloat16*>(obar), status, reinterpret_cast<cudaStream_t>(stream));
}

int bsa_tail_refinement(bsa_shape s, const float* l_T, const bsa_bf16* o_T, const float* lbar, const bsa_bf16* obar,
                        float* d_l, bsa_bf16* d_o, bsa_stream stream) {
  if (!l_T || !o_T || !lbar || !obar || !d_l || !d_o) return BSA_EINVAL;
  if (!aligned16(l_T) || !aligned16(o_T) || !aligned16(lbar) || !aligned16(obar) || !aligned16(d_l) ||
      !aligned16(d_o))
    return BSA_EINVAL;
  if (int r = check_rows_shape(s)) return r;
  if (int r = check_device()) return r;
  return bsa::launch_tail_refine(s, l_T, reinterpret_cast<const __nv_bfloat16*>(o_T), lbar,
                                 reinterpret_cast<const __nv_bfloat16*>(obar), d_l,
                                 reinterpret_cast<__nv_bfloat16*>(d_o), reinterpret_cast<cudaStream_t>(stream));
}

int bsa_tail_reconstruct(bsa_shape s, const float* l_S, const bsa_bf16* o_S, const float* lbar, const bsa_bf16* obar,
                         const float* d_l, const bsa_bf16* d_o, bsa_bf16* o, float* lse, bsa_stream stream) {
  if (!l_S || !o_S || !lbar || !obar || !d_l || !d_o || !o || !lse) return BSA_EINVAL;
  if (!aligned16(l_S) || !aligned16(o_S) || !aligned16(lbar) || !aligned16(obar) || !aligned16(d_l) ||
      !aligned16(d_o) || !aligned16(o) || !aligned16(lse))
    return BSA_EINVAL;
  if (int r = check_rows_shape(s)) return r;
  if (int r = check_device()) return r;
  return bsa::launch_tail_merge(s, l_S, reinterpret_cast<const __nv_bfloat16*>(o_S), lbar,
                                reinterpret_cast<const __nv_bfloat16*>(obar), d_l,
                                reinterpret_cast<const __nv_bfloat16*>(d_o), reinterpret_cast<__nv_bfloat16*>(o), lse,
                                reinterpret_cast<cudaStream_t>(stream));
}

int bsa_complement_lists(bsa_shape s, const uint8_t* mask, int32_t* idx, int32_t* cnt, bsa_stream stream) {
  if (!mask || !idx || !cnt) return BSA_EINVAL;
  if (!aligned16(mask) || !aligned16(idx) || !aligned16(cnt)) return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (int r = check_device()) return r;
  return bsa::launch_complement(s, mask, idx, cnt, reinterpret_cast<cudaStream_t>(stream));
}

int bsa_wait_selftest(int32_t* status, unsigned long long limit_ns, bsa_stream stream) {
  if (!status || !word_ok(status)) return BSA_EINVAL;
  if (limit_ns == 0 || limit_ns > 2000000000ull) return BSA_EINVAL;
  if (int r = check_device()) return r;
  return from_cuda(bsa::launch_wait_selftest(status, limit_ns, reinterpret_cast<cudaStream_t>(stream)));
}

size_t bsa_reorder_workspace_bytes(int T, int Hh, int W) { return bsa::hilbert_workspace_bytes(T, Hh, W); }

int bsa_reorder_tokens(int T, int Hh, int W, int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes,
                       bsa_stream stream) {
  if (!perm || !inv) return BSA_EINVAL;
  const size_t need = bsa::hilbert_workspace_bytes(T, Hh, W);
  if (need == 0) return BSA_ESHAPE;
  if (!ws || ws_bytes < need) return BSA_EWORKSPACE;
  if (!aligned16(perm) || !aligned16(inv) || !aligned16(ws)) return BSA_EINVAL;
  if (int r = check_device()) return r;
  return from_cuda(bsa::launch_hilbert(T, Hh, W, perm, inv, ws, reinterpret_cast<cudaStream_t>(stream)));
}

int bsa_permute_tokens(bsa_shape s, const bsa_bf16* x, const int32_t* perm, bsa_bf16* y, int inverse,
                       bsa_stream stream) {
  if (!x || !perm || !y) return BSA_EINVAL;
  if (!aligned16(x) || !aligned16(y) || !aligned16(perm)) return BSA_EINVAL;
  if (x == y) return BSA_EINVAL;
  if (int r = check_rows_shape(s)) return r;
  if (int r = check_device()) return r;
  return from_cuda(bsa::launch_permute(s, reinterpret_cast<const __nv_bfloat16*>(x), perm,
                                       reinterpret_cast<__nv_bfloat16*>(y), inverse,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

int bsa_sparse_attn_fwd_scatter(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const bsa_bf16* v,
                                const int32_t* kept_idx, const int32_t* kept_cnt, const bsa_bf16* R,
                                const float* alpha, const int32_t* out_rows, bsa_bf16* o, float* lse,
                                int32_t* status, bsa_stream stream);

int bsa_sparse_attn_fwd(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const bsa_bf16* v, const int32_t* kept_idx,
                        const int32_t* kept_cnt, const bsa_bf16* R, const float* alpha, bsa_bf16* o, float* lse,
                        int32_t* status, bsa_stream stream) {
  return bsa_sparse_attn_fwd_scatter(s, q, k, v, kept_idx, kept_cnt, R, alpha, nullptr, o, lse, status, stream);
}

int bsa_sparse_attn_fwd_scatter(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const bsa_bf16* v,
                                const int32_t* kept_idx, const int32_t* kept_cnt, const bsa_bf16* R,
                                const float* alpha, const int32_t* out_rows, bsa_bf16* o, float* lse,
                                int32_t* status, bsa_stream stream) {
  if (!q || !k || !v || !o || !lse) return BSA_EINVAL;
  if ((kept_idx == nullptr) != (kept_cnt == nullptr)) return BSA_EINVAL;
  if ((R == nullptr) != (alpha == nullptr)) return BSA_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return BSA_EINVAL;
  if ((kept_idx && !aligned16(kept_idx)) || (kept_cnt && !aligned16(kept_cnt)) || (R && !aligned16(R)))
    return BSA_EINVAL;
  if (out_rows && !aligned16(out_rows)) return BSA_EINVAL;
  if (!word_ok(status) || !word_ok(alpha)) return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (out_rows && s.blk != 128) return BSA_ESHAPE;
  if (int r = check_device()) return r;
  bsa::AttnArgs a;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.k = reinterpret_cast<const __nv_bfloat16*>(k);
  a.v = reinterpret_cast<const __nv_bfloat16*>(v);
  a.kept_idx = kept_idx;
  a.kept_cnt = kept_cnt;
  a.R = reinterpret_cast<const __nv_bfloat16*>(R);
  a.alpha = alpha;
  a.o = reinterpret_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.status = status;
  a.out_rows = out_rows;
  return bsa::launch_sparse_attn(s, a, reinterpret_cast<cudaStream_t>(stream));
}

int bsa_sparse_attn_fwd_gather(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const bsa_bf16* v,
                               const int32_t* rows, const int32_t* kept_idx, const int32_t* kept_cnt,
                               const bsa_bf16* R, const float* alpha, bsa_bf16* o, float* lse, int32_t* status,
                               bsa_stream stream) {
  if (!q || !k || !v || !rows || !o || !lse) return BSA_EINVAL;
  if ((kept_idx == nullptr) != (kept_cnt == nullptr)) return BSA_EINVAL;
  if ((R == nullptr) != (alpha == nullptr)) return BSA_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(rows))
    return BSA_EINVAL;
  if ((kept_idx && !aligned16(kept_idx)) || (kept_cnt && !aligned16(kept_cnt)) || (R && !aligned16(R)))
    return BSA_EINVAL;
  if (!word_ok(status) || !word_ok(alpha)) return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (s.blk != 128 || s.D != 128) return BSA_ESHAPE;
  if (static_cast<long long>(s.B) * s.H * s.L >= (1ll << 31)) return BSA_ESHAPE;
  if (int r = check_device()) return r;
  bsa::AttnArgs a;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.k = reinterpret_cast<const __nv_bfloat16*>(k);
  a.v = reinterpret_cast<const __nv_bfloat16*>(v);
  a.kept_idx = kept_idx;
  a.kept_cnt = kept_cnt;
  a.R = reinterpret_cast<const __nv_bfloat16*>(R);
  a.alpha = alpha;
  a.o = reinterpret_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.status = status;
  a.in_rows = rows;
  a.out_rows = rows;
  return bsa::launch_sparse_attn(s, a, reinterpret_cast<cudaStream_t>(stream));
}

int bsa_sparse_attn_fwd_intervals(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const bsa_bf16* v,
                                  const int32_t* intervals, const int32_t* n_int, int W, const bsa_bf16* R,
                                  const float* alpha, bsa_bf16* o, float* lse, int32_t* status, bsa_stream stream) {
  if (!q || !k || !v || !intervals || !n_int || !o || !lse) return BSA_EINVAL;
  if ((R == nullptr) != (alpha == nullptr)) return BSA_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return BSA_EINVAL;
  if (!word_ok(intervals) || !word_ok(n_int) || (R && !aligned16(R))) return BSA_EINVAL;
  if (!word_ok(status) || !word_ok(alpha)) return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (s.blk != 128) return BSA_ESHAPE;
  if (W < 1 || W > n_blocks(s.L, s.blk)) return BSA_EINVAL;
  if (int r = check_device()) return r;
  bsa::AttnArgs a;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.k = reinterpret_cast<const __nv_bfloat16*>(k);
  a.v = reinterpret_cast<const __nv_bfloat16*>(v);
  a.kept_idx = nullptr;
  a.kept_cnt = nullptr;
  a.intervals = intervals;
  a.n_int = n_int;
  a.W = W;
  a.R = reinterpret_cast<const __nv_bfloat16*>(R);
  a.alpha = alpha;
  a.o = reinterpret_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.status = status;
  return bsa::launch_sparse_attn(s, a, reinterpret_cast<cudaStream_t>(stream));
}

int bsa_quantize_fp8(bsa_shape s, const bsa_bf16* x, uint8_t* codes, float* scales, bsa_stream stream) {
  if (!x || !codes || !scales) return BSA_EINVAL;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (int r = check_device()) return r;
  return from_cuda(bsa::launch_quantize_fp8(s, reinterpret_cast<const __nv_bfloat16*>(x), codes, scales,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

int bsa_sparse_attn_fwd_fp8(bsa_shape s, const uint8_t* q8, const float* q_scale, const uint8_t* k8,
                            const float* k_scale, const bsa_bf16* v, const int32_t* kept_idx, const int32_t* kept_cnt,
                            const bsa_bf16* R, const float* alpha, bsa_bf16* o, float* lse, int32_t* status,
                            bsa_stream stream) {
  if (!q8 || !q_scale || !k8 || !k_scale || !v || !o || !lse) return BSA_EINVAL;
  if ((kept_idx == nullptr) != (kept_cnt == nullptr)) return BSA_EINVAL;
  if ((R == nullptr) != (alpha == nullptr)) return BSA_EINVAL;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return BSA_EINVAL;
  if ((kept_idx && !aligned16(kept_idx)) || (kept_cnt && !aligned16(kept_cnt)) || (R && !aligned16(R)))
    return BSA_EINVAL;
  if (!word_ok(q_scale) || !word_ok(k_scale) || !word_ok(status) || !word_ok(alpha)) return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (s.blk != 128 || s.D != 128) return BSA_ESHAPE;
  if (int r = check_device()) return r;
  bsa::AttnArgs a;
  a.q = nullptr;
  a.k = nullptr;
  a.v = reinterpret_cast<const __nv_bfloat16*>(v);
  a.kept_idx = kept_idx;
  a.kept_cnt = kept_cnt;
  a.R = reinterpret_cast<const __nv_bfloat16*>(R);
  a.alpha = alpha;
  a.o = reinterpret_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.status = status;
  a.q8 = q8;
  a.k8 = k8;
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  return bsa::launch_sparse_attn(s, a, reinterpret_cast<cudaStream_t>(stream));
}

int bsa_sparse_attn_refresh(bsa_shape s, const bsa_bf16* q, const bsa_bf16* k, const bsa_bf16* v,
                            const int32_t* kept_idx, const int32_t* kept_cnt, bsa_bf16* o_dense, float* lse_dense,
                            bsa_bf16* o_sparse, float* lse_sparse, bsa_bf16* R, float* kept_mass, int32_t* status,
                            bsa_stream stream) {
  if (!q || !k || !v || !kept_idx || !kept_cnt || !o_dense || !lse_dense || !o_sparse || !lse_sparse)
    return BSA_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(kept_idx) || !aligned16(kept_cnt) ||
      !aligned16(o_dense) || !aligned16(lse_dense) || !aligned16(o_sparse) || !aligned16(lse_sparse))
    return BSA_EINVAL;
  if ((R && !aligned16(R)) || (kept_mass && !aligned16(kept_mass))) return BSA_EINVAL;
  if (!word_ok(status)) return BSA_EINVAL;
  if (int r = check_block_shape(s)) return r;
  if (s.blk != 128) return BSA_ESHAPE;
  if (int r = check_device()) return r;
  bsa::AttnArgs a;
  a.q = reinterpret_cast<const __nv_bfloat16*>(q);
  a.k = reinterpret_cast<const __nv_bfloat16*>(k);
  a.v = reinterpret_cast<const __nv_bfloat16*>(v);
  a.kept_idx = kept_idx;
  a.kept_cnt = kept_cnt;
  a.R = nullptr;
  a.alpha = nullptr;
  a.o = reinterpret_cast<__nv_bfloat16*>(o_dense);
  a.lse = lse_dense;
  a.status = status;
  a.o2 = reinterpret_cast<__nv_bfloat16*>(o_sparse);
  a.lse2 = lse_sparse;
  a.r_out = reinterpret_cast<__nv_bfloat16*>(R);
  a.mass = kept_mass;
  return bsa::launch_sparse_attn(s, a, reinterpret_cast<cudaStream_t>(stream));
}

int bsa_refresh_refinement(bsa_shape s, const bsa_bf16* o_dense, const bsa_bf16* o_sparse, bsa_bf16* R,
                           bsa_stream stream) {
  if (!o_dense || !o_sparse || !R) return BSA_EINVAL;
  if (!aligned16(o_dense) || !aligned16(o_sparse) || !aligned16(R)) return BSA_EINVAL;
  if (int r = check_rows_shape(s)) return r;
  if (int r = check_device()) return r;
  const size_t n = static_cast<size_t>(s.B) * s.H * s.L * s.D;
  return from_cuda(bsa::launch_refresh(n, reinterpret_cast<const __nv_bfloat16*>(o_dense),
                                       reinterpret_cast<const __nv_bfloat16*>(o_sparse),
                                       reinterpret_cast<__nv_bfloat16*>(R), reinterpret_cast<cudaStream_t>(stream)));
}

int bsa_apply_correction(bsa_shape s, const bsa_bf16* o_sparse, const bsa_bf16* R, const float* alpha, bsa_bf16* o,
                         bsa_stream stream) {
  if (!o_sparse || !R || !alpha || !o) return BSA_EINVAL;
  if (!aligned16(o_sparse) || !aligned16(R) || !aligned16(o) || !word_ok(alpha)) return BSA_EINVAL;
  if (int r = check_rows_shape(s)) return r;
  if (int r = check_device()) return r;
  return from_cuda(bsa::launch_correct(s, reinterpret_cast<const __nv_bfloat16*>(o_sparse),
                                       reinterpret_cast<const __nv_bfloat16*>(R), alpha,
                                       reinterpret_cast<__nv_bfloat16*>(o), reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
