// Interval (skip-list) form of the kept key blocks (CalibAtt appendix:
// Fig. S9, interval pairs per query-block row; Fig. S10, per-layer trimming
// to the widest row and merging of outlier rows; Table S3, "Merge %").
//
// A row's kept list (ascending block indices) is stored as the maximal runs
// of consecutive indices, each a pair (start, end) with end exclusive.  A row
// with more runs than the width W is merged: the gaps between neighbouring
// runs are filled smallest first (the leftmost of equal gaps first) until W
// intervals remain, so the row keeps a superset of its blocks with the fewest
// blocks added.
//
// One warp per row.  Run starts are found 32 entries at a time (entry t
// starts a run when idx[t] != idx[t-1] + 1) and compacted with a ballot into
// per-warp shared memory.  For a row over the width no sort is needed: the
// W-1 gaps that stay open are the largest ones, ties broken towards the
// right.  A bitwise search over gap sizes finds t*, the size of the (W-1)-th
// largest gap (the largest t with #{gap >= t} >= W-1); every gap above t*
// stays open, and of the gaps equal to t* the rightmost ones do, as many as
// are still missing.
#include "internal.cuh"

namespace bsa {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

__device__ __forceinline__ void flag(int32_t* status, int bits) {
  if (status) atomicOr(status, bits);
}

// kEncode = false: runs per row and their histogram only.
// kEncode = true:  intervals of width W (merging rows with more runs).
template <bool kEncode>
__global__ void __launch_bounds__(256) interval_encode_kernel(const int32_t* __restrict__ kept_idx,
                                                              const int32_t* __restrict__ kept_cnt, int NB,
                                                              long long rows, int W, int cap,
                                                              int32_t* __restrict__ intervals,
                                                              int32_t* __restrict__ n_int,
                                                              int32_t* __restrict__ n_runs,
                                                              int32_t* __restrict__ hist, int32_t* status) {
  extern __shared__ __align__(16) int32_t sh[];
  const int warps = blockDim.x >> 5;
  const int w = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * warps + w;
  if (row >= rows) return;
  int32_t* rs = sh + static_cast<size_t>(w) * 2 * cap;  // run starts
  int32_t* re = rs + cap;                                // run ends (exclusive)
  const int32_t* irow = kept_idx + row * NB;
  const unsigned lt = (1u << lane) - 1u;

  const int cnt = kept_cnt[row];
  bool bad = cnt < 0 || cnt > NB;
  int n = 0;
  int prev = -2;  // index of the previous entry; -2 makes entry 0 a run start
  if (!bad) {
    for (int base = 0; base < cnt; base += 32) {
      const int t = base + lane;
      const bool in = t < cnt;
      const int x = in ? irow[t] : 0;
      int xp = __shfl_up_sync(kFull, x, 1);
      if (lane == 0) xp = prev;
      const bool ok = !in || (x >= 0 && x < NB && x > xp);
      if (__any_sync(kFull, !ok)) {
        bad = true;
        break;
      }
      const bool start = in && x != xp + 1;
      const unsigned bal = __ballot_sync(kFull, start);
      if (kEncode && start) {
        const int pos = n + __popc(bal & lt);
        if (pos < cap) rs[pos] = x;
        if (pos > 0 && pos <= cap) re[pos - 1] = xp + 1;
      }
      n += __popc(bal);
      const int last = min(31, cnt - 1 - base);
      prev = __shfl_sync(kFull, x, last);
    }
  }
  if (bad) {
    if (lane == 0) {
      flag(status, BSA_DEV_BAD_INDEX);
      if (n_runs) n_runs[row] = 0;
      if (kEncode) n_int[row] = 0;
    }
    if (kEncode) {
      int32_t* out = intervals + row * 2 * W;
      for (int t = lane; t < 2 * W; t += 32) out[t] = -1;
    }
    return;
  }
  if (!kEncode) {
    if (lane == 0) {
      n_runs[row] = n;
      if (hist) atomicAdd(hist + n, 1);
    }
    return;
  }
  if (lane == 0) {
    if (n > 0) re[n - 1] = prev + 1;
    if (n_runs) n_runs[row] = n;
    n_int[row] = n < W ? n : W;
  }
  __syncwarp();
  int32_t* out = intervals + row * 2 * W;
  if (n <= W) {
    for (int t = lane; t < W; t += 32) {
      out[2 * t] = t < n ? rs[t] : -1;
      out[2 * t + 1] = t < n ? re[t] : -1;
    }
    return;
  }
  // n > W: keep the K = W - 1 largest gaps open (ties: the rightmost)
  const int K = W - 1;
  const int ng = n - 1;  // gap r lies between run r and run r + 1
  int tstar = 0;
  if (K > 0) {
#pragma unroll 1
    for (int b = 12; b >= 0; --b) {
      const int c = tstar | (1 << b);
      int k = 0;
      for (int r = lane; r < ng; r += 32) k += (rs[r + 1] - re[r]) >= c;
      if (warp_sum_i(k) >= K) tstar = c;
    }
  }
  int above = 0, ties = 0;
  for (int r = lane; r < ng; r += 32) {
    const int g = rs[r + 1] - re[r];
    above += g > tstar;
    ties += g == tstar;
  }
  above = warp_sum_i(above);
  ties = warp_sum_i(ties);
  const int need = K - above;  // open gaps still missing, taken among the ties
  if (lane == 0) {
    out[0] = rs[0];
    out[2 * K + 1] = re[n - 1];
  }
  if (K > 0) {
    int kept = 0, tie_seen = 0;
    for (int base = 0; base < ng; base += 32) {
      const int r = base + lane;
      const int g = r < ng ? rs[r + 1] - re[r] : -1;
      const bool tie = g == tstar;
      const unsigned tb = __ballot_sync(kFull, tie);
      const int tie_incl = tie_seen + __popc(tb & (lt | (1u << lane)));
      const bool open = r < ng && (g > tstar || (tie && ties - tie_incl < need));
      const unsigned ob = __ballot_sync(kFull, open);
      if (open) {
        const int m = kept + __popc(ob & lt);
        out[2 * m + 1] = re[r];
        out[2 * (m + 1)] = rs[r + 1];
      }
      kept += __popc(ob);
      tie_seen += __popc(tb);
    }
  }
}

// One warp per row: validate the row's pairs, then write its blocks, one
// interval at a time across the warp's lanes (coalesced).
__global__ void __launch_bounds__(256) interval_decode_kernel(const int32_t* __restrict__ intervals,
                                                              const int32_t* __restrict__ n_int, int NB,
                                                              long long rows, int W, uint8_t* __restrict__ mask,
                                                              int32_t* __restrict__ kept_idx,
                                                              int32_t* __restrict__ kept_cnt, int32_t* status) {
  const int warps = blockDim.x >> 5;
  const int w = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * warps + w;
  if (row >= rows) return;
  const int32_t* in = intervals + row * 2 * W;
  uint8_t* mrow = mask ? mask + row * NB : nullptr;
  int32_t* irow = kept_idx + row * NB;
  const int n = n_int[row];
  bool bad = n < 0 || n > W;
  int total = 0;
  if (!bad) {
    int carry = 0;  // end of the previous interval
    for (int base = 0; base < n; base += 32) {
      const int t = base + lane;
      const bool v = t < n;
      const int s = v ? in[2 * t] : 0;
      const int e = v ? in[2 * t + 1] : 0;
      int pe = __shfl_up_sync(kFull, e, 1);
      if (lane == 0) pe = carry;
      const bool ok = !v || (s >= pe && s < e && e <= NB);
      if (__any_sync(kFull, !ok)) {
        bad = true;
        break;
      }
      total += warp_sum_i(v ? e - s : 0);
      carry = __shfl_sync(kFull, e, min(31, n - 1 - base));
    }
  }
  if (mrow)
    for (int j = lane; j < NB; j += 32) mrow[j] = 0;
  if (bad) {
    if (lane == 0) {
      flag(status, BSA_DEV_BAD_INDEX);
      kept_cnt[row] = 0;
    }
    return;
  }
  __syncwarp();
  int off = 0;
  for (int base = 0; base < n; base += 32) {
    const int t = base + lane;
    const int s = t < n ? in[2 * t] : 0;
    const int e = t < n ? in[2 * t + 1] : 0;
    const int len = e - s;
    int incl = len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    const int my_off = off + incl - len;
    const int m = min(32, n - base);
    for (int k = 0; k < m; ++k) {
      const int sk = __shfl_sync(kFull, s, k);
      const int ek = __shfl_sync(kFull, e, k);
      const int ko = __shfl_sync(kFull, my_off, k);
      for (int j = sk + lane; j < ek; j += 32) {
        irow[ko + (j - sk)] = j;
        if (mrow) mrow[j] = 1;
      }
    }
    off += __shfl_sync(kFull, incl, 31);
  }
  if (lane == 0) kept_cnt[row] = total;
}

}  // namespace

int max_intervals(int NB) { return (NB + 1) / 2; }

cudaError_t launch_interval_encode(const bsa_shape& s, const int32_t* kept_idx, const int32_t* kept_cnt, int W,
                                   int32_t* intervals, int32_t* n_int, int32_t* n_runs, int32_t* hist,
                                   int32_t* status, cudaStream_t st) {
  const int NB = n_blocks(s.L, s.blk);
  const int cap = max_intervals(NB);
  const long long rows = static_cast<long long>(s.B) * s.H * NB;
  const int warps = 8;
  const long long grid = (rows + warps - 1) / warps;
  if (W == 0) {
    interval_encode_kernel<false><<<static_cast<unsigned>(grid), warps * 32, 0, st>>>(
        kept_idx, kept_cnt, NB, rows, 0, cap, nullptr, nullptr, n_runs, hist, status);
    return cudaGetLastError();
  }
  const size_t smem = static_cast<size_t>(warps) * 2 * cap * sizeof(int32_t);
  if (cudaError_t e = smem_opt_in(reinterpret_cast<const void*>(interval_encode_kernel<true>), smem)) return e;
  interval_encode_kernel<true><<<static_cast<unsigned>(grid), warps * 32, smem, st>>>(
      kept_idx, kept_cnt, NB, rows, W, cap, intervals, n_int, n_runs, nullptr, status);
  return cudaGetLastError();
}

cudaError_t launch_interval_decode(const bsa_shape& s, const int32_t* intervals, const int32_t* n_int, int W,
                                   uint8_t* mask, int32_t* kept_idx, int32_t* kept_cnt, int32_t* status,
                                   cudaStream_t st) {
  const int NB = n_blocks(s.L, s.blk);
  const long long rows = static_cast<long long>(s.B) * s.H * NB;
  const int warps = 8;
  const long long grid = (rows + warps - 1) / warps;
  interval_decode_kernel<<<static_cast<unsigned>(grid), warps * 32, 0, st>>>(intervals, n_int, NB, rows, W, mask,
                                                                            kept_idx, kept_cnt, status);
  return cudaGetLastError();
}

}  // namespace bsa
