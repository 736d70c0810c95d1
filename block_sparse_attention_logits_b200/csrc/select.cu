// Cumulative top-p block selection (head-wise top-p abstract: per-head top-p
// thresholds; GSRS abstract: top-p selection for adaptive sparsity; CalibAtt
// Fig. 5: threshold the top key blocks per query block).
//
// Per row: key_j = float32 bits of clamp(P_j, 0, 1) (order-preserving for
// non-negative floats), u_j = floor(P_j * 2^40) computed exactly from the
// exponent and mantissa, T = ceil(p * sum u) in IEEE double.  The kept set is
// the shortest prefix of the (P desc, index asc) order whose u-sum is >= T.
//
// No sort is needed.  One warp per row finds, by a bitwise search (at most
// 29 steps: the top bits are known), the largest key threshold tau with
// sum_{key >= tau} u >= T.  Every block with key > tau is kept; blocks with
// key == tau are kept in ascending index order while the running mass is
// still below T (a warp prefix scan).  Every decision rests on exact integer
// sums, so the result does not depend on the order of summation and equals
// the sequential definition bit for bit.  Rows of up to 1024 blocks keep
// their keys in registers (select_reg_kernel), which also decides most search
// steps on 32-bit coarse masses and stops the search as soon as a single key
// value is left in play; longer rows stage keys and masses in shared memory.
//
// Restricted form (GSRS abstract: later searches restricted to an early
// candidate set): with a candidate mask the search runs over the candidate
// blocks only -- the others carry key 0 and mass 0 and are never kept, the
// target is p times the candidates' mass, p = 1 keeps every candidate.
#include "internal.cuh"

namespace bsa {
namespace {

constexpr uint32_t kSelected = 0xFFFFFFFFu;  // marker: above every real key
// With T > 0 the threshold is the key of a block with mass, P >= 2^-40
// (key >= 0x2B800000), and no key exceeds 1.0f (0x3F800000): bit 30 of tau is
// 0 and bit 29 is 1, so the search starts at bit 28
constexpr uint32_t kTopBits = 0x20000000u;
constexpr uint32_t kMinMassKey = 0x2B800000u;  // smallest key with u > 0 (P = 2^-40)
// coarse mass a = floor(P * 2^21) = u >> kCoarseShift: a row of at most 1024
// blocks sums to below 2^31, one 32-bit redux
constexpr int kCoarseShift = 19;

__device__ __forceinline__ uint32_t prob_key(float p) {
  // NaN and p <= 0 (incl. -0) -> 0; p > 1 (incl. inf) -> bits of 1.0f
  if (!(p > 0.f)) return 0u;
  if (p > 1.f) p = 1.f;
  return __float_as_uint(p);
}

// floor(P * 2^40) for P given by its (non-negative, <= 1.0) float32 bits.
__device__ __forceinline__ uint64_t fixed_mass(uint32_t key) {
  const int e = static_cast<int>(key >> 23);  // biased exponent
  if (e == 0) return 0ull;                    // zero or subnormal (< 2^-126)
  const uint64_t m = (key & 0x7FFFFFu) | 0x800000u;  // 24-bit significand
  // P * 2^40 = m * 2^(e - 127 - 23 + 40) = m * 2^(e - 110)
  const int sh = e - 110;
  if (sh >= 0) return m << sh;  // e <= 127 -> sh <= 17: fits
  return (-sh >= 24) ? 0ull : (m >> (-sh));
}

// floor(P * 2^21) = floor(floor(P * 2^40) / 2^19), from the same bits:
// m * 2^(e - 129), at most 2^21 (P = 1).
__device__ __forceinline__ uint32_t coarse_mass(uint32_t key) {
  const int e = static_cast<int>(key >> 23);
  if (e == 0) return 0u;
  const uint32_t m = (key & 0x7FFFFFu) | 0x800000u;
  const int sh = 129 - e;  // >= 2 for e <= 127
  return sh >= 24 ? 0u : (m >> sh);
}

// Exact warp sum of per-lane masses below 2^53 (a row's total is at most
// 2^52): three 21-bit limbs, each summed by one redux over 32 lanes (limb sums
// stay below 2^26), then recombined.
__device__ __forceinline__ uint64_t warp_sum(uint64_t v) {
  const uint32_t l0 = static_cast<uint32_t>(v) & 0x1FFFFFu;
  const uint32_t l1 = static_cast<uint32_t>(v >> 21) & 0x1FFFFFu;
  const uint32_t l2 = static_cast<uint32_t>(v >> 42);
  const uint64_t s0 = __reduce_add_sync(0xffffffffu, l0);
  const uint64_t s1 = __reduce_add_sync(0xffffffffu, l1);
  const uint64_t s2 = __reduce_add_sync(0xffffffffu, l2);
  return s0 + (s1 << 21) + (s2 << 42);
}

__global__ void __launch_bounds__(256) select_kernel(const float* __restrict__ probs, const __grid_constant__ TopP tp,
                                                     const uint8_t* __restrict__ cand,
                                                     uint8_t* __restrict__ mask, int32_t* __restrict__ kept_idx,
                                                     int32_t* __restrict__ kept_cnt, int H, int NB, long long rows,
                                                     int nbp) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int warps = blockDim.x >> 5;
  const int w = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t* us = reinterpret_cast<uint64_t*>(smem) + static_cast<size_t>(w) * nbp;
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem + static_cast<size_t>(warps) * nbp * 8) + static_cast<size_t>(w) * nbp;
  const long long row = static_cast<long long>(blockIdx.x) * warps + w;
  if (row >= rows) return;
  const int h = static_cast<int>((row / NB) % H);
  const float p = tp.p[h];
  const float* P = probs + row * NB;
  uint8_t* mrow = mask + row * NB;
  int32_t* irow = kept_idx + row * NB;

  // candidates (optional): the other blocks are never kept; their key and
  // mass are 0, so the search and the target ignore them
  const uint8_t* crow = cand ? cand + row * NB : nullptr;
  if (p == 1.0f && !crow) {
    for (int j = lane; j < NB; j += 32) {
      mrow[j] = 1;
      irow[j] = j;
    }
    if (lane == 0) kept_cnt[row] = NB;
    return;
  }

  uint64_t total = 0;
  for (int j = lane; j < NB; j += 32) {
    const bool in = !crow || crow[j];
    const uint32_t key = in ? prob_key(__ldg(P + j)) : 0u;
    const uint64_t u = fixed_mass(key);
    keys[j] = key;
    us[j] = u;
    total += u;
  }
  total = warp_sum(total);
  __syncwarp();
  const uint64_t T = static_cast<uint64_t>(ceil(static_cast<double>(p) * static_cast<double>(total)));

  uint32_t tau;
  if (p == 1.0f) {
    // every candidate is kept
    for (int j = lane; j < NB; j += 32)
      if (crow[j]) keys[j] = kSelected;
    tau = kSelected - 1u;
  } else if (T == 0) {
    // nothing to reach: keep the first block of the order (max key, lowest
    // index) among the eligible blocks; none if there is no candidate
    uint32_t best_key = 0;
    int best_j = 0x7FFFFFFF;
    for (int j = lane; j < NB; j += 32) {
      const uint32_t kj = keys[j];
      if (crow && !crow[j]) continue;
      if (kj > best_key || (kj == best_key && j < best_j)) {
        best_key = kj;
        best_j = j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint32_t ok = __shfl_xor_sync(0xffffffffu, best_key, o);
      const int oj = __shfl_xor_sync(0xffffffffu, best_j, o);
      if (ok > best_key || (ok == best_key && oj < best_j)) {
        best_key = ok;
        best_j = oj;
      }
    }
    __syncwarp();
    if (lane == 0 && best_j < NB) keys[best_j] = kSelected;
    tau = kSelected - 1u;
  } else {
    // largest tau with sum_{key >= tau} u >= T; its top two bits are known
    tau = kTopBits;
    for (int b = 28; b >= 0; --b) {
      const uint32_t cand = tau | (1u << b);
      uint64_t g = 0;
      for (int j = lane; j < NB; j += 32) g += keys[j] >= cand ? us[j] : 0ull;
      if (warp_sum(g) >= T) tau = cand;
    }
    uint64_t above = 0;
    for (int j = lane; j < NB; j += 32) above += keys[j] > tau ? us[j] : 0ull;
    const uint64_t need = T - warp_sum(above);  // > 0 by maximality of tau
    // blocks equal to tau, in ascending index order, while mass is short
    uint64_t carry = 0;
    for (int base = 0; base < NB && carry < need; base += 32) {
      const int j = base + lane;
      const bool tie = j < NB && keys[j] == tau;
      const uint64_t val = tie ? us[j] : 0ull;
      uint64_t incl = val;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (tie && carry + (incl - val) < need) keys[j] = kSelected;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  __syncwarp();
  // emit mask and the ascending kept list
  int count = 0;
  for (int base = 0; base < NB; base += 32) {
    const int j = base + lane;
    const bool sel = j < NB && keys[j] > tau;
    if (j < NB) mrow[j] = sel ? 1 : 0;
    const uint32_t bal = __ballot_sync(0xffffffffu, sel);
    if (sel) irow[count + __popc(bal & ((1u << lane) - 1u))] = j;
    count += __popc(bal);
  }
  if (lane == 0) kept_cnt[row] = count;
}

// Register-resident form of select_kernel for NB <= 32 R: lane l holds the
// key and the coarse mass of blocks j = 32 r + l (r < R), so the search reads
// no shared memory (the shared-memory form re-reads the whole row at every
// step), and the exact masses are recomputed from the keys where needed.
// The same threshold and the same result bit for bit; fewer steps:
//   * step c is first decided on coarse masses: with A = sum_{key >= c} a,
//     the exact S(c) = sum_{key >= c} u lies in [A 2^19, (A + NB) 2^19), so
//     A 2^19 >= T means S(c) >= T and (A + NB) 2^19 <= T means S(c) < T;
//     only in between is the exact uint64 sum taken;
//   * after every odd bit from bit 15 down, the search stops when the
//     bracket [tau, tau + 2^b) holds a single key value k among the blocks
//     with mass: then S(k) = S(tau) >= T and S(k + 1) = S(tau + 2^b) < T,
//     so k is the threshold the remaining steps would reach;
//   * the tie scan runs only over register slots that hold a block equal to
//     tau.
// Three CTAs per SM up to 640 blocks a row (71 registers at R = 20).
template <int R>
__global__ void __launch_bounds__(256, R <= 20 ? 3 : 2)
    select_reg_kernel(const float* __restrict__ probs, const __grid_constant__ TopP tp,
                      const uint8_t* __restrict__ cand, uint8_t* __restrict__ mask, int32_t* __restrict__ kept_idx,
                      int32_t* __restrict__ kept_cnt, int H, int NB, long long rows) {
  const int warps = blockDim.x >> 5;
  const int w = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * warps + w;
  if (row >= rows) return;
  const int h = static_cast<int>((row / NB) % H);
  const float p = tp.p[h];
  const float* P = probs + row * NB;
  uint8_t* mrow = mask + row * NB;
  int32_t* irow = kept_idx + row * NB;
  const uint8_t* crow = cand ? cand + row * NB : nullptr;
  if (p == 1.0f && !crow) {
    for (int j = lane; j < NB; j += 32) {
      mrow[j] = 1;
      irow[j] = j;
    }
    if (lane == 0) kept_cnt[row] = NB;
    return;
  }

  // every load of the row in flight before the first use: the loads are
  // predicated on the bounds only, and the candidate bytes are applied after
  float pv[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int j = 32 * r + lane;
    pv[r] = j < NB ? __ldg(P + j) : 0.f;
  }
  if (crow) {
    uint8_t cv[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = 32 * r + lane;
      cv[r] = j < NB ? crow[j] : 0;
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (!cv[r]) pv[r] = 0.f;  // key 0, mass 0
  }
  uint32_t key[R];
  uint64_t total = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    key[r] = prob_key(pv[r]);
    total += fixed_mass(key[r]);
  }
  total = warp_sum(total);
  const uint64_t T = static_cast<uint64_t>(ceil(static_cast<double>(p) * static_cast<double>(total)));

  uint32_t tau;
  if (p == 1.0f) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = 32 * r + lane;
      if (j < NB && crow[j]) key[r] = kSelected;
    }
    tau = kSelected - 1u;
  } else if (T == 0) {
    uint32_t best_key = 0;
    int best_j = 0x7FFFFFFF;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = 32 * r + lane;
      if (j >= NB || (crow && !crow[j])) continue;
      if (key[r] > best_key || (key[r] == best_key && j < best_j)) {
        best_key = key[r];
        best_j = j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint32_t ok = __shfl_xor_sync(0xffffffffu, best_key, o);
      const int oj = __shfl_xor_sync(0xffffffffu, best_j, o);
      if (ok > best_key || (ok == best_key && oj < best_j)) {
        best_key = ok;
        best_j = oj;
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (32 * r + lane == best_j) key[r] = kSelected;
    tau = kSelected - 1u;
  } else {
    uint32_t a[R];
#pragma unroll
    for (int r = 0; r < R; ++r) a[r] = coarse_mass(key[r]);
    // largest tau with S(tau) = sum_{key >= tau} u >= T; its top two bits are
    // known.  Before bit b: S(tau) >= T > S(tau + 2^(b+1)).
    tau = kTopBits;
#pragma unroll 1
    for (int b = 28; b >= 0; --b) {
      const uint32_t c = tau | (1u << b);
      uint32_t g[4] = {0u, 0u, 0u, 0u};  // independent partial sums
#pragma unroll
      for (int r = 0; r < R; ++r) g[r & 3] += key[r] >= c ? a[r] : 0u;
      const uint64_t A = __reduce_add_sync(0xffffffffu, (g[0] + g[1]) + (g[2] + g[3]));
      bool ge = (A << kCoarseShift) >= T;
      if (!ge && ((A + static_cast<uint64_t>(NB)) << kCoarseShift) > T) {
        // undecided on coarse masses: the exact sum
        uint64_t e[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int r = 0; r < R; ++r) e[r & 3] += key[r] >= c ? fixed_mass(key[r]) : 0ull;
        ge = warp_sum((e[0] + e[1]) + (e[2] + e[3])) >= T;
      }
      if (ge) tau = c;
      if ((b & 1) && b <= 15) {
        // the bracket is now [tau, tau + 2^b); its keys with mass are >= kMinMassKey
        const uint32_t lo = tau > kMinMassKey ? tau : kMinMassKey;
        const uint32_t hi = tau + (1u << b);
        uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
        for (int r = 0; r < R; ++r)
          if (key[r] >= lo && key[r] < hi) {
            kmin = min(kmin, key[r]);
            kmax = max(kmax, key[r]);
          }
        kmin = __reduce_min_sync(0xffffffffu, kmin);
        kmax = __reduce_max_sync(0xffffffffu, kmax);
        if (kmin == kmax) {  // one key value left (an empty bracket gives kmin > kmax)
          tau = kmin;
          break;
        }
      }
    }
    uint64_t above = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) above += key[r] > tau ? fixed_mass(key[r]) : 0ull;
    const uint64_t need = T - warp_sum(above);  // > 0 by maximality of tau
    // blocks equal to tau, in ascending index order, while mass is short
    uint64_t carry = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = 32 * r + lane;
      const bool tie = j < NB && key[r] == tau;
      if (!__any_sync(0xffffffffu, tie)) continue;  // no block of this slot equals tau
      const uint64_t val = tie ? fixed_mass(key[r]) : 0ull;
      uint64_t incl = val;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (tie && carry + (incl - val) < need) key[r] = kSelected;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  // emit mask and the ascending kept list
  int count = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int j = 32 * r + lane;
    const bool sel = j < NB && key[r] > tau;
    if (j < NB) mrow[j] = sel ? 1 : 0;
    const unsigned bal = __ballot_sync(0xffffffffu, sel);
    if (sel) irow[count + __popc(bal & ((1u << lane) - 1u))] = j;
    count += __popc(bal);
  }
  if (lane == 0) kept_cnt[row] = count;
}

template <int R>
cudaError_t launch_select_reg(const float* probs, const TopP& p, const uint8_t* cand, uint8_t* mask, int32_t* idx,
                              int32_t* cnt, int H, int NB, long long rows, cudaStream_t st) {
  constexpr int kWarps = 8;
  const long long grid = (rows + kWarps - 1) / kWarps;
  select_reg_kernel<R><<<static_cast<unsigned>(grid), kWarps * 32, 0, st>>>(probs, p, cand, mask, idx, cnt, H, NB,
                                                                          rows);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const bsa_shape& s, const float* probs, const TopP& p, const uint8_t* cand, uint8_t* mask,
                          int32_t* idx, int32_t* cnt, cudaStream_t st) {
  const int NB = n_blocks(s.L, s.blk);
  const long long rows = static_cast<long long>(s.B) * s.H * NB;
  if (NB <= 32 * 8) return launch_select_reg<8>(probs, p, cand, mask, idx, cnt, s.H, NB, rows, st);
  if (NB <= 32 * 20) return launch_select_reg<20>(probs, p, cand, mask, idx, cnt, s.H, NB, rows, st);
  if (NB <= 32 * 32) return launch_select_reg<32>(probs, p, cand, mask, idx, cnt, s.H, NB, rows, st);
  const int nbp = (NB + 1) & ~1;
  const size_t per_warp = static_cast<size_t>(nbp) * 12;
  int warps = static_cast<int>((160 * 1024) / per_warp);
  if (warps > 8) warps = 8;
  if (warps < 1) warps = 1;
  const size_t smem = per_warp * warps;
  if (cudaError_t e = smem_opt_in(reinterpret_cast<const void*>(select_kernel), smem)) return e;
  const long long grid = (rows + warps - 1) / warps;
  select_kernel<<<static_cast<unsigned>(grid), warps * 32, smem, st>>>(probs, p, cand, mask, idx, cnt, s.H, NB, rows,
                                                                       nbp);
  return cudaGetLastError();
}

}  // namespace bsa
