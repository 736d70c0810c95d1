// Coarse estimate of the omitted attention tail and its reconstruction
// ("RECAP: Reciprocal Sparse Attention and Hierarchical Caching for Efficient
// Video Diffusion", section 3.2): block means of the keys and values give
// initial estimates of the omitted blocks' normalisation mass and value; the
// log-mass is refined by the key variance (second-order term), the value by
// the pooled value-key covariance (first-order term); a refinement cached at
// a dense refresh completes the fresh coarse estimate.
//
// Per head, with a = q / sqrt(D), omitted blocks T(i) of query block i:
//   coarse block log-mass  log n_j + a . kbar_j + 1/2 sum_d a_d^2 s2_j[d]
//   lbar = log sum_{j in T(i)} exp(block log-mass)
//   obar = sum_j w_j vbar_j + C a        (w_j the normalised block masses)
// with kbar_j, s2_j, vbar_j the block's key mean, per-dimension key variance
// and value mean, and C[e, d] = (1/L) sum over every token of
// (v - vbar_block)[e] (k - kbar_block)[d].
//
// Kernels:
//   tail_moments_kernel   one CTA per (head, block): means and variances, the
//                         bf16 operand tables of the tail kernel, and the
//                         block-centred keys and values ([L, D] per head, the
//                         layout of K and V) for the covariance contraction.
//   cov_kernel            C as a tensor-core contraction over the tokens:
//                         A = centred V^T, B = centred K^T, both read as
//                         MN-major 128-byte-swizzled tiles of 128 tokens x 128
//                         dimensions, accumulated in TMEM; the tokens of a head
//                         are split over several CTAs whose partial sums
//                         cov_reduce adds.
//   coarse_tail_kernel    one CTA per query block: S = Q kbar^T + (Q o Q) s2h^T
//                         over tiles of 128 pseudo-keys (one per key block),
//                         kept blocks masked out, online softmax, O += P vbar,
//                         and C Q^T for the first-order term; the epilogue
//                         writes lbar and obar.
//   tail_refine_kernel    d_l = l_T - lbar, d_o = bf16(o_T - obar) at a refresh.
//   tail_merge_kernel     LSE = logaddexp(l_S, lbar + d_l),
//                         O = w_S O_S + w_T (obar + d_o).
//   complement_kernel     the omitted blocks of every row, from the mask.
#include <cuda.h>

#include <cmath>

#include "internal.cuh"
#include "sm100.cuh"

namespace bsa {
namespace tail {

using namespace sm100;

constexpr int kRows = 128;                       // rows of every MMA tile
constexpr uint64_t kTimeoutNs = 2000000000ull;   // 2 s
constexpr int kTileBytes = kRows * 128 * 2;      // 128 rows x 128 bf16 columns
constexpr int kPanel = kRows * 128;              // one 64-column panel (bytes)

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void flag(int32_t* status, int bits) {
  if (status) atomicOr(status, bits);
}

// Bounded wait; false (and BSA_DEV_TIMEOUT) after 2 s.
__device__ __forceinline__ bool wait_for(uint64_t* bar, uint32_t parity, int32_t* status) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try(bar, parity)) {
    if (globaltimer_ns() - t0 > kTimeoutNs) {
      flag(status, BSA_DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// The same for a whole warp, with one outcome for all its lanes, so that the
// warp-collective TMEM loads and stores that follow never run divergently.
__device__ __forceinline__ bool warp_wait_for(uint64_t* bar, uint32_t parity, int32_t* status) {
  return __all_sync(0xffffffffu, wait_for(bar, parity, status));
}

// --------------------------------------------------------------- moments
// grid (NB, B*H), 256 threads.  Writes (all per head bh, block j):
//   kbar, s2, vbar       float32 [bh][j][d]
//   tabK = bf16(kbar), tabS = bf16(s2 / (2 sqrt(D))), tabV = bf16(vbar)   [bh][j][d]
//   kc, vc               bf16 [bh][t][d]: the block-centred keys and values
// The block's keys, then its values, are read once from HBM with 16-byte
// loads into shared memory; each (dimension, token part) thread sums its part
// and the parts are combined; the centred values go back out 16 bytes per
// store in the input's layout.  HBM-bound: K and V read once, kc and vc
// written once.
constexpr int kMomThreads = 256;

template <int D>
__global__ void __launch_bounds__(kMomThreads) tail_moments_kernel(const __nv_bfloat16* __restrict__ k,
                                                                   const __nv_bfloat16* __restrict__ v, int L,
                                                                   int blk, int NB, float* __restrict__ kbar,
                                                                   float* __restrict__ s2, float* __restrict__ vbar,
                                                                   __nv_bfloat16* __restrict__ tabK,
                                                                   __nv_bfloat16* __restrict__ tabS,
                                                                   __nv_bfloat16* __restrict__ tabV,
                                                                   __nv_bfloat16* __restrict__ kc,
                                                                   __nv_bfloat16* __restrict__ vc) {
  constexpr int VPR = D / 8;                // 16-byte vectors per token row
  constexpr int PARTS = kMomThreads / D;    // token parts per dimension
  constexpr int PER = 128 * VPR / kMomThreads;  // vectors per thread (a full block)
  __shared__ __align__(16) __nv_bfloat16 buf[128 * D];  // one block of keys or values, [t][d]
  __shared__ float part[PARTS][D];
  __shared__ float mean_s[D];
  const int j = blockIdx.x;
  const long long bh = blockIdx.y;
  const int tid = threadIdx.x;
  const int d = tid % D, h = tid / D;
  const int lo = j * blk;
  const int n = min(L, lo + blk) - lo;      // <= blk <= 128
  const size_t o = (static_cast<size_t>(bh) * NB + j) * D + d;
#pragma unroll 1
  for (int which = 0; which < 2; ++which) {
    const size_t base = (bh * L + lo) * D;
    const uint4* src = reinterpret_cast<const uint4*>((which ? v : k) + base);
    uint4* dst = reinterpret_cast<uint4*>((which ? vc : kc) + base);
    uint4* b4 = reinterpret_cast<uint4*>(buf);
    __syncthreads();  // the previous pass has finished with buf
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int e = tid + r * kMomThreads;
      if (e < n * VPR) b4[e] = __ldg(src + e);
    }
    __syncthreads();
    // mean over the block's tokens
    float acc = 0.f;
    for (int t = h; t < n; t += PARTS) acc += __bfloat162float(buf[t * D + d]);
    part[h][d] = acc;
    __syncthreads();
    if (h == 0) {
      float sum = 0.f;
#pragma unroll
      for (int q = 0; q < PARTS; ++q) sum += part[q][d];
      mean_s[d] = sum / static_cast<float>(n);
    }
    __syncthreads();
    const float mu = mean_s[d];
    if (which == 0) {
      // population variance of the keys
      float q2 = 0.f;
      for (int t = h; t < n; t += PARTS) {
        const float x = __bfloat162float(buf[t * D + d]) - mu;
        q2 += x * x;
      }
      __syncthreads();  // every part[] read of the mean is done
      part[h][d] = q2;
      __syncthreads();
      if (h == 0) {
        float sq = 0.f;
#pragma unroll
        for (int q = 0; q < PARTS; ++q) sq += part[q][d];
        const float var = sq / static_cast<float>(n);
        kbar[o] = mu;
        s2[o] = var;
        tabK[o] = __float2bfloat16_rn(mu);
        tabS[o] = __float2bfloat16_rn(var * (0.5f * rsqrtf(static_cast<float>(D))));
      }
    } else if (h == 0) {
      vbar[o] = mu;
      tabV[o] = __float2bfloat16_rn(mu);
    }
    // centred values in the input's layout: each thread its own vectors
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const int e = tid + r * kMomThreads;
      if (e >= n * VPR) continue;
      const uint4 x = b4[e];
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
      const int d0 = (e % VPR) * 8;
      uint32_t c[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float x0 = __uint_as_float(w[q] << 16) - mean_s[d0 + 2 * q];
        const float x1 = __uint_as_float(w[q] & 0xFFFF0000u) - mean_s[d0 + 2 * q + 1];
        const __nv_bfloat162 pr = __floats2bfloat162_rn(x0, x1);
        c[q] = *reinterpret_cast<const uint32_t*>(&pr);
      }
      dst[e] = make_uint4(c[0], c[1], c[2], c[3]);
    }
  }
}

// ------------------------------------------------------------ covariance
// grid (splits, B*H), 160 threads: warps 0-3 read the accumulator, warp 4
// loads tiles and issues the MMAs.  Partial C of split s goes to
// part[(s * BH + bh) * D * D + e * D + d].
struct CovShared {
  uint64_t full[2], empty[2], done;
  uint32_t tmem_base;
};

__global__ void __launch_bounds__(160, 1) cov_kernel(const __grid_constant__ CUtensorMap tmVc,
                                                     const __grid_constant__ CUtensorMap tmKc, int L, int splits,
                                                     float* __restrict__ part, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tiles = smem;                                         // [stage][A | B], 64 KB per stage
  CovShared* sh = reinterpret_cast<CovShared*>(smem + 4 * kTileBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int nchunks = (L + 127) / 128;
  const int per = (nchunks + splits - 1) / splits;
  const int c0 = blockIdx.x * per;
  const int c1 = min(nchunks, c0 + per);
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1);
    }
    mbar_init(&sh->done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sh->tmem_base, 128);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  bool ok = true;
  if (warp == 4) {
    if (c0 < c1) {
      // A = centred V^T (M = value dimension), B = centred K^T (N = key
      // dimension), K = tokens: both tiles are [128 tokens][128 dims], i.e.
      // MN-major
      constexpr uint32_t idC = idesc_bf16_f32(kRows, 128, true, true);
      // two stages: the load of chunk c overlaps the MMA of chunk c-1
      for (int c = c0; c < c1 && ok; ++c) {
        const int u = c - c0;
        const int st = u & 1;
        // load chunk c into stage st once the MMA of chunk c-2 released it
        if (u >= 2) ok = warp_wait_for(&sh->empty[st], ((u - 2) >> 1) & 1, status);
        if (!ok) break;
        if (lane == 0) {
          uint8_t* a = tiles + st * 2 * kTileBytes;
          uint8_t* b = a + kTileBytes;
          mbar_arrive_expect_tx(&sh->full[st], 2 * kTileBytes);
          for (int p = 0; p < 2; ++p) {
            tma_load_3d(a + p * kPanel, &tmVc, &sh->full[st], p * 64, c * 128, bh);
            tma_load_3d(b + p * kPanel, &tmKc, &sh->full[st], p * 64, c * 128, bh);
          }
        }
        __syncwarp();
        ok = warp_wait_for(&sh->full[st], (u >> 1) & 1, status);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a = smem_u32(tiles + st * 2 * kTileBytes);
          const uint32_t b = a + kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // 16 tokens per step: 16 rows of 128 bytes
            mma_ss(tmem, sdesc_sw128(a + kk * 2048, kPanel, 1024), sdesc_sw128(b + kk * 2048, kPanel, 1024), idC,
                   (u > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&sh->empty[st]);
        }
        __syncwarp();
      }
      if (lane == 0) tc_commit(&sh->done);
      __syncwarp();
    } else if (lane == 0) {
      mbar_arrive(&sh->done);
    }
  } else {
    // warps 0-3: row e = 32 * warp + lane of the accumulator
    const bool any = c0 < c1;
    ok = warp_wait_for(&sh->done, 0, status);
    tc_fence_after();
    const int e = warp * 32 + lane;
    float* out = part + ((static_cast<size_t>(blockIdx.x) * gridDim.y + bh) * 128 + e) * 128;
    const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t r[32];
      if (ok && any) {
        tmem_ld32(tl + cc * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) reg_fence(r[x]);
      }
#pragma unroll
      for (int x = 0; x < 32; ++x) out[cc * 32 + x] = (ok && any) ? __uint_as_float(r[x]) : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// C[bh][e][d] = sum over splits / L; also the bf16 table for the tail kernel.
__global__ void cov_reduce_kernel(const float* __restrict__ part, int splits, int BH, int D, float inv_L,
                                  float* __restrict__ C, __nv_bfloat16* __restrict__ tabC) {
  const size_t n = static_cast<size_t>(BH) * D * D;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float s = 0.f;
    for (int sp = 0; sp < splits; ++sp) s += part[static_cast<size_t>(sp) * n + i];
    s *= inv_L;
    C[i] = s;
    tabC[i] = __float2bfloat16_rn(s);
  }
}

// ------------------------------------------------------------ coarse tail
struct TailShared {
  uint64_t q_full, c_full, q2_ready, b_full, b_empty, v_full, v_empty, s_full[2], p_full[2], pv_done, cq_done, drain;
  uint64_t pair[4];        // the two softmax warps of a lane quarter: per tile, then once for the sums
  float xchg[2][2][128];   // [tile parity][column half][row]: a warp's row maxima (then its row sums)
  uint32_t tmem_base;
};
constexpr int kTailSoftmaxWarps = 8;   // two per TMEM lane quarter, one per 64-column half
constexpr int kTailThreads = 32 * kTailSoftmaxWarps + 32;

// grid (NB, B*H), 288 threads: warps 0-7 softmax and epilogue (warp w takes
// the rows of TMEM lane quarter w % 4 and the 64-column half w / 4 of S and of
// O; the two warps of a quarter exchange their row maxima every tile and
// their row sums at the end), warp 8 loads tiles and issues the MMAs.
// Shared memory: Q | Q o Q | C | B1 | B2 | Vbar (32 KB each), the mask row
// (NT * 128 bytes) and the barriers.
// TMEM columns: S0 [0, 128) | S1 [128, 256) | O [256, 384) | CQ [384, 512).
__global__ void __launch_bounds__(kTailThreads, 1)
    coarse_tail_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmC,
                       const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
                       const __grid_constant__ CUtensorMap tmVb, const uint8_t* __restrict__ mask, int L, int blk,
                       int NB, float scale_log2, float log_blk, float* __restrict__ lbar,
                       __nv_bfloat16* __restrict__ obar, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sQ2 = smem + 1 * kTileBytes;
  uint8_t* sC = smem + 2 * kTileBytes;
  uint8_t* sB1 = smem + 3 * kTileBytes;
  uint8_t* sB2 = smem + 4 * kTileBytes;
  uint8_t* sV = smem + 5 * kTileBytes;
  uint8_t* sMask = smem + 6 * kTileBytes;  // NT * 128 bytes: the mask row, 1 past NB
  TailShared* sh = reinterpret_cast<TailShared*>(sMask + ((NB + 127) & ~127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qi = blockIdx.x;
  const int bh = blockIdx.y;
  const int NT = (NB + 127) / 128;  // pseudo-key tiles
  const uint8_t* mrow = mask + (static_cast<size_t>(bh) * NB + qi) * NB;
  for (int j = threadIdx.x; j < NT * kRows; j += blockDim.x) sMask[j] = j < NB ? mrow[j] : 1;
  if (threadIdx.x == 0) {
    mbar_init(&sh->q_full, 1);
    mbar_init(&sh->c_full, 1);
    mbar_init(&sh->q2_ready, 32 * kTailSoftmaxWarps);
    mbar_init(&sh->b_full, 1);
    mbar_init(&sh->b_empty, 1);
    mbar_init(&sh->v_full, 1);
    mbar_init(&sh->v_empty, 1);
    mbar_init(&sh->s_full[0], 1);
    mbar_init(&sh->s_full[1], 1);
    mbar_init(&sh->p_full[0], 32 * kTailSoftmaxWarps);
    mbar_init(&sh->p_full[1], 32 * kTailSoftmaxWarps);
    for (int qq = 0; qq < 4; ++qq) mbar_init(&sh->pair[qq], 64);
    mbar_init(&sh->pv_done, 1);
    mbar_init(&sh->cq_done, 1);
    mbar_init(&sh->drain, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  constexpr uint32_t COL_S = 0, COL_O = 256, COL_CQ = 384;

  if (warp == kTailSoftmaxWarps) {
    // ------------------------------------------------ loads and MMA issue
    constexpr uint32_t idS = idesc_bf16_f32(kRows, 128, false, false);
    constexpr uint32_t idPV = idesc_bf16_f32(kRows, 128, false, true);
    bool ok = true;
    if (lane == 0) {
      mbar_arrive_expect_tx(&sh->q_full, kTileBytes);
      for (int p = 0; p < 2; ++p) tma_load_3d(sQ + p * kPanel, &tmQ, &sh->q_full, p * 64, qi * kRows, bh);
      mbar_arrive_expect_tx(&sh->c_full, kTileBytes);
      for (int p = 0; p < 2; ++p) tma_load_3d(sC + p * kPanel, &tmC, &sh->c_full, p * 64, 0, bh);
      mbar_arrive_expect_tx(&sh->b_full, 2 * kTileBytes);
      mbar_arrive_expect_tx(&sh->v_full, kTileBytes);
      for (int p = 0; p < 2; ++p) {
        tma_load_3d(sB1 + p * kPanel, &tmB1, &sh->b_full, p * 64, 0, bh);
        tma_load_3d(sB2 + p * kPanel, &tmB2, &sh->b_full, p * 64, 0, bh);
        tma_load_3d(sV + p * kPanel, &tmVb, &sh->v_full, p * 64, 0, bh);
      }
    }
    __syncwarp();
    const uint32_t aQ = smem_u32(sQ), aQ2 = smem_u32(sQ2), aC = smem_u32(sC);
    const uint32_t aB1 = smem_u32(sB1), aB2 = smem_u32(sB2), aV = smem_u32(sV);
    // C Q^T as soon as Q and C are in
    ok = warp_wait_for(&sh->q_full, 0, status) && warp_wait_for(&sh->c_full, 0, status);
    tc_fence_after();
    if (ok && lane == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * kPanel + (kk & 3) * 32;
        mma_ss(tmem + COL_CQ, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aC + off, 16, 1024), idS,
               kk > 0 ? 1u : 0u);
      }
      tc_commit(&sh->cq_done);
    }
    __syncwarp();
    if (ok) ok = warp_wait_for(&sh->q2_ready, 0, status);
    // S runs one tile ahead in two TMEM buffers (S, then P of tile t in
    // buffer t % 2): S(t+1) is computed while the softmax works on tile t.
    // The pseudo-key operands B1, B2 of the next tile are loaded as soon as S
    // has read this tile's, the values Vbar as soon as PV has.  S(t+1)
    // overwrites the buffer that held P(t-1), so it waits for PV(t-1).  Every
    // barrier a waiter could otherwise see two phases ahead is kept per
    // buffer (s_full, p_full).
    int b_loads = 1, v_loads = 1, b_seen = 0, v_seen = 0;  // tile loads issued / waited for
    auto issue_s = [&](int t) -> bool {                     // S(t) into buffer t % 2
      if (!warp_wait_for(&sh->b_full, t & 1, status)) return false;
      ++b_seen;
      if (t >= 2 && !warp_wait_for(&sh->pv_done, (t - 2) & 1, status)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t dS = tmem + COL_S + (t & 1) * kRows;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kPanel + (kk & 3) * 32;
          mma_ss(dS, sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aB1 + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kPanel + (kk & 3) * 32;
          mma_ss(dS, sdesc_sw128(aQ2 + off, 16, 1024), sdesc_sw128(aB2 + off, 16, 1024), idS, 1u);
        }
        tc_commit(&sh->s_full[t & 1]);
        tc_commit(&sh->b_empty);
      }
      __syncwarp();
      if (t + 1 < NT) {
        // the next tile's B1, B2 once S(t) has read this tile's
        if (!warp_wait_for(&sh->b_empty, t & 1, status)) return false;
        if (lane == 0) {
          mbar_arrive_expect_tx(&sh->b_full, 2 * kTileBytes);
          for (int p = 0; p < 2; ++p) {
            tma_load_3d(sB1 + p * kPanel, &tmB1, &sh->b_full, p * 64, (t + 1) * kRows, bh);
            tma_load_3d(sB2 + p * kPanel, &tmB2, &sh->b_full, p * 64, (t + 1) * kRows, bh);
          }
        }
        ++b_loads;
        __syncwarp();
      }
      return true;
    };
    if (ok) ok = issue_s(0);
    for (int t = 0; t < NT && ok; ++t) {
      if (t + 1 < NT && !(ok = issue_s(t + 1))) break;
      if (!(ok = warp_wait_for(&sh->p_full[t & 1], (t >> 1) & 1, status))) break;
      if (!(ok = warp_wait_for(&sh->v_full, t & 1, status))) break;
      ++v_seen;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t aP = tmem + COL_S + (t & 1) * kRows;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + COL_O, aP + kk * 8, sdesc_sw128(aV + kk * 2048, kRows * 128, 1024), idPV,
                 (t > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&sh->pv_done);
        tc_commit(&sh->v_empty);
      }
      __syncwarp();
      if (t + 1 < NT) {
        if (!(ok = warp_wait_for(&sh->v_empty, t & 1, status))) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&sh->v_full, kTileBytes);
          for (int p = 0; p < 2; ++p)
            tma_load_3d(sV + p * kPanel, &tmVb, &sh->v_full, p * 64, (t + 1) * kRows, bh);
        }
        ++v_loads;
        __syncwarp();
      }
    }
    if (!ok && lane == 0) {
      // let every MMA this thread issued finish before TMEM is released, and
      // every tile load land before the shared memory is (bounded waits)
      tc_commit(&sh->drain);
      wait_for(&sh->drain, 0, nullptr);
      if (b_loads > b_seen) wait_for(&sh->b_full, (b_loads - 1) & 1, nullptr);
      if (v_loads > v_seen) wait_for(&sh->v_full, (v_loads - 1) & 1, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------- softmax and epilogue
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;  // the thread's row
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t colS = COL_S + half * 64;  // this warp's 64 columns of S ...
    const uint32_t colO = COL_O + half * 64;  // ... of O ...
    const uint32_t colC = COL_CQ + half * 64;  // ... and of C Q^T
    bool ok = warp_wait_for(&sh->q_full, 0, status);
    if (ok) {
      // Q o Q in the same swizzled positions (an elementwise map keeps the layout)
      const uint4* src = reinterpret_cast<const uint4*>(sQ);
      uint4* dst = reinterpret_cast<uint4*>(sQ2);
      for (int c = threadIdx.x; c < kTileBytes / 16; c += 32 * kTailSoftmaxWarps) {
        uint4 x = src[c];
        uint32_t* w = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
          w[e] = pack_bf16x2(lo * lo, hi * hi);
        }
        dst[c] = x;
      }
      fence_proxy_async_smem();
    }
    mbar_arrive(&sh->q2_ready);
    const float bias_last = log2f(static_cast<float>(L - (NB - 1) * blk) / static_cast<float>(blk));
    float m = -INFINITY, l = 0.f;  // l: this half's share of the row sum
    int xp = 0;                    // completions of this quarter's pair barrier so far
    for (int t = 0; t < NT && ok; ++t) {
      if (!(ok = warp_wait_for(&sh->s_full[t & 1], (t >> 1) & 1, status))) break;
      tc_fence_after();
      const uint32_t bufS = (t & 1) * kRows;  // this tile's S buffer
      uint32_t s[64];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc)
        tmem_ld32(tmem + lane_off + bufS + colS + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(s + cc * 32));
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 64; ++e) reg_fence(s[e]);
      // kept blocks and blocks past NB (mask byte 1) are not in the tail; the
      // mask bytes come 16 at a time, the maxima in four chains
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      const uint4* mrow4 = reinterpret_cast<const uint4*>(sMask + t * kRows + half * 64);
      const int e_last = NB - 1 - t * kRows - half * 64;  // the ragged last block, if in this half
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 mw = mrow4[c];
        const uint32_t mwd[4] = {mw.x, mw.y, mw.z, mw.w};
#pragma unroll
        for (int b = 0; b < 16; ++b) {
          const int e = c * 16 + b;
          float x = __uint_as_float(s[e]) * scale_log2;
          if (e == e_last) x += bias_last;
          if ((mwd[b >> 2] >> (8 * (b & 3))) & 0xFFu) x = -INFINITY;
          s[e] = __float_as_uint(x);
          mx4[e & 3] = fmaxf(mx4[e & 3], x);
        }
      }
      // the other half-row's maximum, through shared memory (buffer by tile
      // parity: a warp can be at most one exchange ahead of its partner)
      sh->xchg[t & 1][half][r] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      mbar_arrive(&sh->pair[quarter]);
      if (!(ok = warp_wait_for(&sh->pair[quarter], xp & 1, status))) break;
      ++xp;
      const float mx = fmaxf(sh->xchg[t & 1][0][r], sh->xchg[t & 1][1][r]);
      const float m_new = fmaxf(m, mx);
      const bool grow_m = t > 0 && m_new > m;
      if (__any_sync(0xffffffffu, grow_m)) {
        // rescale this half of O once the previous PV has completed; the whole
        // warp takes part in the TMEM accesses, rows whose maximum did not grow
        // with 1
        if (!(ok = warp_wait_for(&sh->pv_done, (t - 1) & 1, status))) break;
        tc_fence_after();
        const float f = grow_m ? ex2_approx(m - m_new) : 1.f;  // 0 while m is -inf
        l *= f;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + colO + cc * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            reg_fence(o[x]);
            o[x] = __float_as_uint(__uint_as_float(o[x]) * f);
          }
          tmem_st32(tmem + lane_off + colO + cc * 32, o);
        }
        tmem_wait_st();
      }
      m = m_new;
      uint32_t p[32];
      float l4[4] = {0.f, 0.f, 0.f, 0.f};  // four independent partial sums
      const float mm = m == -INFINITY ? 0.f : m;  // a row with no tail block so far: every x is -inf
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float p0 = ex2_approx(__uint_as_float(s[2 * c]) - mm);
        const float p1 = ex2_approx(__uint_as_float(s[2 * c + 1]) - mm);
        l4[c & 3] += p0 + p1;
        p[c] = pack_bf16x2(p0, p1);
      }
      l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      // P columns 32*half .. 32*half+31 (both halves have loaded their S:
      // the exchange above follows every load)
      tmem_st32(tmem + lane_off + COL_S + bufS + half * 32, p);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sh->p_full[t & 1]);
    }
    // the full row sum, through the same exchange
    if (ok) {
      sh->xchg[xp & 1][half][r] = l;
      mbar_arrive(&sh->pair[quarter]);
      ok = warp_wait_for(&sh->pair[quarter], xp & 1, status);
      l = sh->xchg[xp & 1][0][r] + sh->xchg[xp & 1][1][r];
    }
    // epilogue: this half of the row's obar
    if (ok) ok = warp_wait_for(&sh->pv_done, (NT - 1) & 1, status) && warp_wait_for(&sh->cq_done, 0, status);
    tc_fence_after();
    const int grow = qi * kRows + r;
    if (ok) {
      const bool store = grow < L;
      const size_t row = static_cast<size_t>(bh) * L + (store ? grow : 0);
      const bool empty = !(l > 0.f);
      if (store && half == 0) lbar[row] = empty ? -INFINITY : (m + log2f(l)) * 0.69314718055994531f + log_blk;
      const float inv_l = empty ? 0.f : 1.f / l;
      const float inv_sqrt_d = rsqrtf(128.f);
      __nv_bfloat16* out = obar + row * 128 + half * 64;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t o[32], cq[32];
        tmem_ld32(tmem + lane_off + colO + cc * 32, o);
        tmem_ld32(tmem + lane_off + colC + cc * 32, cq);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          reg_fence(o[x]);
          reg_fence(cq[x]);
        }
        if (!store) continue;
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const float a0 = empty ? 0.f : __uint_as_float(o[2 * x]) * inv_l + __uint_as_float(cq[2 * x]) * inv_sqrt_d;
          const float a1 =
              empty ? 0.f : __uint_as_float(o[2 * x + 1]) * inv_l + __uint_as_float(cq[2 * x + 1]) * inv_sqrt_d;
          pk[x] = pack_bf16x2(a0, a1);
        }
        uint4* dst = reinterpret_cast<uint4*>(out + cc * 32);
#pragma unroll
        for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------- elementwise
// one thread per (row, 8 columns)
__global__ void tail_refine_kernel(size_t rows, int D, const float* __restrict__ l_T,
                                   const __nv_bfloat16* __restrict__ o_T, const float* __restrict__ lbar,
                                   const __nv_bfloat16* __restrict__ obar, float* __restrict__ d_l,
                                   __nv_bfloat16* __restrict__ d_o) {
  const int per_row = D / 8;
  const size_t n = rows * per_row;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t row = i / per_row;
    const int c = static_cast<int>(i - row * per_row) * 8;
    const bool empty = isinf(lbar[row]) && lbar[row] < 0.f;
    if (c == 0) d_l[row] = empty ? 0.f : l_T[row] - lbar[row];
    const uint4 a = *reinterpret_cast<const uint4*>(o_T + row * D + c);
    const uint4 b = *reinterpret_cast<const uint4*>(obar + row * D + c);
    const uint32_t* pa = reinterpret_cast<const uint32_t*>(&a);
    const uint32_t* pb = reinterpret_cast<const uint32_t*>(&b);
    uint4 r;
    uint32_t* pr = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = __uint_as_float(pa[e] << 16) - __uint_as_float(pb[e] << 16);
      const float hi = __uint_as_float(pa[e] & 0xFFFF0000u) - __uint_as_float(pb[e] & 0xFFFF0000u);
      pr[e] = empty ? 0u : pack_bf16x2(lo, hi);
    }
    *reinterpret_cast<uint4*>(d_o + row * D + c) = r;
  }
}

__global__ void tail_merge_kernel(size_t rows, int D, const float* __restrict__ l_S,
                                  const __nv_bfloat16* __restrict__ o_S, const float* __restrict__ lbar,
                                  const __nv_bfloat16* __restrict__ obar, const float* __restrict__ d_l,
                                  const __nv_bfloat16* __restrict__ d_o, __nv_bfloat16* __restrict__ o,
                                  float* __restrict__ lse) {
  const int per_row = D / 8;
  const size_t n = rows * per_row;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t row = i / per_row;
    const int c = static_cast<int>(i - row * per_row) * 8;
    const float ls = l_S[row];
    const float lh = lbar[row] + d_l[row];
    const float mx = fmaxf(ls, lh);
    float ws = 0.f, wt = 0.f, out_lse = -INFINITY;
    if (mx > -INFINITY) {
      const float es = expf(ls - mx), et = expf(lh - mx);
      const float tot = es + et;
      out_lse = mx + logf(tot);
      ws = es / tot;
      wt = et / tot;
    }
    if (c == 0) lse[row] = out_lse;
    const uint4 a = *reinterpret_cast<const uint4*>(o_S + row * D + c);
    const uint4 b = *reinterpret_cast<const uint4*>(obar + row * D + c);
    const uint4 dd = *reinterpret_cast<const uint4*>(d_o + row * D + c);
    const uint32_t* pa = reinterpret_cast<const uint32_t*>(&a);
    const uint32_t* pb = reinterpret_cast<const uint32_t*>(&b);
    const uint32_t* pd = reinterpret_cast<const uint32_t*>(&dd);
    uint4 r;
    uint32_t* pr = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float s0 = ws > 0.f ? __uint_as_float(pa[e] << 16) : 0.f;
      const float s1 = ws > 0.f ? __uint_as_float(pa[e] & 0xFFFF0000u) : 0.f;
      const float t0 = __uint_as_float(pb[e] << 16) + __uint_as_float(pd[e] << 16);
      const float t1 = __uint_as_float(pb[e] & 0xFFFF0000u) + __uint_as_float(pd[e] & 0xFFFF0000u);
      pr[e] = pack_bf16x2(ws * s0 + wt * t0, ws * s1 + wt * t1);
    }
    *reinterpret_cast<uint4*>(o + row * D + c) = r;
  }
}

// one warp per row: the blocks with mask 0, ascending
__global__ void __launch_bounds__(256) complement_kernel(const uint8_t* __restrict__ mask, int NB, long long rows,
                                                         int32_t* __restrict__ idx, int32_t* __restrict__ cnt) {
  const int warps = blockDim.x >> 5;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * warps + w;
  if (row >= rows) return;
  const uint8_t* m = mask + row * NB;
  int32_t* out = idx + row * NB;
  int count = 0;
  for (int base = 0; base < NB; base += 32) {
    const int j = base + lane;
    const bool sel = j < NB && m[j] == 0;
    const unsigned bal = __ballot_sync(0xffffffffu, sel);
    if (sel) out[count + __popc(bal & ((1u << lane) - 1u))] = j;
    count += __popc(bal);
  }
  if (lane == 0) cnt[row] = count;
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D bf16 map (cols, rows, BH) with a row stride of `stride` elements; boxes
// of 64 columns x 128 rows, 128-byte swizzle; rows beyond `rows` read as 0.
bool map3(CUtensorMap* m, const void* base, int cols, int rows, int BH, size_t stride) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(stride) * 2, static_cast<cuuint64_t>(stride) * rows * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kRows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// CTAs per head for the covariance contraction: enough to cover the SMs
int splits_for(int BH) {
  const int s = (sm_count() + BH - 1) / BH;
  return s < 1 ? 1 : (s > 16 ? 16 : s);
}

}  // namespace tail

// Workspace layout (bytes, each part 1024-aligned):
//   kc, vc     bf16 [BH][L][D]
//   tabK, tabS, tabV  bf16 [BH][NB][D]
//   tabC       bf16 [BH][D][D]
//   part       f32  [splits][BH][D][D]
struct TailWs {
  size_t kc, vc, tabK, tabS, tabV, tabC, part, total;
  int splits;
};

static TailWs tail_ws_layout(const bsa_shape& s, int splits) {
  auto up = [](size_t x) { return (x + 1023) & ~size_t(1023); };
  TailWs w;
  const size_t BH = static_cast<size_t>(s.B) * s.H;
  const int NB = n_blocks(s.L, s.blk);
  w.splits = splits;
  size_t o = 0;
  w.kc = o; o += up(BH * s.L * s.D * 2);
  w.vc = o; o += up(BH * s.L * s.D * 2);
  w.tabK = o; o += up(BH * NB * s.D * 2);
  w.tabS = o; o += up(BH * NB * s.D * 2);
  w.tabV = o; o += up(BH * NB * s.D * 2);
  w.tabC = o; o += up(BH * s.D * s.D * 2);
  w.part = o; o += up(static_cast<size_t>(splits) * BH * s.D * s.D * 4);
  w.total = o;
  return w;
}

size_t tail_workspace_bytes(const bsa_shape& s) { return tail_ws_layout(s, 16).total; }

int launch_tail_stats(const bsa_shape& s, const __nv_bfloat16* k, const __nv_bfloat16* v, float* kbar, float* s2,
                      float* vbar, float* C, void* ws, int32_t* status, cudaStream_t st) {
  if (s.D != 128) return BSA_ESHAPE;
  const int BH = s.B * s.H;
  const int NB = n_blocks(s.L, s.blk);
  const int splits = tail::splits_for(BH);
  const TailWs w = tail_ws_layout(s, splits);
  uint8_t* base = static_cast<uint8_t*>(ws);
  auto* kc = reinterpret_cast<__nv_bfloat16*>(base + w.kc);
  auto* vc = reinterpret_cast<__nv_bfloat16*>(base + w.vc);
  tail::tail_moments_kernel<128><<<dim3(NB, BH), tail::kMomThreads, 0, st>>>(
      k, v, s.L, s.blk, NB, kbar, s2, vbar, reinterpret_cast<__nv_bfloat16*>(base + w.tabK),
      reinterpret_cast<__nv_bfloat16*>(base + w.tabS), reinterpret_cast<__nv_bfloat16*>(base + w.tabV), kc, vc);
  if (cudaGetLastError() != cudaSuccess) return BSA_ECUDA;
  CUtensorMap mVc, mKc;
  if (!tail::map3(&mVc, vc, 128, s.L, BH, 128) || !tail::map3(&mKc, kc, 128, s.L, BH, 128)) return BSA_ECUDA;
  constexpr int kCovSmem = 4 * tail::kTileBytes + 1024 + 1024;
  if (smem_opt_in(reinterpret_cast<const void*>(tail::cov_kernel), kCovSmem) != cudaSuccess) return BSA_ECUDA;
  float* part = reinterpret_cast<float*>(base + w.part);
  tail::cov_kernel<<<dim3(splits, BH), 160, kCovSmem, st>>>(mVc, mKc, s.L, splits, part, status);
  if (cudaGetLastError() != cudaSuccess) return BSA_ECUDA;
  tail::cov_reduce_kernel<<<512, 256, 0, st>>>(part, splits, BH, 128, 1.0f / static_cast<float>(s.L), C,
                                                reinterpret_cast<__nv_bfloat16*>(base + w.tabC));
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ECUDA;
}

int launch_coarse_tail(const bsa_shape& s, const __nv_bfloat16* q, const uint8_t* mask, const void* ws,
                       float* lbar, __nv_bfloat16* obar, int32_t* status, cudaStream_t st) {
  if (s.D != 128) return BSA_ESHAPE;
  const int BH = s.B * s.H;
  const int NB = n_blocks(s.L, s.blk);
  if (s.blk != 128) return BSA_ESHAPE;  // one 128-row query tile per query block
  const TailWs w = tail_ws_layout(s, tail::splits_for(BH));
  const uint8_t* base = static_cast<const uint8_t*>(ws);
  CUtensorMap mQ, mC, mB1, mB2, mV;
  if (!tail::map3(&mQ, q, 128, s.L, BH, 128) || !tail::map3(&mC, base + w.tabC, 128, 128, BH, 128) ||
      !tail::map3(&mB1, base + w.tabK, 128, NB, BH, 128) || !tail::map3(&mB2, base + w.tabS, 128, NB, BH, 128) ||
      !tail::map3(&mV, base + w.tabV, 128, NB, BH, 128))
    return BSA_ECUDA;
  const int smem = 6 * tail::kTileBytes + ((NB + 127) & ~127) + static_cast<int>(sizeof(tail::TailShared)) + 1024;
  if (smem_opt_in(reinterpret_cast<const void*>(tail::coarse_tail_kernel), smem) != cudaSuccess) return BSA_ECUDA;
  const float scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(128.0));
  tail::coarse_tail_kernel<<<dim3(NB, BH), tail::kTailThreads, smem, st>>>(mQ, mC, mB1, mB2, mV, mask, s.L, s.blk, NB, scale_log2,
                                                             std::log(static_cast<float>(s.blk)), lbar, obar, status);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ECUDA;
}

int launch_tail_refine(const bsa_shape& s, const float* l_T, const __nv_bfloat16* o_T, const float* lbar,
                       const __nv_bfloat16* obar, float* d_l, __nv_bfloat16* d_o, cudaStream_t st) {
  const size_t rows = static_cast<size_t>(s.B) * s.H * s.L;
  tail::tail_refine_kernel<<<1184, 256, 0, st>>>(rows, s.D, l_T, o_T, lbar, obar, d_l, d_o);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ECUDA;
}

int launch_tail_merge(const bsa_shape& s, const float* l_S, const __nv_bfloat16* o_S, const float* lbar,
                      const __nv_bfloat16* obar, const float* d_l, const __nv_bfloat16* d_o, __nv_bfloat16* o,
                      float* lse, cudaStream_t st) {
  const size_t rows = static_cast<size_t>(s.B) * s.H * s.L;
  tail::tail_merge_kernel<<<1184, 256, 0, st>>>(rows, s.D, l_S, o_S, lbar, obar, d_l, d_o, o, lse);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ECUDA;
}

int launch_complement(const bsa_shape& s, const uint8_t* mask, int32_t* idx, int32_t* cnt, cudaStream_t st) {
  const int NB = n_blocks(s.L, s.blk);
  const long long rows = static_cast<long long>(s.B) * s.H * NB;
  tail::complement_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(mask, NB, rows, idx, cnt);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ECUDA;
}

}  // namespace bsa
