// Block importance scoring: block-mean pooling of Q and K (RECAP section
// 3.2, coarse estimates from block means; DFSAttn abstract, block scoring)
// and the per-query-block softmax of pooled logits that top-p acts on
// (head-wise top-p and GSRS abstracts).
//
//   pool:    one CTA per (block, head, Q|K); 16-byte vector loads, fp32
//            accumulation, a shared-memory tree over the row groups; the
//            partial last block divides by its own token count.  HBM-bound.
//   softmax: one CTA per (64 query blocks, head); pooled means staged
//            transposed in shared memory, a 4x4 register tile of logits per
//            thread, raw logits written to `probs`, then each warp
//            normalises its rows in place: a row of up to 1024 blocks is read
//            once into registers (every load in flight), P written once.
#include <cuda_bf16.h>

#include "internal.cuh"

namespace bsa {
namespace {

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(w[i] << 16);
    acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// With `perm` (gathering form) token t of the block is row perm[t] of the
// input, and the gathered rows are also written to q_out / k_out in order
// (when given).
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k, float* __restrict__ qp,
                                                   float* __restrict__ kp, int L, int blk, int NB,
                                                   const int32_t* __restrict__ perm, __nv_bfloat16* __restrict__ q_out,
                                                   __nv_bfloat16* __restrict__ k_out) {
  constexpr int TPR = D / 8;        // threads per token row (8 bf16 each)
  constexpr int RPI = 256 / TPR;    // rows in flight per iteration
  __shared__ float part[RPI][D + 1];
  const __nv_bfloat16* x = blockIdx.z ? k : q;
  float* out = blockIdx.z ? kp : qp;
  const int i = blockIdx.x;
  const size_t bh = blockIdx.y;
  const int t0 = i * blk;
  const int n = min(blk, L - t0);
  const int c = threadIdx.x % TPR;
  const int r = threadIdx.x / TPR;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (perm) {
    const uint4* src = reinterpret_cast<const uint4*>(x + bh * L * D) + c;
    __nv_bfloat16* copy = blockIdx.z ? k_out : q_out;
    if (copy) {
      uint4* dst = reinterpret_cast<uint4*>(copy + (bh * L + t0) * D) + c;
#pragma unroll 4
      for (int row = r; row < n; row += RPI) {
        const uint4 v = __ldg(src + static_cast<size_t>(__ldg(perm + t0 + row)) * TPR);
        dst[static_cast<size_t>(row) * TPR] = v;
        add_bf16x8(acc, v);
      }
    } else {
#pragma unroll 4
      for (int row = r; row < n; row += RPI)
        add_bf16x8(acc, __ldg(src + static_cast<size_t>(__ldg(perm + t0 + row)) * TPR));
    }
  } else {
    const uint4* base = reinterpret_cast<const uint4*>(x + (bh * L + t0) * D) + c;
#pragma unroll 4
    for (int row = r; row < n; row += RPI) add_bf16x8(acc, __ldg(base + static_cast<size_t>(row) * TPR));
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[r][c * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float sum = 0.f;
#pragma unroll
    for (int g = 0; g < RPI; ++g) sum += part[g][threadIdx.x];
    out[(bh * NB + i) * D + threadIdx.x] = sum / static_cast<float>(n);
  }
}

constexpr int kTile = 64;   // query blocks per CTA, key blocks per tile
constexpr int kPad = 68;    // row pitch (floats) of the transposed tiles: 16-byte aligned

// Logits of a 64-query-block strip against all key blocks, 64 key blocks at a
// time: Q and K means staged transposed ([d][block]) in shared memory, each
// thread a 4x4 register tile (two 16-byte shared loads per 16 FMAs); raw
// scaled logits go to `probs`, then each warp normalises 8 of the strip's rows
// in place (max, exp and sum, divide).
template <int D, int PER>
__global__ void __launch_bounds__(256, 3) block_softmax_kernel(const float* __restrict__ qp,
                                                            const float* __restrict__ kp, float* __restrict__ probs,
                                                            const uint8_t* __restrict__ cand, int NB, float scale) {
  extern __shared__ __align__(16) float sm[];
  float* qT = sm;              // [D][kPad]
  float* kT = sm + D * kPad;   // [D][kPad]
  const size_t bh = blockIdx.y;
  const int i0 = blockIdx.x * kTile;
  const int tid = threadIdx.x;
  // fill: consecutive threads take consecutive d of one block row (coalesced)
  for (int e = tid; e < kTile * D; e += 256) {
    const int rr = e / D, d = e % D;
    qT[d * kPad + rr] = (i0 + rr < NB) ? __ldg(qp + (bh * NB + i0 + rr) * D + d) : 0.f;
  }
  const int r0 = (tid >> 4) * 4;  // the thread's 4 query rows ...
  const int c0 = (tid & 15) * 4;  // ... and 4 key columns within the tile
  for (int j0 = 0; j0 < NB; j0 += kTile) {
    __syncthreads();
    for (int e = tid; e < kTile * D; e += 256) {
      const int cc = e / D, d = e % D;
      kT[d * kPad + cc] = (j0 + cc < NB) ? __ldg(kp + (bh * NB + j0 + cc) * D + d) : 0.f;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) {
      const float4 qa = *reinterpret_cast<const float4*>(qT + d * kPad + r0);
      const float4 kb = *reinterpret_cast<const float4*>(kT + d * kPad + c0);
      const float qv[4] = {qa.x, qa.y, qa.z, qa.w};
      const float kv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(qv[a], kv[b], acc[a][b]);
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int i = i0 + r0 + a;
      if (i >= NB) break;
      float* row = probs + (bh * NB + i) * NB;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int j = j0 + c0 + b;
        if (j < NB) row[j] = acc[a][b] * scale;
      }
    }
  }
  __syncthreads();
  // row softmax: warp w normalises rows w, w+8, ...
  const int w = tid >> 5, lane = tid & 31;
  if constexpr (PER > 0) {
    // the row in registers: one read and one write per element
    for (int rr = w; rr < kTile; rr += 8) {
      const int i = i0 + rr;
      if (i >= NB) break;
      float* row = probs + (bh * NB + i) * NB;
      const uint8_t* crow = cand ? cand + (bh * NB + i) * NB : nullptr;
      float x[PER];
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int j = lane + 32 * e;
        x[e] = (j < NB && (!crow || crow[j])) ? row[j] : -INFINITY;
      }
      float m = -INFINITY;
#pragma unroll
      for (int e = 0; e < PER; ++e) m = fmaxf(m, x[e]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float sum = 0.f;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        x[e] = x[e] == -INFINITY ? 0.f : expf(x[e] - m);
        sum += x[e];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      // a row without candidates (sum 0) stays all zeros
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int j = lane + 32 * e;
        if (j < NB) row[j] = sum > 0.f ? x[e] / sum : 0.f;
      }
    }
  } else {
    for (int rr = w; rr < kTile; rr += 8) {
      const int i = i0 + rr;
      if (i >= NB) break;
      float* row = probs + (bh * NB + i) * NB;
      const uint8_t* crow = cand ? cand + (bh * NB + i) * NB : nullptr;
      float m = -INFINITY;
      for (int j = lane; j < NB; j += 32)
        if (!crow || crow[j]) m = fmaxf(m, row[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float sum = 0.f;
      for (int j = lane; j < NB; j += 32) {
        const float e = (!crow || crow[j]) ? expf(row[j] - m) : 0.f;
        row[j] = e;
        sum += e;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      // a row without candidates (sum 0) stays all zeros
      for (int j = lane; j < NB; j += 32) row[j] = sum > 0.f ? row[j] / sum : 0.f;
    }
  }
}

// Query-key drift of one head (head-wise top-p abstract, Temporal Mask Reuse):
// max of ||x - x_ref||_F / ||x_ref||_F over x = block means of Q and of K,
// with 0/0 -> 0 and a change from an all-zero reference -> +inf.  One CTA per
// (b, h); float64 sums of squares.
__global__ void __launch_bounds__(256) drift_kernel(const float* __restrict__ qr, const float* __restrict__ kr,
                                                    const float* __restrict__ q, const float* __restrict__ k,
                                                    float* __restrict__ drift, long long n) {
  const size_t base = static_cast<size_t>(blockIdx.x) * n;
  double s[4] = {0.0, 0.0, 0.0, 0.0};  // |dq|^2, |q_ref|^2, |dk|^2, |k_ref|^2
  for (long long e = threadIdx.x; e < n; e += 256) {
    const double a = qr[base + e], b = q[base + e], c = kr[base + e], d = k[base + e];
    s[0] += (b - a) * (b - a);
    s[1] += a * a;
    s[2] += (d - c) * (d - c);
    s[3] += c * c;
  }
  __shared__ double part[4][8];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    double v = s[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) part[t][threadIdx.x >> 5] = v;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot[4];
    for (int t = 0; t < 4; ++t) {
      tot[t] = 0.0;
      for (int w = 0; w < 8; ++w) tot[t] += part[t][w];
    }
    double r = 0.0;
    for (int t = 0; t < 4; t += 2) {
      const double rel = tot[t] == 0.0 ? 0.0 : (tot[t + 1] == 0.0 ? INFINITY : sqrt(tot[t] / tot[t + 1]));
      r = rel > r ? rel : r;
    }
    drift[blockIdx.x] = static_cast<float>(r);
  }
}

}  // namespace

cudaError_t launch_pool(const bsa_shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k, float* qp, float* kp,
                        cudaStream_t st, const int32_t* perm, __nv_bfloat16* q_out, __nv_bfloat16* k_out) {
  const int NB = n_blocks(s.L, s.blk);
  dim3 grid(NB, s.B * s.H, 2);
  if (s.D == 128)
    pool_kernel<128><<<grid, 256, 0, st>>>(q, k, qp, kp, s.L, s.blk, NB, perm, q_out, k_out);
  else
    pool_kernel<64><<<grid, 256, 0, st>>>(q, k, qp, kp, s.L, s.blk, NB, perm, q_out, k_out);
  return cudaGetLastError();
}

namespace {

// PER: values of a row per lane in the register row pass (0: rows longer
// than 1024 blocks, three passes over the row in `probs`)
template <int D, int PER>
cudaError_t launch_softmax(dim3 grid, const float* qp, const float* kp, float* probs, const uint8_t* cand, int NB,
                           float scale, cudaStream_t st) {
  // 69.6 KB of transposed tiles at D = 128: above the default 48 KB
  constexpr size_t smem = 2 * D * kPad * 4;
  if (cudaError_t e = smem_opt_in(reinterpret_cast<const void*>(block_softmax_kernel<D, PER>), smem)) return e;
  block_softmax_kernel<D, PER><<<grid, 256, smem, st>>>(qp, kp, probs, cand, NB, scale);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_softmax(const bsa_shape& s, const float* qp, const float* kp, float* probs,
                                 const uint8_t* cand, cudaStream_t st) {
  const int NB = n_blocks(s.L, s.blk);
  dim3 grid((NB + kTile - 1) / kTile, s.B * s.H);
  const float scale = static_cast<float>(1.0 / sqrt(static_cast<double>(s.D)));
  if (s.D == 128) {
    if (NB <= 256) return launch_softmax<128, 8>(grid, qp, kp, probs, cand, NB, scale, st);
    if (NB <= 640) return launch_softmax<128, 20>(grid, qp, kp, probs, cand, NB, scale, st);
    if (NB <= 1024) return launch_softmax<128, 32>(grid, qp, kp, probs, cand, NB, scale, st);
    return launch_softmax<128, 0>(grid, qp, kp, probs, cand, NB, scale, st);
  }
  if (NB <= 256) return launch_softmax<64, 8>(grid, qp, kp, probs, cand, NB, scale, st);
  if (NB <= 640) return launch_softmax<64, 20>(grid, qp, kp, probs, cand, NB, scale, st);
  if (NB <= 1024) return launch_softmax<64, 32>(grid, qp, kp, probs, cand, NB, scale, st);
  return launch_softmax<64, 0>(grid, qp, kp, probs, cand, NB, scale, st);
}

cudaError_t launch_drift(const bsa_shape& s, const float* qp_ref, const float* kp_ref, const float* qp,
                         const float* kp, float* drift, cudaStream_t st) {
  const long long n = static_cast<long long>(n_blocks(s.L, s.blk)) * s.D;
  drift_kernel<<<s.B * s.H, 256, 0, st>>>(qp_ref, kp_ref, qp, kp, drift, n);
  return cudaGetLastError();
}

}  // namespace bsa
