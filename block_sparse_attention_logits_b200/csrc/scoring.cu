// Block importance scoring: block-mean pooling of Q and K (RECAP section
// 3.2, coarse estimates from block means; DFSAttn abstract, block scoring)
// and the per-query-block softmax of pooled logits that top-p acts on
// (head-wise top-p and GSRS abstracts).
//
//   pool:    one CTA per (block, head, Q|K); 16-byte vector loads, fp32
//            accumulation, a shared-memory tree over the row groups; the
//            partial last block divides by its own token count.  HBM-bound.
//   softmax: one CTA per (16 query blocks, head); pooled rows staged in
//            shared memory, two query rows per thread, raw logits
//            written to `probs`, then each warp normalises its rows in place.
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

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k, float* __restrict__ qp,
                                                   float* __restrict__ kp, int L, int blk, int NB) {
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
  const uint4* base = reinterpret_cast<const uint4*>(x + (bh * L + t0) * D) + c;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int row = r; row < n; row += RPI) add_bf16x8(acc, __ldg(base + static_cast<size_t>(row) * TPR));
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

constexpr int kRows = 16;  // query blocks per CTA
constexpr int kCols = 32;  // key blocks per shared-memory chunk

template <int D>
__global__ void __launch_bounds__(256) block_softmax_kernel(const float* __restrict__ qp,
                                                            const float* __restrict__ kp, float* __restrict__ probs,
                                                            int NB, float scale) {
  __shared__ __align__(16) float qs[kRows][D + 4];
  __shared__ __align__(16) float ks[kCols][D + 4];
  const size_t bh = blockIdx.y;
  const int i0 = blockIdx.x * kRows;
  const int tid = threadIdx.x;
  for (int e = tid; e < kRows * D; e += 256) {
    const int rr = e / D, d = e % D;
    qs[rr][d] = (i0 + rr < NB) ? qp[(bh * NB + i0 + rr) * D + d] : 0.f;
  }
  // thread -> query rows {ra, ra+8} and one key column of each 32-column
  // chunk: threads 0..127 take columns 0..15, threads 128..255 columns 16..31
  const int tr = tid >> 4;
  const int ra = tr & 7, rb = ra + 8;
  const int col = (tid & 15) + (tr >= 8 ? 16 : 0);
  for (int j0 = 0; j0 < NB; j0 += kCols) {
    __syncthreads();
    for (int e = tid; e < kCols * D; e += 256) {
      const int cc = e / D, d = e % D;
      ks[cc][d] = (j0 + cc < NB) ? kp[(bh * NB + j0 + cc) * D + d] : 0.f;
    }
    __syncthreads();
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; d += 4) {
      const float4 kv = *reinterpret_cast<const float4*>(&ks[col][d]);
      const float4 a = *reinterpret_cast<const float4*>(&qs[ra][d]);
      const float4 b = *reinterpret_cast<const float4*>(&qs[rb][d]);
      s0 = fmaf(a.x, kv.x, s0);
      s0 = fmaf(a.y, kv.y, s0);
      s0 = fmaf(a.z, kv.z, s0);
      s0 = fmaf(a.w, kv.w, s0);
      s1 = fmaf(b.x, kv.x, s1);
      s1 = fmaf(b.y, kv.y, s1);
      s1 = fmaf(b.z, kv.z, s1);
      s1 = fmaf(b.w, kv.w, s1);
    }
    const int j = j0 + col;
    if (j < NB) {
      if (i0 + ra < NB) probs[(bh * NB + i0 + ra) * NB + j] = s0 * scale;
      if (i0 + rb < NB) probs[(bh * NB + i0 + rb) * NB + j] = s1 * scale;
    }
  }
  __syncthreads();
  // row softmax: warp w handles rows w and w+8
  const int w = tid >> 5, lane = tid & 31;
  for (int rr = w; rr < kRows; rr += 8) {
    const int i = i0 + rr;
    if (i >= NB) break;
    float* row = probs + (bh * NB + i) * NB;
    float m = -INFINITY;
    for (int j = lane; j < NB; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = 0.f;
    for (int j = lane; j < NB; j += 32) {
      const float e = expf(row[j] - m);
      row[j] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    for (int j = lane; j < NB; j += 32) row[j] = row[j] / sum;
  }
}

}  // namespace

cudaError_t launch_pool(const bsa_shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k, float* qp, float* kp,
                        cudaStream_t st) {
  const int NB = n_blocks(s.L, s.blk);
  dim3 grid(NB, s.B * s.H, 2);
  if (s.D == 128)
    pool_kernel<128><<<grid, 256, 0, st>>>(q, k, qp, kp, s.L, s.blk, NB);
  else
    pool_kernel<64><<<grid, 256, 0, st>>>(q, k, qp, kp, s.L, s.blk, NB);
  return cudaGetLastError();
}

cudaError_t launch_block_softmax(const bsa_shape& s, const float* qp, const float* kp, float* probs,
                                 cudaStream_t st) {
  const int NB = n_blocks(s.L, s.blk);
  dim3 grid((NB + kRows - 1) / kRows, s.B * s.H);
  const float scale = static_cast<float>(1.0 / sqrt(static_cast<double>(s.D)));
  if (s.D == 128)
    block_softmax_kernel<128><<<grid, 256, 0, st>>>(qp, kp, probs, NB, scale);
  else
    block_softmax_kernel<64><<<grid, 256, 0, st>>>(qp, kp, probs, NB, scale);
  return cudaGetLastError();
}

}  // namespace bsa
