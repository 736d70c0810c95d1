// E4M3 quantization of Q or K per token block, for the FP8 Q.K^T attention
// (the abstract on the page titled RECAP runs its sparse attention in FP8 with
// fused kernels; the pages give no format or scaling rule, so the reading is:
// OCP E4M3, one scale per (batch, head, 128-token block), scale = amax / 448).
//
//   codes = E4M3_rn_satfinite(x * (448 / amax))     (448 / amax and the product
//   scale = amax / 448                               each rounded to float32;
//                                                    an all-zero block: scale 1)
//
// One CTA per (block, head): 16-byte loads of the block's bf16 values (kept in
// registers), a block-wide maximum of |x|, then cvt.rn.satfinite.e4m3x2 of
// each pair.  HBM-bound: 2 bytes read and 1 written per element.
#include <cuda_bf16.h>

#include "internal.cuh"

namespace bsa {
namespace {

constexpr int kThr = 256;

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  // cvt packs its first source into the upper byte
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// D / 8 16-byte vectors per token row; a block of at most 128 rows is 16 * D
// vectors, 8 * D / 128 per thread.
template <int D>
__global__ void __launch_bounds__(kThr) quantize_fp8_kernel(const __nv_bfloat16* __restrict__ x,
                                                            uint8_t* __restrict__ codes, float* __restrict__ scales,
                                                            int L, int blk, int NB) {
  constexpr int VPR = D / 8;                 // vectors per row
  constexpr int PER = 128 * VPR / kThr;      // vectors per thread (full block)
  const int j = blockIdx.x;
  const size_t bh = blockIdx.y;
  const int t0 = j * blk;
  const int n = min(blk, L - t0);
  const int nvec = n * VPR;
  const uint4* src = reinterpret_cast<const uint4*>(x + (bh * L + t0) * D);
  uint4 v[PER];
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int e = threadIdx.x + k * kThr;
    v[k] = e < nvec ? __ldg(src + e) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w[q] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w[q] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __shared__ float part[kThr / 32];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = part[0];
#pragma unroll
  for (int w = 1; w < kThr / 32; ++w) amax = fmaxf(amax, part[w]);
  const float inv = amax > 0.f ? 448.f / amax : 1.f;
  if (threadIdx.x == 0) scales[bh * NB + j] = amax > 0.f ? amax / 448.f : 1.f;
  uint2* dst = reinterpret_cast<uint2*>(codes + (bh * L + t0) * D);
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int e = threadIdx.x + k * kThr;
    if (e >= nvec) continue;
    const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
    uint32_t b[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      b[q] = e4m3x2(__uint_as_float(w[q] << 16) * inv, __uint_as_float(w[q] & 0xFFFF0000u) * inv);
    dst[e] = make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
  }
}

}  // namespace

cudaError_t launch_quantize_fp8(const bsa_shape& s, const __nv_bfloat16* x, uint8_t* codes, float* scales,
                                cudaStream_t st) {
  const int NB = n_blocks(s.L, s.blk);
  dim3 grid(NB, s.B * s.H);
  if (s.D == 128)
    quantize_fp8_kernel<128><<<grid, kThr, 0, st>>>(x, codes, scales, s.L, s.blk, NB);
  else
    quantize_fp8_kernel<64><<<grid, kThr, 0, st>>>(x, codes, scales, s.L, s.blk, NB);
  return cudaGetLastError();
}

}  // namespace bsa
