// Cached dense refinement (RECAP sections 1, 3.4, 4.3: a dense refresh renews
// the refinement that later sparse steps reuse) and its standalone
// alpha-scaled application (RECAP section 1 / abstract: fresh sparse
// statistics regulate how strongly the aging refinement is applied).
// Both are HBM-bound elementwise passes over 16-byte vectors of 8 bf16.
#include <cuda_bf16.h>

#include "internal.cuh"

namespace bsa {
namespace {

__device__ __forceinline__ float lo_bf(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(256) refresh_kernel(const uint4* __restrict__ od, const uint4* __restrict__ os,
                                                      uint4* __restrict__ R, long long nvec) {
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < nvec; i += static_cast<long long>(gridDim.x) * 256) {
    const uint4 a = __ldcs(od + i);
    const uint4 b = __ldcs(os + i);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) r[j] = pack2(lo_bf(aw[j]) - lo_bf(bw[j]), hi_bf(aw[j]) - hi_bf(bw[j]));
    R[i] = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

__global__ void __launch_bounds__(256) correct_kernel(const uint4* os, const uint4* __restrict__ R,
                                                      const float* __restrict__ alpha, uint4* o, long long nvec,
                                                      long long vec_per_head, int H) {
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < nvec; i += static_cast<long long>(gridDim.x) * 256) {
    const float a = __ldg(alpha + (i / vec_per_head) % H);
    const uint4 x = __ldcs(os + i);
    const uint4 y = __ldcs(R + i);
    const uint32_t xw[4] = {x.x, x.y, x.z, x.w}, yw[4] = {y.x, y.y, y.z, y.w};
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      r[j] = pack2(fmaf(a, lo_bf(yw[j]), lo_bf(xw[j])), fmaf(a, hi_bf(yw[j]), hi_bf(xw[j])));
    o[i] = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

unsigned grid_for(long long nvec) {
  long long b = (nvec + 255) / 256;
  const long long cap = 148ll * 16;
  return static_cast<unsigned>(b > cap ? cap : (b < 1 ? 1 : b));
}

}  // namespace

cudaError_t launch_refresh(size_t n, const __nv_bfloat16* od, const __nv_bfloat16* os, __nv_bfloat16* R,
                           cudaStream_t st) {
  const long long nvec = static_cast<long long>(n / 8);
  refresh_kernel<<<grid_for(nvec), 256, 0, st>>>(reinterpret_cast<const uint4*>(od),
                                                 reinterpret_cast<const uint4*>(os), reinterpret_cast<uint4*>(R),
                                                 nvec);
  return cudaGetLastError();
}

cudaError_t launch_correct(const bsa_shape& s, const __nv_bfloat16* os, const __nv_bfloat16* R, const float* alpha,
                           __nv_bfloat16* o, cudaStream_t st) {
  const long long vec_per_head = static_cast<long long>(s.L) * s.D / 8;
  const long long nvec = vec_per_head * s.B * s.H;
  correct_kernel<<<grid_for(nvec), 256, 0, st>>>(reinterpret_cast<const uint4*>(os),
                                                 reinterpret_cast<const uint4*>(R), alpha,
                                                 reinterpret_cast<uint4*>(o), nvec, vec_per_head, s.H);
  return cudaGetLastError();
}

}  // namespace bsa
