// Hilbert-curve token order and token permutation (DFSAttn abstract:
// Hilbert curve-based token reordering for fine-grained block sparsity).
//
// The curve is J. Skilling's n-dimensional Hilbert curve ("Programming the
// Hilbert curve", AIP Conf. Proc. 707, 2004) on the smallest 2^k cube that
// holds the (T, Hh, W) grid, axes (t, y, x) with t most significant.  Instead
// of computing an index per token and sorting, the GPU walks the curve: for
// every cube index d it decodes the point (Skilling's transpose -> axes
// direction) and, if the point lies inside the grid, emits it at its rank.
// Ranks come from a two-pass stream compaction over chunks of the index
// range: pass 1 counts grid points per chunk into the caller's workspace,
// pass 2 adds up the counts of the preceding chunks and writes perm / inv.

#include "internal.cuh"

namespace bsa {
namespace {

constexpr int kChunk = 4096;   // cube indices per CTA
constexpr int kThr = 256;      // threads per CTA
constexpr int kPer = kChunk / kThr;
constexpr int kMaxExtent = 256;  // => at most 2^24 cube cells

int cube_bits(int T, int Hh, int W) {
  int m = T > Hh ? T : Hh;
  m = m > W ? m : W;
  int k = 1;
  while ((1 << k) < m) ++k;
  return k;
}

// Hilbert index d (3*k bits) -> axes (t, y, x).
__device__ __forceinline__ void hilbert_axes(uint32_t d, int k, uint32_t& a0, uint32_t& a1, uint32_t& a2) {
  // de-interleave: at level b the bits of axes 0, 1, 2 sit at 3b+2, 3b+1, 3b
  uint32_t x[3] = {0u, 0u, 0u};
  for (int b = 0; b < k; ++b) {
    x[0] |= ((d >> (3 * b + 2)) & 1u) << b;
    x[1] |= ((d >> (3 * b + 1)) & 1u) << b;
    x[2] |= ((d >> (3 * b)) & 1u) << b;
  }
  // Gray decode
  uint32_t t = x[2] >> 1;
  x[2] ^= x[1];
  x[1] ^= x[0];
  x[0] ^= t;
  // undo excess work, from the lowest level upwards
  const uint32_t top = 2u << (k - 1);
  for (uint32_t q = 2; q != top; q <<= 1) {
    const uint32_t p = q - 1;
    for (int i = 2; i >= 0; --i) {
      if (x[i] & q) {
        x[0] ^= p;
      } else {
        t = (x[0] ^ x[i]) & p;
        x[0] ^= t;
        x[i] ^= t;
      }
    }
  }
  a0 = x[0];
  a1 = x[1];
  a2 = x[2];
}

__device__ __forceinline__ bool in_grid(uint32_t d, int k, int T, int Hh, int W, int& flat) {
  uint32_t t, y, x;
  hilbert_axes(d, k, t, y, x);
  if (t >= static_cast<uint32_t>(T) || y >= static_cast<uint32_t>(Hh) || x >= static_cast<uint32_t>(W)) return false;
  flat = (static_cast<int>(t) * Hh + static_cast<int>(y)) * W + static_cast<int>(x);
  return true;
}

__device__ __forceinline__ int block_exclusive_scan(int v, int* sh, int& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh[w] = incl;
  __syncthreads();
  if (w == 0) {
    int s = lane < kThr / 32 ? sh[lane] : 0;
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += y;
    }
    if (lane < kThr / 32) sh[lane] = si - s;
    if (lane == kThr / 32 - 1) sh[kThr / 32] = si;
  }
  __syncthreads();
  total = sh[kThr / 32];
  const int r = sh[w] + incl - v;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kThr) hilbert_count_kernel(int k, int T, int Hh, int W, uint32_t cells,
                                                             int* __restrict__ counts) {
  __shared__ int sh[kThr / 32 + 1];
  const uint32_t d0 = blockIdx.x * kChunk + threadIdx.x * kPer;
  int c = 0;
  for (int e = 0; e < kPer; ++e) {
    int flat;
    if (d0 + e < cells && in_grid(d0 + e, k, T, Hh, W, flat)) ++c;
  }
  int total;
  block_exclusive_scan(c, sh, total);
  if (threadIdx.x == 0) counts[blockIdx.x] = total;
}

__global__ void __launch_bounds__(kThr) hilbert_emit_kernel(int k, int T, int Hh, int W, uint32_t cells,
                                                            const int* __restrict__ counts, int32_t* __restrict__ perm,
                                                            int32_t* __restrict__ inv) {
  __shared__ int sh[kThr / 32 + 1];
  __shared__ int base_sh;
  // rank of this chunk's first grid point = points in all earlier chunks
  int part = 0;
  for (int c = threadIdx.x; c < static_cast<int>(blockIdx.x); c += kThr) part += counts[c];
  int total;
  block_exclusive_scan(part, sh, total);
  if (threadIdx.x == 0) base_sh = total;
  __syncthreads();
  const int base = base_sh;
  const uint32_t d0 = blockIdx.x * kChunk + threadIdx.x * kPer;
  int flats[kPer];
  int c = 0;
  for (int e = 0; e < kPer; ++e) {
    int flat = -1;
    if (d0 + e < cells && in_grid(d0 + e, k, T, Hh, W, flat)) ++c;
    flats[e] = flat;
  }
  int chunk_total;
  int rank = base + block_exclusive_scan(c, sh, chunk_total);
  for (int e = 0; e < kPer; ++e) {
    if (flats[e] >= 0) {
      perm[rank] = flats[e];
      inv[flats[e]] = rank;
      ++rank;
    }
  }
}

template <int VEC>
__global__ void __launch_bounds__(256) permute_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm,
                                                      uint4* __restrict__ y, long long BH, int L, int inverse) {
  // VEC = D / 8 sixteen-byte vectors per token row
  const long long total = BH * L * VEC;
  for (long long idx = blockIdx.x * 256ll + threadIdx.x; idx < total; idx += static_cast<long long>(gridDim.x) * 256) {
    const int vec = static_cast<int>(idx % VEC);
    const long long rowflat = idx / VEC;
    const int i = static_cast<int>(rowflat % L);
    const long long bh = rowflat / L;
    const int pi = __ldg(perm + i);
    const long long src = inverse ? i : pi;
    const long long dst = inverse ? pi : i;
    y[(bh * L + dst) * VEC + vec] = __ldg(x + (bh * L + src) * VEC + vec);
  }
}

__global__ void __launch_bounds__(256) permute_kernel_any(const uint4* __restrict__ x,
                                                          const int32_t* __restrict__ perm, uint4* __restrict__ y,
                                                          long long BH, int L, int vecs, int inverse) {
  const long long total = BH * L * vecs;
  for (long long idx = blockIdx.x * 256ll + threadIdx.x; idx < total; idx += static_cast<long long>(gridDim.x) * 256) {
    const int vec = static_cast<int>(idx % vecs);
    const long long rowflat = idx / vecs;
    const int i = static_cast<int>(rowflat % L);
    const long long bh = rowflat / L;
    const int pi = __ldg(perm + i);
    const long long src = inverse ? i : pi;
    const long long dst = inverse ? pi : i;
    y[(bh * L + dst) * vecs + vec] = __ldg(x + (bh * L + src) * vecs + vec);
  }
}

}  // namespace

size_t hilbert_workspace_bytes(int T, int Hh, int W) {
  if (T < 1 || Hh < 1 || W < 1 || T > kMaxExtent || Hh > kMaxExtent || W > kMaxExtent) return 0;
  const int k = cube_bits(T, Hh, W);
  const uint64_t cells = 1ull << (3 * k);
  const uint64_t chunks = (cells + kChunk - 1) / kChunk;
  return static_cast<size_t>(chunks * sizeof(int));
}

cudaError_t launch_hilbert(int T, int Hh, int W, int32_t* perm, int32_t* inv, void* ws, cudaStream_t st) {
  const int k = cube_bits(T, Hh, W);
  const uint32_t cells = 1u << (3 * k);
  const unsigned chunks = (cells + kChunk - 1) / kChunk;
  int* counts = static_cast<int*>(ws);
  hilbert_count_kernel<<<chunks, kThr, 0, st>>>(k, T, Hh, W, cells, counts);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  hilbert_emit_kernel<<<chunks, kThr, 0, st>>>(k, T, Hh, W, cells, counts, perm, inv);
  return cudaGetLastError();
}

cudaError_t launch_permute(const bsa_shape& s, const __nv_bfloat16* x, const int32_t* perm, __nv_bfloat16* y,
                           int inverse, cudaStream_t st) {
  const long long BH = static_cast<long long>(s.B) * s.H;
  const int vecs = s.D / 8;
  const long long total = BH * s.L * vecs;
  long long blocks = (total + 255) / 256;
  const long long cap = 148ll * 16;
  if (blocks > cap) blocks = cap;
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  uint4* yv = reinterpret_cast<uint4*>(y);
  if (vecs == 16)
    permute_kernel<16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(xv, perm, yv, BH, s.L, inverse);
  else if (vecs == 8)
    permute_kernel<8><<<static_cast<unsigned>(blocks), 256, 0, st>>>(xv, perm, yv, BH, s.L, inverse);
  else
    permute_kernel_any<<<static_cast<unsigned>(blocks), 256, 0, st>>>(xv, perm, yv, BH, s.L, vecs, inverse);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free variant (bsa_reorder_tokens_noalloc).
//
// Some callers cannot allocate device memory for the two-pass scratch: a host
// framework that owns all device memory through its own allocator and hands
// this library only its input and output buffers, with no way to ask for more;
// a process whose caching allocator has already reserved nearly all of HBM, so
// a fresh cudaMalloc can fail; or a latency-critical loop that cannot afford
// cudaMalloc's implicit device synchronisation.  For them the per-chunk counts
// live in a file-scope device array instead of a caller workspace.
//
// Limit: kNoAllocChunks counts (16 KB), which covers every grid this call
// accepts (extents <= 256, so at most 2^24 cube cells = 4096 chunks).  Every
// GPU that loads the library holds the array until the process exits.
// Nothing in it has to start at zero: pass 1 writes every count pass 2 reads.
// All calls share the array and it keeps the last call's counts, so calls
// that overlap on the GPU (two streams, two host threads) race: serialise them.
constexpr int kNoAllocChunks = 4096;
static __device__ __align__(256) int g_reorder_counts[kNoAllocChunks];

}  // namespace bsa

extern "C" int bsa_reorder_tokens_noalloc(int T, int Hh, int W, int32_t* perm, int32_t* inv, bsa_stream stream) {
  if (!perm || !inv) return BSA_EINVAL;
  const size_t need = bsa::hilbert_workspace_bytes(T, Hh, W);
  if (need == 0 || need > sizeof(int) * static_cast<size_t>(bsa::kNoAllocChunks)) return BSA_ESHAPE;
  if ((reinterpret_cast<uintptr_t>(perm) & 15u) || (reinterpret_cast<uintptr_t>(inv) & 15u)) return BSA_EINVAL;
  int major = 0, dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10)
    return BSA_ENODEV;
  // Device address of g_reorder_counts on the current device: in host code
  // the array's name is only a host-side stand-in.  Looked up by the first
  // call on each device (make that call before any stream capture) and again
  // whenever the device's context has changed (after cudaDeviceReset).
  void* counts = nullptr;
  if (int r = bsa::symbol_address(reinterpret_cast<const void*>(&bsa::g_reorder_counts), &counts)) return r;
  return bsa::launch_hilbert(T, Hh, W, perm, inv, counts, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? BSA_OK
             : BSA_ECUDA;
}
