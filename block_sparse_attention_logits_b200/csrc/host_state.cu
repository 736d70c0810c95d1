// Host-side per-device state shared by the launchers: the opt-in to more than
// 48 KB of dynamic shared memory, the SM count, and device addresses of the
// library's own device arrays.
//
// Each of these belongs to one device, and the first and last to one CUDA
// context of it: cudaFuncSetAttribute applies to the current device only, and
// after cudaDeviceReset the device's primary context (with the module and its
// arrays) is rebuilt, so attributes are lost and addresses may move.  Entries
// are therefore keyed by device ordinal and remember the context they were
// made in; a call under another context (a second device, or the same device
// after a reset) redoes the set-up.  The rules live in device_cache.h (plain
// C++, tested on the host with fake device calls); this file binds them to
// the CUDA runtime.
#include <cuda.h>
#include <cuda_runtime.h>

#include "device_cache.h"
#include "internal.cuh"

namespace bsa {
namespace {

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// The calling thread's current context (null before the runtime has made the
// device's primary context current, or without the driver entry point).
void* current_ctx() {
  CtxGetCurrentFn fn = ctx_get_current();
  CUcontext c = nullptr;
  if (fn && fn(&c) == CUDA_SUCCESS) return c;
  return nullptr;
}

int get_device(int* dev) { return static_cast<int>(cudaGetDevice(dev)); }
int set_smem(const void* func, size_t bytes) {
  return static_cast<int>(
      cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)));
}
int device_sms(int dev, int* n) {
  return static_cast<int>(cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev));
}
int lookup_symbol(const void* sym, void** addr) { return static_cast<int>(cudaGetSymbolAddress(addr, sym)); }

const DeviceOps kOps = {get_device, current_ctx, set_smem, device_sms, lookup_symbol,
                        static_cast<int>(cudaErrorInvalidDevice), static_cast<int>(cudaErrorUnknown)};
DeviceCache<64, 64, 4> g_cache;

}  // namespace

cudaError_t smem_opt_in(const void* func, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return static_cast<cudaError_t>(g_cache.smem_opt_in(kOps, func, bytes));
}

int sm_count() {
  int n = 0;
  return g_cache.sm_count(kOps, &n) == 0 ? n : 148;
}

int symbol_address(const void* symbol, void** out) {
  const int e = g_cache.symbol_address(kOps, symbol, out);
  if (e == static_cast<int>(cudaErrorInvalidDevice)) return BSA_ENODEV;
  return e == 0 ? BSA_OK : BSA_ECUDA;
}

}  // namespace bsa
