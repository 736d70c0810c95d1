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
// after a reset) redoes the set-up.  Every table is guarded by one mutex, so
// host threads may launch concurrently.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.cuh"

namespace bsa {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxFuncs = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

std::mutex g_mu;

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
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

struct OptIn {
  const void* func;
  void* ctx;
  size_t bytes;
};
OptIn g_optin[kMaxDevices][kMaxFuncs];
int g_sms[kMaxDevices];
void* g_sym_ctx[kMaxDevices][4];
void* g_sym_addr[kMaxDevices][4];
const void* g_sym_key[4];

}  // namespace

cudaError_t smem_opt_in(const void* func, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  void* ctx = current_ctx();
  OptIn* slot = nullptr;
  for (OptIn& o : g_optin[dev]) {
    if (o.func == func) {
      slot = &o;
      break;
    }
    if (!slot && o.func == nullptr) slot = &o;  // first free entry, used if func is new
  }
  if (!slot) return cudaErrorUnknown;  // more kernels than the table holds (not reached: < 20 kernels)
  if (slot->func == func && ctx != nullptr && slot->ctx == ctx && slot->bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  slot->func = func;
  slot->ctx = current_ctx();  // the attribute call made the primary context current if it was not
  slot->bytes = slot->ctx == ctx ? (bytes > slot->bytes ? bytes : slot->bytes) : bytes;
  return cudaSuccess;
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_sms[dev] <= 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

int symbol_address(const void* symbol, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSA_ENODEV;
  std::lock_guard<std::mutex> lock(g_mu);
  int k = 0;
  for (; k < 4; ++k)
    if (g_sym_key[k] == symbol || g_sym_key[k] == nullptr) break;
  if (k == 4) return BSA_ECUDA;
  g_sym_key[k] = symbol;
  void* ctx = current_ctx();
  if (g_sym_addr[dev][k] == nullptr || ctx == nullptr || g_sym_ctx[dev][k] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess || p == nullptr) return BSA_ECUDA;
    g_sym_addr[dev][k] = p;
    g_sym_ctx[dev][k] = current_ctx();
  }
  *out = g_sym_addr[dev][k];
  return BSA_OK;
}

}  // namespace bsa
