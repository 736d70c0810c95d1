// Per-device, per-context host tables of the launchers, as plain C++ with the
// device calls passed in, so that the caching rules can be tested on a host
// without a GPU (tests/test_device_cache.py builds this header with fake
// calls).  host_state.cu instantiates it with the CUDA runtime.
//
// Rules:
//   * an opt-in to a kernel's dynamic shared memory holds for one device and
//     one context: a call on another device, or on the same device under
//     another context (after cudaDeviceReset), sets the attribute again, and
//     so does a call asking for more bytes than were set;
//   * a device array's address is looked up again when the context differs
//     from the one it was looked up in;
//   * the SM count is read once per device.
// Every method takes the table's mutex, so host threads may call
// concurrently.  Return values: 0 on success, else the failing call's code.
#pragma once

#include <cstddef>
#include <mutex>

namespace bsa {

struct DeviceOps {
  int (*get_device)(int* dev);                         // current device ordinal
  void* (*current_ctx)();                              // current context (may be null)
  int (*set_smem)(const void* func, size_t bytes);     // dynamic shared memory opt-in
  int (*sm_count)(int dev, int* n);                    // number of SMs of a device
  int (*symbol_address)(const void* sym, void** addr); // device address of a library array
  int invalid_device;                                  // code for an ordinal outside the table
  int table_full;                                      // code for a full table
};

template <int kMaxDevices, int kMaxFuncs, int kMaxSymbols>
class DeviceCache {
 public:
  int smem_opt_in(const DeviceOps& ops, const void* func, size_t bytes) {
    int dev = -1;
    if (int e = ops.get_device(&dev)) return e;
    if (dev < 0 || dev >= kMaxDevices) return ops.invalid_device;
    std::lock_guard<std::mutex> lock(mu_);
    void* ctx = ops.current_ctx();
    OptIn* slot = nullptr;
    for (OptIn& o : optin_[dev]) {
      if (o.func == func) {
        slot = &o;
        break;
      }
      if (!slot && o.func == nullptr) slot = &o;  // first free entry, used if func is new
    }
    if (!slot) return ops.table_full;
    if (slot->func == func && ctx != nullptr && slot->ctx == ctx && slot->bytes >= bytes) return 0;
    if (int e = ops.set_smem(func, bytes)) return e;
    // the attribute now holds exactly `bytes`; the call makes the primary
    // context current if none was
    slot->func = func;
    slot->ctx = ops.current_ctx();
    slot->bytes = bytes;
    return 0;
  }

  int sm_count(const DeviceOps& ops, int* n) {
    int dev = -1;
    if (int e = ops.get_device(&dev)) return e;
    if (dev < 0 || dev >= kMaxDevices) return ops.invalid_device;
    std::lock_guard<std::mutex> lock(mu_);
    if (sms_[dev] <= 0) {
      int m = 0;
      if (int e = ops.sm_count(dev, &m)) return e;
      if (m <= 0) return ops.invalid_device;
      sms_[dev] = m;
    }
    *n = sms_[dev];
    return 0;
  }

  int symbol_address(const DeviceOps& ops, const void* sym, void** out) {
    int dev = -1;
    if (int e = ops.get_device(&dev)) return e;
    if (dev < 0 || dev >= kMaxDevices) return ops.invalid_device;
    std::lock_guard<std::mutex> lock(mu_);
    int k = 0;
    for (; k < kMaxSymbols; ++k)
      if (sym_key_[k] == sym || sym_key_[k] == nullptr) break;
    if (k == kMaxSymbols) return ops.table_full;
    sym_key_[k] = sym;
    void* ctx = ops.current_ctx();
    Sym& s = sym_[dev][k];
    if (s.addr == nullptr || ctx == nullptr || s.ctx != ctx) {
      void* p = nullptr;
      if (int e = ops.symbol_address(sym, &p)) return e;
      if (p == nullptr) return ops.table_full;
      s.addr = p;
      s.ctx = ops.current_ctx();
    }
    *out = s.addr;
    return 0;
  }

 private:
  struct OptIn {
    const void* func = nullptr;
    void* ctx = nullptr;
    size_t bytes = 0;
  };
  struct Sym {
    void* ctx = nullptr;
    void* addr = nullptr;
  };
  std::mutex mu_;
  OptIn optin_[kMaxDevices][kMaxFuncs];
  int sms_[kMaxDevices] = {};
  Sym sym_[kMaxDevices][kMaxSymbols];
  const void* sym_key_[kMaxSymbols] = {};
};

}  // namespace bsa
