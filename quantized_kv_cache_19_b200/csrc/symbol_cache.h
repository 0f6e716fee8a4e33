// Device addresses of the library's own __device__ variables (the status word, the static scratch
// of the allocation-free entry point), remembered per device together with the id of the CUDA
// context they were looked up in.
//
// In host code the name of a __device__ variable is a host-side stand-in, not a device address;
// the address comes from cudaGetSymbolAddress and belongs to one context. After the context is
// destroyed (cudaDeviceReset, or a primary context released and re-created by another component of
// the process) the old address points at memory that no longer exists, so an entry is valid only
// while the current context is the one it was taken in: a lookup from any other context, or when
// the context id is unknown (0), asks again. Plain C++ (no CUDA types) so that the policy can be
// tested on a machine without a GPU. Thread-safe: one mutex guards every entry.
#pragma once

#include <mutex>

namespace qkv {

class SymbolAddressCache {
 public:
  static constexpr int kMaxDevices = 64;

  // Address for device `dev` in the context with unique id `ctx_id` (0 = unknown). `lookup(void**)`
  // fetches the address in the current context and returns 0 on success, else an error code that
  // get() passes on (the entry is then left as it was). Returns -1 for a device index out of range.
  template <class Lookup>
  int get(int dev, unsigned long long ctx_id, Lookup&& lookup, void** out) {
    if (dev < 0 || dev >= kMaxDevices) return -1;
    std::lock_guard<std::mutex> guard(mu_);
    Entry& e = entries_[dev];
    if (e.addr == nullptr || ctx_id == 0 || e.ctx != ctx_id) {
      void* p = nullptr;
      const int rc = lookup(&p);
      if (rc != 0) return rc;
      e.addr = p;
      e.ctx = ctx_id;
      ++lookups_;
    }
    *out = e.addr;
    return 0;
  }

  // Number of lookups made so far (for tests of the policy).
  long lookups() {
    std::lock_guard<std::mutex> guard(mu_);
    return lookups_;
  }

 private:
  struct Entry {
    unsigned long long ctx = 0;
    void* addr = nullptr;
  };
  std::mutex mu_;
  Entry entries_[kMaxDevices];
  long lookups_ = 0;
};

}  // namespace qkv
