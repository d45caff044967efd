// host_common.cuh -- host helpers shared by every entry point: alignment,
// per-device lookups done once, and the test-hook settings
// (host code of libssscan.so; the library is one translation unit, ss_scan.cu)
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstdint>

namespace ssscan {
namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Test hooks (ss_scan_debug.h): consumed by the next ss_scan_fwd call.
std::atomic<long long> g_dbg_workers{0};
std::atomic<long long> g_dbg_skip_publish{-1};
std::atomic<long long> g_dbg_spin_limit{0};
std::atomic<long long> g_dbg_step_simple{0};
std::atomic<long long> g_dbg_segments{0};

// Per-device answers that never change, looked up once (every launch plans its
// schedule, and every workspace query plans all kernel variants).
constexpr int kDevCache = 64;

int device_sms() {
  static std::atomic<int> cache[kDevCache];
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kDevCache && (sms = cache[dev].load()) > 0) return sms;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kDevCache) cache[dev].store(sms);
  return sms;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Run `setup` (attribute settings of a kernel family) once per device: the
// dynamic shared memory limit is a per-device setting, so a process that
// drives several GPUs needs it on each.  `Tag` keeps one cache per family.
// Returns the cached value: 1 set up, -1 failed.
template <class Tag, class F>
int once_per_device(F setup) {
  static std::atomic<int> state[kDevCache];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (dev < 0 || dev >= kDevCache) return setup() ? 1 : -1;  // not cached
  int v = state[dev].load();
  if (v == 0) {
    v = setup() ? 1 : -1;  // idempotent: a concurrent first call may repeat it
    state[dev].store(v);
  }
  return v;
}

bool supported_dstate(int n) { return n == 16 || n == 32 || n == 64 || n == 128; }

}  // namespace
}  // namespace ssscan
