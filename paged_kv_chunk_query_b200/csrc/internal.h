// Internal definitions shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>
#include <vector>

#include "../../include/oomb.h"

// Device status word bits (see oomb_get_device_status).
#define OOMB_DEV_BAD_PAGE 1u
#define OOMB_DEV_WAIT_LIMIT 2u
#define OOMB_DEV_BAD_COUNT 4u

struct oomb_wb_engine;  // gradient write-back worker (offload.cu)

struct oomb_pool {
  oomb_pool_desc desc{};
  void* kv = nullptr;          // bf16 [pages][Hkv][2][P][d]
  float* grad = nullptr;       // fp32, same shape (optional)
  float* summary = nullptr;    // fp32 [pages][Hkv][d]
  uint32_t* d_status = nullptr;  // device status word (device and pinned pools)
  // kernel-side addresses of kv / grad (pinned pools: the mapped device
  // pointers of the host pages; device pools: kv / grad themselves)
  void* kv_dev = nullptr;
  float* grad_dev = nullptr;
  std::vector<int32_t> free_stack;  // top = back()
  std::vector<uint8_t> used;
  std::mutex mu;
  // gradient write-back engine (device pools), created on first use
  oomb_wb_engine* wb = nullptr;

  size_t block_elems() const {  // K+V of one (page, head)
    return static_cast<size_t>(2) * desc.page_size * desc.head_dim;
  }
  size_t kv_elems() const {
    return static_cast<size_t>(desc.num_pages) * desc.num_kv_heads * block_elems();
  }
  size_t summary_elems() const {
    return static_cast<size_t>(desc.num_pages) * desc.num_kv_heads * desc.head_dim;
  }
};

namespace oomb {

inline bool cuda_ok(cudaError_t e) { return e == cudaSuccess; }

// Maps the last CUDA error (sticky or not) to a status.
inline oomb_status check_launch() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? OOMB_OK : OOMB_ERR_CUDA;
}

inline bool supported_head_dim(int d) { return d == 64 || d == 128; }
inline bool supported_page_size(int p) { return p == 16 || p == 32 || p == 64 || p == 128; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Scoped device switch for calls on a pool's device.
struct DeviceGuard {
  int prev = -1;
  bool changed = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) {
      changed = cudaSetDevice(dev) == cudaSuccess;
    }
  }
  ~DeviceGuard() {
    if (changed) cudaSetDevice(prev);
  }
};

// Runs `set` (a per-device setting such as a kernel's shared-memory limit) the
// first time it is needed on the current device and remembers success in
// `done` (one bit per device ordinal < 64; later devices run it every call).
// Concurrent first calls may both run `set`, which must be idempotent.
template <class F>
inline bool once_per_device(std::atomic<uint64_t>& done, F set) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const uint64_t bit = dev >= 0 && dev < 64 ? (1ull << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return true;
  if (!set()) return false;
  if (bit) done.fetch_or(bit, std::memory_order_release);
  return true;
}

// Common validation of an attention call; fills the derived sizes.
struct AttnShape {
  int C, Hq, Hkv, G, D, P, n_qtiles, n_cur_pages;
};
void destroy_wb_engine(oomb_pool* pool);  // drains and joins the worker

oomb_status validate_attn(const oomb_pool* pool, const oomb_attn_args* a, bool backward,
                          AttnShape* s);

}  // namespace oomb
