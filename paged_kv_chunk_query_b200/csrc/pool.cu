// Page pools, page allocator, status and waits (host side of the C ABI).
//
// The KV cache and its gradients live in pages that need not be contiguous,
// so a chunk's keys are appended without reallocating or copying what is
// already stored ("Out of the Memory Barrier", [pt] §2B "Gerenciamento de KV
// Cache Paginado"; [it] §2B).  The pages say nothing about which free page is
// handed out next; this allocator keeps its free list as a stack (LIFO on
// free) that initially yields ids ascending, or in the order of a Fisher-Yates
// shuffle driven by SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) when a
// seed is given, so that page tables are reproducible bit for bit.
#include <chrono>
#include <cstdlib>
#include <cstring>
#include <new>
#include <thread>

#include "internal.h"

namespace {

uint64_t splitmix64_next(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ull;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

void release_buffers(oomb_pool* p) {
  const int loc = p->desc.location;
  auto free_one = [&](void* ptr) {
    if (!ptr) return;
    if (loc == OOMB_LOC_DEVICE) cudaFree(ptr);
    else if (loc == OOMB_LOC_PINNED_HOST) cudaFreeHost(ptr);
    else std::free(ptr);
  };
  free_one(p->kv);
  free_one(p->grad);
  if (loc == OOMB_LOC_PINNED_HOST) {
    if (p->summary) cudaFree(p->summary);
  } else {
    free_one(p->summary);
  }
  if (p->d_status) cudaFree(p->d_status);
  p->kv = nullptr;
  p->grad = nullptr;
  p->summary = nullptr;
  p->d_status = nullptr;
}

}  // namespace

extern "C" {

oomb_status oomb_pool_create(const oomb_pool_desc* desc, oomb_pool** out_pool) {
  if (!desc || !out_pool) return OOMB_ERR_INVALID_ARG;
  *out_pool = nullptr;
  if (desc->num_pages <= 0 || desc->num_kv_heads <= 0) return OOMB_ERR_INVALID_ARG;
  if (desc->location < OOMB_LOC_DEVICE || desc->location > OOMB_LOC_HOST)
    return OOMB_ERR_INVALID_ARG;
  if (!oomb::supported_head_dim(desc->head_dim) || !oomb::supported_page_size(desc->page_size))
    return OOMB_ERR_UNSUPPORTED;

  oomb_pool* p = new (std::nothrow) oomb_pool();
  if (!p) return OOMB_ERR_INVALID_ARG;
  p->desc = *desc;

  const size_t kv_bytes = p->kv_elems() * 2;
  const size_t grad_bytes = p->kv_elems() * 4;
  const size_t sum_bytes = p->summary_elems() * 4;
  bool ok = true;
  if (desc->location == OOMB_LOC_DEVICE) {
    oomb::DeviceGuard g(desc->device);
    ok = ok && cudaMalloc(&p->kv, kv_bytes) == cudaSuccess;
    ok = ok && cudaMemset(p->kv, 0, kv_bytes) == cudaSuccess;
    if (desc->with_grad) {
      ok = ok && cudaMalloc(reinterpret_cast<void**>(&p->grad), grad_bytes) == cudaSuccess;
      ok = ok && cudaMemset(p->grad, 0, grad_bytes) == cudaSuccess;
    }
    ok = ok && cudaMalloc(reinterpret_cast<void**>(&p->summary), sum_bytes) == cudaSuccess;
    ok = ok && cudaMemset(p->summary, 0, sum_bytes) == cudaSuccess;
    ok = ok && cudaMalloc(reinterpret_cast<void**>(&p->d_status), sizeof(uint32_t)) == cudaSuccess;
    ok = ok && cudaMemset(p->d_status, 0, sizeof(uint32_t)) == cudaSuccess;
    ok = ok && cudaDeviceSynchronize() == cudaSuccess;
    p->kv_dev = p->kv;
    p->grad_dev = p->grad;
  } else if (desc->location == OOMB_LOC_PINNED_HOST) {
    oomb::DeviceGuard g(desc->device);
    // mapped: the block-copy kernels read and write these pages directly over
    // the host link
    const unsigned flags = cudaHostAllocPortable | cudaHostAllocMapped;
    ok = ok && cudaHostAlloc(&p->kv, kv_bytes, flags) == cudaSuccess;
    if (desc->with_grad)
      ok = ok && cudaHostAlloc(reinterpret_cast<void**>(&p->grad), grad_bytes, flags) ==
                     cudaSuccess;
    ok = ok && cudaHostGetDevicePointer(&p->kv_dev, p->kv, 0) == cudaSuccess;
    if (ok && p->grad)
      ok = cudaHostGetDevicePointer(reinterpret_cast<void**>(&p->grad_dev), p->grad, 0) ==
           cudaSuccess;
    // Page representatives stay in device memory: Top-K reads them on the GPU.
    ok = ok && cudaMalloc(reinterpret_cast<void**>(&p->summary), sum_bytes) == cudaSuccess;
    ok = ok && cudaMemset(p->summary, 0, sum_bytes) == cudaSuccess;
    ok = ok && cudaMalloc(reinterpret_cast<void**>(&p->d_status), sizeof(uint32_t)) == cudaSuccess;
    ok = ok && cudaMemset(p->d_status, 0, sizeof(uint32_t)) == cudaSuccess;
    ok = ok && cudaDeviceSynchronize() == cudaSuccess;
    if (ok) {
      std::memset(p->kv, 0, kv_bytes);
      if (p->grad) std::memset(p->grad, 0, grad_bytes);
    }
  } else {
    p->kv = std::calloc(kv_bytes, 1);
    p->summary = static_cast<float*>(std::calloc(sum_bytes, 1));
    if (desc->with_grad) p->grad = static_cast<float*>(std::calloc(grad_bytes, 1));
    ok = p->kv && p->summary && (!desc->with_grad || p->grad);
  }
  if (!ok) {
    release_buffers(p);
    delete p;
    cudaGetLastError();  // do not leave a sticky allocation error behind
    return desc->location == OOMB_LOC_HOST ? OOMB_ERR_INVALID_ARG : OOMB_ERR_CUDA;
  }

  // Free list: order[0] is handed out first, so it goes on top of the stack.
  const int n = desc->num_pages;
  std::vector<int32_t> order(n);
  for (int i = 0; i < n; ++i) order[i] = i;
  if (desc->alloc_seed != 0) {
    uint64_t state = desc->alloc_seed;
    for (int i = n - 1; i > 0; --i) {
      const uint64_t j = splitmix64_next(state) % static_cast<uint64_t>(i + 1);
      std::swap(order[i], order[static_cast<int>(j)]);
    }
  }
  p->free_stack.assign(order.rbegin(), order.rend());
  p->used.assign(n, 0);
  *out_pool = p;
  return OOMB_OK;
}

oomb_status oomb_pool_destroy(oomb_pool* pool) {
  if (!pool) return OOMB_OK;
  {
    oomb::DeviceGuard g(pool->desc.device);
    if (pool->desc.location != OOMB_LOC_HOST) cudaDeviceSynchronize();
    oomb::destroy_wb_engine(pool);  // finishes queued gradient additions first
    release_buffers(pool);
  }
  delete pool;
  return OOMB_OK;
}

oomb_status oomb_pool_alloc_page(oomb_pool* pool, int32_t* out_page_id) {
  if (!pool || !out_page_id) return OOMB_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(pool->mu);
  if (pool->free_stack.empty()) return OOMB_ERR_OUT_OF_PAGES;
  const int32_t id = pool->free_stack.back();
  pool->free_stack.pop_back();
  pool->used[id] = 1;
  *out_page_id = id;
  return OOMB_OK;
}

oomb_status oomb_pool_free_page(oomb_pool* pool, int32_t page_id) {
  if (!pool) return OOMB_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(pool->mu);
  if (page_id < 0 || page_id >= pool->desc.num_pages || !pool->used[page_id])
    return OOMB_ERR_BAD_PAGE;
  pool->used[page_id] = 0;
  pool->free_stack.push_back(page_id);
  return OOMB_OK;
}

oomb_status oomb_pool_num_free(const oomb_pool* pool, int32_t* out_num_free) {
  if (!pool || !out_num_free) return OOMB_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(const_cast<oomb_pool*>(pool)->mu);
  *out_num_free = static_cast<int32_t>(pool->free_stack.size());
  return OOMB_OK;
}

oomb_status oomb_pool_buffers(const oomb_pool* pool, void** kv, float** grad, float** summary) {
  if (!pool) return OOMB_ERR_INVALID_ARG;
  if (kv) *kv = pool->kv;
  if (grad) *grad = pool->grad;
  if (summary) *summary = pool->summary;
  return OOMB_OK;
}

oomb_status oomb_pool_get_desc(const oomb_pool* pool, oomb_pool_desc* out_desc) {
  if (!pool || !out_desc) return OOMB_ERR_INVALID_ARG;
  *out_desc = pool->desc;
  return OOMB_OK;
}

oomb_status oomb_wait(void* event, int64_t timeout_us) {
  if (!event) return OOMB_ERR_INVALID_ARG;
  const auto t0 = std::chrono::steady_clock::now();
  cudaEvent_t ev = static_cast<cudaEvent_t>(event);
  while (true) {
    cudaError_t e = cudaEventQuery(ev);
    if (e == cudaSuccess) return OOMB_OK;
    if (e != cudaErrorNotReady) return OOMB_ERR_CUDA;
    const auto us = std::chrono::duration_cast<std::chrono::microseconds>(
                        std::chrono::steady_clock::now() - t0)
                        .count();
    if (us >= timeout_us) return OOMB_ERR_TIMEOUT;
    std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
}

oomb_status oomb_get_device_status(oomb_pool* pool, uint32_t* out_word) {
  if (!pool) return OOMB_ERR_INVALID_ARG;
  if (out_word) *out_word = 0;
  if (pool->desc.location == OOMB_LOC_HOST || !pool->d_status) return OOMB_OK;
  oomb::DeviceGuard g(pool->desc.device);
  uint32_t word = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return OOMB_ERR_CUDA;
  if (cudaMemcpy(&word, pool->d_status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return OOMB_ERR_CUDA;
  if (cudaMemset(pool->d_status, 0, sizeof(uint32_t)) != cudaSuccess) return OOMB_ERR_CUDA;
  if (out_word) *out_word = word;
  return word ? OOMB_ERR_DEVICE_CHECK : OOMB_OK;
}

const char* oomb_status_string(oomb_status status) {
  switch (status) {
    case OOMB_OK: return "ok";
    case OOMB_ERR_INVALID_ARG: return "invalid argument";
    case OOMB_ERR_OUT_OF_PAGES: return "out of pages";
    case OOMB_ERR_BAD_PAGE: return "bad page id";
    case OOMB_ERR_CUDA: return "CUDA error";
    case OOMB_ERR_TIMEOUT: return "timeout";
    case OOMB_ERR_UNSUPPORTED: return "unsupported shape";
    case OOMB_ERR_DEVICE_CHECK: return "device check failed";
  }
  return "unknown status";
}

int32_t oomb_version(void) { return 100; }

}  // extern "C"

namespace oomb {

oomb_status validate_attn(const oomb_pool* pool, const oomb_attn_args* a, bool backward,
                          AttnShape* s) {
  if (!pool || !a || !s) return OOMB_ERR_INVALID_ARG;
  if (pool->desc.location != OOMB_LOC_DEVICE) return OOMB_ERR_INVALID_ARG;
  const int P = pool->desc.page_size, D = pool->desc.head_dim, Hkv = pool->desc.num_kv_heads;
  if (a->chunk_len <= 0 || a->chunk_len % P != 0) return OOMB_ERR_INVALID_ARG;
  if (a->num_q_heads <= 0 || a->num_q_heads % Hkv != 0) return OOMB_ERR_INVALID_ARG;
  if (a->max_past < 0 || (a->max_past > 0 && (!a->past_pages || !a->past_counts)))
    return OOMB_ERR_INVALID_ARG;
  if (a->lists_per_qtile < 0 || a->lists_per_qtile > 2) return OOMB_ERR_INVALID_ARG;
  if (a->lists_per_qtile == 2 && a->max_past > 0 && !a->past_masks) return OOMB_ERR_INVALID_ARG;
  if (a->segment < OOMB_SEG_WHOLE || a->segment > OOMB_SEG_LAST) return OOMB_ERR_INVALID_ARG;
  if (a->segment != OOMB_SEG_WHOLE) {
    if (a->lists_per_qtile) return OOMB_ERR_INVALID_ARG;
    if (!a->o_acc || !aligned16(a->o_acc)) return OOMB_ERR_INVALID_ARG;
    if (backward && (!a->dq_acc || !aligned16(a->dq_acc))) return OOMB_ERR_INVALID_ARG;
  }
  if (!a->q || !a->o || !a->lse || !a->cur_pages) return OOMB_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->o)) return OOMB_ERR_INVALID_ARG;
  if (!backward && a->fwd_ws && !aligned16(a->fwd_ws)) return OOMB_ERR_INVALID_ARG;
  if (!(a->softmax_scale > 0.f)) return OOMB_ERR_INVALID_ARG;
  if (backward) {
    if (!a->d_o || !a->dq || !a->delta_ws || !pool->grad) return OOMB_ERR_INVALID_ARG;
    if (!aligned16(a->d_o) || !aligned16(a->dq)) return OOMB_ERR_INVALID_ARG;
  }
  s->C = a->chunk_len;
  s->Hq = a->num_q_heads;
  s->Hkv = Hkv;
  s->G = a->num_q_heads / Hkv;
  s->D = D;
  s->P = P;
  s->n_qtiles = (a->chunk_len + 127) / 128;
  s->n_cur_pages = a->chunk_len / P;
  return OOMB_OK;
}

}  // namespace oomb
