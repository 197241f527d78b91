// Offload: KV blocks between pinned host and device pools, gradient write-back.
//
// "Out of the Memory Barrier" ([pt] §2D "Offloading Assíncrono de KV Cache
// para CPU": dedicated CUDA streams and pinned memory move data between CPU
// and GPU while computation runs; for sparse attention the transfer overlaps
// other work because the page ids are known early; [es] §2B "Descarga
// Asíncrona a CPU": the KV cache AND its gradients are moved; [it] §2C).
//
// A block is the K and V of one (page, KV head): 2 * P * d values, contiguous
// in both pools.  Copies are issued as one cudaMemcpyAsync per run of blocks
// that are consecutive in both pools.  Gradient write-back copies the device
// blocks' fp32 gradients to a pinned staging slot (one copy per run of
// consecutive source blocks), zero-fills the device blocks for their next
// use, and hands the slot to a library worker thread that adds it into the
// host pool with several CPU threads once the copy has landed.
#include <algorithm>
#include <chrono>
#include <condition_variable>
#include <deque>
#include <mutex>
#include <thread>
#include <vector>

#include "internal.h"

namespace {

bool same_shape(const oomb_pool* a, const oomb_pool* b) {
  return a->desc.page_size == b->desc.page_size && a->desc.num_kv_heads == b->desc.num_kv_heads &&
         a->desc.head_dim == b->desc.head_dim;
}

bool blocks_valid(const oomb_pool* pool, const int32_t* blocks, int n) {
  const int64_t nb = static_cast<int64_t>(pool->desc.num_pages) * pool->desc.num_kv_heads;
  for (int i = 0; i < n; ++i)
    if (blocks[i] < 0 || blocks[i] >= nb) return false;
  return true;
}

// One pass over a destination list, in order: OOMB_ERR_BAD_PAGE at the first
// id outside the pool, OOMB_ERR_INVALID_ARG at the first id seen twice.
oomb_status distinct_blocks(const oomb_pool* pool, const int32_t* blocks, int n) {
  const int64_t nb = static_cast<int64_t>(pool->desc.num_pages) * pool->desc.num_kv_heads;
  std::vector<uint8_t> seen(static_cast<size_t>(nb), 0);
  for (int i = 0; i < n; ++i) {
    if (blocks[i] < 0 || blocks[i] >= nb) return OOMB_ERR_BAD_PAGE;
    if (seen[blocks[i]]) return OOMB_ERR_INVALID_ARG;
    seen[blocks[i]] = 1;
  }
  return OOMB_OK;
}

// Runs [i, j) with src and dst both consecutive.
template <class F>
void for_each_run(const int32_t* src, const int32_t* dst, int n, F f) {
  int i = 0;
  while (i < n) {
    int j = i + 1;
    while (j < n && src[j] == src[j - 1] + 1 && dst[j] == dst[j - 1] + 1) ++j;
    f(src[i], dst[i], j - i);
    i = j;
  }
}

int host_threads() {
  const unsigned hc = std::thread::hardware_concurrency();
  return static_cast<int>(std::max(1u, std::min(hc, 16u)));
}

}  // namespace

// Gradient write-back engine of a device pool: two pinned staging slots used
// in turn, and one worker thread that, job by job in submission order, waits
// for a slot's device->host copy to finish and adds the slot into the host
// pool with several CPU threads.  The worker never calls back into a stream,
// so the copy stream is not held up by the additions.  A job whose copy did
// not complete is not added: the worker only frees its slot and records the
// failure, which the next oomb_grad_writeback_sync reports.
struct oomb_wb_engine {
  struct Job {
    int slot;
    float* host_grad;           // nullptr: nothing to add, only wait and free the slot
    std::vector<int32_t> dst;
    size_t block_floats;
  };
  std::mutex mu;
  std::condition_variable cv;
  std::deque<Job> jobs;
  bool stop = false;
  int pending = 0;              // jobs submitted and not yet added
  bool failed = false;          // a job's copy failed since the last sync
  float* slot_ptr[2] = {nullptr, nullptr};
  size_t slot_bytes[2] = {0, 0};
  bool slot_busy[2] = {false, false};
  cudaEvent_t slot_ev[2] = {nullptr, nullptr};
  int next_slot = 0;
  int device = 0;
  // host-only self-test: no CUDA call; every copy "completes" with this status
  bool fake_copies = false;
  cudaError_t fake_copy_status = cudaSuccess;
  std::thread worker;

  cudaError_t wait_copy(int slot) {
    if (fake_copies) return fake_copy_status;
    return cudaEventSynchronize(slot_ev[slot]);
  }

  void run() {
    if (!fake_copies) cudaSetDevice(device);
    while (true) {
      Job job;
      {
        std::unique_lock<std::mutex> lk(mu);
        cv.wait(lk, [&] { return stop || !jobs.empty(); });
        if (jobs.empty()) return;
        job = std::move(jobs.front());
        jobs.pop_front();
      }
      const bool copied = wait_copy(job.slot) == cudaSuccess;
      if (copied && job.host_grad) {
        const float* stage = slot_ptr[job.slot];
        const size_t n = job.dst.size();
        const int T = std::max(1, std::min<int>(host_threads(), static_cast<int>(n)));
        auto work = [&](int t) {
          for (size_t b = t; b < n; b += T) {
            float* out = job.host_grad + static_cast<size_t>(job.dst[b]) * job.block_floats;
            const float* in = stage + b * job.block_floats;
            for (size_t e = 0; e < job.block_floats; ++e) out[e] += in[e];
          }
        };
        std::vector<std::thread> pool;
        for (int t = 1; t < T; ++t) pool.emplace_back(work, t);
        work(0);
        for (auto& th : pool) th.join();
      }
      {
        std::lock_guard<std::mutex> lk(mu);
        if (!copied) failed = true;
        slot_busy[job.slot] = false;
        --pending;
      }
      cv.notify_all();
    }
  }

  // Waits for every queued job; reports (and clears) a failed copy.
  oomb_status sync(int64_t timeout_us) {
    std::unique_lock<std::mutex> lk(mu);
    if (!cv.wait_for(lk, std::chrono::microseconds(timeout_us), [&] { return pending == 0; }))
      return OOMB_ERR_TIMEOUT;
    const bool f = failed;
    failed = false;
    return f ? OOMB_ERR_CUDA : OOMB_OK;
  }

  void shutdown() {
    {
      std::lock_guard<std::mutex> lk(mu);
      stop = true;
    }
    cv.notify_all();
    if (worker.joinable()) worker.join();
  }
};

namespace oomb {

void destroy_wb_engine(oomb_pool* pool) {
  oomb_wb_engine* e = pool->wb;
  if (!e) return;
  e->shutdown();
  for (int i = 0; i < 2; ++i) {
    if (e->slot_ptr[i]) cudaFreeHost(e->slot_ptr[i]);
    if (e->slot_ev[i]) cudaEventDestroy(e->slot_ev[i]);
  }
  delete e;
  pool->wb = nullptr;
}

}  // namespace oomb

namespace {

oomb_wb_engine* wb_engine(oomb_pool* pool) {
  if (!pool->wb) {
    oomb_wb_engine* e = new oomb_wb_engine();
    e->device = pool->desc.device;
    for (int i = 0; i < 2; ++i)
      if (cudaEventCreateWithFlags(&e->slot_ev[i], cudaEventDisableTiming) != cudaSuccess) {
        for (int k = 0; k < i; ++k) cudaEventDestroy(e->slot_ev[k]);
        delete e;
        return nullptr;
      }
    e->worker = std::thread([e] { e->run(); });
    pool->wb = e;
  }
  return pool->wb;
}

}  // namespace

extern "C" oomb_status oomb_page_prefetch(const oomb_pool* src_pool, oomb_pool* dst_pool,
                                          const int32_t* h_src_blocks,
                                          const int32_t* h_dst_blocks, int32_t n_blocks,
                                          void* stream, void* done_event) {
  if (!src_pool || !dst_pool || n_blocks < 0) return OOMB_ERR_INVALID_ARG;
  if (n_blocks > 0 && (!h_src_blocks || !h_dst_blocks)) return OOMB_ERR_INVALID_ARG;
  if (!same_shape(src_pool, dst_pool)) return OOMB_ERR_INVALID_ARG;
  const int ls = src_pool->desc.location, ld = dst_pool->desc.location;
  if (ls == OOMB_LOC_HOST || ld == OOMB_LOC_HOST) return OOMB_ERR_INVALID_ARG;
  if (!blocks_valid(src_pool, h_src_blocks, n_blocks) ||
      !blocks_valid(dst_pool, h_dst_blocks, n_blocks))
    return OOMB_ERR_BAD_PAGE;
  oomb::DeviceGuard guard(dst_pool->desc.location == OOMB_LOC_DEVICE ? dst_pool->desc.device
                                                                     : src_pool->desc.device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bbytes = src_pool->block_elems() * 2;
  const size_t sbytes = static_cast<size_t>(src_pool->desc.head_dim) * 4;
  const auto* sb = static_cast<const uint8_t*>(src_pool->kv);
  auto* db = static_cast<uint8_t*>(dst_pool->kv);
  bool ok = true;
  for_each_run(h_src_blocks, h_dst_blocks, n_blocks, [&](int s0, int d0, int len) {
    if (!ok) return;
    ok = cudaMemcpyAsync(db + d0 * bbytes, sb + s0 * bbytes, len * bbytes, cudaMemcpyDefault, s) ==
         cudaSuccess;
    // a block stored into a host pool takes its page representative along
    if (ok && ld == OOMB_LOC_PINNED_HOST)
      ok = cudaMemcpyAsync(reinterpret_cast<uint8_t*>(dst_pool->summary) + d0 * sbytes,
                           reinterpret_cast<const uint8_t*>(src_pool->summary) + s0 * sbytes,
                           len * sbytes, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
  });
  if (ok && done_event) ok = cudaEventRecord(static_cast<cudaEvent_t>(done_event), s) == cudaSuccess;
  return ok ? OOMB_OK : OOMB_ERR_CUDA;
}

extern "C" oomb_status oomb_grad_writeback(oomb_pool* device_pool, oomb_pool* host_pool,
                                           const int32_t* h_src_blocks,
                                           const int32_t* h_dst_blocks, int32_t n_blocks,
                                           void* stream) {
  if (!device_pool || !host_pool || n_blocks < 0) return OOMB_ERR_INVALID_ARG;
  if (n_blocks == 0) return OOMB_OK;
  if (!h_src_blocks || !h_dst_blocks) return OOMB_ERR_INVALID_ARG;
  if (!same_shape(device_pool, host_pool)) return OOMB_ERR_INVALID_ARG;
  if (!blocks_valid(device_pool, h_src_blocks, n_blocks)) return OOMB_ERR_BAD_PAGE;
  // the worker's CPU threads add different blocks at once: a destination
  // listed twice would lose one of its additions
  const oomb_status dst_ok = distinct_blocks(host_pool, h_dst_blocks, n_blocks);
  if (dst_ok != OOMB_OK) return dst_ok;
  if (device_pool->desc.location != OOMB_LOC_DEVICE ||
      host_pool->desc.location != OOMB_LOC_PINNED_HOST || !device_pool->grad || !host_pool->grad)
    return OOMB_ERR_INVALID_ARG;
  oomb::DeviceGuard guard(device_pool->desc.device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bfloats = device_pool->block_elems();
  const size_t need = static_cast<size_t>(n_blocks) * bfloats * 4;
  oomb_wb_engine* e = wb_engine(device_pool);
  if (!e) return OOMB_ERR_CUDA;
  int slot;
  {
    // take the next staging slot once the worker has finished adding from it
    std::unique_lock<std::mutex> lk(e->mu);
    slot = e->next_slot;
    if (!e->cv.wait_for(lk, std::chrono::seconds(120), [&] { return !e->slot_busy[slot]; }))
      return OOMB_ERR_TIMEOUT;
    e->next_slot ^= 1;
    if (e->slot_bytes[slot] < need) {
      if (e->slot_ptr[slot]) cudaFreeHost(e->slot_ptr[slot]);
      e->slot_ptr[slot] = nullptr;
      e->slot_bytes[slot] = 0;
      if (cudaHostAlloc(reinterpret_cast<void**>(&e->slot_ptr[slot]), need,
                        cudaHostAllocPortable) != cudaSuccess)
        return OOMB_ERR_CUDA;
      e->slot_bytes[slot] = need;
    }
    e->slot_busy[slot] = true;
  }
  float* stage = e->slot_ptr[slot];
  bool ok = true;
  // device -> pinned slot in list order, one copy per run of consecutive source blocks
  int done = 0;
  for (int i = 0; i < n_blocks && ok;) {
    int j = i + 1;
    while (j < n_blocks && h_src_blocks[j] == h_src_blocks[j - 1] + 1) ++j;
    ok = cudaMemcpyAsync(stage + static_cast<size_t>(done) * bfloats,
                         device_pool->grad + static_cast<size_t>(h_src_blocks[i]) * bfloats,
                         (j - i) * bfloats * 4, cudaMemcpyDeviceToHost, s) == cudaSuccess;
    done += j - i;
    i = j;
  }
  const bool copies_ok = ok;
  const bool recorded = cudaEventRecord(e->slot_ev[slot], s) == cudaSuccess;
  if (!copies_ok || !recorded) {
    // Nothing is added and no device block is zeroed: the device gradients
    // stay as they were.  Copies already queued may still be writing into
    // the slot, so it stays busy until they are done.
    if (recorded) {
      std::lock_guard<std::mutex> lk(e->mu);
      e->jobs.push_back(oomb_wb_engine::Job{slot, nullptr, {}, bfloats});
      ++e->pending;
    } else {
      cudaStreamSynchronize(s);
      std::lock_guard<std::mutex> lk(e->mu);
      e->slot_busy[slot] = false;
    }
    e->cv.notify_all();
    return OOMB_ERR_CUDA;
  }
  {
    std::lock_guard<std::mutex> lk(e->mu);
    e->jobs.push_back(oomb_wb_engine::Job{
        slot, host_pool->grad, std::vector<int32_t>(h_dst_blocks, h_dst_blocks + n_blocks),
        bfloats});
    ++e->pending;
  }
  e->cv.notify_all();
  // The device blocks start from zero for their next contributions; the
  // copies ahead of these fills on the stream have captured the values.
  for (int i = 0; i < n_blocks && ok;) {
    int j = i + 1;
    while (j < n_blocks && h_src_blocks[j] == h_src_blocks[j - 1] + 1) ++j;
    ok = cudaMemsetAsync(device_pool->grad + static_cast<size_t>(h_src_blocks[i]) * bfloats, 0,
                         (j - i) * bfloats * 4, s) == cudaSuccess;
    i = j;
  }
  return ok ? OOMB_OK : OOMB_ERR_CUDA;
}

extern "C" oomb_status oomb_grad_writeback_sync(oomb_pool* device_pool, int64_t timeout_us) {
  if (!device_pool) return OOMB_ERR_INVALID_ARG;
  oomb_wb_engine* e = device_pool->wb;
  if (!e) return OOMB_OK;
  return e->sync(timeout_us);
}

extern "C" oomb_status oomb_selftest_writeback_copy(float* host_grad, int32_t n_blocks,
                                                    int32_t block_floats, int32_t fail_copy) {
  if (!host_grad || n_blocks <= 0 || block_floats <= 0) return OOMB_ERR_INVALID_ARG;
  // A host-only engine: its staging slot holds 1.0 in every element and its
  // copy "completes" with success or with an error, as asked.
  oomb_wb_engine e;
  e.fake_copies = true;
  e.fake_copy_status = fail_copy ? cudaErrorLaunchFailure : cudaSuccess;
  const size_t nf = static_cast<size_t>(n_blocks) * block_floats;
  std::vector<float> slot(nf, 1.0f);
  e.slot_ptr[0] = slot.data();
  e.slot_bytes[0] = nf * 4;
  e.slot_busy[0] = true;
  std::vector<int32_t> dst(n_blocks);
  for (int i = 0; i < n_blocks; ++i) dst[i] = i;
  e.worker = std::thread([&e] { e.run(); });
  {
    std::lock_guard<std::mutex> lk(e.mu);
    e.jobs.push_back(oomb_wb_engine::Job{0, host_grad, dst, static_cast<size_t>(block_floats)});
    ++e.pending;
  }
  e.cv.notify_all();
  const oomb_status st = e.sync(10'000'000);
  e.shutdown();
  e.slot_ptr[0] = nullptr;
  return st;
}
