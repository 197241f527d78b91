// Block movement kernels driven by block lists in device memory.
//
// "Out of the Memory Barrier" ([pt] §2D "Offloading Assíncrono de KV Cache
// para CPU": pinned memory and dedicated streams move pages while computation
// runs, and for sparse attention the page ids are known ahead of the compute,
// so the transfer hides under it; [es] §2B "Descarga Asíncrona a CPU": the KV
// cache AND its gradients are offloaded; [it] §2C).
//
// On this GPU the ids of a sparse step are known on the device as soon as
// Top-K has run.  So the lists are built there (prefetch_lists_kernel) and the
// moves run as kernels that read or write pinned host pages in place (mapped
// memory over the host link): one launch per list instead of one copy per
// block, and no host round trip between Top-K and the prefetch.  Between two
// device pools the same kernels are HBM gathers / scatter-adds.
//
// A block is the K and V of one (page, KV head): 2 * P * d values, contiguous.
//   block_copy_kernel   dst.kv[d_i] = src.kv[s_i], dst.summary[d_i] = src.summary[s_i]
//   grad_add_kernel     dst.grad[d_i] += src.grad[s_i]; optionally src.grad[s_i] = 0
//   prefetch_lists_kernel  selection -> (src, dst) block lists + staging page lists
// Entries with a negative id are padding and skipped; an id beyond its pool
// sets the device status bit and is skipped.
#include "internal.h"

namespace {

constexpr int kMoveThreads = 256;
constexpr int kUnroll = 4;  // 16-byte accesses in flight per thread

int sm_count(int device) {
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0)
    n = 148;
  return n;
}

// grid size: a few CTAs already saturate the host link (measured on B200:
// 8 CTAs copy at 51 GB/s, 16 add at 40 GB/s each way), and fewer CTAs leave
// more SMs to the attention kernels these moves run beside; an HBM gather
// wants several CTAs per SM.
int move_grid(int n_blocks, bool over_host_link, bool read_modify_write, int device) {
  const int cap = over_host_link ? (read_modify_write ? 16 : 8) : 4 * sm_count(device);
  return n_blocks < cap ? n_blocks : cap;
}

__device__ __forceinline__ bool block_ok(int id, int nb, uint32_t* status) {
  if (id < nb) return true;
  if (threadIdx.x == 0) atomicOr(status, OOMB_DEV_BAD_PAGE);
  return false;
}

__global__ void __launch_bounds__(kMoveThreads) block_copy_kernel(
    const uint4* __restrict__ src, uint4* __restrict__ dst, const float* __restrict__ src_sum,
    float* __restrict__ dst_sum, const int32_t* __restrict__ sb, const int32_t* __restrict__ db,
    int n, int src_nb, int dst_nb, int vec_per_block, int sum_per_block, uint32_t* status) {
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    const int s = sb[i], d = db[i];
    if (s < 0 || d < 0) continue;  // padding
    if (!block_ok(s, src_nb, status) || !block_ok(d, dst_nb, status)) continue;
    const uint4* in = src + static_cast<size_t>(s) * vec_per_block;
    uint4* out = dst + static_cast<size_t>(d) * vec_per_block;
    for (int base = threadIdx.x; base < vec_per_block; base += kUnroll * kMoveThreads) {
      uint4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int e = base + u * kMoveThreads;
        if (e < vec_per_block) v[u] = in[e];
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int e = base + u * kMoveThreads;
        if (e < vec_per_block) out[e] = v[u];
      }
    }
    for (int e = threadIdx.x; e < sum_per_block; e += kMoveThreads)
      dst_sum[static_cast<size_t>(d) * sum_per_block + e] =
          src_sum[static_cast<size_t>(s) * sum_per_block + e];
  }
}

// kAtomic: the destination is device memory, added with vector atomics (so
// repeated destination ids stay correct); otherwise (pinned host pages) a
// plain read-modify-write, which needs distinct destinations.
template <bool kAtomic>
__global__ void __launch_bounds__(kMoveThreads) grad_add_kernel(
    float4* __restrict__ src, float4* __restrict__ dst, const int32_t* __restrict__ sb,
    const int32_t* __restrict__ db, int n, int src_nb, int dst_nb, int vec_per_block,
    int zero_src, uint32_t* status) {
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    const int s = sb[i], d = db[i];
    if (s < 0 || d < 0) continue;
    if (!block_ok(s, src_nb, status) || !block_ok(d, dst_nb, status)) continue;
    float4* in = src + static_cast<size_t>(s) * vec_per_block;
    float4* out = dst + static_cast<size_t>(d) * vec_per_block;
    for (int base = threadIdx.x; base < vec_per_block; base += kUnroll * kMoveThreads) {
      float4 a[kUnroll], b[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int e = base + u * kMoveThreads;
        if (e < vec_per_block) {
          a[u] = in[e];
          if (!kAtomic) b[u] = out[e];
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int e = base + u * kMoveThreads;
        if (e < vec_per_block) {
          if (kAtomic) {
            atomicAdd(out + e, a[u]);
          } else {
            out[e] = make_float4(b[u].x + a[u].x, b[u].y + a[u].y, b[u].z + a[u].z,
                                 b[u].w + a[u].w);
          }
          if (zero_src) in[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
  }
}

// One thread per entry e = i * Hkv + g (slot-major: the blocks of slot i are
// consecutive in the staging pool).
__global__ void prefetch_lists_kernel(const int32_t* __restrict__ sel_logical,
                                      const int32_t* __restrict__ sel_count, int max_sel, int Hkv,
                                      const int32_t* __restrict__ page_table, int table_len,
                                      int src_pages, const int32_t* __restrict__ slot_pages,
                                      int dst_pages, int32_t* __restrict__ src_blocks,
                                      int32_t* __restrict__ dst_blocks,
                                      int32_t* __restrict__ past_pages, uint32_t* status) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= max_sel * Hkv) return;
  const int i = e / Hkv, g = e % Hkv;
  int cnt = sel_count[g];
  if (cnt < 0 || cnt > max_sel) {
    if (i == 0) atomicOr(status, OOMB_DEV_BAD_COUNT);
    cnt = cnt < 0 ? 0 : max_sel;
  }
  int src = -1, dst = -1, past = 0;
  const int slot = slot_pages[i];
  const bool slot_ok = slot >= 0 && slot < dst_pages;
  if (!slot_ok) atomicOr(status, OOMB_DEV_BAD_PAGE);
  if (i < cnt && slot_ok) {
    const int lp = sel_logical[static_cast<size_t>(g) * max_sel + i];
    const int phys = (lp >= 0 && lp < table_len) ? page_table[lp] : -1;
    if (phys >= 0 && phys < src_pages) {
      src = phys * Hkv + g;
      dst = slot * Hkv + g;
      past = slot;
    } else {
      atomicOr(status, OOMB_DEV_BAD_PAGE);
    }
  }
  src_blocks[e] = src;
  dst_blocks[e] = dst;
  past_pages[static_cast<size_t>(g) * max_sel + i] = past;
}

bool same_shape(const oomb_pool* a, const oomb_pool* b) {
  return a->desc.page_size == b->desc.page_size && a->desc.num_kv_heads == b->desc.num_kv_heads &&
         a->desc.head_dim == b->desc.head_dim;
}

int64_t num_blocks(const oomb_pool* p) {
  return static_cast<int64_t>(p->desc.num_pages) * p->desc.num_kv_heads;
}

}  // namespace

extern "C" oomb_status oomb_block_copy(const oomb_pool* src_pool, oomb_pool* dst_pool,
                                       const int32_t* d_src_blocks, const int32_t* d_dst_blocks,
                                       int32_t n_blocks, void* stream) {
  if (!src_pool || !dst_pool || n_blocks < 0) return OOMB_ERR_INVALID_ARG;
  if (src_pool->desc.location == OOMB_LOC_HOST || dst_pool->desc.location == OOMB_LOC_HOST)
    return OOMB_ERR_INVALID_ARG;
  if (!same_shape(src_pool, dst_pool)) return OOMB_ERR_INVALID_ARG;
  if (n_blocks == 0) return OOMB_OK;
  if (!d_src_blocks || !d_dst_blocks) return OOMB_ERR_INVALID_ARG;
  if (num_blocks(src_pool) > INT32_MAX || num_blocks(dst_pool) > INT32_MAX)
    return OOMB_ERR_UNSUPPORTED;
  const int dev = dst_pool->desc.location == OOMB_LOC_DEVICE ? dst_pool->desc.device
                                                             : src_pool->desc.device;
  oomb::DeviceGuard guard(dev);
  const bool link = src_pool->desc.location != OOMB_LOC_DEVICE ||
                    dst_pool->desc.location != OOMB_LOC_DEVICE;
  const int vec = static_cast<int>(src_pool->block_elems() * 2 / 16);
  block_copy_kernel<<<move_grid(n_blocks, link, false, dev), kMoveThreads, 0,
                      static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src_pool->kv_dev), static_cast<uint4*>(dst_pool->kv_dev),
      src_pool->summary, dst_pool->summary, d_src_blocks, d_dst_blocks, n_blocks,
      static_cast<int>(num_blocks(src_pool)), static_cast<int>(num_blocks(dst_pool)), vec,
      src_pool->desc.head_dim, dst_pool->d_status);
  return oomb::check_launch();
}

extern "C" oomb_status oomb_grad_block_add(oomb_pool* src_pool, oomb_pool* dst_pool,
                                           const int32_t* d_src_blocks,
                                           const int32_t* d_dst_blocks, int32_t n_blocks,
                                           int32_t zero_src, void* stream) {
  if (!src_pool || !dst_pool || n_blocks < 0) return OOMB_ERR_INVALID_ARG;
  if (src_pool->desc.location != OOMB_LOC_DEVICE || dst_pool->desc.location == OOMB_LOC_HOST)
    return OOMB_ERR_INVALID_ARG;
  if (!src_pool->grad || !dst_pool->grad || !same_shape(src_pool, dst_pool))
    return OOMB_ERR_INVALID_ARG;
  if (n_blocks == 0) return OOMB_OK;
  if (!d_src_blocks || !d_dst_blocks) return OOMB_ERR_INVALID_ARG;
  if (num_blocks(src_pool) > INT32_MAX || num_blocks(dst_pool) > INT32_MAX)
    return OOMB_ERR_UNSUPPORTED;
  const int dev = src_pool->desc.device;
  oomb::DeviceGuard guard(dev);
  const bool host_dst = dst_pool->desc.location == OOMB_LOC_PINNED_HOST;
  const int vec = static_cast<int>(src_pool->block_elems() * 4 / 16);
  const int grid = move_grid(n_blocks, host_dst, true, dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* in = reinterpret_cast<float4*>(src_pool->grad_dev);
  auto* out = reinterpret_cast<float4*>(dst_pool->grad_dev);
  const int snb = static_cast<int>(num_blocks(src_pool)), dnb = static_cast<int>(num_blocks(dst_pool));
  if (host_dst)
    grad_add_kernel<false><<<grid, kMoveThreads, 0, s>>>(in, out, d_src_blocks, d_dst_blocks,
                                                         n_blocks, snb, dnb, vec, zero_src != 0,
                                                         dst_pool->d_status);
  else
    grad_add_kernel<true><<<grid, kMoveThreads, 0, s>>>(in, out, d_src_blocks, d_dst_blocks,
                                                        n_blocks, snb, dnb, vec, zero_src != 0,
                                                        dst_pool->d_status);
  return oomb::check_launch();
}

extern "C" oomb_status oomb_prefetch_lists(const oomb_pool* src_pool, oomb_pool* dst_pool,
                                           const int32_t* d_sel_logical,
                                           const int32_t* d_sel_count, int32_t max_sel,
                                           const int32_t* d_page_table, int32_t table_len,
                                           const int32_t* d_slot_pages, int32_t* d_src_blocks,
                                           int32_t* d_dst_blocks, int32_t* d_past_pages,
                                           void* stream) {
  if (!src_pool || !dst_pool || max_sel <= 0 || table_len < 0) return OOMB_ERR_INVALID_ARG;
  if (src_pool->desc.location == OOMB_LOC_HOST || dst_pool->desc.location == OOMB_LOC_HOST)
    return OOMB_ERR_INVALID_ARG;
  if (!same_shape(src_pool, dst_pool)) return OOMB_ERR_INVALID_ARG;
  if (!d_sel_logical || !d_sel_count || !d_slot_pages || !d_src_blocks || !d_dst_blocks ||
      !d_past_pages || (table_len > 0 && !d_page_table))
    return OOMB_ERR_INVALID_ARG;
  const int Hkv = src_pool->desc.num_kv_heads;
  if (static_cast<int64_t>(max_sel) * Hkv > (1 << 24) || num_blocks(src_pool) > INT32_MAX ||
      num_blocks(dst_pool) > INT32_MAX)
    return OOMB_ERR_UNSUPPORTED;
  const int dev = dst_pool->desc.location == OOMB_LOC_DEVICE ? dst_pool->desc.device
                                                             : src_pool->desc.device;
  oomb::DeviceGuard guard(dev);
  const int n = max_sel * Hkv;
  prefetch_lists_kernel<<<(n + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      d_sel_logical, d_sel_count, max_sel, Hkv, d_page_table, table_len, src_pool->desc.num_pages,
      d_slot_pages, dst_pool->desc.num_pages, d_src_blocks, d_dst_blocks, d_past_pages,
      dst_pool->d_status);
  return oomb::check_launch();
}
