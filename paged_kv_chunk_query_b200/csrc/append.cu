// kv_append: one chunk's K/V into pool pages, page representatives, grad zeroing.
//
// The page representative is the mean of the page's keys ("Out of the Memory
// Barrier", [es] §2B "Atención Escasa a Nivel de Página": an average
// representative vector per key page), kept in fp32 per (page, KV head) and
// taken over the keys as stored (bf16).  The written pages' gradient blocks
// are zero-filled so the backward can add into them in place.
#include "internal.h"
#include "ptx.cuh"

namespace {

template <int D>
__global__ void __launch_bounds__(256) kv_append_kernel(
    const int32_t* __restrict__ page_ids, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ kv,
    float* __restrict__ grad, float* __restrict__ summary, uint32_t* status, int P, int Hkv,
    int num_pages) {
  constexpr int VPR = D / 8;        // 16-byte vectors per row
  constexpr int RG = 256 / VPR;     // row groups
  __shared__ float part[RG][D];
  const int i = blockIdx.x, g = blockIdx.y, t = threadIdx.x;
  const int page = page_ids[i];
  if (page < 0 || page >= num_pages) {
    if (t == 0) atomicOr(status, OOMB_DEV_BAD_PAGE);
    return;
  }
  const int vec = t % VPR, rg = t / VPR;
  const size_t blk = (static_cast<size_t>(page) * Hkv + g) * 2;  // K block index
  __nv_bfloat16* kdst = kv + blk * P * D;
  __nv_bfloat16* vdst = kdst + static_cast<size_t>(P) * D;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int r = rg; r < P; r += RG) {
    const size_t src = (static_cast<size_t>(i) * P + r) * Hkv + g;
    const uint4 kk = *reinterpret_cast<const uint4*>(k + src * D + vec * 8);
    const uint4 vv = *reinterpret_cast<const uint4*>(v + src * D + vec * 8);
    *reinterpret_cast<uint4*>(kdst + static_cast<size_t>(r) * D + vec * 8) = kk;
    *reinterpret_cast<uint4*>(vdst + static_cast<size_t>(r) * D + vec * 8) = vv;
    const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(&kk);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __bfloat162float(kb[e]);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rg][vec * 8 + e] = acc[e];
  __syncthreads();
  if (t < D) {
    float s = 0.f;
    for (int r = 0; r < RG; ++r) s += part[r][t];  // fixed order: deterministic
    summary[(static_cast<size_t>(page) * Hkv + g) * D + t] = s / static_cast<float>(P);
  }
  if (grad) {
    float4* gz = reinterpret_cast<float4*>(grad + blk * P * D);
    const int n4 = 2 * P * D / 4;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e = t; e < n4; e += 256) gz[e] = z;
  }
}

}  // namespace

extern "C" oomb_status oomb_kv_append(oomb_pool* pool, const int32_t* d_page_ids,
                                      int32_t n_pages, const void* d_k, const void* d_v,
                                      void* stream) {
  if (!pool || pool->desc.location != OOMB_LOC_DEVICE) return OOMB_ERR_INVALID_ARG;
  if (n_pages < 0) return OOMB_ERR_INVALID_ARG;
  if (n_pages == 0) return OOMB_OK;
  if (!d_page_ids || !d_k || !d_v) return OOMB_ERR_INVALID_ARG;
  if (!oomb::aligned16(d_k) || !oomb::aligned16(d_v)) return OOMB_ERR_INVALID_ARG;
  const oomb_pool_desc& d = pool->desc;
  oomb::DeviceGuard guard(d.device);
  dim3 grid(n_pages, d.num_kv_heads);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d.head_dim == 128)
    kv_append_kernel<128><<<grid, 256, 0, s>>>(
        d_page_ids, static_cast<const __nv_bfloat16*>(d_k),
        static_cast<const __nv_bfloat16*>(d_v), static_cast<__nv_bfloat16*>(pool->kv),
        pool->grad, pool->summary, pool->d_status, d.page_size, d.num_kv_heads, d.num_pages);
  else
    kv_append_kernel<64><<<grid, 256, 0, s>>>(
        d_page_ids, static_cast<const __nv_bfloat16*>(d_k),
        static_cast<const __nv_bfloat16*>(d_v), static_cast<__nv_bfloat16*>(pool->kv),
        pool->grad, pool->summary, pool->d_status, d.page_size, d.num_kv_heads, d.num_pages);
  return oomb::check_launch();
}
