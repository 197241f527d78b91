// Page-level Top-K selection for one chunk (memory-bound, sm_100a).
//
// "Out of the Memory Barrier" ([pt] §2C: Top-K retrieval of the key pages most
// relevant to the queries; [es] §2B "Atención Escasa a Nivel de Página": an
// average representative vector per key page, the pages most relevant to the
// current queries are kept; [it] §2D: most recent or selected pages).
//   q_bar_g   = mean over the chunk's C rows and the G query heads of group g (fp32)
//   score_p,g = q_bar_g . k_bar_p,g  with k_bar the page's fp32 mean key
// Candidates are logical pages [0, n_past - R); the K largest scores are kept,
// ties going to the lower logical id; pages [n_past - R, n_past) are always
// kept; the output lists ascending logical ids.
//
// Kernel 1 (qmean_partial): grid (splits, Hkv); each CTA streams a slice of the
//   chunk's rows with 16-byte loads and writes one fp32 partial sum per d.
// Kernel 2 (select): one CTA per group; reduces the partials in a fixed order,
//   scores every past page (one warp per page, float4 loads of the summary),
//   finds the K-th largest 64-bit key (ordered score, inverted id) with an
//   8-pass radix select, then compacts the kept ids in ascending order.
#include <cuda_bf16.h>

#include "internal.h"

namespace {

constexpr int kSelectThreads = 1024;

int topk_splits(int C) {
  int s = C / 32;
  if (s < 1) s = 1;
  if (s > 128) s = 128;
  return s;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

template <int D>
__global__ void __launch_bounds__(256) qmean_partial_kernel(const __nv_bfloat16* __restrict__ q,
                                                            float* __restrict__ partial, int C,
                                                            int Hq, int G, int splits) {
  constexpr int VPR = D / 8;      // 16-byte vectors per row
  constexpr int RG = 256 / VPR;   // rows in flight per pass
  __shared__ float red[RG][D];
  const int split = blockIdx.x, g = blockIdx.y, t = threadIdx.x;
  const int vec = t % VPR, rg = t / VPR;
  const int per = (C + splits - 1) / splits;
  const int tok0 = split * per, tok1 = min(C, tok0 + per);
  const int rows = max(0, tok1 - tok0) * G;  // rows (token, head in group) of this slice
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int rr = rg; rr < rows; rr += RG) {
    const int tok = tok0 + rr / G, hh = g * G + rr % G;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(
        q + (static_cast<size_t>(tok) * Hq + hh) * D + vec * 8));
    const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __bfloat162float(b[e]);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rg][vec * 8 + e] = acc[e];
  __syncthreads();
  if (t < D) {
    float s = 0.f;
    for (int r = 0; r < RG; ++r) s += red[r][t];
    partial[(static_cast<size_t>(split) * gridDim.y + g) * D + t] = s;
  }
}

__device__ __forceinline__ uint32_t order_f32(float f) {
  // monotone map of fp32 onto uint32 (larger float -> larger integer)
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int D>
__global__ void __launch_bounds__(kSelectThreads) topk_select_kernel(
    const float* __restrict__ partial, int splits, const float* __restrict__ summary,
    const int32_t* __restrict__ page_table, int n_past, int top_k, int n_recent, int Hkv,
    int num_pool_pages, float inv_rows, unsigned long long* __restrict__ keys,
    int32_t* __restrict__ out_logical, int32_t* __restrict__ out_physical,
    int32_t* __restrict__ out_count, float* __restrict__ out_scores, uint32_t* status) {
  __shared__ float qbar[D];
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long kth_sh;
  __shared__ int need_sh;
  __shared__ int warp_sum[kSelectThreads / 32];
  __shared__ int running_sh;
  const int g = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int max_sel = top_k + n_recent;
  const int n_cand = max(0, n_past - n_recent);
  const int k_eff = min(top_k, n_cand);

  if (t < D) {
    float s = 0.f;
    for (int i = 0; i < splits; ++i) s += partial[(static_cast<size_t>(i) * Hkv + g) * D + t];
    qbar[t] = s * inv_rows;
  }
  __syncthreads();

  // scores: one warp per page
  unsigned long long* gkeys = keys + static_cast<size_t>(g) * n_past;
  for (int p = warp; p < n_past; p += kSelectThreads / 32) {
    int phys = page_table[p];
    if (phys < 0 || phys >= num_pool_pages) {
      if (lane == 0) atomicOr(status, OOMB_DEV_BAD_PAGE);
      phys = 0;
    }
    const float* srow = summary + (static_cast<size_t>(phys) * Hkv + g) * D;
    float acc = 0.f;
    if (D == 128) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(srow) + lane);
      acc = a.x * qbar[4 * lane] + a.y * qbar[4 * lane + 1] + a.z * qbar[4 * lane + 2] +
            a.w * qbar[4 * lane + 3];
    } else {
      const float2 a = __ldg(reinterpret_cast<const float2*>(srow) + lane);
      acc = a.x * qbar[2 * lane] + a.y * qbar[2 * lane + 1];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      if (out_scores) out_scores[static_cast<size_t>(g) * n_past + p] = acc;
      gkeys[p] = (static_cast<unsigned long long>(order_f32(acc)) << 32) |
                 static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(p));
    }
  }
  __syncthreads();

  // K-th largest candidate key (keys are unique: ids differ)
  if (t == 0) {
    kth_sh = 0ull;  // with k_eff >= n_cand every candidate is kept
    need_sh = k_eff;
  }
  __syncthreads();
  if (k_eff > 0 && k_eff < n_cand) {
    unsigned long long prefix = 0ull, mask = 0ull;
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = t; i < 256; i += kSelectThreads) hist[i] = 0u;
      __syncthreads();
      for (int p = t; p < n_cand; p += kSelectThreads) {
        const unsigned long long k = gkeys[p];
        if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255ull], 1u);
      }
      __syncthreads();
      if (t == 0) {
        int need = need_sh, cum = 0, sel = 0;
        for (int d = 255; d >= 0; --d) {
          if (cum + static_cast<int>(hist[d]) >= need) {
            sel = d;
            need -= cum;
            break;
          }
          cum += hist[d];
        }
        need_sh = need;
        kth_sh = prefix | (static_cast<unsigned long long>(sel) << shift);
      }
      __syncthreads();
      prefix = kth_sh;
      mask |= 255ull << shift;
    }
  }
  const unsigned long long kth = kth_sh;

  // compaction in ascending logical id
  if (t == 0) running_sh = 0;
  __syncthreads();
  for (int base = 0; base < n_past; base += kSelectThreads) {
    const int p = base + t;
    int keep = 0;
    if (p < n_cand) keep = (k_eff >= n_cand) || (k_eff > 0 && gkeys[p] >= kth);
    else if (p < n_past) keep = 1;
    const unsigned ballot = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) warp_sum[warp] = __popc(ballot);
    __syncthreads();
    int before = running_sh;
    for (int w = 0; w < warp; ++w) before += warp_sum[w];
    before += __popc(ballot & ((1u << lane) - 1u));
    if (keep && before < max_sel) {
      out_logical[static_cast<size_t>(g) * max_sel + before] = p;
      if (out_physical) {
        int phys = page_table[p];
        out_physical[static_cast<size_t>(g) * max_sel + before] =
            (phys >= 0 && phys < num_pool_pages) ? phys : 0;
      }
    }
    __syncthreads();
    if (t == 0) {
      int tot = 0;
      for (int w = 0; w < kSelectThreads / 32; ++w) tot += warp_sum[w];
      running_sh += tot;
    }
    __syncthreads();
  }
  if (t == 0) out_count[g] = min(running_sh, max_sel);
}

}  // namespace

extern "C" size_t oomb_page_topk_workspace_size(int32_t chunk_len, int32_t num_q_heads,
                                                int32_t num_kv_heads, int32_t head_dim,
                                                int32_t n_past) {
  (void)num_q_heads;
  if (chunk_len <= 0 || num_kv_heads <= 0 || head_dim <= 0 || n_past < 0) return 0;
  const size_t partial = static_cast<size_t>(topk_splits(chunk_len)) * num_kv_heads * head_dim * 4;
  const size_t keys = static_cast<size_t>(num_kv_heads) * (n_past > 0 ? n_past : 1) * 8;
  return align256(partial) + align256(keys);
}

extern "C" oomb_status oomb_page_topk(const oomb_pool* pool, const void* d_q, int32_t chunk_len,
                                      int32_t num_q_heads, const int32_t* d_page_table,
                                      int32_t n_past, int32_t top_k, int32_t n_recent,
                                      int32_t* d_out_logical, int32_t* d_out_physical,
                                      int32_t* d_out_count, float* d_out_scores,
                                      void* d_workspace, size_t workspace_bytes, void* stream) {
  // device pools and pinned-host pools (whose summaries live on the device)
  if (!pool || pool->desc.location == OOMB_LOC_HOST) return OOMB_ERR_INVALID_ARG;
  const oomb_pool_desc& d = pool->desc;
  const int Hkv = d.num_kv_heads, D = d.head_dim;
  if (!d_q || !d_out_logical || !d_out_count || !d_workspace) return OOMB_ERR_INVALID_ARG;
  if (chunk_len <= 0 || num_q_heads <= 0 || num_q_heads % Hkv != 0) return OOMB_ERR_INVALID_ARG;
  if (n_past < 0 || n_past > 65536 || top_k < 0 || n_recent < 0 || top_k + n_recent > 4096 ||
      top_k + n_recent == 0)
    return OOMB_ERR_INVALID_ARG;
  if (n_past > 0 && !d_page_table) return OOMB_ERR_INVALID_ARG;
  if (!oomb::aligned16(d_q) || !oomb::aligned16(d_workspace)) return OOMB_ERR_INVALID_ARG;
  if (workspace_bytes < oomb_page_topk_workspace_size(chunk_len, num_q_heads, Hkv, D, n_past))
    return OOMB_ERR_INVALID_ARG;
  oomb::DeviceGuard guard(d.device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int splits = topk_splits(chunk_len);
  float* partial = static_cast<float*>(d_workspace);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(
      static_cast<uint8_t*>(d_workspace) +
      align256(static_cast<size_t>(splits) * Hkv * D * 4));
  const int G = num_q_heads / Hkv;
  const float inv_rows = 1.0f / (static_cast<float>(chunk_len) * static_cast<float>(G));
  dim3 g1(splits, Hkv);
  if (D == 128) {
    qmean_partial_kernel<128><<<g1, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(d_q), partial,
                                                 chunk_len, num_q_heads, G, splits);
    topk_select_kernel<128><<<Hkv, kSelectThreads, 0, s>>>(
        partial, splits, pool->summary, d_page_table, n_past, top_k, n_recent, Hkv, d.num_pages,
        inv_rows, keys, d_out_logical, d_out_physical, d_out_count, d_out_scores, pool->d_status);
  } else {
    qmean_partial_kernel<64><<<g1, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(d_q), partial,
                                                chunk_len, num_q_heads, G, splits);
    topk_select_kernel<64><<<Hkv, kSelectThreads, 0, s>>>(
        partial, splits, pool->summary, d_page_table, n_past, top_k, n_recent, Hkv, d.num_pages,
        inv_rows, keys, d_out_logical, d_out_physical, d_out_count, d_out_scores, pool->d_status);
  }
  return oomb::check_launch();
}
