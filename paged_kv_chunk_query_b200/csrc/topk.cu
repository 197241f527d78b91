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
// Kernel 1 (qmean_partial): grid (128 slices, Hkv); each CTA streams a slice of
//   the chunk's rows with 16-byte loads, 8 in flight per thread, and writes one
//   fp32 partial sum per d.
// Kernel 2 (page_score): grid (pages / 64, Hkv); each CTA reduces the partials
//   in a fixed order into q_bar, then each warp scores 8 pages (float4 loads of
//   the summaries, shuffle reduction).
// Kernel 3 (select): one CTA per group; finds the K-th largest 64-bit key
//   (ordered score, inverted id) by 8-bit radix passes from the top with a
//   parallel bin scan, stopping once the boundary bin is kept whole, then
//   compacts the kept ids in ascending order.
#include <cuda_bf16.h>

#include <mutex>

#include "internal.h"

namespace {

constexpr int kSplits = 128;         // query-mean slices per group (~3.5 CTAs per SM at Hkv 4)
constexpr int kMeanThreads = 256;
constexpr int kScoreThreads = 256;   // 8 warps x 8 pages per CTA
constexpr int kPagesPerScoreCta = 64;
constexpr int kSelectThreads = 1024;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// ---------------------------------------------------------------- query mean
// grid (kSplits, Hkv): CTA (s, g) sums rows (token, head in g) of token slice
// s.  Each thread keeps 8 independent 16-byte loads in flight (about 32 KiB
// per CTA), enough with 3-4 CTAs per SM to stream Q at HBM speed.
template <int D>
__global__ void __launch_bounds__(kMeanThreads) qmean_partial_kernel(
    const __nv_bfloat16* __restrict__ q, float* __restrict__ partial, int C, int Hq, int G) {
  constexpr int VPR = D / 8;               // 16-byte vectors per row
  constexpr int RG = kMeanThreads / VPR;   // rows per pass
  constexpr int U = 8;                     // loads in flight per thread
  __shared__ float red[RG][D];
  const int split = blockIdx.x, g = blockIdx.y, t = threadIdx.x;
  const int vec = t % VPR, rg = t / VPR;
  const int per = (C + kSplits - 1) / kSplits;
  const int tok0 = split * per, tok1 = min(C, tok0 + per);
  const int rows = max(0, tok1 - tok0) * G;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int base = rg; base < rows; base += RG * U) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int rr = base + u * RG;
      if (rr < rows) {
        const int tok = tok0 + rr / G, hh = g * G + rr % G;
        v[u] = __ldg(reinterpret_cast<const uint4*>(q + (static_cast<size_t>(tok) * Hq + hh) * D +
                                                    vec * 8));
      } else {
        v[u] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const __nv_bfloat16* bv = reinterpret_cast<const __nv_bfloat16*>(&v[u]);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __bfloat162float(bv[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rg][vec * 8 + e] = acc[e];
  __syncthreads();
  if (t < D) {
    float s = 0.f;
    for (int r = 0; r < RG; ++r) s += red[r][t];  // fixed order: deterministic
    partial[(static_cast<size_t>(split) * gridDim.y + g) * D + t] = s;
  }
}

__device__ __forceinline__ uint32_t order_f32(float f) {
  // monotone map of fp32 onto uint32 (larger float -> larger integer)
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- page scores
// grid (ceil(n_past / 64), Hkv).  Every CTA reduces the kSplits partials of its
// group in the same fixed order (so all CTAs use the identical q_bar), then
// each warp scores 8 pages.  Key = (ordered score << 32) | (~logical id).
template <int D>
__global__ void __launch_bounds__(kScoreThreads) page_score_kernel(
    const float* __restrict__ partial, const float* __restrict__ summary,
    const int32_t* __restrict__ page_table, int n_past, int Hkv, int num_pool_pages,
    float inv_rows, unsigned long long* __restrict__ keys, float* __restrict__ out_scores,
    uint32_t* status) {
  constexpr int kParts = kScoreThreads / D;  // threads per d in the q_bar reduction
  __shared__ float part_sum[kParts][D];
  __shared__ float qbar[D];
  const int g = blockIdx.y, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  {
    constexpr int PER = kSplits / kParts;  // partials per thread, all loads in flight
    const int d = t % D, part = t / D;
    float v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i)
      v[i] = __ldg(partial + (static_cast<size_t>(part * PER + i) * Hkv + g) * D + d);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) s += v[i];
    part_sum[part][d] = s;
    __syncthreads();
    if (t < D) {
      float s2 = 0.f;
#pragma unroll
      for (int i = 0; i < kParts; ++i) s2 += part_sum[i][t];
      qbar[t] = s2 * inv_rows;
    }
    __syncthreads();
  }
  constexpr int PW = kPagesPerScoreCta / (kScoreThreads / 32);  // pages per warp
  const int p0 = blockIdx.x * kPagesPerScoreCta + warp * PW;
  constexpr int EPL = D / 32;  // elements per lane
  float qv[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) qv[e] = qbar[lane * EPL + e];
  float acc[PW];
#pragma unroll
  for (int i = 0; i < PW; ++i) {
    const int p = p0 + i;
    acc[i] = 0.f;
    if (p < n_past) {
      int phys = __ldg(page_table + p);
      if (phys < 0 || phys >= num_pool_pages) {
        if (lane == 0) atomicOr(status, OOMB_DEV_BAD_PAGE);
        phys = 0;
      }
      const float* srow = summary + (static_cast<size_t>(phys) * Hkv + g) * D + lane * EPL;
      if (EPL == 4) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(srow));
        acc[i] = a.x * qv[0] + a.y * qv[1] + a.z * qv[2] + a.w * qv[3];
      } else {
        const float2 a = __ldg(reinterpret_cast<const float2*>(srow));
        acc[i] = a.x * qv[0] + a.y * qv[1];
      }
    }
  }
#pragma unroll
  for (int i = 0; i < PW; ++i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
  }
  if (lane < PW) {
    float mine = 0.f;
#pragma unroll
    for (int i = 0; i < PW; ++i)
      if (lane == i) mine = acc[i];
    const int p = p0 + lane;
    if (p < n_past) {
      if (out_scores) out_scores[static_cast<size_t>(g) * n_past + p] = mine;
      keys[static_cast<size_t>(g) * n_past + p] =
          (static_cast<unsigned long long>(order_f32(mine)) << 32) |
          static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(p));
    }
  }
}

// ---------------------------------------------------------------- select
// One CTA per group: the K-th largest candidate key by 8-bit radix passes from
// the top, each with a parallel suffix scan over the 256 bins; stops early once
// the boundary bin is taken whole.  Then compacts kept ids in ascending order.
__global__ void __launch_bounds__(kSelectThreads) topk_select_kernel(
    const unsigned long long* __restrict__ keys_all, const int32_t* __restrict__ page_table,
    int n_past, int top_k, int n_recent, int num_pool_pages, int32_t* __restrict__ out_logical,
    int32_t* __restrict__ out_physical, int32_t* __restrict__ out_count) {
  __shared__ unsigned int hist[256];
  __shared__ unsigned int warp_tot[8];
  __shared__ unsigned long long kth_sh;
  __shared__ int need_sh, done_sh;
  __shared__ int warp_sum[kSelectThreads / 32];
  __shared__ int running_sh;
  const int g = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int max_sel = top_k + n_recent;
  const int n_cand = max(0, n_past - n_recent);
  const int k_eff = min(top_k, n_cand);
  const unsigned long long* keys = keys_all + static_cast<size_t>(g) * n_past;

  if (t == 0) {
    kth_sh = 0ull;  // with k_eff >= n_cand every candidate is kept
    need_sh = k_eff;
    done_sh = 0;
  }
  __syncthreads();
  if (k_eff > 0 && k_eff < n_cand) {
    unsigned long long prefix = 0ull, mask = 0ull;
    for (int shift = 56; shift >= 0; shift -= 8) {
      if (t < 256) hist[t] = 0u;
      __syncthreads();
      for (int p = t; p < n_cand; p += kSelectThreads) {
        const unsigned long long k = keys[p];
        if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255ull], 1u);
      }
      __syncthreads();
      // inclusive suffix sum over bins 255..0: thread t < 256 owns bin 255 - t
      unsigned int incl = 0;
      if (t < 256) {
        const unsigned int v = hist[255 - t];
        incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const unsigned int y = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += y;
        }
        if (lane == 31) warp_tot[warp] = incl;
      }
      __syncthreads();
      if (t < 256) {
        for (int w = 0; w < warp; ++w) incl += warp_tot[w];
        const int bin = 255 - t;
        const unsigned int v = hist[bin];
        const unsigned int excl = incl - v;
        const int need = need_sh;
        if (excl < static_cast<unsigned>(need) && static_cast<unsigned>(need) <= incl) {
          kth_sh = prefix | (static_cast<unsigned long long>(bin) << shift);
          need_sh = need - static_cast<int>(excl);
          if (v == static_cast<unsigned>(need) - excl) done_sh = 1;  // bin taken whole
        }
      }
      __syncthreads();
      prefix = kth_sh;
      mask |= 255ull << shift;
      if (done_sh) break;
    }
  }
  const unsigned long long kth = kth_sh;

  if (t == 0) running_sh = 0;
  __syncthreads();
  for (int base = 0; base < n_past; base += kSelectThreads) {
    const int p = base + t;
    int keep = 0;
    if (p < n_cand) keep = (k_eff >= n_cand) || (k_eff > 0 && keys[p] >= kth);
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
        const int phys = page_table[p];
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
  const size_t partial = static_cast<size_t>(kSplits) * num_kv_heads * head_dim * 4;
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
  float* partial = static_cast<float*>(d_workspace);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(
      static_cast<uint8_t*>(d_workspace) + align256(static_cast<size_t>(kSplits) * Hkv * D * 4));
  const int G = num_q_heads / Hkv;
  const float inv_rows = 1.0f / (static_cast<float>(chunk_len) * static_cast<float>(G));
  const auto* q = static_cast<const __nv_bfloat16*>(d_q);
  dim3 g1(kSplits, Hkv), g2((n_past + kPagesPerScoreCta - 1) / kPagesPerScoreCta, Hkv);
  if (D == 128) {
    qmean_partial_kernel<128><<<g1, kMeanThreads, 0, s>>>(q, partial, chunk_len, num_q_heads, G);
    if (n_past > 0)
      page_score_kernel<128><<<g2, kScoreThreads, 0, s>>>(partial, pool->summary, d_page_table,
                                                          n_past, Hkv, d.num_pages, inv_rows,
                                                          keys, d_out_scores, pool->d_status);
  } else {
    qmean_partial_kernel<64><<<g1, kMeanThreads, 0, s>>>(q, partial, chunk_len, num_q_heads, G);
    if (n_past > 0)
      page_score_kernel<64><<<g2, kScoreThreads, 0, s>>>(partial, pool->summary, d_page_table,
                                                         n_past, Hkv, d.num_pages, inv_rows, keys,
                                                         d_out_scores, pool->d_status);
  }
  topk_select_kernel<<<Hkv, kSelectThreads, 0, s>>>(keys, d_page_table, n_past, top_k, n_recent,
                                                     d.num_pages, d_out_logical, d_out_physical,
                                                     d_out_count);
  return oomb::check_launch();
}

// ---------------------------------------------------------------- no-allocation variant
// Some callers of this library cannot allocate device memory: a host
// framework that owns every device allocation and forbids side allocations,
// or a latency-critical loop in which a cudaMalloc (which may synchronise the
// device) is not acceptable.  oomb_page_topk_static serves them: it is
// oomb_page_topk with its scratch (query-mean partials and 64-bit page keys)
// taken from the file-scope device array below instead of a caller workspace.
// Every GPU that loads the library holds this array until the process exits.
// All calls share it and it keeps the last call's contents; the kernels write
// every scratch word before reading it, so nothing needs clearing, but calls
// that overlap on the GPU (on different streams) race on it.
namespace {

static __device__ __align__(256) uint8_t g_topk_static_scratch[OOMB_TOPK_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once
// per device; the host-side name is only a stand-in, not a device address).
oomb_status static_scratch(int device, void** out) {
  if (device < 0 || device >= kMaxDevices) return OOMB_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_addr[device]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_topk_static_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return OOMB_ERR_CUDA;
    }
    g_static_addr[device] = p;
  }
  *out = g_static_addr[device];
  return OOMB_OK;
}

}  // namespace

extern "C" oomb_status oomb_page_topk_static(const oomb_pool* pool, const void* d_q,
                                             int32_t chunk_len, int32_t num_q_heads,
                                             const int32_t* d_page_table, int32_t n_past,
                                             int32_t top_k, int32_t n_recent,
                                             int32_t* d_out_logical, int32_t* d_out_physical,
                                             int32_t* d_out_count, float* d_out_scores,
                                             void* stream) {
  if (!pool || pool->desc.location == OOMB_LOC_HOST) return OOMB_ERR_INVALID_ARG;
  const oomb_pool_desc& d = pool->desc;
  const int Hkv = d.num_kv_heads, D = d.head_dim;
  if (!d_q || !d_out_logical || !d_out_count) return OOMB_ERR_INVALID_ARG;
  if (chunk_len <= 0 || num_q_heads <= 0 || num_q_heads % Hkv != 0) return OOMB_ERR_INVALID_ARG;
  if (n_past < 0 || n_past > 65536 || top_k < 0 || n_recent < 0 || top_k + n_recent > 4096 ||
      top_k + n_recent == 0)
    return OOMB_ERR_INVALID_ARG;
  if (n_past > 0 && !d_page_table) return OOMB_ERR_INVALID_ARG;
  if (!oomb::aligned16(d_q)) return OOMB_ERR_INVALID_ARG;
  // the scratch array has a fixed size: larger problems must use oomb_page_topk
  if (oomb_page_topk_workspace_size(chunk_len, num_q_heads, Hkv, D, n_past) >
      OOMB_TOPK_STATIC_SCRATCH_BYTES)
    return OOMB_ERR_UNSUPPORTED;
  oomb::DeviceGuard guard(d.device);
  void* scratch = nullptr;
  const oomb_status st = static_scratch(d.device, &scratch);
  if (st != OOMB_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* partial = static_cast<float*>(scratch);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(
      static_cast<uint8_t*>(scratch) + align256(static_cast<size_t>(kSplits) * Hkv * D * 4));
  const int G = num_q_heads / Hkv;
  const float inv_rows = 1.0f / (static_cast<float>(chunk_len) * static_cast<float>(G));
  const auto* q = static_cast<const __nv_bfloat16*>(d_q);
  dim3 g1(kSplits, Hkv), g2((n_past + kPagesPerScoreCta - 1) / kPagesPerScoreCta, Hkv);
  if (D == 128) {
    qmean_partial_kernel<128><<<g1, kMeanThreads, 0, s>>>(q, partial, chunk_len, num_q_heads, G);
    if (n_past > 0)
      page_score_kernel<128><<<g2, kScoreThreads, 0, s>>>(partial, pool->summary, d_page_table,
                                                          n_past, Hkv, d.num_pages, inv_rows,
                                                          keys, d_out_scores, pool->d_status);
  } else {
    qmean_partial_kernel<64><<<g1, kMeanThreads, 0, s>>>(q, partial, chunk_len, num_q_heads, G);
    if (n_past > 0)
      page_score_kernel<64><<<g2, kScoreThreads, 0, s>>>(partial, pool->summary, d_page_table,
                                                         n_past, Hkv, d.num_pages, inv_rows, keys,
                                                         d_out_scores, pool->d_status);
  }
  topk_select_kernel<<<Hkv, kSelectThreads, 0, s>>>(keys, d_page_table, n_past, top_k, n_recent,
                                                     d.num_pages, d_out_logical, d_out_physical,
                                                     d_out_count);
  return oomb::check_launch();
}
