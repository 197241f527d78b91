// Q/K/V projection of a chunk with a paged epilogue (tcgen05 + TMA, sm_100a).
//
// "Out of the Memory Barrier" ([pt] §2D: with sparse attention the pages a
// chunk needs are known as soon as its queries exist, so their transfer can
// run while the rest of the chunk's work does; [es] §2B).  In a layer that
// rest is the projection producing K and V, so the projection runs in two
// launches: the Q part (after which Top-K can select and the prefetch can
// start) and the K/V part, which writes K and V straight into the chunk's
// pool pages with their page means — the work of oomb_kv_append folded into
// the GEMM's epilogue.
//
// Y = X W^T with X [C][hidden] bf16 and W [(Hq + 2 Hkv) d][hidden] bf16 (rows:
// Q heads, K heads, V heads), fp32 accumulation, outputs rounded to bf16.
// One CTA per 128 x 256 output tile (tokens x outputs; each k-step loads 48 KB
// for 128 x 256 x 64 products, a quarter less L2 traffic per FLOP than 128 x
// 128): warp 0 loads X and W slices of 64 hidden elements by TMA into a ring
// of 4 stages, warp 1 issues the UMMAs (both
// operands K-major in shared memory, accumulator in TMEM), warps 2-5 read the
// accumulator (TMEM lane = token) and write Q rows, or K/V rows into pool
// pages, and add their sums: the page means of K (over the page's P tokens)
// and the per-group sums of Q (over the chunk's tokens and the group's heads).
#include "internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace {

using namespace oomb;

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kTileA = kBM * kBK * 2, kTileB = kBN * kBK * 2;
constexpr int kStageBytes = kTileA + kTileB;
constexpr int kProjSmem = kStages * kStageBytes + 1024;
constexpr int kProjThreads = 192;

struct ProjParams {
  __nv_bfloat16* q;        // [C][Hq][d], or null
  float* qsum;             // [Hkv][d] fp32 sums of Q per group, or null
  const int32_t* page_ids;  // [C / P] physical pages of the chunk
  __nv_bfloat16* kv;       // pool K/V
  float* summary;          // pool page means
  uint32_t* status;
  int C, Hq, Hkv, G, D, P, num_pages, n_base, n_end, k_tiles;
};

// Butterfly over the 32 lanes: on return lane l holds the sum over all lanes of
// v[l] (31 shuffles for 32 columns).
__device__ __forceinline__ float column_sums(float* v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

__global__ void __launch_bounds__(kProjThreads, 1)
    proj_kernel(const ProjParams p, const __grid_constant__ CUtensorMap xmap,
                const __grid_constant__ CUtensorMap wmap) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t bar_full[kStages], bar_empty[kStages], bar_acc, bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh, issued_sh, used_sh;

  const int warp = warp_id(), lane = lane_id();
  const int m0 = blockIdx.x * kBM, n0 = p.n_base + blockIdx.y * kBN;
  if (threadIdx.x == 0) {
    abort_sh = issued_sh = used_sh = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_empty[i], 1);
    }
    mbar_init(&bar_acc, 1);
    mbar_init(&bar_drain, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;

  if (warp == 0) {
    if (lane == 0) {  // TMA producer
      prefetch_tensormap(&xmap);
      prefetch_tensormap(&wmap);
      int issued = 0;
      for (int kt = 0; kt < p.k_tiles; ++kt) {
        const int st = kt % kStages;
        if (!mbar_wait(&bar_empty[st], ((kt / kStages) & 1) ^ 1, abort_flag)) break;
        uint8_t* a = smem + st * kStageBytes;
        mbar_arrive_expect_tx(&bar_full[st], kStageBytes);
        tma_load_2d(a, &xmap, &bar_full[st], kt * kBK, m0);
        tma_load_2d(a + kTileA, &wmap, &bar_full[st], kt * kBK, n0);
        ++issued;
      }
      if (*abort_flag) atomicOr(p.status, OOMB_DEV_WAIT_LIMIT);
      issued_sh = issued;
    }
  } else if (warp == 1) {
    if (lane == 0) {  // UMMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 0);
      const uint32_t base = smem_u32(smem);
      bool ok = true;
      int used = 0;
      for (int kt = 0; kt < p.k_tiles; ++kt) {
        const int st = kt % kStages;
        if (!(ok = mbar_wait(&bar_full[st], (kt / kStages) & 1, abort_flag))) break;
        ++used;
        tc_fence_after();
        const uint32_t a = base + st * kStageBytes, b = a + kTileA;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_ss(tmem, sw128_desc(a + kk * 32, 16, 1024), sw128_desc(b + kk * 32, 16, 1024),
                  idesc, (kt > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&bar_empty[st]);
      }
      if (ok) umma_commit(&bar_acc);
      if (!ok) {
        *abort_flag = 1;
        atomicOr(p.status, OOMB_DEV_WAIT_LIMIT);
      }
      umma_commit(&bar_drain);
      mbar_wait_drain(&bar_drain, 0);
      used_sh = used;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int lg = warp & 3;                 // TMEM lane quarter of this warp
    const int row = lg * 32 + lane, t = m0 + row;
    const bool valid = t < p.C;
    const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
    bool ok = warp_wait(&bar_acc, 0, abort_flag);
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(p.status, OOMB_DEV_WAIT_LIMIT);
    } else {
      tc_fence_after();
      const int nq = p.Hq * p.D, nk = p.Hkv * p.D;
      int page = -1;
      if (valid && p.n_end > nq) {  // the page ids exist only when K/V columns are written
        page = p.page_ids[t / p.P];
        if (page < 0 || page >= p.num_pages) {
          atomicOr(p.status, OOMB_DEV_BAD_PAGE);
          page = -1;
        }
      }
#pragma unroll 1
      for (int cc = 0; cc < kBN / 32; ++cc) {
        const int n = n0 + cc * 32;          // first output column of this chunk
        uint32_t a[32];
        tmem_ld32(tmem + lane_off + cc * 32, a);
        tmem_ld_wait();
        if (n >= p.n_end) continue;          // columns past the launch's range (warp-uniform)
        // round to bf16; the sums below are taken over the rounded values
        uint32_t pk[16];
        float v[32];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          pk[e] = pack_bf16(__uint_as_float(a[2 * e]), __uint_as_float(a[2 * e + 1]));
          const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&pk[e]);
          v[2 * e] = valid ? __low2float(b2) : 0.f;
          v[2 * e + 1] = valid ? __high2float(b2) : 0.f;
        }
        if (n < nq) {                        // Q columns of head h
          const int h = n / p.D, dim0 = n % p.D;
          if (valid && p.q) {
            uint4* dst = reinterpret_cast<uint4*>(p.q + (static_cast<size_t>(t) * p.Hq + h) * p.D + dim0);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
          if (p.qsum) {
            const float s = column_sums(v);
            atomicAdd(p.qsum + (h / p.G) * p.D + dim0 + lane, s);
          }
        } else {                             // K or V columns of KV head g
          const int nn = n - nq;
          const int which = nn >= nk ? 1 : 0;  // 0 = K, 1 = V
          const int g = (nn - which * nk) / p.D, dim0 = (nn - which * nk) % p.D;
          if (page >= 0) {
            const size_t blk = (static_cast<size_t>(page) * p.Hkv + g) * 2 + which;
            uint4* dst = reinterpret_cast<uint4*>(p.kv + (blk * p.P + t % p.P) * p.D + dim0);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
          if (which == 0) {
            // page means of K: this warp's 32 rows hold 32 / P pages (P < 32),
            // one page, or part of one (P > 32); sum per page, then add
            const int span = p.P < 32 ? p.P : 32;
            for (int j = 0; j < 32 / span; ++j) {
              float w[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) w[e] = (lane / span == j) ? v[e] : 0.f;
              const float s = column_sums(w);
              const int tj = m0 + lg * 32 + j * span;  // first token of that page part
              if (tj < p.C) {
                const int pg = p.page_ids[tj / p.P];
                if (pg >= 0 && pg < p.num_pages)
                  atomicAdd(p.summary + (static_cast<size_t>(pg) * p.Hkv + g) * p.D + dim0 + lane,
                            s / static_cast<float>(p.P));
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (abort_sh && warp == 0 && lane == 0) {
    for (int i = used_sh; i < issued_sh; ++i)
      mbar_wait_drain(&bar_full[i % kStages], (i / kStages) & 1);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kBN);
  }
}

// Zero the page means and gradient blocks of the chunk's pages (the epilogue
// adds into the means).  grid (pages, Hkv).
__global__ void proj_prepare_kernel(const int32_t* __restrict__ page_ids, float* summary,
                                    float* grad, int Hkv, int D, int P, int num_pages,
                                    uint32_t* status) {
  const int page = page_ids[blockIdx.x], g = blockIdx.y;
  if (page < 0 || page >= num_pages) {
    if (threadIdx.x == 0) atomicOr(status, OOMB_DEV_BAD_PAGE);
    return;
  }
  const size_t blk = static_cast<size_t>(page) * Hkv + g;
  for (int e = threadIdx.x; e < D; e += blockDim.x) summary[blk * D + e] = 0.f;
  if (grad) {
    float4* gz = reinterpret_cast<float4*>(grad + blk * 2 * P * D);
    const int n4 = 2 * P * D / 4;
    for (int e = threadIdx.x; e < n4; e += blockDim.x) gz[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

bool make_rows_map(CUtensorMap* m, const void* base, int inner, int rows, int box_rows) {
  const uint64_t dims[2] = {static_cast<uint64_t>(inner), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(inner) * 2};
  const uint32_t box[2] = {kBK, static_cast<uint32_t>(box_rows)};
  return make_bf16_map(m, base, 2, dims, strides, box);
}

}  // namespace

extern "C" oomb_status oomb_qkv_project(oomb_pool* pool, const void* d_x, const void* d_w,
                                        int32_t chunk_len, int32_t hidden, int32_t num_q_heads,
                                        int32_t part, void* d_q, float* d_qsum,
                                        const int32_t* d_page_ids, void* stream) {
  if (!pool || pool->desc.location != OOMB_LOC_DEVICE || !d_x || !d_w) return OOMB_ERR_INVALID_ARG;
  const oomb_pool_desc& d = pool->desc;
  const int Hkv = d.num_kv_heads, D = d.head_dim, P = d.page_size;
  if (part < OOMB_PROJ_Q || part > OOMB_PROJ_QKV) return OOMB_ERR_INVALID_ARG;
  if (chunk_len <= 0 || chunk_len % P != 0 || hidden <= 0 || hidden % kBK != 0)
    return OOMB_ERR_INVALID_ARG;
  if (num_q_heads <= 0 || num_q_heads % Hkv != 0) return OOMB_ERR_INVALID_ARG;
  const bool do_q = part != OOMB_PROJ_KV, do_kv = part != OOMB_PROJ_Q;
  if (do_q && !d_q && !d_qsum) return OOMB_ERR_INVALID_ARG;
  if (do_kv && !d_page_ids) return OOMB_ERR_INVALID_ARG;
  if (!aligned16(d_x) || !aligned16(d_w) || (d_q && !aligned16(d_q))) return OOMB_ERR_INVALID_ARG;
  DeviceGuard guard(d.device);
  static std::atomic<uint64_t> attr_done{0};
  if (!once_per_device(attr_done, [] {
        return cudaFuncSetAttribute(proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kProjSmem) == cudaSuccess;
      }))
    return OOMB_ERR_CUDA;
  const int nq = num_q_heads * D, n_out = nq + 2 * Hkv * D;
  CUtensorMap xmap, wmap;
  if (!make_rows_map(&xmap, d_x, hidden, chunk_len, kBM) ||
      !make_rows_map(&wmap, d_w, hidden, n_out, kBN))
    return OOMB_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ProjParams p;
  p.q = static_cast<__nv_bfloat16*>(d_q);
  p.qsum = d_qsum;
  p.page_ids = d_page_ids;
  p.kv = static_cast<__nv_bfloat16*>(pool->kv);
  p.summary = pool->summary;
  p.status = pool->d_status;
  p.C = chunk_len;
  p.Hq = num_q_heads;
  p.Hkv = Hkv;
  p.G = num_q_heads / Hkv;
  p.D = D;
  p.P = P;
  p.num_pages = d.num_pages;
  p.k_tiles = hidden / kBK;
  p.n_base = do_q ? 0 : nq;
  p.n_end = do_kv ? n_out : nq;
  if (do_q && d_qsum &&
      cudaMemsetAsync(d_qsum, 0, static_cast<size_t>(Hkv) * D * sizeof(float), s) != cudaSuccess)
    return OOMB_ERR_CUDA;
  if (do_kv) {
    proj_prepare_kernel<<<dim3(chunk_len / P, Hkv), 128, 0, s>>>(
        d_page_ids, pool->summary, pool->grad, Hkv, D, P, d.num_pages, pool->d_status);
    if (check_launch() != OOMB_OK) return OOMB_ERR_CUDA;
  }
  const dim3 grid((chunk_len + kBM - 1) / kBM, (p.n_end - p.n_base + kBN - 1) / kBN);
  proj_kernel<<<grid, kProjThreads, kProjSmem, s>>>(p, xmap, wmap);
  return check_launch();
}
