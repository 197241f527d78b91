// Chunk attention backward over the paged KV cache (tcgen05 + TMA, sm_100a).
//
// "Out of the Memory Barrier" ([pt] §2B "Kernels Personalizados": gradients
// accumulated in place, outside autograd; [es] §2B: the operators are opaque
// to autograd and need no intermediate buffers; [it] §2B: in-place
// accumulation with atomic_add).  For the loss sum(O * dO):
//   D_i  = dO_i . O_i                         (preprocess)
//   P_ij = exp(S_ij - LSE_i),  dS_ij = P_ij (dO_i . v_j - D_i)
//   dK_j += scale sum_i dS_ij q_i,  dV_j += sum_i P_ij dO_i   (KV-major kernel,
//           summed over every query head of the group, then added into the
//           fp32 gradient pool with vector atomics)
//   dQ_i  = scale sum_j dS_ij k_j                               (Q-major kernel)
// The dQ kernel recomputes S and dP rather than reducing dQ across KV tiles:
// the chunk's rows are few (C * G per group) and the keys many, so a KV-major
// dQ would need a large reduction per chunk.
#include "internal.h"
#include "ptx.cuh"
#include "tiles.cuh"
#include "tmap.h"

namespace {

using namespace oomb;

constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* d_o;
  const float* lse;
  float* delta;
  __nv_bfloat16* dq;
  float* grad;
  const int32_t* past_pages;
  const int32_t* past_counts;
  const int32_t* cur_pages;
  uint32_t* status;
  int max_past, C, Hq, Hkv, G, P, num_pool_pages, max_past_tiles;
  int lpq;  // 1: one past list per (query tile, group); dK/dV: blockIdx.z = query tile
            // 2: per query page (union lists + membership masks), as 1 otherwise
  int seg;  // OOMB_SEG_*: whole key set, or a segment accumulated into dq_acc
  float* dq_acc;
  const uint8_t* masks;  // lpq 2: query-page membership bits of each list entry
  int lg_p;              // log2(P)
  float scale, scale_log2;
};

// ------------------------------------------------------------------ preprocess
// delta[h][q] = sum_d dO[q][h][d] * O[q][h][d], fp32; D/8 lanes per row, 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const BwdParams p) {
  constexpr int LPR = D / 8;
  constexpr int RPB = 256 / LPR;  // rows per block per pass
  const int t = threadIdx.x;
  const int row = blockIdx.x * RPB + t / LPR;
  const int sub = t % LPR;
  const int rows = p.C * p.Hq;
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = *reinterpret_cast<const uint4*>(p.o + static_cast<size_t>(row) * D + sub * 8);
    const uint4 b = *reinterpret_cast<const uint4*>(p.d_o + static_cast<size_t>(row) * D + sub * 8);
    const __nv_bfloat16* av = reinterpret_cast<const __nv_bfloat16*>(&a);
    const __nv_bfloat16* bv = reinterpret_cast<const __nv_bfloat16*>(&b);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc += __bfloat162float(av[e]) * __bfloat162float(bv[e]);
  }
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && sub == 0) {
    const int q = row / p.Hq, h = row % p.Hq;
    p.delta[static_cast<size_t>(h) * p.C + q] = acc;
  }
}

// ------------------------------------------------------------------ dK / dV
// One CTA per (KV tile of 128 keys, KV head g); loops over the group's query
// tiles (G heads x 128-row tiles; for the chunk's own keys only the causally
// reachable tiles).  Warps 0-7 compute: warps w and w+4 share keys
// 32(w%4)..+31 (TMEM lanes); warp w < 4 takes query columns 0-63 (and d
// columns [0, D/2) in the epilogue), warp w >= 4 the other halves.  Warp 8
// loads (TMA), warp 9 issues UMMA.
// TMEM: S^T [0,128) (then P^T bf16: query half k in [64k, 64k+32)), dP^T
// [128,256) (then dS^T likewise), dV [256,256+D), dK [256+D, 256+2D).
template <int D>
struct KvCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kNS = 2;
  static constexpr int kStageBytes = 2 * kTileBytes + 1024;  // Q, dO, LSE[128], delta[128]
  static constexpr int kSmem = 2 * kTileBytes + kNS * kStageBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColST = 0, kColDPT = 128, kColDV = 256, kColDK = 256 + D;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    bwd_dkdv_kernel(const BwdParams p, const __grid_constant__ CUtensorMap qmap,
                    const __grid_constant__ CUtensorMap domap,
                    const __grid_constant__ CUtensorMap kvmap) {
  using Cfg = KvCfg<D>;
  const int g = blockIdx.y;
  // with one list per query tile this CTA serves query tile blockIdx.z only
  // (the chunk's own tiles then come from a separate launch without lists)
  const int qsel = p.lpq ? static_cast<int>(blockIdx.z) : 0;
  const int li = (p.lpq ? qsel * p.Hkv : 0) + g;
  const KvSchedule sch = kv_schedule(p.past_counts ? p.past_counts + (li - g) : nullptr, g,
                                     p.max_past, p.P, p.status);
  const bool is_past = static_cast<int>(blockIdx.x) < p.max_past_tiles;
  if (is_past && static_cast<int>(blockIdx.x) >= sch.n_past_tiles) return;  // beyond the list
  const int u = is_past ? 0 : static_cast<int>(blockIdx.x) - p.max_past_tiles;  // current tile
  const int j = is_past ? static_cast<int>(blockIdx.x) : sch.n_past_tiles + u;    // schedule index
  const int n_qtiles = (p.C + kTile - 1) / kTile;
  const int t0 = p.lpq ? qsel : (is_past ? 0 : u);  // first query tile that can see these keys
  const int n_qt = p.lpq ? 1 : n_qtiles - t0;
  const int n_iter = p.G * n_qt;
  const int n_cur_pages = p.C / p.P;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + Cfg::kTileBytes;
  uint8_t* sStage = sV + Cfg::kTileBytes;
  auto sQ = [&](int s) { return sStage + s * Cfg::kStageBytes; };
  auto sDO = [&](int s) { return sStage + s * Cfg::kStageBytes + Cfg::kTileBytes; };
  auto sL = [&](int s) {
    return reinterpret_cast<float*>(sStage + s * Cfg::kStageBytes + 2 * Cfg::kTileBytes);
  };
  auto sDl = [&](int s) {
    return reinterpret_cast<float*>(sStage + s * Cfg::kStageBytes + 2 * Cfg::kTileBytes + 512);
  };

  __shared__ uint64_t bar_kv, bar_qf[Cfg::kNS], bar_qe[Cfg::kNS];
  __shared__ uint64_t bar_st, bar_sl, bar_dpt, bar_p, bar_ds, bar_acc, bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh, q_issued_sh, q_used_sh, kv_issued_sh;

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    abort_sh = 0;
    q_issued_sh = q_used_sh = kv_issued_sh = 0;
    mbar_init(&bar_kv, 1);
    for (int i = 0; i < Cfg::kNS; ++i) {
      mbar_init(&bar_qf[i], 1);
      mbar_init(&bar_qe[i], 1);
    }
    mbar_init(&bar_st, 1);
    mbar_init(&bar_sl, 8);
    mbar_init(&bar_dpt, 1);
    mbar_init(&bar_p, 8);
    mbar_init(&bar_ds, 8);
    mbar_init(&bar_acc, 1);
    mbar_init(&bar_drain, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;
  const int32_t* past_list = p.past_pages ? p.past_pages + static_cast<size_t>(li) * p.max_past
                                          : nullptr;

  if (warp == 8) {
    if (lane == 0) {
      prefetch_tensormap(&qmap);
      prefetch_tensormap(&domap);
      prefetch_tensormap(&kvmap);
      const int per = kTile / p.P;
      mbar_arrive_expect_tx(&bar_kv, 2 * Cfg::kTileBytes);
      for (int s = 0; s < per; ++s) {
        const int pg = tile_page(j, s, sch, past_list, p.cur_pages, n_cur_pages, p.P,
                                 p.num_pool_pages, p.status);
        for (int hf = 0; hf < Cfg::kHalves; ++hf) {
          tma_load_4d(sK + hf * kTile * 128 + s * p.P * 128, &kvmap, &bar_kv, hf * 64, 0, 2 * g,
                      pg);
          tma_load_4d(sV + hf * kTile * 128 + s * p.P * 128, &kvmap, &bar_kv, hf * 64, 0,
                      2 * g + 1, pg);
        }
      }
      kv_issued_sh = 1;
      int issued = 0;
      for (int i = 0; i < n_iter; ++i) {
        const int s = i % Cfg::kNS;
        const int head = g * p.G + i / n_qt, t = t0 + i % n_qt;
        const int nvalid = min(kTile, p.C - t * kTile);
        if (!mbar_wait(&bar_qe[s], ((i / Cfg::kNS) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&bar_qf[s], 2 * Cfg::kTileBytes + 2 * nvalid * 4);
        for (int hf = 0; hf < Cfg::kHalves; ++hf) {
          tma_load_3d(sQ(s) + hf * kTile * 128, &qmap, &bar_qf[s], hf * 64, head, t * kTile);
          tma_load_3d(sDO(s) + hf * kTile * 128, &domap, &bar_qf[s], hf * 64, head, t * kTile);
        }
        const size_t row0 = static_cast<size_t>(head) * p.C + t * kTile;
        bulk_load(sL(s), p.lse + row0, nvalid * 4, &bar_qf[s]);
        bulk_load(sDl(s), p.delta + row0, nvalid * 4, &bar_qf[s]);
        ++issued;
      }
      if (*abort_flag) atomicOr(p.status, OOMB_DEV_WAIT_LIMIT);
      q_issued_sh = issued;
    }
  } else if (warp == 9) {
    if (lane == 0) {
      // Order per query tile i: S^T_{i+1} as soon as the compute warps hold S^T_i
      // in registers; dV_i once P^T_i is in TMEM, dK_i once dS^T_i is; then
      // dP^T_{i+1}.
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      int used = 0;
      auto issue_s = [&](int i) -> bool {  // S^T_i = K Q_i^T
        const int s = i % Cfg::kNS;
        if (!mbar_wait(&bar_qf[s], (i / Cfg::kNS) & 1, abort_flag)) return false;
        ++used;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQ(s));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * (kTile * 128) + (kk % 4) * 32;
          umma_ss(tmem + Cfg::kColST, sw128_desc(k_addr + off, 16, 1024),
                  sw128_desc(q_addr + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(&bar_st);
        return true;
      };
      auto issue_dp = [&](int i) {  // dP^T_i = V dO_i^T (its stage is already resident)
        const uint32_t do_addr = smem_u32(sDO(i % Cfg::kNS));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * (kTile * 128) + (kk % 4) * 32;
          umma_ss(tmem + Cfg::kColDPT, sw128_desc(v_addr + off, 16, 1024),
                  sw128_desc(do_addr + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(&bar_dpt);
      };
      bool ok = mbar_wait(&bar_kv, 0, abort_flag);
      if (ok && n_iter > 0) {
        ok = issue_s(0);
        if (ok) issue_dp(0);
      }
      for (int i = 0; ok && i < n_iter; ++i) {
        const int s = i % Cfg::kNS;
        if (i + 1 < n_iter) {
          if (!(ok = mbar_wait(&bar_sl, i & 1, abort_flag))) break;
          if (!(ok = issue_s(i + 1))) break;
        }
        // dV += P^T_i dO_i as soon as P^T_i is in TMEM (while the compute warps
        // still form dS^T_i); dK += dS^T_i Q_i once dS^T_i is there.  Both A
        // operands are packed in the (already read) dP^T columns.
        if (!(ok = mbar_wait(&bar_p, i & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQ(s)), do_addr = smem_u32(sDO(s));
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ts(tmem + Cfg::kColDV, tmem + Cfg::kColDPT + (kk / 4) * 64 + (kk % 4) * 8,
                  sw128_desc(do_addr + kk * 16 * 128, kTile * 128, 1024), idesc_acc,
                  (i > 0 || kk > 0) ? 1u : 0u);
        if (!(ok = mbar_wait(&bar_ds, i & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ts(tmem + Cfg::kColDK, tmem + Cfg::kColDPT + (kk / 4) * 64 + 32 + (kk % 4) * 8,
                  sw128_desc(q_addr + kk * 16 * 128, kTile * 128, 1024), idesc_acc,
                  (i > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&bar_qe[s]);
        if (i + 1 < n_iter) issue_dp(i + 1);
      }
      if (ok && n_iter > 0) umma_commit(&bar_acc);
      if (!ok) {
        *abort_flag = 1;
        atomicOr(p.status, OOMB_DEV_WAIT_LIMIT);
      }
      umma_commit(&bar_drain);
      mbar_wait_drain(&bar_drain, 0);
      q_used_sh = used;
    }
  } else {
    const int lg = warp & 3, half = warp >> 2;  // lane group, query/d column half
    const int r = lg * 32 + lane;               // key row (TMEM lane)
    const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
    const uint32_t cs = half * 64;              // this half's columns in S^T / dP^T
    bool key_valid;
    if (is_past) key_valid = j * kTile + r < sch.n_past_pages * p.P;
    else key_valid = u * kTile + r < p.C;
    const int key_local = u * kTile + r;  // causal position (current tiles only)
    // Groups of 16 query columns of this half that may hold a valid (key,
    // query) pair, constant over the loop (P >= 16, so a group lies in one
    // query page): none for a key row past the list; with per-query-page
    // lists, the groups whose query page listed this key row's page (bit
    // (cs + 16 k) / P of the entry's membership mask).
    uint32_t grp = key_valid ? 0xFu : 0u;
    if (p.masks && is_past && key_valid) {
      const uint32_t qm =
          p.masks[static_cast<size_t>(li) * p.max_past + ((j * kTile + r) >> p.lg_p)];
      grp = 0;
      for (int k = 0; k < 4; ++k) grp |= ((qm >> ((half * 64 + 16 * k) >> p.lg_p)) & 1u) << k;
    }
    bool ok = true;
    for (int i = 0; i < n_iter; ++i) {
      const int s = i % Cfg::kNS;
      const int t = t0 + i % n_qt;
      if (!(ok = warp_wait(&bar_st, i & 1, abort_flag))) break;
      if (!(ok = warp_wait(&bar_qf[s], (i / Cfg::kNS) & 1, abort_flag))) break;
      tc_fence_after();
      float pr[64];
      tmem_ld32(tmem + lane_off + Cfg::kColST + cs, reinterpret_cast<uint32_t*>(pr));
      tmem_ld32(tmem + lane_off + Cfg::kColST + cs + 32, reinterpret_cast<uint32_t*>(pr + 32));
      tmem_ld_wait();
      // S^T_i is in registers: the next S^T may overwrite its columns
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_sl);
      const float* L = sL(s) + cs;
      // query column c (of this half) is valid if inside the chunk and, for the
      // chunk's own keys, causally at or after the key
      const int cmax = min(kTile, p.C - t * kTile) - static_cast<int>(cs);
      const int cmin = (is_past ? 0 : key_local - t * kTile) - static_cast<int>(cs);
      const bool full = grp == 0xFu && cmin <= 0 && cmax >= 64;
      // P^T = 2^(S^T*scale*log2e - LSE*log2e); LSE read 4 at a time (broadcast)
#pragma unroll
      for (int c4 = 0; c4 < 16; ++c4) {
        const float4 l4 = *reinterpret_cast<const float4*>(L + 4 * c4);
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 4 * c4 + e;
          pr[c] = fast_exp2(fmaf(pr[c], p.scale_log2, -lv[e] * kLog2e));
        }
      }
      if (!full) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          pr[c] = (c < cmax && c >= cmin && ((grp >> (c >> 4)) & 1u)) ? pr[c] : 0.f;
      }
      if (!(ok = warp_wait(&bar_dpt, i & 1, abort_flag))) break;
      tc_fence_after();
      uint32_t dp[64];
      tmem_ld32(tmem + lane_off + Cfg::kColDPT + cs, dp);
      tmem_ld32(tmem + lane_off + Cfg::kColDPT + cs + 32, dp + 32);
      tmem_ld_wait();
      {
        // P^T (bf16) into this half's first 32 dP^T columns, already read: the
        // dV product can start while dS^T is formed
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = pack_bf16(pr[2 * c], pr[2 * c + 1]);
        tmem_st16(tmem + lane_off + Cfg::kColDPT + cs, pk);
        tmem_st16(tmem + lane_off + Cfg::kColDPT + cs + 16, pk + 16);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_p);
      }
      const float* Dl = sDl(s) + cs;
      uint32_t dsk[32];
#pragma unroll
      for (int e4 = 0; e4 < 16; ++e4) {
        const float4 d4 = *reinterpret_cast<const float4*>(Dl + 4 * e4);
        const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
        float ds[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c0 = 4 * e4 + e;
          ds[e] = pr[c0] * (__uint_as_float(dp[c0]) - dv[e]);
          // masked columns may hold stale delta values: force an exact zero
          if (!full) ds[e] = pr[c0] != 0.f ? ds[e] : 0.f;
        }
        dsk[2 * e4] = pack_bf16(ds[0], ds[1]);
        dsk[2 * e4 + 1] = pack_bf16(ds[2], ds[3]);
      }
      // dS^T (bf16) into this half's last 32 dP^T columns, already read
      tmem_st16(tmem + lane_off + Cfg::kColDPT + cs + 32, dsk);
      tmem_st16(tmem + lane_off + Cfg::kColDPT + cs + 48, dsk + 16);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_ds);
    }
    if (ok && n_iter > 0) ok = warp_wait(&bar_acc, 0, abort_flag);
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(p.status, OOMB_DEV_WAIT_LIMIT);
    } else if (n_iter > 0) {
      tc_fence_after();
      int page = -1;
      if (key_valid)
        page = tile_page(j, r / p.P, sch, past_list, p.cur_pages, n_cur_pages, p.P,
                         p.num_pool_pages, p.status);
      const bool write = key_valid && page >= 0 && page < p.num_pool_pages;
      const size_t blk = (static_cast<size_t>(write ? page : 0) * p.Hkv + g) * 2;
      const int d0 = half * (D / 2);
      float* gk = p.grad + (blk * p.P + r % p.P) * D + d0;
      float* gv = p.grad + ((blk + 1) * p.P + r % p.P) * D + d0;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t a[32], bb[32];
        tmem_ld32(tmem + lane_off + Cfg::kColDK + d0 + c * 32, a);
        tmem_ld32(tmem + lane_off + Cfg::kColDV + d0 + c * 32, bb);
        tmem_ld_wait();
        if (write) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            atomicAdd(reinterpret_cast<float4*>(gk + c * 32 + 4 * e),
                      make_float4(__uint_as_float(a[4 * e]) * p.scale,
                                  __uint_as_float(a[4 * e + 1]) * p.scale,
                                  __uint_as_float(a[4 * e + 2]) * p.scale,
                                  __uint_as_float(a[4 * e + 3]) * p.scale));
            atomicAdd(reinterpret_cast<float4*>(gv + c * 32 + 4 * e),
                      make_float4(__uint_as_float(bb[4 * e]), __uint_as_float(bb[4 * e + 1]),
                                  __uint_as_float(bb[4 * e + 2]), __uint_as_float(bb[4 * e + 3])));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8 && lane == 0) {
    // Loads that were issued but never consumed must land before the CTA exits.
    if (kv_issued_sh && (abort_sh || n_iter == 0)) mbar_wait_drain(&bar_kv, 0);
    if (abort_sh)
      for (int i = q_used_sh; i < q_issued_sh; ++i)
        mbar_wait_drain(&bar_qf[i % Cfg::kNS], (i / Cfg::kNS) & 1);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// ------------------------------------------------------------------ dQ
// One CTA per (128-row query tile, head).  Q and dO are copied into TMEM once
// and serve as the A operands of S = Q K_j^T and dP = dO V_j^T, so those
// UMMAs read only K_j or V_j from shared memory.  S_{j+1} is computed while
// the compute warps work on tile j; dS_j (bf16) goes into the dP columns the
// warps have already read and feeds dQ += dS_j K_j.
// Warps 0-7 compute (warps w and w+4 share rows 32(w%4)..+31; w < 4 takes key
// columns 0-63 and copies Q into TMEM, w >= 4 the other half and dO), warp 8
// loads Q, dO and the K tiles, warp 10 the V tiles, warp 9 issues UMMA:
//   S(0) dP(0) | S(j+1) dQ(j) dP(j+1) for j = 0, 1, ...
// TMEM: S [0,128), dP [128,256) (dS of key half k: [128+64k, +32)), dQ
// [256, 256+D), Q [384, 384+D/2), dO [448, 448+D/2).
template <int D>
struct QCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kNK = 3, kNV = 2;
  static constexpr int kSmem = kTileBytes * (2 + kNK + kNV) + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256, kColQ = 384, kColDO = 448;
};

template <int D>
__global__ void __launch_bounds__(352, 1)
    bwd_dq_kernel(const BwdParams p, const __grid_constant__ CUtensorMap qmap,
                  const __grid_constant__ CUtensorMap domap,
                  const __grid_constant__ CUtensorMap kvmap) {
  using Cfg = QCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sDO = sQ + Cfg::kTileBytes;
  uint8_t* sK = sDO + Cfg::kTileBytes;
  uint8_t* sV = sK + Cfg::kNK * Cfg::kTileBytes;

  __shared__ uint64_t bar_q, bar_qt, bar_kf[Cfg::kNK], bar_ke[Cfg::kNK], bar_vf[Cfg::kNV],
      bar_ve[Cfg::kNV];
  __shared__ uint64_t bar_s, bar_sl, bar_dp, bar_ds, bar_fin, bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh, k_issued_sh, v_issued_sh, k_used_sh, v_used_sh;

  const int warp = warp_id(), lane = lane_id();
  const int qt = blockIdx.x, h = blockIdx.y, g = h / p.G;
  const int li = (p.lpq ? qt * p.Hkv : 0) + g;
  const KvSchedule sch = kv_schedule(p.past_counts ? p.past_counts + (li - g) : nullptr, g,
                                     p.max_past, p.P, p.status);
  // past tiles + (unless this call is a past-only segment) the chunk's tiles
  const bool with_cur = p.seg == OOMB_SEG_WHOLE || p.seg == OOMB_SEG_LAST;
  const int T = sch.n_past_tiles + (with_cur ? qt + 1 : 0);
  const int n_cur_pages = p.C / p.P;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    k_issued_sh = v_issued_sh = k_used_sh = v_used_sh = 0;
    mbar_init(&bar_q, 1);
    mbar_init(&bar_qt, 8);
    for (int i = 0; i < Cfg::kNK; ++i) {
      mbar_init(&bar_kf[i], 1);
      mbar_init(&bar_ke[i], 1);
    }
    for (int i = 0; i < Cfg::kNV; ++i) {
      mbar_init(&bar_vf[i], 1);
      mbar_init(&bar_ve[i], 1);
    }
    mbar_init(&bar_s, 1);
    mbar_init(&bar_sl, 8);
    mbar_init(&bar_dp, 1);
    mbar_init(&bar_ds, 8);
    mbar_init(&bar_fin, 1);
    mbar_init(&bar_drain, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  volatile int* abort_flag = &abort_sh;

  if (warp == 8 || warp == 10) {
    if (lane == 0) {
      const bool is_k = warp == 8;
      if (is_k) {
        prefetch_tensormap(&qmap);
        prefetch_tensormap(&domap);
        mbar_arrive_expect_tx(&bar_q, 2 * Cfg::kTileBytes);
        for (int hf = 0; hf < Cfg::kHalves; ++hf) {
          tma_load_3d(sQ + hf * kTile * 128, &qmap, &bar_q, hf * 64, h, qt * kTile);
          tma_load_3d(sDO + hf * kTile * 128, &domap, &bar_q, hf * 64, h, qt * kTile);
        }
      }
      prefetch_tensormap(&kvmap);
      const int32_t* past_list =
          p.past_pages ? p.past_pages + static_cast<size_t>(li) * p.max_past : nullptr;
      const int per = kTile / p.P;
      const int nst = is_k ? Cfg::kNK : Cfg::kNV;
      uint64_t* full = is_k ? bar_kf : bar_vf;
      uint64_t* empty = is_k ? bar_ke : bar_ve;
      uint8_t* base = is_k ? sK : sV;
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        int pg[8];
        for (int s = 0; s < per; ++s)
          pg[s] = tile_page(j, s, sch, past_list, p.cur_pages, n_cur_pages, p.P,
                            p.num_pool_pages, is_k ? p.status : nullptr);
        const int st = j % nst;
        if (!mbar_wait(&empty[st], ((j / nst) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&full[st], Cfg::kTileBytes);
        for (int s = 0; s < per; ++s)
          for (int hf = 0; hf < Cfg::kHalves; ++hf)
            tma_load_4d(base + st * Cfg::kTileBytes + hf * kTile * 128 + s * p.P * 128, &kvmap,
                        &full[st], hf * 64, 0, 2 * g + (is_k ? 0 : 1), pg[s]);
        ++issued;
      }
      if (*abort_flag) atomicOr(p.status, OOMB_DEV_WAIT_LIMIT);
      if (is_k) k_issued_sh = issued;
      else v_issued_sh = issued;
    }
  } else if (warp == 9) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      int k_used = 0, v_used = 0;
      auto issue_s = [&](int j) -> bool {  // S(j) = Q K_j^T, Q from TMEM
        const int ks = j % Cfg::kNK;
        if (!mbar_wait(&bar_kf[ks], (j / Cfg::kNK) & 1, abort_flag)) return false;
        ++k_used;
        tc_fence_after();
        const uint32_t kb = k_addr + ks * Cfg::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * (kTile * 128) + (kk % 4) * 32;
          umma_ts(tmem + Cfg::kColS, tmem + Cfg::kColQ + kk * 8, sw128_desc(kb + off, 16, 1024),
                  idesc_s, kk > 0);
        }
        umma_commit(&bar_s);
        return true;
      };
      auto issue_dp = [&](int j) -> bool {  // dP(j) = dO V_j^T, dO from TMEM
        const int vs = j % Cfg::kNV;
        if (!mbar_wait(&bar_vf[vs], (j / Cfg::kNV) & 1, abort_flag)) return false;
        ++v_used;
        tc_fence_after();
        const uint32_t vb = v_addr + vs * Cfg::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * (kTile * 128) + (kk % 4) * 32;
          umma_ts(tmem + Cfg::kColDP, tmem + Cfg::kColDO + kk * 8,
                  sw128_desc(vb + off, 16, 1024), idesc_s, kk > 0);
        }
        umma_commit(&bar_ve[vs]);
        umma_commit(&bar_dp);
        return true;
      };
      bool ok = mbar_wait(&bar_qt, 0, abort_flag);  // Q and dO are in TMEM
      if (T > 0) ok = ok && issue_s(0) && issue_dp(0);
      for (int j = 0; ok && j < T; ++j) {
        if (j + 1 < T) {
          if (!(ok = mbar_wait(&bar_sl, j & 1, abort_flag))) break;  // S(j) in registers
          if (!(ok = issue_s(j + 1))) break;
        }
        if (!(ok = mbar_wait(&bar_ds, j & 1, abort_flag))) break;
        tc_fence_after();
        const int ks = j % Cfg::kNK;
        const uint32_t kb = k_addr + ks * Cfg::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ts(tmem + Cfg::kColDQ, tmem + Cfg::kColDP + (kk / 4) * 64 + (kk % 4) * 8,
                  sw128_desc(kb + kk * 16 * 128, kTile * 128, 1024), idesc_dq,
                  (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&bar_ke[ks]);
        if (j + 1 < T && !(ok = issue_dp(j + 1))) break;
      }
      if (ok) umma_commit(&bar_fin);
      if (!ok) {
        *abort_flag = 1;
        atomicOr(p.status, OOMB_DEV_WAIT_LIMIT);
      }
      umma_commit(&bar_drain);
      mbar_wait_drain(&bar_drain, 0);
      k_used_sh = k_used;
      v_used_sh = v_used;
    }
  } else if (warp < 8) {
    const int lg = warp & 3, half = warp >> 2;  // lane group, key/d column half
    const int r = lg * 32 + lane;               // query row (TMEM lane)
    const int q_local = qt * kTile + r;
    const bool row_valid = q_local < p.C;
    const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
    const uint32_t cs = half * 64;
    const float lse2 = row_valid ? p.lse[static_cast<size_t>(h) * p.C + q_local] * kLog2e : 0.f;
    const float dl = row_valid ? p.delta[static_cast<size_t>(h) * p.C + q_local] : 0.f;
    const int n_past_keys = sch.n_past_pages * p.P;
    // half 0 copies its Q row, half 1 its dO row, into TMEM (packed bf16 pairs)
    bool ok = warp_wait(&bar_q, 0, abort_flag);
    if (ok) {
      const uint8_t* src = half == 0 ? sQ : sDO;
      const uint32_t col = half == 0 ? Cfg::kColQ : Cfg::kColDO;
#pragma unroll
      for (int hf = 0; hf < Cfg::kHalves; ++hf) {
        uint32_t v[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 x = *reinterpret_cast<const uint4*>(src + hf * kTile * 128 +
                                                          sw128_offset(r, ch * 8));
          v[4 * ch] = x.x;
          v[4 * ch + 1] = x.y;
          v[4 * ch + 2] = x.z;
          v[4 * ch + 3] = x.w;
        }
        tmem_st32(tmem + lane_off + col + hf * 32, v);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_qt);
    }
    for (int j = 0; ok && j < T; ++j) {
      if (!(ok = warp_wait(&bar_s, j & 1, abort_flag))) break;
      tc_fence_after();
      float pr[64];
      tmem_ld32(tmem + lane_off + Cfg::kColS + cs, reinterpret_cast<uint32_t*>(pr));
      tmem_ld32(tmem + lane_off + Cfg::kColS + cs + 32, reinterpret_cast<uint32_t*>(pr + 32));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_sl);  // the next S may overwrite these columns
      int lim;
      if (j < sch.n_past_tiles) lim = n_past_keys - j * kTile;
      else lim = min(p.C, q_local + 1) - (j - sch.n_past_tiles) * kTile;
      if (!row_valid) lim = 0;
      lim -= static_cast<int>(cs);
#pragma unroll
      for (int c = 0; c < 64; ++c) pr[c] = fast_exp2(fmaf(pr[c], p.scale_log2, -lse2));
      if (lim < 64) {
#pragma unroll
        for (int c = 0; c < 64; ++c) pr[c] = c < lim ? pr[c] : 0.f;
      }
      if (p.masks && j < sch.n_past_tiles) {
        // per-query-page lists: pages this row's query page did not select
        const int per = kTile >> p.lg_p;
        const uint8_t* mrow = p.masks + static_cast<size_t>(li) * p.max_past + j * per;
        const int qb = r >> p.lg_p;
        // bit k: this half's columns [16k, 16k + 16) (one page: P >= 16) are kept
        uint32_t keep = 0;
        for (int k = 0; k < 4; ++k) {
          const int sl = (static_cast<int>(cs) + 16 * k) >> p.lg_p;
          if (j * per + sl < sch.n_past_pages && ((mrow[sl] >> qb) & 1u)) keep |= 1u << k;
        }
        if (keep != 0xFu) {
#pragma unroll
          for (int c = 0; c < 64; ++c) pr[c] = ((keep >> (c >> 4)) & 1u) ? pr[c] : 0.f;
        }
      }
      if (!(ok = warp_wait(&bar_dp, j & 1, abort_flag))) break;
      tc_fence_after();
      uint32_t dp[64];
      tmem_ld32(tmem + lane_off + Cfg::kColDP + cs, dp);
      tmem_ld32(tmem + lane_off + Cfg::kColDP + cs + 32, dp + 32);
      tmem_ld_wait();
      uint32_t ds[32];
#pragma unroll
      for (int e = 0; e < 32; ++e)
        ds[e] = pack_bf16(pr[2 * e] * (__uint_as_float(dp[2 * e]) - dl),
                          pr[2 * e + 1] * (__uint_as_float(dp[2 * e + 1]) - dl));
      tmem_st16(tmem + lane_off + Cfg::kColDP + cs, ds);
      tmem_st16(tmem + lane_off + Cfg::kColDP + cs + 16, ds + 16);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_ds);
    }
    if (ok) ok = warp_wait(&bar_fin, 0, abort_flag);
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(p.status, OOMB_DEV_WAIT_LIMIT);
    } else {
      tc_fence_after();
      const int d0 = half * (D / 2);
      const size_t ridx = (static_cast<size_t>(q_local) * p.Hq + h) * D + d0;
      // segments: FIRST writes dq_acc, NEXT adds into it, LAST adds and writes dq
      const bool add = p.seg == OOMB_SEG_NEXT || p.seg == OOMB_SEG_LAST;
      const bool write_bf16 = p.seg == OOMB_SEG_WHOLE || p.seg == OOMB_SEG_LAST;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t a[32];
        if (T > 0) {  // no tile: this call's dQ is zero (TMEM never written)
          tmem_ld32(tmem + lane_off + Cfg::kColDQ + d0 + c * 32, a);
          tmem_ld_wait();
        }
        if (row_valid) {
          float x[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = T > 0 ? __uint_as_float(a[e]) * p.scale : 0.f;
          if (add) {
            const float4* acc = reinterpret_cast<const float4*>(p.dq_acc + ridx + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 a4 = acc[e];
              x[4 * e] += a4.x;
              x[4 * e + 1] += a4.y;
              x[4 * e + 2] += a4.z;
              x[4 * e + 3] += a4.w;
            }
          }
          if (write_bf16) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
            uint4* dst = reinterpret_cast<uint4*>(p.dq + ridx + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          } else {
            float4* dst = reinterpret_cast<float4*>(p.dq_acc + ridx + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (abort_sh && warp == 8 && lane == 0) {
    for (int i = k_used_sh; i < k_issued_sh; ++i)
      mbar_wait_drain(&bar_kf[i % Cfg::kNK], (i / Cfg::kNK) & 1);
    for (int i = v_used_sh; i < v_issued_sh; ++i)
      mbar_wait_drain(&bar_vf[i % Cfg::kNV], (i / Cfg::kNV) & 1);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// ------------------------------------------------------------------ host
bool make_row_map(CUtensorMap* m, const void* base, int D, int Hq, int C) {
  const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(Hq),
                            static_cast<uint64_t>(C)};
  const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(Hq) * D * 2};
  const uint32_t box[3] = {64, 1, kTile};
  return make_bf16_map(m, base, 3, dims, strides, box);
}

bool make_pool_map(CUtensorMap* m, const oomb_pool* pool) {
  const oomb_pool_desc& d = pool->desc;
  const int D = d.head_dim;
  const uint64_t dims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(d.page_size),
                            static_cast<uint64_t>(2 * d.num_kv_heads),
                            static_cast<uint64_t>(d.num_pages)};
  const uint64_t strides[3] = {static_cast<uint64_t>(D) * 2,
                               static_cast<uint64_t>(d.page_size) * D * 2,
                               static_cast<uint64_t>(2 * d.num_kv_heads) * d.page_size * D * 2};
  const uint32_t box[4] = {64, static_cast<uint32_t>(d.page_size), 1, 1};
  return make_bf16_map(m, pool->kv, 4, dims, strides, box);
}

template <int D>
oomb_status launch_bwd(oomb_pool* pool, const oomb_attn_args* a, const AttnShape& s, int step,
                       cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};
  if (!once_per_device(attr_done, [] {
        return cudaFuncSetAttribute(bwd_dkdv_kernel<D>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    KvCfg<D>::kSmem) == cudaSuccess &&
               cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    QCfg<D>::kSmem) == cudaSuccess;
      }))
    return OOMB_ERR_CUDA;
  BwdParams p;
  p.o = static_cast<const __nv_bfloat16*>(a->o);
  p.d_o = static_cast<const __nv_bfloat16*>(a->d_o);
  p.lse = a->lse;
  p.delta = a->delta_ws;
  p.dq = static_cast<__nv_bfloat16*>(a->dq);
  p.grad = pool->grad;
  p.past_pages = a->past_pages;
  p.past_counts = a->past_counts;
  p.cur_pages = a->cur_pages;
  p.status = pool->d_status;
  p.max_past = a->max_past;
  p.C = s.C;
  p.Hq = s.Hq;
  p.Hkv = s.Hkv;
  p.G = s.G;
  p.P = s.P;
  p.num_pool_pages = pool->desc.num_pages;
  p.max_past_tiles = (a->max_past * s.P + kTile - 1) / kTile;
  p.scale = a->softmax_scale;
  p.scale_log2 = a->softmax_scale * kLog2e;
  p.lpq = a->lists_per_qtile;
  p.seg = a->segment;
  p.dq_acc = a->dq_acc;
  p.masks = a->lists_per_qtile == 2 ? a->past_masks : nullptr;
  p.lg_p = __builtin_ctz(static_cast<unsigned>(s.P));

  if (step < 0 || step == OOMB_BWD_PREPROCESS) {
    constexpr int RPB = 256 / (D / 8);
    const int rows = s.C * s.Hq;
    bwd_preprocess_kernel<D><<<(rows + RPB - 1) / RPB, 256, 0, stream>>>(p);
    if (check_launch() != OOMB_OK) return OOMB_ERR_CUDA;
  }
  if (step < 0 || step == OOMB_BWD_DKDV || step == OOMB_BWD_DQ) {
    CUtensorMap qmap, domap, kvmap;
    if (!make_row_map(&qmap, a->q, D, s.Hq, s.C) || !make_row_map(&domap, a->d_o, D, s.Hq, s.C) ||
        !make_pool_map(&kvmap, pool))
      return OOMB_ERR_CUDA;
    if ((step < 0 || step == OOMB_BWD_DKDV) && !p.lpq) {
      // a past-only segment has no tile of the chunk itself
      const bool with_cur = p.seg == OOMB_SEG_WHOLE || p.seg == OOMB_SEG_LAST;
      dim3 grid(p.max_past_tiles + (with_cur ? s.n_qtiles : 0), s.Hkv);
      if (grid.x > 0) {
        bwd_dkdv_kernel<D><<<grid, 320, KvCfg<D>::kSmem, stream>>>(p, qmap, domap, kvmap);
        if (check_launch() != OOMB_OK) return OOMB_ERR_CUDA;
      }
    }
    if ((step < 0 || step == OOMB_BWD_DKDV) && p.lpq) {
      // the chunk's own tiles, for every query tile that reaches them
      BwdParams pc = p;
      pc.lpq = 0;
      pc.max_past = pc.max_past_tiles = 0;
      pc.past_pages = pc.past_counts = nullptr;
      pc.masks = nullptr;
      bwd_dkdv_kernel<D><<<dim3(s.n_qtiles, s.Hkv), 320, KvCfg<D>::kSmem, stream>>>(
          pc, qmap, domap, kvmap);
      if (check_launch() != OOMB_OK) return OOMB_ERR_CUDA;
      // each query tile's listed pages: one z-slice per query tile
      if (p.max_past_tiles > 0) {
        bwd_dkdv_kernel<D><<<dim3(p.max_past_tiles, s.Hkv, s.n_qtiles), 320, KvCfg<D>::kSmem,
                             stream>>>(p, qmap, domap, kvmap);
        if (check_launch() != OOMB_OK) return OOMB_ERR_CUDA;
      }
    }
    if (step < 0 || step == OOMB_BWD_DQ) {
      dim3 grid(s.n_qtiles, s.Hq);
      bwd_dq_kernel<D><<<grid, 352, QCfg<D>::kSmem, stream>>>(p, qmap, domap, kvmap);
      if (check_launch() != OOMB_OK) return OOMB_ERR_CUDA;
    }
  }
  return OOMB_OK;
}

oomb_status bwd_entry(oomb_pool* pool, const oomb_attn_args* args, int step, void* stream) {
  AttnShape s;
  oomb_status st = validate_attn(pool, args, true, &s);
  if (st != OOMB_OK) return st;
  if (!aligned16(args->lse) || !aligned16(args->delta_ws)) return OOMB_ERR_INVALID_ARG;
  DeviceGuard guard(pool->desc.device);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return s.D == 128 ? launch_bwd<128>(pool, args, s, step, cs)
                    : launch_bwd<64>(pool, args, s, step, cs);
}

}  // namespace

extern "C" oomb_status oomb_chunk_attn_bwd(oomb_pool* pool, const oomb_attn_args* args,
                                           void* stream) {
  return bwd_entry(pool, args, -1, stream);
}

extern "C" oomb_status oomb_chunk_attn_bwd_step(oomb_pool* pool, const oomb_attn_args* args,
                                                int32_t step, void* stream) {
  if (step < OOMB_BWD_PREPROCESS || step > OOMB_BWD_DQ) return OOMB_ERR_INVALID_ARG;
  return bwd_entry(pool, args, step, stream);
}
