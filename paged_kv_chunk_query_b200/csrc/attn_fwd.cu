// Chunk attention forward over the paged KV cache (tcgen05 + TMA, sm_100a).
//
// "Out of the Memory Barrier" ([pt] §2B "Kernels Personalizados"; [es] §2B;
// [it] §2B): attention runs directly on the paged cache.  One CTA owns 128
// query rows of one head and walks the KV tiles of its group: the listed past
// pages (all visible) and then the chunk's own pages (causal).
//
// Warp roles (224 threads):
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r).  First copies
//              its Q row from shared memory into TMEM (A operand of QK^T);
//              then per tile reads S from TMEM, keeps the running max / sum,
//              writes P (bf16) back into the same TMEM columns, rescales O
//              when the max grows, and finally normalises O and writes O and
//              the LSE.
//   warp 4     TMA producer of Q and the K tiles, warp 6 of the V tiles, page
//              by page through a 4-D tensor map over the pool (page id =
//              outermost coordinate).
//   warp 5     UMMA issuer (one thread): S_j = Q K_j^T (Q from TMEM) into one of
//              two TMEM S buffers, O += P_j V_j with P read from TMEM (A
//              operand) and V from shared memory (MN-major B operand).
// TMEM: S0 [0,128), S1 [128,256), O [256, 256+D), Q [384, 384+D/2).
//
// Online softmax in base 2: s2 = S * scale * log2(e).  The running maximum is
// only moved when a tile's maximum exceeds it by more than 8 (a factor 256),
// so O is rescaled rarely; the final O / l and LSE = ln2 * (m + log2 l) are
// exact whichever maximum was used.
//
// Grid: one CTA per (query tile, head) unit, one CTA per SM.  When the units
// do not fill whole waves and the caller gives a workspace, the units of the
// last wave are split along their key tiles over the SMs that wave would
// leave idle; each part writes a normalised O and its LSE, and
// fwd_merge_kernel combines them by log-sum-exp.
#include <algorithm>

#include "internal.h"
#include "ptx.cuh"
#include "tiles.cuh"
#include "tmap.h"

namespace {

using namespace oomb;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;

struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  const int32_t* past_pages;
  const int32_t* past_counts;
  const int32_t* cur_pages;
  uint32_t* status;
  int max_past, C, Hq, G, P, num_pool_pages;
  int lpq;  // 1: one past list per (query tile, group); 2: per query page (union + masks)
  int seg;  // OOMB_SEG_*: whole key set, or a segment merged into o_acc / lse
  float* o_acc;
  const uint8_t* masks;  // lpq 2: query-page membership bits of each list entry
  int lg_p;              // log2(P)
  float scale_log2;
  // units (query tile, head) u = h * n_qtiles + qt.  CTAs [0, n_full) take unit
  // = blockIdx.x whole; with n_split > 0 the remaining units (the last wave's)
  // are split: CTA n_full + k takes part k % n_split of the key tiles of unit
  // n_full + k / n_split and writes its normalised O and LSE to part_o /
  // part_lse [k][128 rows] for fwd_merge_kernel.
  int n_qtiles, n_full, n_split;
  float* part_o;
  float* part_lse;
};

// Partial-result capacity of the forward workspace: parts of at most this many
// CTAs (a wave on 148 SMs fits).
constexpr int kMaxFwdParts = 256;

template <int D>
struct FwdCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kTile * D * 2;  // Q, K or V tile
  static constexpr int kNK = 3;
  static constexpr int kNV = 3;
  static constexpr int kSmem = kTileBytes * (1 + kNK + kNV) + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;
  static constexpr uint32_t kColQ = 384;  // Q as a bf16 A operand (D/2 columns)
};

template <int D>
__global__ void __launch_bounds__(224, 1)
    attn_fwd_kernel(const FwdParams p, const __grid_constant__ CUtensorMap qmap,
                    const __grid_constant__ CUtensorMap kvmap) {
  using Cfg = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + Cfg::kTileBytes;
  uint8_t* sV = sK + Cfg::kNK * Cfg::kTileBytes;

  __shared__ uint64_t bar_q, bar_qt, bar_drain, bar_o, bar_fin;
  __shared__ uint64_t bar_kf[Cfg::kNK], bar_ke[Cfg::kNK], bar_vf[Cfg::kNV], bar_ve[Cfg::kNV];
  __shared__ uint64_t bar_s[2], bar_p[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ int k_issued_sh, v_issued_sh, k_used_sh, v_used_sh;

  const int warp = warp_id(), lane = lane_id();
  // this CTA's unit, and its part of the unit's key tiles (part < 0: all)
  const int cid = blockIdx.x;
  int unit = cid, part = -1;
  if (p.n_split > 0 && cid >= p.n_full) {
    unit = p.n_full + (cid - p.n_full) / p.n_split;
    part = (cid - p.n_full) % p.n_split;
  }
  const int qt = unit % p.n_qtiles, h = unit / p.n_qtiles, g = h / p.G;
  // list of (query tile, group) or of the group
  const int li = (p.lpq ? qt * (p.Hq / p.G) : 0) + g;
  const KvSchedule sch = kv_schedule(p.past_counts ? p.past_counts + (li - g) : nullptr, g,
                                     p.max_past, p.P, p.status);
  // past tiles + (unless this call is a past-only segment) the chunk's tiles up
  // to the diagonal; a past-only segment with an empty list has no tile
  const bool with_cur = p.seg == OOMB_SEG_WHOLE || p.seg == OOMB_SEG_LAST;
  const int T_all = sch.n_past_tiles + (with_cur ? qt + 1 : 0);
  // key tiles [j0, j0 + T) in the unit's order (past, then the chunk's own);
  // loops count j from 0 and tile j is the unit's tile j0 + j
  const int j0 = part < 0 ? 0 : part * T_all / p.n_split;
  const int T = part < 0 ? T_all : (part + 1) * T_all / p.n_split - j0;
  const int n_cur_pages = p.C / p.P;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    k_issued_sh = v_issued_sh = k_used_sh = v_used_sh = 0;
    mbar_init(&bar_q, 1);
    mbar_init(&bar_qt, 4);
    mbar_init(&bar_drain, 1);
    mbar_init(&bar_o, 1);
    mbar_init(&bar_fin, 1);
    for (int i = 0; i < Cfg::kNK; ++i) {
      mbar_init(&bar_kf[i], 1);
      mbar_init(&bar_ke[i], 1);
    }
    for (int i = 0; i < Cfg::kNV; ++i) {
      mbar_init(&bar_vf[i], 1);
      mbar_init(&bar_ve[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_s[i], 1);
      mbar_init(&bar_p[i], 4);
    }
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

  if (warp == 4 || warp == 6) {
    // ------------------------------------------------------------ producers
    // warp 4 loads Q and the K tiles, warp 6 the V tiles, so a K load never
    // queues behind a V slot that frees only after a late PV.
    if (lane == 0) {
      const bool is_k = warp == 4;
      if (is_k) {
        prefetch_tensormap(&qmap);
        mbar_arrive_expect_tx(&bar_q, Cfg::kTileBytes);
        for (int hf = 0; hf < Cfg::kHalves; ++hf)
          tma_load_3d(sQ + hf * kTile * 128, &qmap, &bar_q, hf * 64, h, qt * kTile);
      }
      prefetch_tensormap(&kvmap);
      const int32_t* past_list = p.past_pages + static_cast<size_t>(li) * p.max_past;
      const int per = kTile / p.P;
      const int nst = is_k ? Cfg::kNK : Cfg::kNV;
      uint64_t* full = is_k ? bar_kf : bar_vf;
      uint64_t* empty = is_k ? bar_ke : bar_ve;
      uint8_t* base = is_k ? sK : sV;
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        int pg[8];
        for (int s = 0; s < per; ++s)
          pg[s] = tile_page(j0 + j, s, sch, past_list, p.cur_pages, n_cur_pages, p.P,
                            p.num_pool_pages, is_k ? p.status : nullptr);
        const int st = j % nst;
        if (!mbar_wait(&empty[st], ((j / nst) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&full[st], Cfg::kTileBytes);
        uint8_t* dst = base + st * Cfg::kTileBytes;
        for (int s = 0; s < per; ++s)
          for (int hf = 0; hf < Cfg::kHalves; ++hf)
            tma_load_4d(dst + hf * kTile * 128 + s * p.P * 128, &kvmap, &full[st], hf * 64, 0,
                        2 * g + (is_k ? 0 : 1), pg[s]);
        ++issued;
      }
      if (*abort_flag) atomicOr(p.status, OOMB_DEV_WAIT_LIMIT);
      if (is_k) k_issued_sh = issued;
      else v_issued_sh = issued;
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      int k_used = 0, v_used = 0;
      bool ok = mbar_wait(&bar_qt, 0, abort_flag);  // Q copied into TMEM
      for (int j = 0; ok && j <= T; ++j) {
        if (j < T) {
          const int ks = j % Cfg::kNK;
          if (!(ok = mbar_wait(&bar_kf[ks], (j / Cfg::kNK) & 1, abort_flag))) break;
          ++k_used;
          tc_fence_after();
          const uint32_t sd = tmem + (j & 1) * 128;
          const uint32_t kb = k_addr + ks * Cfg::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk / 4) * (kTile * 128) + (kk % 4) * 32;
            umma_ts(sd, tmem + Cfg::kColQ + kk * 8, sw128_desc(kb + off, 16, 1024), idesc_s,
                    kk > 0);
          }
          umma_commit(&bar_ke[ks]);
          umma_commit(&bar_s[j & 1]);
        }
        if (j >= 1) {
          const int jp = j - 1, b = jp & 1, vs = jp % Cfg::kNV;
          if (!(ok = mbar_wait(&bar_p[b], (jp >> 1) & 1, abort_flag))) break;
          if (!(ok = mbar_wait(&bar_vf[vs], (jp / Cfg::kNV) & 1, abort_flag))) break;
          ++v_used;
          tc_fence_after();
          const uint32_t vb = v_addr + vs * Cfg::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ts(tmem + Cfg::kColO, tmem + b * 128 + kk * 8,
                    sw128_desc(vb + kk * 16 * 128, kTile * 128, 1024), idesc_pv,
                    (jp > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&bar_ve[vs]);
          umma_commit(&bar_o);
          if (jp == T - 1) umma_commit(&bar_fin);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(p.status, OOMB_DEV_WAIT_LIMIT);
      }
      // every UMMA of this CTA has completed once bar_drain fires
      umma_commit(&bar_drain);
      mbar_wait_drain(&bar_drain, 0);
      k_used_sh = k_used;
      v_used_sh = v_used;
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int r = threadIdx.x;  // 0..127
    const int q_local = qt * kTile + r;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int n_past_keys = sch.n_past_pages * p.P;
    float m_used = -INFINITY, l = 0.f;
    // Q row r into TMEM (packed bf16 pairs, A operand of S = Q K^T): the S
    // UMMAs then read only K from shared memory
    bool ok = warp_wait(&bar_q, 0, abort_flag);
    if (ok) {
#pragma unroll
      for (int hf = 0; hf < Cfg::kHalves; ++hf) {
        uint32_t qv[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 v = *reinterpret_cast<const uint4*>(sQ + hf * kTile * 128 +
                                                          sw128_offset(r, ch * 8));
          qv[4 * ch] = v.x;
          qv[4 * ch + 1] = v.y;
          qv[4 * ch + 2] = v.z;
          qv[4 * ch + 3] = v.w;
        }
        tmem_st32(tmem + lane_off + Cfg::kColQ + hf * 32, qv);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_qt);
    }
    for (int j = 0; ok && j < T; ++j) {
      const int b = j & 1;
      if (!(ok = warp_wait(&bar_s[b], (j >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      float s[kTile];
#pragma unroll
      for (int c = 0; c < kTile / 32; ++c)
        tmem_ld32(tmem + lane_off + b * 128 + c * 32, reinterpret_cast<uint32_t*>(s + c * 32));
      tmem_ld_wait();
      const int jt = j0 + j;  // the unit's tile
      int lim;
      if (jt < sch.n_past_tiles) {
        lim = n_past_keys - jt * kTile;
      } else {
        const int key0 = (jt - sch.n_past_tiles) * kTile;
        lim = min(p.C, q_local + 1) - key0;
      }
      if (lim < kTile) {  // diagonal or ragged tile: keys at and past `lim` are masked
#pragma unroll
        for (int c = 0; c < kTile; ++c) s[c] = c < lim ? s[c] : -INFINITY;
      }
      if (p.masks && jt < sch.n_past_tiles) {
        // per-query-page lists: a listed page this row's query page did not
        // select is masked (its bit in the entry's membership mask is clear)
        const int per = kTile >> p.lg_p;
        const uint8_t* mrow = p.masks + static_cast<size_t>(li) * p.max_past + jt * per;
        const int qb = r >> p.lg_p;
        // bit k: columns [16k, 16k + 16) (one page: P >= 16) are kept
        uint32_t keep = 0;
        for (int k = 0; k < kTile / 16; ++k) {
          const int sl = (16 * k) >> p.lg_p;
          if (jt * per + sl < sch.n_past_pages && ((mrow[sl] >> qb) & 1u)) keep |= 1u << k;
        }
        if (keep != 0xFFu) {
#pragma unroll
          for (int c = 0; c < kTile; ++c) s[c] = ((keep >> (c >> 4)) & 1u) ? s[c] : -INFINITY;
        }
      }
      // row max with 8 independent chains (raw logits; scale > 0 keeps the order)
      float m8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) m8[e] = s[e];
#pragma unroll
      for (int c = 8; c < kTile; ++c) m8[c & 7] = fmaxf(m8[c & 7], s[c]);
      const float mt = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                             fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * p.scale_log2;
      const bool need = mt > m_used + kRescaleThreshold;
      const float m_new = need ? mt : m_used;
      const float alpha = need ? fast_exp2(m_used - m_new) : 1.f;
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O holds sum_{<j} 2^(s - m_used) v; PV_{j-1} must land before rescaling.
        // S_j's commit implies PV_{j-2} completed and PV_j waits for P_j, so
        // bar_o is in phase j-1 or j here and the parity names PV_{j-1}.
        if (!(ok = warp_wait(&bar_o, (j - 1) & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + Cfg::kColO + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tmem + lane_off + Cfg::kColO + c * 32, o);
        }
        tmem_st_wait();
      }
      m_used = m_new;
      const float neg_mref = m_used == -INFINITY ? 0.f : -m_used;
      // p = 2^(S*scale*log2e - m); masked logits are -inf and give 0
      float l8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) l8[e] = 0.f;
      uint32_t pk[kTile / 2];
#pragma unroll
      for (int c = 0; c < kTile / 2; ++c) {
        const float p0 = fast_exp2(fmaf(s[2 * c], p.scale_log2, neg_mref));
        const float p1 = fast_exp2(fmaf(s[2 * c + 1], p.scale_log2, neg_mref));
        l8[c & 7] += p0 + p1;
        pk[c] = pack_bf16(p0, p1);
      }
      l = l * alpha + (((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7])));
#pragma unroll
      for (int c = 0; c < kTile / 2 / 16; ++c)
        tmem_st16(tmem + lane_off + b * 128 + c * 16, pk + c * 16);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_p[b]);
    }
    if (ok && T > 0) ok = warp_wait(&bar_fin, 0, abort_flag);
    if (!ok) {
      *abort_flag = 1;
      if (lane == 0) atomicOr(p.status, OOMB_DEV_WAIT_LIMIT);
    } else {
      tc_fence_after();
      const bool valid = q_local < p.C;
      // this call's result: O_s = O_tmem / l with LSE_s (natural log)
      const float lse_s = (T > 0 && l > 0.f) ? kLn2 * (m_used + log2f(l)) : -INFINITY;
      float* lse_ptr = p.lse + static_cast<size_t>(h) * p.C + q_local;
      // merge with the running (o_acc, lse) of earlier segments:
      //   LSE = ln(e^LSE_old + e^LSE_s), O = e^(LSE_old - LSE) O_old + e^(LSE_s - LSE) O_s
      // (a part of a split unit leaves that to fwd_merge_kernel)
      const bool as_part = part >= 0;
      const bool merge = (p.seg == OOMB_SEG_NEXT || p.seg == OOMB_SEG_LAST) && !as_part;
      float w_o = 0.f, w_s = 1.f, lse_new = lse_s;
      if (merge && valid) {
        const float lse_o = *lse_ptr;
        const float mx = fmaxf(lse_o, lse_s);
        if (mx == -INFINITY) {
          lse_new = -INFINITY;
          w_s = 0.f;
        } else {
          const float eo = lse_o == -INFINITY ? 0.f : expf(lse_o - mx);
          const float es = lse_s == -INFINITY ? 0.f : expf(lse_s - mx);
          lse_new = mx + logf(eo + es);
          w_o = eo / (eo + es);
          w_s = es / (eo + es);
        }
      }
      const float scale_s = (T > 0 && l > 0.f) ? w_s / l : 0.f;
      const size_t ridx = (static_cast<size_t>(q_local) * p.Hq + h) * D;
      const bool write_bf16 = p.seg == OOMB_SEG_WHOLE || p.seg == OOMB_SEG_LAST;
      // a part of a split unit: its normalised O and LSE into the workspace
      // (every row; the merge writes the valid ones)
      const size_t prow = as_part ? static_cast<size_t>(cid - p.n_full) * kTile + r : 0;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (T > 0) {
          tmem_ld32(tmem + lane_off + Cfg::kColO + c * 32, o);
          tmem_ld_wait();
        }
        if (as_part) {
          float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D + c * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float x0 = T > 0 ? __uint_as_float(o[4 * e]) * scale_s : 0.f;
            const float x1 = T > 0 ? __uint_as_float(o[4 * e + 1]) * scale_s : 0.f;
            const float x2 = T > 0 ? __uint_as_float(o[4 * e + 2]) * scale_s : 0.f;
            const float x3 = T > 0 ? __uint_as_float(o[4 * e + 3]) * scale_s : 0.f;
            dst[e] = make_float4(x0, x1, x2, x3);
          }
        } else if (valid) {
          float x[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = T > 0 ? __uint_as_float(o[e]) * scale_s : 0.f;
          if (merge && w_o > 0.f) {
            const float4* acc = reinterpret_cast<const float4*>(p.o_acc + ridx + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 a4 = acc[e];
              x[4 * e] = fmaf(a4.x, w_o, x[4 * e]);
              x[4 * e + 1] = fmaf(a4.y, w_o, x[4 * e + 1]);
              x[4 * e + 2] = fmaf(a4.z, w_o, x[4 * e + 2]);
              x[4 * e + 3] = fmaf(a4.w, w_o, x[4 * e + 3]);
            }
          }
          if (write_bf16) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
            uint4* dst = reinterpret_cast<uint4*>(p.o + ridx + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          } else {
            float4* dst = reinterpret_cast<float4*>(p.o_acc + ridx + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
          }
        }
      }
      if (as_part) p.part_lse[prow] = lse_s;
      else if (valid) *lse_ptr = merge ? lse_new : lse_s;
    }
  }

  tc_fence_before();
  __syncthreads();
  // After an abort, wait (bounded) for TMA loads still landing in shared memory.
  if (abort_sh && warp == 4 && lane == 0) {
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

// The parts of the split units merged: grid (n_tail, kTile / kMergeRows<D>),
// 128 threads, a thread 4 consecutive d of one row.  For each row
//   LSE = ln sum_k e^LSE_k,  O = sum_k e^(LSE_k - LSE) O_k
// over the unit's n_split parts in part order (a part whose keys were all
// masked for the row has LSE_k = -inf and weight 0; its O is written as 0).
// That is the call's result; a segmented call then merges it with the
// running (o_acc, lse) as the forward's epilogue does, and the row is written
// as o (bf16: whole key set, last segment) or o_acc (fp32: first and middle
// segments) with its lse.  Parts are read in batches of 4 with every load of
// a batch issued before its first use.
template <int D>
constexpr int kMergeRows = 128 / (D / 4);  // rows per merge CTA

template <int D>
__global__ void __launch_bounds__(128) fwd_merge_kernel(const FwdParams p) {
  constexpr int TPR = D / 4;  // threads per row
  constexpr int U = 4;        // parts per batch
  const int ti = blockIdx.x;
  const int row = blockIdx.y * kMergeRows<D> + threadIdx.x / TPR, seg = threadIdx.x % TPR;
  const int unit = p.n_full + ti;
  const int qt = unit % p.n_qtiles, h = unit / p.n_qtiles;
  const int q_local = qt * kTile + row;
  // rows past the chunk's end are merged too (their parts exist) but neither
  // read nor written; every lane stays to the warp barrier below
  const bool active = q_local < p.C;
  const int n = p.n_split;
  const size_t base = static_cast<size_t>(ti) * n;
  // part k of this row: LSE at lse_k[k * kTile], O at o_k[k * kPartStride]
  const float* lse_k = p.part_lse + base * kTile + row;
  const float4* o_k = reinterpret_cast<const float4*>(p.part_o + (base * kTile + row) * D) + seg;
  constexpr size_t kPartStride = static_cast<size_t>(kTile) * D / 4;
  float mx = -INFINITY;
#pragma unroll 8
  for (int k = 0; k < n; ++k) mx = fmaxf(mx, lse_k[static_cast<size_t>(k) * kTile]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  if (mx != -INFINITY) {
    for (int k0 = 0; k0 < n; k0 += U) {
      float lk[U];
      float4 a[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int k = min(k0 + u, n - 1);  // past the last part: a repeat, weight 0 below
        lk[u] = lse_k[static_cast<size_t>(k) * kTile];
        a[u] = o_k[k * kPartStride];
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float wk = (k0 + u < n && lk[u] != -INFINITY) ? expf(lk[u] - mx) : 0.f;
        den += wk;
        acc.x = fmaf(wk, a[u].x, acc.x);
        acc.y = fmaf(wk, a[u].y, acc.y);
        acc.z = fmaf(wk, a[u].z, acc.z);
        acc.w = fmaf(wk, a[u].w, acc.w);
      }
    }
  }
  // this call's result for the row: O_s = acc / den, LSE_s
  const float lse_s = mx == -INFINITY ? -INFINITY : mx + logf(den);
  float w_s = den > 0.f ? 1.f / den : 0.f, w_o = 0.f, lse_out = lse_s;
  float* lse_ptr = p.lse + static_cast<size_t>(h) * p.C + q_local;
  const size_t ridx = (static_cast<size_t>(q_local) * p.Hq + h) * D + seg * 4;
  if (p.seg == OOMB_SEG_NEXT || p.seg == OOMB_SEG_LAST) {
    // merged with the running (o_acc, lse) of earlier segments, as the
    // forward's own epilogue does for a whole unit
    const float lse_o = active ? *lse_ptr : -INFINITY;
    const float m2 = fmaxf(lse_o, lse_s);
    if (m2 == -INFINITY) {
      lse_out = -INFINITY;
      w_s = 0.f;
    } else {
      const float eo = lse_o == -INFINITY ? 0.f : expf(lse_o - m2);
      const float es = lse_s == -INFINITY ? 0.f : expf(lse_s - m2);
      lse_out = m2 + logf(eo + es);
      w_o = eo / (eo + es);
      w_s *= es / (eo + es);
    }
  }
  float4 x = make_float4(acc.x * w_s, acc.y * w_s, acc.z * w_s, acc.w * w_s);
  if (active && w_o > 0.f) {
    const float4 a4 = *reinterpret_cast<const float4*>(p.o_acc + ridx);
    x = make_float4(fmaf(a4.x, w_o, x.x), fmaf(a4.y, w_o, x.y), fmaf(a4.z, w_o, x.z),
                    fmaf(a4.w, w_o, x.w));
  }
  if (active) {
    if (p.seg == OOMB_SEG_WHOLE || p.seg == OOMB_SEG_LAST)
      *reinterpret_cast<uint2*>(p.o + ridx) =
          make_uint2(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w));
    else
      *reinterpret_cast<float4*>(p.o_acc + ridx) = x;
  }
  // every lane of the row has read the old lse before it is replaced
  __syncwarp();
  if (active && seg == 0) *lse_ptr = lse_out;
}

int sm_count(int device) {
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || n <= 0)
    n = 148;
  return n;
}

template <int D>
oomb_status launch_fwd(oomb_pool* pool, const oomb_attn_args* a, const AttnShape& s,
                       cudaStream_t stream) {
  using Cfg = FwdCfg<D>;
  static std::atomic<uint64_t> attr_done{0};
  if (!once_per_device(attr_done, [] {
        return cudaFuncSetAttribute(attn_fwd_kernel<D>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Cfg::kSmem) == cudaSuccess;
      }))
    return OOMB_ERR_CUDA;
  CUtensorMap qmap, kvmap;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(s.Hq),
                              static_cast<uint64_t>(s.C)};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2,
                                 static_cast<uint64_t>(s.Hq) * D * 2};
    const uint32_t box[3] = {64, 1, kTile};
    if (!make_bf16_map(&qmap, a->q, 3, dims, strides, box)) return OOMB_ERR_CUDA;
  }
  {
    const oomb_pool_desc& d = pool->desc;
    const uint64_t dims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(d.page_size),
                              static_cast<uint64_t>(2 * d.num_kv_heads),
                              static_cast<uint64_t>(d.num_pages)};
    const uint64_t strides[3] = {static_cast<uint64_t>(D) * 2,
                                 static_cast<uint64_t>(d.page_size) * D * 2,
                                 static_cast<uint64_t>(2 * d.num_kv_heads) * d.page_size * D * 2};
    const uint32_t box[4] = {64, static_cast<uint32_t>(d.page_size), 1, 1};
    if (!make_bf16_map(&kvmap, pool->kv, 4, dims, strides, box)) return OOMB_ERR_CUDA;
  }
  FwdParams p;
  p.o = static_cast<__nv_bfloat16*>(a->o);
  p.lse = a->lse;
  p.past_pages = a->past_pages;
  p.past_counts = a->past_counts;
  p.cur_pages = a->cur_pages;
  p.status = pool->d_status;
  p.max_past = a->max_past;
  p.C = s.C;
  p.Hq = s.Hq;
  p.G = s.G;
  p.P = s.P;
  p.num_pool_pages = pool->desc.num_pages;
  p.scale_log2 = a->softmax_scale * kLog2e;
  p.lpq = a->lists_per_qtile;
  p.seg = a->segment;
  p.o_acc = a->o_acc;
  p.masks = a->lists_per_qtile == 2 ? a->past_masks : nullptr;
  p.lg_p = __builtin_ctz(static_cast<unsigned>(s.P));
  // one CTA per unit (one per SM); with a workspace the last, partial wave's
  // units are split over the SMs it leaves free
  const int units = s.n_qtiles * s.Hq;
  int n_tail = 0;
  p.n_qtiles = s.n_qtiles;
  p.n_full = units;
  p.n_split = 0;
  p.part_o = a->fwd_ws;
  p.part_lse = a->fwd_ws ? a->fwd_ws + static_cast<size_t>(kMaxFwdParts) * kTile * D : nullptr;
  if (a->fwd_ws) {
    const int ns = sm_count(pool->desc.device);
    const int tail = units % ns;
    if (tail > 0) {
      const int parts = std::min(ns / tail, kMaxFwdParts / tail);
      if (parts >= 2) {
        n_tail = tail;
        p.n_full = units - tail;
        p.n_split = parts;
      }
    }
  }
  attn_fwd_kernel<D><<<p.n_full + n_tail * p.n_split, 224, Cfg::kSmem, stream>>>(p, qmap, kvmap);
  if (n_tail > 0) {
    fwd_merge_kernel<D><<<dim3(n_tail, kTile / kMergeRows<D>), 128, 0, stream>>>(p);
  }
  return check_launch();
}

}  // namespace

extern "C" size_t oomb_chunk_attn_fwd_workspace_size(int32_t head_dim) {
  if (head_dim != 64 && head_dim != 128) return 0;
  return static_cast<size_t>(kMaxFwdParts) * kTile * (head_dim + 1) * sizeof(float);
}

extern "C" oomb_status oomb_chunk_attn_fwd(oomb_pool* pool, const oomb_attn_args* args,
                                           void* stream) {
  oomb::AttnShape s;
  oomb_status st = oomb::validate_attn(pool, args, false, &s);
  if (st != OOMB_OK) return st;
  oomb::DeviceGuard guard(pool->desc.device);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return s.D == 128 ? launch_fwd<128>(pool, args, s, cs) : launch_fwd<64>(pool, args, s, cs);
}
