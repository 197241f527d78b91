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
// The kernels take a batch of independent problems (blockIdx.z), each a
// range of query rows and its own number of past pages; the per-chunk entry
// points run a batch of one.
// Kernel 1 (qmean_partial): grid (slices, Hkv, problems); each CTA streams the
//   G heads of one group (contiguous in a token row) over a slice of its
//   problem's rows, one thread per 16-byte column, 16 rows in flight, and
//   writes one fp32 partial per d.  It also zeroes the select tickets.
// One problem (oomb_page_topk, two launches): kernel 2 (page_score_select,
//   fused select) is a programmatic dependent launch: grid (pages / 64, Hkv),
//   each warp loads the summaries of its 8 pages while kernel 1 finishes,
//   then every CTA sums the slice partials of its group in one fixed order
//   into q_bar (so all CTAs of a group score against the identical q_bar),
//   scores its pages into 64-bit keys (ordered score, inverted id), and the
//   last CTA of the group to take a ticket runs the select.
// A batch (oomb_page_topk_batched, four dependent launches): a Q-sum kernel
//   reduces each (problem, group)'s partials once, in the same order; the
//   scores kernel without the select (few registers, full occupancy); then
//   one select CTA per (problem, group).
// From Q sums made by the producer of Q (oomb_page_topk_qsum): the fused
//   scores + select kernel alone, one launch.
// The select (up to 4,096 past pages: keys in registers, 16 contiguous pages
//   per thread): a 256-bucket histogram of the fp32 score on a linear scale
//   between the candidates' minimum and maximum finds the bucket of the K-th
//   largest key; one warp ranks that bucket's keys when there are at most 64
//   of them, exact 8-bit radix passes over them otherwise; one CTA-wide scan
//   compacts the kept ids in ascending order; beyond 4,096 pages, 8-bit
//   passes over the keys re-read from L2.
#include <cuda_bf16.h>

#include <algorithm>
#include <climits>
#include <mutex>

#include "internal.h"

namespace {

constexpr int kSplits = 128;         // max query-mean slices per (problem, group)
constexpr int kMeanThreads = 256;    // query mean: one thread per 16-byte column of a group's heads
constexpr int kScoreThreads = 256;   // 8 warps x 8 pages per CTA
constexpr int kPagesPerScoreCta = 64;
constexpr int kKeysPerThread = 16;   // register-resident select: up to 4,096 past pages

// Programmatic dependent launch (sm_90+): the query-mean kernel lets the
// scores kernel launch once all of its CTAs have started; the scores kernel
// does the work that does not read the query mean's output, then waits for
// that grid to complete and its writes to be visible.  Without a dependent
// launch the wait returns at once.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Ticket of a CTA that has written its keys: one acquire-release atomic add
// at GPU scope by one thread, between two CTA barriers.  The release covers
// the whole CTA's earlier writes (the first barrier orders them before it,
// and release is cumulative); the CTA that draws the last ticket acquires
// every earlier CTA's release, and its second barrier orders all of its
// threads' later loads after that acquire.
__device__ __forceinline__ unsigned int ticket_acq_rel(unsigned int* p) {
  unsigned int old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
  return old;
}

// Row stride of the 64-bit key array: even, so that every row starts on a
// 16-byte boundary and key pairs load as one vector.
__host__ __device__ __forceinline__ int key_stride(int max_past) {
  return ((max_past > 0 ? max_past : 1) + 1) & ~1;
}


size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Slices per (problem, group): about 32 query rows (x G heads) per slice, at
// most kSplits.  A 4096-row chunk gets 128.
int choose_splits(int max_rows) {
  const int s = (max_rows + 31) / 32;
  return s < 1 ? 1 : (s > kSplits ? kSplits : s);
}

// A batch of independent selections.  Problem b takes query rows
// [row_start[b], row_start[b+1]) and candidates among logical pages
// [0, n_past[b]) of one page table.  With null arrays there is one problem:
// rows [0, rows0) and n_past0 pages.  Values the device arrays hold out of
// range are clamped and flagged (bad count).
struct Problems {
  const int32_t* row_start;
  const int32_t* n_past;
  int rows0, n_past0, max_past, num_rows, splits;
  uint32_t* status;
};

__device__ __forceinline__ void problem_rows(const Problems& pb, int b, int& r0, int& r1) {
  if (!pb.row_start) {
    r0 = 0;
    r1 = pb.rows0;
    return;
  }
  r0 = pb.row_start[b];
  r1 = pb.row_start[b + 1];
  if (r0 < 0 || r1 < r0 || r1 > pb.num_rows) {
    atomicOr(pb.status, OOMB_DEV_BAD_COUNT);
    r0 = min(max(r0, 0), pb.num_rows);
    r1 = min(max(r1, r0), pb.num_rows);
  }
}

__device__ __forceinline__ int problem_npast(const Problems& pb, int b) {
  if (!pb.n_past) return pb.n_past0;
  const int n = pb.n_past[b];
  if (n < 0 || n > pb.max_past) {
    atomicOr(pb.status, OOMB_DEV_BAD_COUNT);
    return n < 0 ? 0 : pb.max_past;
  }
  return n;
}

// ---------------------------------------------------------------- query mean
// grid (splits, Hkv, problems): CTA (s, g, b) streams slice s of problem b's
// tokens, the G heads of group g (G * d * 2 contiguous bytes of each token
// row), one thread per 16-byte column, 16 rows in flight per thread; then sums
// the G heads in shared memory (fixed order) and writes one fp32 partial per
// d.  Each partial is the same sum, in the same order, for any grid shape:
// rows in slice order per column, then heads in order.
template <int D>
__global__ void __launch_bounds__(kMeanThreads, 1) qmean_partial_kernel(
    const __nv_bfloat16* __restrict__ q, float* __restrict__ partial, const Problems pb, int Hq,
    int G, unsigned int* __restrict__ tickets, int n_tickets) {
  extern __shared__ float col_sum[];  // [G][D]
  constexpr int VPR = D / 8;          // 16-byte vectors per (token, head) row
  constexpr int U = 16;               // rows in flight per thread
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z, t = threadIdx.x;
  const int Hkv = gridDim.y;
  pdl_launch_dependents();
  // the next kernel on the stream counts finished CTAs from zero
  if (split == 0 && g == 0 && b == 0)
    for (int i = t; i < n_tickets; i += blockDim.x) tickets[i] = 0u;
  const int ncol = G * VPR;           // 16-byte vectors of the group's heads in a token row
  const size_t row_vecs = static_cast<size_t>(Hq) * VPR;
  int r0, r1;
  problem_rows(pb, b, r0, r1);
  const int per = (r1 - r0 + pb.splits - 1) / pb.splits;
  const int tok0 = r0 + split * per, tok1 = min(r1, tok0 + per);
  const uint4* base = reinterpret_cast<const uint4*>(q) + static_cast<size_t>(g) * ncol;
  for (int col = t; col < ncol; col += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    int tok = tok0;
    for (; tok + U <= tok1; tok += U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = __ldg(base + (tok + u) * row_vecs + col);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const __nv_bfloat16* bv = reinterpret_cast<const __nv_bfloat16*>(&v[u]);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += __bfloat162float(bv[e]);
      }
    }
    for (; tok < tok1; ++tok) {
      const uint4 v = __ldg(base + tok * row_vecs + col);
      const __nv_bfloat16* bv = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __bfloat162float(bv[e]);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) col_sum[col * 8 + e] = acc[e];  // (head in group, d) = col * 8 + e
  }
  __syncthreads();
  for (int dd = t; dd < D; dd += blockDim.x) {
    float s = 0.f;
    for (int hh = 0; hh < G; ++hh) s += col_sum[hh * D + dd];  // fixed order
    partial[((static_cast<size_t>(b) * pb.splits + split) * Hkv + g) * D + dd] = s;
  }
}

__device__ __forceinline__ uint32_t order_f32(float f) {
  // monotone map of fp32 onto uint32 (larger float -> larger integer)
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- select
// Shared state of one CTA's radix select (256 bins, 8 warps of bin scan).
// A boundary bucket of at most this many keys is ranked by one warp instead
// of by radix passes.
constexpr int kSmallBucket = 64;

struct RadixShared {
  unsigned int hist[256];
  unsigned int warp_tot[8];
  int warp_cnt[32];
  unsigned long long kth;
  int need, done;
  unsigned int n_small;                   // boundary-bucket keys gathered so far
  unsigned long long small[kSmallBucket];  // and the keys
};

// One radix step's bin search, once hist[] holds the counts, by the 8-bit
// digit at `shift`, of the keys still in play (those equal to the K-th key's
// prefix found so far): the bin, scanned from 255 down, that holds the
// need-th largest of them.  Sets kth (prefix plus that digit), need (the rank
// left inside the bin) and done (the bin is kept whole, so the lower digits
// do not matter).  Thread t < 256 owns bin 255 - t.  Ends on a barrier.
__device__ __forceinline__ void radix_pick_bin(RadixShared& sh, unsigned long long prefix,
                                               int shift) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  // every thread reads the remaining count here, before the barrier that
  // precedes its one update below (a read after the update could let a
  // second bin match)
  const int need = sh.need;
  // inclusive suffix sum over bins 255..0
  unsigned int incl = 0;
  if (t < 256) {
    incl = sh.hist[255 - t];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) sh.warp_tot[warp] = incl;
  }
  __syncthreads();
  if (t < 256) {
    for (int w = 0; w < warp; ++w) incl += sh.warp_tot[w];
    const int bin = 255 - t;
    const unsigned int v = sh.hist[bin];
    const unsigned int excl = incl - v;
    if (excl < static_cast<unsigned>(need) && static_cast<unsigned>(need) <= incl) {
      sh.kth = prefix | (static_cast<unsigned long long>(bin) << shift);
      sh.need = need - static_cast<int>(excl);
      if (v == static_cast<unsigned>(need) - excl) sh.done = 1;  // bin taken whole
    }
  }
  __syncthreads();
}

// The K-th largest candidate key of one (problem, group) by 8-bit radix passes
// from the top, stopping early once the boundary bin is taken whole; then the
// kept ids compacted in ascending order.  Keys are read from L2 on every pass
// (coherent loads: other CTAs of this launch wrote them).  Any n_past.  Run
// by one CTA of NT threads (NT >= 256).
template <int NT>
__device__ void select_pages_cta(const unsigned long long* keys,
                                 const int32_t* __restrict__ page_table, int n_past, int top_k,
                                 int n_recent, int num_pool_pages, int32_t* __restrict__ out_l,
                                 int32_t* __restrict__ out_p, int32_t* __restrict__ out_count) {
  __shared__ RadixShared sh;
  __shared__ int running_sh;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int max_sel = top_k + n_recent;
  const int n_cand = max(0, n_past - n_recent);
  const int k_eff = min(top_k, n_cand);

  if (t == 0) {
    sh.kth = 0ull;  // with k_eff >= n_cand every candidate is kept
    sh.need = k_eff;
    sh.done = 0;
  }
  __syncthreads();
  if (k_eff > 0 && k_eff < n_cand) {
    unsigned long long prefix = 0ull, mask = 0ull;
    for (int shift = 56; shift >= 0; shift -= 8) {
      if (t < 256) sh.hist[t] = 0u;
      __syncthreads();
      // eight keys per thread in flight before their histogram updates
      for (int base = 0; base < n_cand; base += 8 * NT) {
        unsigned long long kv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int p = base + u * NT + t;
          kv[u] = p < n_cand ? __ldcg(keys + p) : 0ull;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int p = base + u * NT + t;
          if (p < n_cand && (kv[u] & mask) == prefix)
            atomicAdd(&sh.hist[(kv[u] >> shift) & 255ull], 1u);
        }
      }
      __syncthreads();
      radix_pick_bin(sh, prefix, shift);
      prefix = sh.kth;
      mask |= 255ull << shift;
      if (sh.done) break;
    }
  }
  const unsigned long long kth = sh.kth;

  if (t == 0) running_sh = 0;
  __syncthreads();
  for (int base = 0; base < n_past; base += NT) {
    const int p = base + t;
    int keep = 0;
    if (p < n_cand) keep = (k_eff >= n_cand) || (k_eff > 0 && __ldcg(keys + p) >= kth);
    else if (p < n_past) keep = 1;
    const unsigned ballot = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) sh.warp_cnt[warp] = __popc(ballot);
    __syncthreads();
    int before = running_sh;
    for (int w = 0; w < warp; ++w) before += sh.warp_cnt[w];
    before += __popc(ballot & ((1u << lane) - 1u));
    if (keep && before < max_sel) {
      out_l[before] = p;
      if (out_p) {
        const int phys = page_table[p];
        out_p[before] = (phys >= 0 && phys < num_pool_pages) ? phys : 0;
      }
    }
    __syncthreads();
    if (t == 0) {
      int tot = 0;
      for (int w = 0; w < NT / 32; ++w) tot += sh.warp_cnt[w];
      running_sh += tot;
    }
    __syncthreads();
  }
  if (t == 0) *out_count = min(running_sh, max_sel);
}

// Score of a key: the inverse of order_f32 on its upper 32 bits.
__device__ __forceinline__ float key_score(unsigned long long k) {
  const uint32_t u = static_cast<uint32_t>(k >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// Bucket of a score on a linear scale from smin (bucket 0) over 256 buckets.
// Non-decreasing in s: a key in a higher bucket has a strictly higher score.
__device__ __forceinline__ int score_bucket(float s, float smin, float scale) {
  const float x = (s - smin) * scale;
  return x >= 255.f ? 255 : (x > 0.f ? static_cast<int>(x) : 0);
}

// The same selection with the keys held in registers, for n_past <= NT * KPT:
// thread t owns logical pages [t * KPT, (t + 1) * KPT), loaded once together
// with their physical ids (key rows start 16-byte aligned, so pairs load as
// one vector).  The first digit is not a byte of the key (whose top bytes,
// sign and exponent, most scores share, so that nearly every key would land
// in one or two bins) but a bucket of the score on a linear scale between
// the candidates' minimum and maximum: the bucket holding the K-th largest
// key is found from its histogram; the keys above it are kept, and only the
// keys inside it go through exact radix passes over the 64-bit key, starting
// at the highest bit in which they differ.  The kept ids come out ascending
// from one CTA-wide scan of the per-thread counts.
template <int NT, int KPT>
__device__ void select_pages_regs(const unsigned long long* keys,
                                  const int32_t* __restrict__ page_table, int n_past, int top_k,
                                  int n_recent, int num_pool_pages, int32_t* __restrict__ out_l,
                                  int32_t* __restrict__ out_p, int32_t* __restrict__ out_count) {
  static_assert(NT == 256 && KPT % 2 == 0 && KPT <= 32, "select layout");
  constexpr int NW = NT / 32;
  __shared__ RadixShared sh;
  __shared__ float wmin[NW], wmax[NW];
  __shared__ unsigned long long wlo[NW], whi[NW];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int max_sel = top_k + n_recent;
  const int n_cand = max(0, n_past - n_recent);
  const int k_eff = min(top_k, n_cand);
  const int p0 = t * KPT;

  unsigned long long kv[KPT];
  int phys[KPT];
#pragma unroll
  for (int j = 0; j < KPT; ++j) phys[j] = p0 + j < n_past && out_p ? page_table[p0 + j] : 0;
#pragma unroll
  for (int j = 0; j < KPT; j += 2) {
    if (p0 + j + 1 < n_cand) {
      const ulonglong2 v = __ldcg(reinterpret_cast<const ulonglong2*>(keys + p0 + j));
      kv[j] = v.x;
      kv[j + 1] = v.y;
    } else {
      kv[j] = p0 + j < n_cand ? __ldcg(keys + p0 + j) : 0ull;
      kv[j + 1] = 0ull;
    }
  }
  const bool keep_all = k_eff >= n_cand;
  const bool run = k_eff > 0 && !keep_all;  // uniform over the CTA
  unsigned int above_bits = 0u, member_bits = 0u;
  bool bucket_whole = false;
  unsigned long long kth = 0ull;
  if (run) {
    // score range of the candidates
    float lo = __int_as_float(0x7f800000), hi = -lo;
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if (p0 + j < n_cand) {
        const float sc = key_score(kv[j]);
        lo = fminf(lo, sc);
        hi = fmaxf(hi, sc);
      }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (lane == 0) {
      wmin[warp] = lo;
      wmax[warp] = hi;
    }
    if (t == 0) {
      sh.need = k_eff;
      sh.done = 0;
      sh.n_small = 0u;
    }
    sh.hist[t] = 0u;
    __syncthreads();
    float smin = wmin[0], smax = wmax[0];
    for (int w = 1; w < NW; ++w) {
      smin = fminf(smin, wmin[w]);
      smax = fmaxf(smax, wmax[w]);
    }
    const float range = smax - smin;
    const float scale = range > 0.f && range < __int_as_float(0x7f800000) ? 256.f / range : 0.f;
    // histogram of the score buckets, then the bucket of the K-th largest key
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if (p0 + j < n_cand) atomicAdd(&sh.hist[score_bucket(key_score(kv[j]), smin, scale)], 1u);
    __syncthreads();
    radix_pick_bin(sh, 0ull, 0);
    const int B = static_cast<int>(sh.kth);
    bucket_whole = sh.done != 0;
    unsigned long long klo = ~0ull, khi = 0ull;
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if (p0 + j < n_cand) {
        const int bj = score_bucket(key_score(kv[j]), smin, scale);
        above_bits |= static_cast<unsigned int>(bj > B) << j;
        if (bj == B) {
          member_bits |= 1u << j;
          klo = min(klo, kv[j]);
          khi = max(khi, kv[j]);
        }
      }
    const unsigned int n_member = sh.hist[B];  // uniform: read after the pick's barrier
    if (!bucket_whole && n_member <= static_cast<unsigned int>(kSmallBucket)) {
      // exact K-th key among the boundary bucket's few keys (at least two, all
      // distinct): gathered into shared memory, then the key that exactly
      // need - 1 others exceed, found by one warp
#pragma unroll
      for (int j = 0; j < KPT; ++j)
        if ((member_bits >> j) & 1u) sh.small[atomicAdd(&sh.n_small, 1u)] = kv[j];
      __syncthreads();
      if (warp == 0) {
        const int need = sh.need;
        for (int i = lane; i < static_cast<int>(n_member); i += 32) {
          const unsigned long long x = sh.small[i];
          int greater = 0;
          for (int m = 0; m < static_cast<int>(n_member); ++m) greater += sh.small[m] > x;
          if (greater == need - 1) sh.kth = x;
        }
      }
      __syncthreads();
      kth = sh.kth;
    } else if (!bucket_whole) {
      // exact K-th key among the boundary bucket's keys (at least two of
      // them, all distinct): 8-bit digits from the highest differing bit
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        klo = min(klo, __shfl_xor_sync(0xffffffffu, klo, off));
        khi = max(khi, __shfl_xor_sync(0xffffffffu, khi, off));
      }
      if (lane == 0) {
        wlo[warp] = klo;
        whi[warp] = khi;
      }
      __syncthreads();
      klo = wlo[0];
      khi = whi[0];
      for (int w = 1; w < NW; ++w) {
        klo = min(klo, wlo[w]);
        khi = max(khi, whi[w]);
      }
      const int top = 63 - __clzll(static_cast<long long>(klo ^ khi));
      unsigned long long mask = ~((2ull << top) - 1ull);  // the bits above `top`, common
      unsigned long long prefix = klo & mask;
      for (int s = top - 7; s > -8; s -= 8) {
        const int shift = s > 0 ? s : 0;
        const unsigned long long dmask = (1ull << (s >= 0 ? 8 : 8 + s)) - 1ull;
        sh.hist[t] = 0u;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < KPT; ++j)
          if (((member_bits >> j) & 1u) && (kv[j] & mask) == prefix)
            atomicAdd(&sh.hist[(kv[j] >> shift) & dmask], 1u);
        __syncthreads();
        radix_pick_bin(sh, prefix, shift);
        prefix = sh.kth;
        mask |= dmask << shift;
        if (sh.done) break;
      }
      kth = sh.kth;
    }
  }

  unsigned int keep_bits = 0u;
  int cnt = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const int p = p0 + j;
    bool keep;
    if (p < n_cand) {
      const bool member = (member_bits >> j) & 1u;
      keep = keep_all || ((above_bits >> j) & 1u) || (member && (bucket_whole || kv[j] >= kth));
    } else {
      keep = p < n_past;
    }
    keep_bits |= static_cast<unsigned int>(keep) << j;
    cnt += keep;
  }
  int incl = cnt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) sh.warp_cnt[warp] = incl;
  __syncthreads();
  int before = incl - cnt, total = 0;
  for (int w = 0; w < NW; ++w) {
    const int c = sh.warp_cnt[w];
    if (w < warp) before += c;
    total += c;
  }
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    if ((keep_bits >> j) & 1u) {
      if (before < max_sel) {
        out_l[before] = p0 + j;
        if (out_p) out_p[before] = (phys[j] >= 0 && phys[j] < num_pool_pages) ? phys[j] : 0;
      }
      ++before;
    }
  }
  if (t == 0) *out_count = min(total, max_sel);
}

// ---------------------------------------------------------------- q_bar sums
// The query-mean partials of (problem b, group g) summed in one fixed order:
// thread t of 256 sums splits [64 (t / 128), ...) of column t % 128 in eight
// chains (split i goes to chain i mod 8, in increasing i; blocks of B loads
// in flight, the tail as one more block with zeros, x + 0 = x), the chains
// in a fixed tree; qs[half][d] = that half's sum.  The caller adds the halves
// (qs[0] + qs[1]).  B (loads in flight, a multiple of 8) changes only the
// registers used, not the result.
template <int D, int B>
__device__ __forceinline__ void reduce_partials(const float* __restrict__ partial, int splits,
                                                int Hkv, int b, int g, float (*qs)[D]) {
  static_assert(B % 8 == 0, "chains");
  const int t = threadIdx.x, dd = t % 128, half = t / 128;
  if (dd >= D) return;
  const float* pp = partial + static_cast<size_t>(b) * splits * Hkv * D + g * D + dd;
  const int lo = min(splits, half * 64), hi = min(splits, lo + 64);
  float s8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) s8[e] = 0.f;
  int i = lo;
  for (; i + B <= hi; i += B) {
    float v[B];
#pragma unroll
    for (int e = 0; e < B; ++e) v[e] = __ldg(pp + static_cast<size_t>(i + e) * Hkv * D);
#pragma unroll
    for (int e = 0; e < B; ++e) s8[e & 7] += v[e];
  }
  if (i < hi) {
    float v[B];
#pragma unroll
    for (int e = 0; e < B; ++e)
      v[e] = i + e < hi ? __ldg(pp + static_cast<size_t>(i + e) * Hkv * D) : 0.f;
#pragma unroll
    for (int e = 0; e < B; ++e) s8[e & 7] += v[e];
  }
  qs[half][dd] = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
}

// A batch's Q sums, once per (group, problem): grid (Hkv, problems), 256
// threads, a dependent launch after the query mean.  Writes qs[0] + qs[1]
// into qsum [problems][Hkv][d]; the scores kernel then reads them as Q sums
// (adding 0 for the second half), so every problem gets bit for bit the q_bar
// of the one-problem path, whose CTAs each reduce the partials themselves.
template <int D>
__global__ void __launch_bounds__(kScoreThreads) qsum_reduce_kernel(
    const float* __restrict__ partial, int splits, float* __restrict__ qsum) {
  __shared__ float qs[2][D];
  const int g = blockIdx.x, b = blockIdx.y, Hkv = gridDim.x, t = threadIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  reduce_partials<D, 32>(partial, splits, Hkv, b, g, qs);
  __syncthreads();
  if (t < D) qsum[(static_cast<size_t>(b) * Hkv + g) * D + t] = qs[0][t] + qs[1][t];
}

// ---------------------------------------------------------------- scores + select
// grid (max(1, ceil(max_past / 64)), Hkv, problems), kScoreThreads threads.
// Each warp first loads the summaries of its 8 pages (they do not depend on
// q_bar, so these loads overlap its reduction).  q_bar, FROM_QSUM false:
// thread t sums splits [64 (t / D), ...) of column t % D of the query-mean
// partials in a fixed order (eight chains, sixteen loads in flight), the two
// halves are added in a fixed order and divided by rows * G.  FROM_QSUM true:
// q_bar = qsum[problem][group] / (rows * G), qsum being the group's sum of Q
// over the rows and G heads made elsewhere (the projection's epilogue).
// Key = (ordered score << 32) | (~logical id), stored at
// [problem][group][key_stride(max_past)].  The CTA whose ticket is the last
// of its (problem, group) then runs the select and sets the ticket back to
// zero, so a completed call leaves every ticket at zero.
template <int D, bool FROM_QSUM, bool FUSED_SELECT>
__global__ void __launch_bounds__(kScoreThreads, FUSED_SELECT ? 2 : 5) page_score_select_kernel(
    const float* __restrict__ partial, const float* __restrict__ qsum,
    const float* __restrict__ summary, const int32_t* __restrict__ page_table, const Problems pb,
    int G, int Hkv, int num_pool_pages, unsigned long long* __restrict__ keys,
    float* __restrict__ out_scores, unsigned int* __restrict__ tickets, int top_k, int n_recent,
    int32_t* __restrict__ out_logical, int32_t* __restrict__ out_physical,
    int32_t* __restrict__ out_count) {
  static_assert(kScoreThreads == 2 * 128 && D <= 128, "q_bar reduction layout");
  constexpr int PW = kPagesPerScoreCta / (kScoreThreads / 32);  // pages per warp
  constexpr int EPL = D / 32;                                   // elements per lane
  __shared__ float qs[2][D];
  __shared__ int last_sh;
  const int g = blockIdx.y, b = blockIdx.z, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int n_past = problem_npast(pb, b);
  const int n_ctas = max(1, (n_past + kPagesPerScoreCta - 1) / kPagesPerScoreCta);
  if (!FUSED_SELECT) pdl_launch_dependents();
  if (static_cast<int>(blockIdx.x) >= n_ctas) return;  // beyond this problem's pages

  // this warp's page summaries (EPL fp32 per lane and page).  One problem:
  // loaded first, so that the loads overlap the q_bar reduction (and the
  // query-mean kernel's tail); a batch: loaded after q_bar, which keeps the
  // registers, and so the occupancy of its many short CTAs, low.
  const int p0 = blockIdx.x * kPagesPerScoreCta + warp * PW;
  float sv[PW][EPL];
  auto load_summaries = [&]() {
    int phys[PW];
#pragma unroll
    for (int i = 0; i < PW; ++i) phys[i] = p0 + i < n_past ? __ldg(page_table + p0 + i) : 0;
#pragma unroll
    for (int i = 0; i < PW; ++i) {
      if (phys[i] < 0 || phys[i] >= num_pool_pages) {
        if (lane == 0) atomicOr(pb.status, OOMB_DEV_BAD_PAGE);
        phys[i] = 0;
      }
      const float* srow = summary + (static_cast<size_t>(phys[i]) * Hkv + g) * D + lane * EPL;
      if (EPL == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(srow));
        sv[i][0] = v.x;
        sv[i][1] = v.y;
        sv[i][2] = v.z;
        sv[i][3] = v.w;
      } else {
        const float2 v = __ldg(reinterpret_cast<const float2*>(srow));
        sv[i][0] = v.x;
        sv[i][1] = v.y;
      }
    }
  };
  if (FUSED_SELECT) load_summaries();

  // the query-mean partials and the tickets it zeroed are read from here on
  pdl_wait();
  // q_bar of (problem b, group g)
  if (FROM_QSUM) {
    if (t < D) qs[0][t] = __ldg(qsum + (static_cast<size_t>(b) * Hkv + g) * D + t);
    else if (t >= 128 && t - 128 < D) qs[1][t - 128] = 0.f;
  } else {
    reduce_partials<D, 32>(partial, pb.splits, Hkv, b, g, qs);
  }
  __syncthreads();
  if (!FUSED_SELECT) load_summaries();
  int r0, r1;
  problem_rows(pb, b, r0, r1);
  const float rows = static_cast<float>(r1 - r0) * static_cast<float>(G);
  const size_t row = (static_cast<size_t>(b) * Hkv + g);
  unsigned long long* key_row = keys + row * key_stride(pb.max_past);
  float qv[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int dd = lane * EPL + e;
    qv[e] = rows > 0.f ? (qs[0][dd] + qs[1][dd]) / rows : 0.f;
  }
  float acc[PW];
#pragma unroll
  for (int i = 0; i < PW; ++i) {
    acc[i] = 0.f;
    if (p0 + i < n_past) {
      if (EPL == 4)
        acc[i] = sv[i][0] * qv[0] + sv[i][1] * qv[1] + sv[i][2] * qv[2] + sv[i][3] * qv[3];
      else
        acc[i] = sv[i][0] * qv[0] + sv[i][1] * qv[1];
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
      if (out_scores) out_scores[row * pb.max_past + p] = mine;
      key_row[p] =
          (static_cast<unsigned long long>(order_f32(mine)) << 32) |
          static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(p));
    }
  }
  if (!FUSED_SELECT) return;  // topk_select_kernel selects after this grid
  // the last CTA of this (problem, group) to get here selects; its ticket
  // makes every other CTA's keys visible to it (see ticket_acq_rel)
  __syncthreads();
  if (t == 0) last_sh = ticket_acq_rel(&tickets[row]) == static_cast<unsigned>(n_ctas - 1);
  __syncthreads();
  if (!last_sh) return;
  const int max_sel = top_k + n_recent;
  int32_t* out_p = out_physical ? out_physical + row * max_sel : nullptr;
  if (n_past <= kScoreThreads * kKeysPerThread)
    select_pages_regs<kScoreThreads, kKeysPerThread>(key_row, page_table, n_past, top_k, n_recent,
                                                     num_pool_pages, out_logical + row * max_sel,
                                                     out_p, out_count + row);
  else
    select_pages_cta<kScoreThreads>(key_row, page_table, n_past, top_k, n_recent, num_pool_pages,
                                    out_logical + row * max_sel, out_p, out_count + row);
  if (t == 0) tickets[row] = 0u;  // every CTA of this (problem, group) has counted
}

// The select alone, one CTA per (group, problem): grid (Hkv, problems), a
// dependent launch after the scores kernel (of a batch of problems, whose
// scoring CTAs then carry no select code and run at full occupancy).
__global__ void __launch_bounds__(kScoreThreads) topk_select_kernel(
    const unsigned long long* keys, const int32_t* __restrict__ page_table, const Problems pb,
    int num_pool_pages, int top_k, int n_recent, int32_t* __restrict__ out_logical,
    int32_t* __restrict__ out_physical, int32_t* __restrict__ out_count) {
  const int g = blockIdx.x, b = blockIdx.y, Hkv = gridDim.x;
  const int n_past = problem_npast(pb, b);
  const size_t row = static_cast<size_t>(b) * Hkv + g;
  const unsigned long long* key_row = keys + row * key_stride(pb.max_past);
  const int max_sel = top_k + n_recent;
  int32_t* out_p = out_physical ? out_physical + row * max_sel : nullptr;
  pdl_wait();  // the keys of the scores kernel
  if (n_past <= kScoreThreads * kKeysPerThread)
    select_pages_regs<kScoreThreads, kKeysPerThread>(key_row, page_table, n_past, top_k, n_recent,
                                                     num_pool_pages, out_logical + row * max_sel,
                                                     out_p, out_count + row);
  else
    select_pages_cta<kScoreThreads>(key_row, page_table, n_past, top_k, n_recent, num_pool_pages,
                                    out_logical + row * max_sel, out_p, out_count + row);
}

// Workspace: partials [problems][splits <= 128][Hkv][d] fp32, a region of
// [problems][Hkv][d] fp32 whose first problems * Hkv words are the select
// tickets, then keys [problems][Hkv][key_stride(max_past)] u64.
size_t workspace_bytes_for(int64_t problems, int Hkv, int D, int max_past) {
  const size_t partial = static_cast<size_t>(problems) * kSplits * Hkv * D * 4;
  const size_t qbar = static_cast<size_t>(problems) * Hkv * D * 4;
  const size_t keys = static_cast<size_t>(problems) * Hkv * key_stride(max_past) * 8;
  return align256(partial) + align256(qbar) + align256(keys);
}

// Launches the scores kernel (q_bar from the query-mean partials, or from Q
// sums when qsum is set) and, for a batch, the select kernel after it.
// dependent: the scores kernel is a programmatic dependent launch of the
// kernel before it on the stream (which made its partials or sums).
oomb_status launch_score_select(const oomb_pool* pool, const float* partial, const float* qsum,
                                bool dependent, const Problems& pb, int n_problems, int G,
                                const int32_t* d_page_table, int top_k, int n_recent,
                                int32_t* d_out_logical, int32_t* d_out_physical,
                                int32_t* d_out_count, float* d_out_scores, unsigned int* tickets,
                                unsigned long long* keys, cudaStream_t s) {
  const oomb_pool_desc& d = pool->desc;
  const int Hkv = d.num_kv_heads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(std::max(1, (pb.max_past + kPagesPerScoreCta - 1) / kPagesPerScoreCta),
                     Hkv, n_problems);
  cfg.blockDim = dim3(kScoreThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  const float* summary = pool->summary;
  const int num_pages = d.num_pages;
  // one problem: the last scoring CTA of a group selects; a batch: the
  // scoring CTAs only score and a select kernel follows
  const bool fused = n_problems == 1;
  cudaError_t e;
#define OOMB_SCORE_ARGS                                                                    \
  partial, qsum, summary, d_page_table, pb, G, Hkv, num_pages, keys, d_out_scores, tickets, \
      top_k, n_recent, d_out_logical, d_out_physical, d_out_count
  // (a batch always scores from Q sums: launch_topk reduces its partials once)
#define OOMB_SCORE_LAUNCH(DD)                                                                   \
  (!qsum   ? cudaLaunchKernelEx(&cfg, page_score_select_kernel<DD, false, true>, OOMB_SCORE_ARGS) \
   : fused ? cudaLaunchKernelEx(&cfg, page_score_select_kernel<DD, true, true>, OOMB_SCORE_ARGS)  \
           : cudaLaunchKernelEx(&cfg, page_score_select_kernel<DD, true, false>, OOMB_SCORE_ARGS))
  if (!qsum && !fused) return OOMB_ERR_INVALID_ARG;
  e = d.head_dim == 128 ? OOMB_SCORE_LAUNCH(128) : OOMB_SCORE_LAUNCH(64);
#undef OOMB_SCORE_LAUNCH
#undef OOMB_SCORE_ARGS
  if (e == cudaSuccess && !fused) {
    cudaLaunchConfig_t sel = cfg;
    sel.gridDim = dim3(Hkv, n_problems, 1);
    sel.numAttrs = 1;  // dependent of the scores kernel
    const unsigned long long* ckeys = keys;
    e = cudaLaunchKernelEx(&sel, topk_select_kernel, ckeys, d_page_table, pb, num_pages, top_k,
                           n_recent, d_out_logical, d_out_physical, d_out_count);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return OOMB_ERR_CUDA;
  }
  return oomb::check_launch();
}

// Launches the selection of `n_problems` problems from Q on `s`: the query
// mean, then for one problem the fused scores + select kernel, for a batch
// the Q-sum reduction, the scores kernel and the select kernel.
oomb_status launch_topk(const oomb_pool* pool, const void* d_q, int num_q_heads,
                        const Problems& pb_in, int n_problems, const int32_t* d_page_table,
                        int top_k, int n_recent, int32_t* d_out_logical, int32_t* d_out_physical,
                        int32_t* d_out_count, float* d_out_scores, void* scratch,
                        cudaStream_t s) {
  const oomb_pool_desc& d = pool->desc;
  const int Hkv = d.num_kv_heads, D = d.head_dim, G = num_q_heads / Hkv;
  Problems pb = pb_in;
  pb.status = pool->d_status;
  const size_t partial_bytes = align256(static_cast<size_t>(n_problems) * kSplits * Hkv * D * 4);
  const size_t qbar_bytes = align256(static_cast<size_t>(n_problems) * Hkv * D * 4);
  float* partial = static_cast<float*>(scratch);
  // the region after the partials: the tickets of the one-problem path, or a
  // batch's Q sums
  unsigned int* tickets =
      reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(scratch) + partial_bytes);
  float* batch_qsum = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + partial_bytes);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(
      static_cast<uint8_t*>(scratch) + partial_bytes + qbar_bytes);
  const int n_tickets = n_problems * Hkv;
  const auto* q = static_cast<const __nv_bfloat16*>(d_q);
  // one thread per 16-byte column of a group's heads, a multiple of 32, at most 256
  const int ncol = G * D / 8;
  const int mean_threads = ncol >= kMeanThreads ? kMeanThreads : ((ncol + 31) / 32) * 32;
  const size_t mean_smem = static_cast<size_t>(G) * D * 4;
  dim3 g1(pb.splits, Hkv, n_problems);
  if (D == 128)
    qmean_partial_kernel<128><<<g1, mean_threads, mean_smem, s>>>(q, partial, pb, num_q_heads, G,
                                                                  tickets, n_tickets);
  else
    qmean_partial_kernel<64><<<g1, mean_threads, mean_smem, s>>>(q, partial, pb, num_q_heads, G,
                                                                 tickets, n_tickets);
  if (n_problems == 1)
    return launch_score_select(pool, partial, nullptr, true, pb, 1, G, d_page_table, top_k,
                               n_recent, d_out_logical, d_out_physical, d_out_count,
                               d_out_scores, tickets, keys, s);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(Hkv, n_problems, 1);
  cfg.blockDim = dim3(kScoreThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float* cpartial = partial;
  const int splits = pb.splits;
  const cudaError_t e =
      D == 128 ? cudaLaunchKernelEx(&cfg, qsum_reduce_kernel<128>, cpartial, splits, batch_qsum)
               : cudaLaunchKernelEx(&cfg, qsum_reduce_kernel<64>, cpartial, splits, batch_qsum);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return OOMB_ERR_CUDA;
  }
  return launch_score_select(pool, nullptr, batch_qsum, true, pb, n_problems, G, d_page_table,
                             top_k, n_recent, d_out_logical, d_out_physical, d_out_count,
                             d_out_scores, tickets, keys, s);
}

// Host-side checks shared by the entry points.
oomb_status check_topk_args(const oomb_pool* pool, const void* d_q, int num_q_heads,
                            const int32_t* d_page_table, int max_past, int top_k, int n_recent,
                            const int32_t* d_out_logical, const int32_t* d_out_count) {
  // device pools and pinned-host pools (whose summaries live on the device)
  if (!pool || pool->desc.location == OOMB_LOC_HOST) return OOMB_ERR_INVALID_ARG;
  const int Hkv = pool->desc.num_kv_heads;
  if (!d_q || !d_out_logical || !d_out_count) return OOMB_ERR_INVALID_ARG;
  if (num_q_heads <= 0 || num_q_heads % Hkv != 0) return OOMB_ERR_INVALID_ARG;
  // the query mean keeps one fp32 row of every head in 48 KiB of shared memory
  if (static_cast<size_t>(num_q_heads) * pool->desc.head_dim * 4 > 48 * 1024)
    return OOMB_ERR_UNSUPPORTED;
  if (max_past < 0 || max_past > 65536 || top_k < 0 || n_recent < 0 ||
      top_k + n_recent > 4096 || top_k + n_recent == 0)
    return OOMB_ERR_INVALID_ARG;
  if (max_past > 0 && !d_page_table) return OOMB_ERR_INVALID_ARG;
  if (!oomb::aligned16(d_q)) return OOMB_ERR_INVALID_ARG;
  return OOMB_OK;
}

}  // namespace

extern "C" size_t oomb_page_topk_workspace_size(int32_t chunk_len, int32_t num_q_heads,
                                                int32_t num_kv_heads, int32_t head_dim,
                                                int32_t n_past) {
  (void)num_q_heads;
  if (chunk_len <= 0 || num_kv_heads <= 0 || head_dim <= 0 || n_past < 0) return 0;
  return workspace_bytes_for(1, num_kv_heads, head_dim, n_past);
}

extern "C" oomb_status oomb_page_topk(const oomb_pool* pool, const void* d_q, int32_t chunk_len,
                                      int32_t num_q_heads, const int32_t* d_page_table,
                                      int32_t n_past, int32_t top_k, int32_t n_recent,
                                      int32_t* d_out_logical, int32_t* d_out_physical,
                                      int32_t* d_out_count, float* d_out_scores,
                                      void* d_workspace, size_t workspace_bytes, void* stream) {
  oomb_status st = check_topk_args(pool, d_q, num_q_heads, d_page_table, n_past, top_k, n_recent,
                                   d_out_logical, d_out_count);
  if (st != OOMB_OK) return st;
  if (chunk_len <= 0 || !d_workspace || !oomb::aligned16(d_workspace)) return OOMB_ERR_INVALID_ARG;
  const oomb_pool_desc& d = pool->desc;
  if (workspace_bytes < workspace_bytes_for(1, d.num_kv_heads, d.head_dim, n_past))
    return OOMB_ERR_INVALID_ARG;
  oomb::DeviceGuard guard(d.device);
  const Problems pb{nullptr, nullptr, chunk_len, n_past, n_past, chunk_len,
                    choose_splits(chunk_len), nullptr};
  return launch_topk(pool, d_q, num_q_heads, pb, 1, d_page_table, top_k, n_recent, d_out_logical,
                     d_out_physical, d_out_count, d_out_scores, d_workspace,
                     static_cast<cudaStream_t>(stream));
}

namespace {

// Selection from per-group sums of Q made by the producer of Q (the
// projection's epilogue): the scores + select kernel alone, one launch.  Its
// workspace holds the Hkv tickets (zero before the first call; every
// completed call leaves them at zero) and the keys.
size_t qsum_workspace_bytes(int Hkv, int n_past) {
  return align256(static_cast<size_t>(Hkv) * 4) +
         align256(static_cast<size_t>(Hkv) * key_stride(n_past) * 8);
}

}  // namespace

extern "C" size_t oomb_page_topk_qsum_workspace_size(int32_t num_kv_heads, int32_t n_past) {
  if (num_kv_heads <= 0 || n_past < 0) return 0;
  return qsum_workspace_bytes(num_kv_heads, n_past);
}

extern "C" oomb_status oomb_page_topk_qsum(const oomb_pool* pool, const float* d_qsum,
                                           int32_t chunk_len, int32_t num_q_heads,
                                           const int32_t* d_page_table, int32_t n_past,
                                           int32_t top_k, int32_t n_recent,
                                           int32_t* d_out_logical, int32_t* d_out_physical,
                                           int32_t* d_out_count, float* d_out_scores,
                                           void* d_workspace, size_t workspace_bytes,
                                           void* stream) {
  oomb_status st = check_topk_args(pool, d_qsum, num_q_heads, d_page_table, n_past, top_k,
                                   n_recent, d_out_logical, d_out_count);
  if (st != OOMB_OK) return st;
  if (chunk_len <= 0 || !d_workspace || !oomb::aligned16(d_workspace)) return OOMB_ERR_INVALID_ARG;
  const oomb_pool_desc& d = pool->desc;
  if (workspace_bytes < qsum_workspace_bytes(d.num_kv_heads, n_past)) return OOMB_ERR_INVALID_ARG;
  oomb::DeviceGuard guard(d.device);
  const Problems pb{nullptr, nullptr, chunk_len, n_past, n_past, chunk_len, 1, pool->d_status};
  auto* tickets = static_cast<unsigned int*>(d_workspace);
  auto* keys = reinterpret_cast<unsigned long long*>(
      static_cast<uint8_t*>(d_workspace) + align256(static_cast<size_t>(d.num_kv_heads) * 4));
  return launch_score_select(pool, nullptr, d_qsum, false, pb, 1, num_q_heads / d.num_kv_heads,
                             d_page_table, top_k, n_recent, d_out_logical, d_out_physical,
                             d_out_count, d_out_scores, tickets, keys,
                             static_cast<cudaStream_t>(stream));
}

extern "C" size_t oomb_page_topk_batched_workspace_size(int32_t n_problems, int32_t num_kv_heads,
                                                        int32_t head_dim, int32_t max_past) {
  if (n_problems <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_past < 0) return 0;
  return workspace_bytes_for(n_problems, num_kv_heads, head_dim, max_past);
}

extern "C" oomb_status oomb_page_topk_batched(
    const oomb_pool* pool, const void* d_q, int32_t num_rows, int32_t num_q_heads,
    int32_t n_problems, const int32_t* d_row_start, int32_t max_rows, const int32_t* d_n_past,
    int32_t max_past, const int32_t* d_page_table, int32_t top_k, int32_t n_recent,
    int32_t* d_out_logical, int32_t* d_out_physical, int32_t* d_out_count, float* d_out_scores,
    void* d_workspace, size_t workspace_bytes, void* stream) {
  oomb_status st = check_topk_args(pool, d_q, num_q_heads, d_page_table, max_past, top_k,
                                   n_recent, d_out_logical, d_out_count);
  if (st != OOMB_OK) return st;
  if (n_problems <= 0 || n_problems > 65535 || num_rows <= 0 || max_rows <= 0 ||
      max_rows > num_rows || !d_row_start || !d_n_past || !d_workspace ||
      !oomb::aligned16(d_workspace))
    return OOMB_ERR_INVALID_ARG;
  const oomb_pool_desc& d = pool->desc;
  if (workspace_bytes < workspace_bytes_for(n_problems, d.num_kv_heads, d.head_dim, max_past))
    return OOMB_ERR_INVALID_ARG;
  oomb::DeviceGuard guard(d.device);
  const Problems pb{d_row_start, d_n_past, 0, 0, max_past, num_rows, choose_splits(max_rows),
                    nullptr};
  return launch_topk(pool, d_q, num_q_heads, pb, n_problems, d_page_table, top_k, n_recent,
                     d_out_logical, d_out_physical, d_out_count, d_out_scores, d_workspace,
                     static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- recent-only lists
// Layers that are sparse by construction attend to the most recent pages
// ([it] §2D): group g's list is the last `window` of the n_past logical pages,
// ascending, mapped to physical ids.  One thread per (group, slot).
namespace {

__global__ void local_pages_kernel(const int32_t* __restrict__ page_table, int n_past, int window,
                                   int Hkv, int num_pool_pages, int32_t* __restrict__ out_pages,
                                   int32_t* __restrict__ out_count, uint32_t* status) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= Hkv * window) return;
  const int g = e / window, i = e % window;
  const int n = min(window, n_past), lo = n_past - n;
  int id = 0;
  if (i < n) {
    id = page_table[lo + i];
    if (id < 0 || id >= num_pool_pages) {
      atomicOr(status, OOMB_DEV_BAD_PAGE);
      id = 0;
    }
  }
  out_pages[static_cast<size_t>(g) * window + i] = id;
  if (i == 0) out_count[g] = n;
}

}  // namespace

extern "C" oomb_status oomb_local_pages(const oomb_pool* pool, const int32_t* d_page_table,
                                        int32_t n_past, int32_t window, int32_t* d_out_pages,
                                        int32_t* d_out_count, void* stream) {
  if (!pool || pool->desc.location == OOMB_LOC_HOST || !d_out_pages || !d_out_count)
    return OOMB_ERR_INVALID_ARG;
  if (n_past < 0 || window <= 0 || (n_past > 0 && !d_page_table)) return OOMB_ERR_INVALID_ARG;
  const int Hkv = pool->desc.num_kv_heads;
  if (static_cast<int64_t>(window) * Hkv > (1 << 26)) return OOMB_ERR_UNSUPPORTED;
  oomb::DeviceGuard guard(pool->desc.device);
  const int n = window * Hkv;
  local_pages_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      d_page_table, n_past, window, Hkv, pool->desc.num_pages, d_out_pages, d_out_count,
      pool->d_status);
  return oomb::check_launch();
}

// ---------------------------------------------------------------- per-query-page lists
// One thread per (128-row query tile, group): merges the ascending logical
// lists of the tile's query pages (at most 8) into one ascending union,
// writing each union entry's physical id and the bit set of the query pages
// that listed it.
namespace {

__global__ void qpage_lists_kernel(const int32_t* __restrict__ sel_logical,
                                   const int32_t* __restrict__ sel_physical,
                                   const int32_t* __restrict__ sel_count, int n_qpages,
                                   int per_tile, int n_qtiles, int Hkv, int max_sel,
                                   int32_t* __restrict__ out_pages, uint8_t* __restrict__ out_masks,
                                   int32_t* __restrict__ out_count, int max_union,
                                   uint32_t* status) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n_qtiles * Hkv) return;
  const int t = e / Hkv, g = e % Hkv;
  const int b0 = t * per_tile, nb = min(per_tile, n_qpages - b0);
  int cur[8], cnt[8];
  for (int b = 0; b < nb; ++b) {
    int c = sel_count[static_cast<size_t>(b0 + b) * Hkv + g];
    if (c < 0 || c > max_sel) {
      atomicOr(status, OOMB_DEV_BAD_COUNT);
      c = c < 0 ? 0 : max_sel;
    }
    cnt[b] = c;
    cur[b] = 0;
  }
  const size_t out0 = static_cast<size_t>(e) * max_union;
  int n = 0;
  while (true) {
    int lo = INT_MAX, phys = 0;
    for (int b = 0; b < nb; ++b) {
      if (cur[b] < cnt[b]) {
        const size_t i = (static_cast<size_t>(b0 + b) * Hkv + g) * max_sel + cur[b];
        const int l = sel_logical[i];
        if (l < lo) {
          lo = l;
          phys = sel_physical[i];
        }
      }
    }
    if (lo == INT_MAX) break;
    uint32_t m = 0;
    for (int b = 0; b < nb; ++b) {
      if (cur[b] < cnt[b] &&
          sel_logical[(static_cast<size_t>(b0 + b) * Hkv + g) * max_sel + cur[b]] == lo) {
        m |= 1u << b;
        ++cur[b];
      }
    }
    out_pages[out0 + n] = phys;
    out_masks[out0 + n] = static_cast<uint8_t>(m);
    ++n;
  }
  out_count[e] = n;
}

}  // namespace

extern "C" oomb_status oomb_qpage_lists(oomb_pool* pool, const int32_t* d_sel_logical,
                                        const int32_t* d_sel_physical, const int32_t* d_sel_count,
                                        int32_t chunk_len, int32_t max_sel, int32_t* d_out_pages,
                                        uint8_t* d_out_masks, int32_t* d_out_count,
                                        int32_t max_union, void* stream) {
  if (!pool || pool->desc.location == OOMB_LOC_HOST) return OOMB_ERR_INVALID_ARG;
  const int P = pool->desc.page_size, Hkv = pool->desc.num_kv_heads;
  if (chunk_len <= 0 || chunk_len % P != 0 || max_sel <= 0) return OOMB_ERR_INVALID_ARG;
  if (!d_sel_logical || !d_sel_physical || !d_sel_count || !d_out_pages || !d_out_masks ||
      !d_out_count)
    return OOMB_ERR_INVALID_ARG;
  const int per_tile = 128 / P;  // query pages per 128-row tile (1 .. 8)
  const int n_qpages = chunk_len / P;
  if (static_cast<int64_t>(max_union) < static_cast<int64_t>(std::min(per_tile, n_qpages)) *
                                            max_sel)
    return OOMB_ERR_INVALID_ARG;
  const int n_qtiles = (chunk_len + 127) / 128;
  oomb::DeviceGuard guard(pool->desc.device);
  const int n = n_qtiles * Hkv;
  qpage_lists_kernel<<<(n + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      d_sel_logical, d_sel_physical, d_sel_count, n_qpages, per_tile, n_qtiles, Hkv, max_sel,
      d_out_pages, d_out_masks, d_out_count, max_union, pool->d_status);
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
// every scratch word before reading it (the first launch zeroes the select
// tickets the second counts on), so the caller clears nothing, but calls
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
  oomb_status st = check_topk_args(pool, d_q, num_q_heads, d_page_table, n_past, top_k, n_recent,
                                   d_out_logical, d_out_count);
  if (st != OOMB_OK) return st;
  if (chunk_len <= 0) return OOMB_ERR_INVALID_ARG;
  const oomb_pool_desc& d = pool->desc;
  // the scratch array has a fixed size: larger problems must use oomb_page_topk
  if (workspace_bytes_for(1, d.num_kv_heads, d.head_dim, n_past) > OOMB_TOPK_STATIC_SCRATCH_BYTES)
    return OOMB_ERR_UNSUPPORTED;
  oomb::DeviceGuard guard(d.device);
  void* scratch = nullptr;
  st = static_scratch(d.device, &scratch);
  if (st != OOMB_OK) return st;
  const Problems pb{nullptr, nullptr, chunk_len, n_past, n_past, chunk_len,
                    choose_splits(chunk_len), nullptr};
  return launch_topk(pool, d_q, num_q_heads, pb, 1, d_page_table, top_k, n_recent, d_out_logical,
                     d_out_physical, d_out_count, d_out_scores, scratch,
                     static_cast<cudaStream_t>(stream));
}
