// KV-tile schedule of one chunk over the paged cache, shared by the attention
// kernels.
//
// A KV tile is 128 consecutive keys of one KV head: 128/P pages.  Tiles
// [0, n_past_tiles) walk the group's list of past pages in list order; the
// next tiles walk the chunk's own pages.  Pages are full (every page of the
// list holds P valid keys), so a past tile is valid page by page; the chunk's
// own keys are valid below chunk_len and, for row q, at local positions <= q.
#pragma once
#include <cstdint>

#include "internal.h"

namespace oomb {

constexpr int kTile = 128;  // rows per Q tile and keys per KV tile

struct KvSchedule {
  int n_past_pages;  // pages of the group's past list (clamped to max_past)
  int n_past_tiles;  // ceil(n_past_pages * P / 128)
};

__device__ __forceinline__ KvSchedule kv_schedule(const int32_t* past_counts, int g, int max_past,
                                                  int P, uint32_t* status) {
  KvSchedule s;
  int n = 0;
  if (max_past > 0) {
    n = past_counts[g];
    if (n < 0 || n > max_past) {
      if (threadIdx.x == 0) atomicOr(status, OOMB_DEV_BAD_COUNT);
      n = n < 0 ? 0 : max_past;
    }
  }
  s.n_past_pages = n;
  s.n_past_tiles = (n * P + kTile - 1) / kTile;
  return s;
}

// Physical page of slot `slot` (0 .. 128/P-1) of KV tile j, or `oob` (an id
// past the pool's end: the TMA zero-fills it) when the slot holds no page.
// Invalid ids in the lists are reported and replaced by `oob`.
__device__ __forceinline__ int tile_page(int j, int slot, const KvSchedule& s,
                                         const int32_t* past_list, const int32_t* cur_pages,
                                         int n_cur_pages, int P, int oob, uint32_t* status) {
  const int per = kTile / P;
  int id = oob;
  bool listed = false;
  if (j < s.n_past_tiles) {
    const int li = j * per + slot;
    if (li < s.n_past_pages) {
      id = past_list[li];
      listed = true;
    }
  } else {
    const int ci = (j - s.n_past_tiles) * per + slot;
    if (ci < n_cur_pages) {
      id = cur_pages[ci];
      listed = true;
    }
  }
  if (listed && (id < 0 || id >= oob)) {
    if (status) atomicOr(status, OOMB_DEV_BAD_PAGE);
    id = oob;
  }
  return id;
}

}  // namespace oomb
