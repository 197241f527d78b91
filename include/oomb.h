/*
 * oomb.h — C ABI of the paged chunk-attention library (liboomb.so).
 *
 * One chunk's queries attend to a paged KV cache that holds every earlier
 * chunk plus the chunk itself (causal), on one NVIDIA B200 (sm_100a).  The
 * method is the one summarised in "Out of the Memory Barrier: A Highly Memory
 * Efficient Training System for LLMs with Million-Token Contexts"
 * (gist.science/{pt,es,it}/paper/2602.02108):
 *   - chunk-recurrent training, activations recomputed in the backward
 *     ([pt] §2A, [es] §2A, [it] §2A);
 *   - KV cache AND its gradients in non-contiguous pages, no reallocation or
 *     copy on append ([pt] §2B, [es] §2B "Gestión de Memoria Paginada",
 *     [it] §2B);
 *   - custom forward/backward operators on the paged cache that add gradients
 *     in place with atomic adds, outside autograd ([pt] §2B "Kernels
 *     Personalizados", [es] §2B, [it] §2B);
 *   - page-level Top-K sparse attention by a mean representative vector
 *     ([pt] §2C, [es] §2B "Atención Escasa a Nivel de Página", [it] §2D);
 *   - asynchronous CPU offload of KV and gradients with pinned memory and
 *     dedicated streams ([pt] §2D, [es] §2B "Descarga Asíncrona", [it] §2C).
 *
 * Conventions
 *   - Every call returns an oomb_status; nothing throws across the ABI.
 *   - Argument errors are detected on the host before any launch and leave
 *     all buffers untouched.
 *   - Work is stream-ordered on the stream passed (a cudaStream_t given as
 *     void*; NULL = the legacy default stream).  Asynchronous CUDA errors
 *     surface at a later call as OOMB_ERR_CUDA.
 *   - Kernels never trap or assert.  A kernel that finds an invalid page id
 *     skips the access and sets the pool's device status word; a kernel whose
 *     internal wait runs past its limit sets it too and returns.  Read it with
 *     oomb_get_device_status().
 *   - Caller-owned buffers (q, o, lse, dO, dq, page lists, workspaces) are
 *     plain device pointers; the library keeps no caller pointer past a call.
 *   - The library owns pool memory; a page id stays valid until freed.
 *
 * Layouts (row-major, innermost last)
 *   KV pool     [num_pages][num_kv_heads][2][page_size][head_dim] bf16
 *               (index 0 of the size-2 axis = K, 1 = V)
 *   grad pool   same shape, fp32 (dK, dV)
 *   summaries   [num_pages][num_kv_heads][head_dim] fp32 (mean key of a page)
 *   q, o, dO, dq  [chunk_len][num_q_heads][head_dim] bf16 (token-major)
 *   lse, delta  [num_q_heads][chunk_len] fp32, natural log
 *   query head h reads KV head h / (num_q_heads / num_kv_heads).
 *
 * Supported shapes: head_dim 64 or 128; page_size 16, 32, 64 or 128;
 * chunk_len a positive multiple of page_size; num_q_heads a multiple of
 * num_kv_heads.
 */
#ifndef OOMB_H
#define OOMB_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum oomb_status {
  OOMB_OK = 0,
  OOMB_ERR_INVALID_ARG = 1,   /* bad pointer, size, shape or combination       */
  OOMB_ERR_OUT_OF_PAGES = 2,  /* alloc_page on an exhausted pool               */
  OOMB_ERR_BAD_PAGE = 3,      /* page id out of range, or freeing a free page  */
  OOMB_ERR_CUDA = 4,          /* a CUDA runtime call failed                    */
  OOMB_ERR_TIMEOUT = 5,       /* oomb_wait ran past its limit                  */
  OOMB_ERR_UNSUPPORTED = 6,   /* shape outside the supported set               */
  OOMB_ERR_DEVICE_CHECK = 7   /* a kernel recorded a bounds or wait failure    */
} oomb_status;

typedef enum oomb_location {
  OOMB_LOC_DEVICE = 0,       /* HBM of desc.device (cudaMalloc)               */
  OOMB_LOC_PINNED_HOST = 1,  /* page-locked host memory (cudaHostAlloc)       */
  OOMB_LOC_HOST = 2          /* ordinary host memory; needs no GPU            */
} oomb_location;

typedef struct oomb_pool oomb_pool; /* opaque, owned by the library */

typedef struct oomb_pool_desc {
  int32_t num_pages;    /* > 0 */
  int32_t page_size;    /* tokens per page: 16, 32, 64 or 128 */
  int32_t num_kv_heads; /* > 0 */
  int32_t head_dim;     /* 64 or 128 */
  int32_t location;     /* oomb_location */
  int32_t with_grad;    /* non-zero: allocate the fp32 gradient pool too */
  uint64_t alloc_seed;  /* 0: pages handed out ascending; otherwise in the order of
                           a Fisher-Yates shuffle driven by SplitMix64(alloc_seed) */
  int32_t device;       /* CUDA device ordinal (ignored for OOMB_LOC_HOST) */
} oomb_pool_desc;

/* ---------------------------------------------------------------- pools
 * Paged memory for the KV cache and its gradients ([pt] §2B, [it] §2B: pages
 * are non-contiguous, so appending needs no reallocation or copy).
 * The free list is a stack: pages freed are handed out again first (LIFO).
 * Pool buffers are zero-filled at creation. */
oomb_status oomb_pool_create(const oomb_pool_desc* desc, oomb_pool** out_pool);
oomb_status oomb_pool_destroy(oomb_pool* pool); /* NULL is accepted */
/* Pops the next free page id; OOMB_ERR_OUT_OF_PAGES when none is left. */
oomb_status oomb_pool_alloc_page(oomb_pool* pool, int32_t* out_page_id);
/* Returns a page to the free list; OOMB_ERR_BAD_PAGE if out of range or already free. */
oomb_status oomb_pool_free_page(oomb_pool* pool, int32_t page_id);
oomb_status oomb_pool_num_free(const oomb_pool* pool, int32_t* out_num_free);
/* Borrowed views of the pool's buffers (any output may be NULL; grad is NULL
 * without with_grad).  Valid until oomb_pool_destroy.  The summaries of a
 * pinned-host pool are in device memory (Top-K reads them on the GPU); its KV
 * and gradients are in pinned host memory. */
oomb_status oomb_pool_buffers(const oomb_pool* pool, void** kv, float** grad, float** summary);
oomb_status oomb_pool_get_desc(const oomb_pool* pool, oomb_pool_desc* out_desc);

/* ---------------------------------------------------------------- append
 * Writes one chunk's keys and values into pages of a device pool, computes each
 * written page's fp32 mean key per KV head (the page representative, [es] §2B)
 * and zero-fills the written pages' gradient blocks.
 *   d_page_ids  device int32[n_pages]: physical page of the chunk's i-th page
 *   d_k, d_v    device bf16 [n_pages*page_size][num_kv_heads][head_dim] */
oomb_status oomb_kv_append(oomb_pool* pool, const int32_t* d_page_ids, int32_t n_pages,
                           const void* d_k, const void* d_v, void* stream);

/* ---------------------------------------------------------------- attention
 * Row i of the chunk (query head h, KV head g = h / G) attends to every token
 * of the past pages listed for group g (unmasked) and to the chunk's own keys
 * at local positions <= i (causal):
 *   S_ij = scale q_i.k_j,  LSE_i = ln sum_j exp(S_ij),  O_i = sum_j exp(S_ij - LSE_i) v_j.
 * Dense attention lists every past page for every group; page-sparse lists
 * the pages oomb_page_topk kept. */
typedef struct oomb_attn_args {
  const void* q;      /* device bf16 [chunk_len][num_q_heads][head_dim]            */
  void* o;            /* device bf16, same layout: fwd output, bwd input           */
  float* lse;         /* device fp32 [num_q_heads][chunk_len]: fwd output, bwd input */
  const void* d_o;    /* device bf16, layout of q: bwd input (dL/dO)               */
  void* dq;           /* device bf16, layout of q: bwd output (overwritten)        */
  float* delta_ws;    /* device fp32 [num_q_heads][chunk_len]: bwd workspace       */
  int32_t chunk_len;
  int32_t num_q_heads;
  const int32_t* past_pages;  /* device int32 [num_kv_heads][max_past] physical ids  */
  const int32_t* past_counts; /* device int32 [num_kv_heads], each in [0, max_past]   */
  int32_t max_past;           /* row stride of past_pages; 0 for the first chunk     */
  const int32_t* cur_pages;   /* device int32 [chunk_len/page_size] physical ids      */
  float softmax_scale;        /* usually 1/sqrt(head_dim)                             */
  /* 0: one past list per group for the whole chunk (layouts above).
   * 1: one past list per 128-row query tile and group (a coarser form of
   *    mode 2 below, one list for two 64-token query pages):
   *    past_pages [n_qtiles][num_kv_heads][max_past] and
   *    past_counts [n_qtiles][num_kv_heads], n_qtiles = ceil(chunk_len / 128);
   *    rows of query tile t attend to list t (plus the chunk, causally).  The
   *    outputs of oomb_page_topk_batched with one problem per query tile have
   *    exactly this layout.
   * 2: one past list per QUERY PAGE (page_size consecutive rows of the chunk)
   *    and group ([pt] §2C), given per 128-row query tile as the union of the
   *    lists of its 128/page_size query pages: past_pages and past_counts as
   *    for 1 (the union, ascending logical page order), and past_masks
   *    [n_qtiles][num_kv_heads][max_past] with bit b of entry i set iff that
   *    page is in the list of the tile's query page b (rows 128 t + b page_size
   *    .. + page_size - 1).  A row attends to the entries whose bit for its
   *    query page is set (plus the chunk, causally).  oomb_qpage_lists builds
   *    these from oomb_page_topk_batched's per-query-page selections. */
  int32_t lists_per_qtile;
  /* Segmented attention: the past streamed through a bounded device window
   * ([pt] §2D: pages move between host and GPU while computation runs; a
   * dense chunk then takes its past in pieces).
   *   OOMB_SEG_WHOLE (0): the call covers the listed past pages and the chunk
   *     itself (causal); outputs as described above.
   *   OOMB_SEG_FIRST (1) / OOMB_SEG_NEXT (2): the call covers only the listed
   *     past pages (not the chunk).  Forward: writes (FIRST) or merges into
   *     (NEXT) the running normalised output o_acc and lse; o is not written.
   *     Backward: dK/dV of the listed pages are added to the pool as usual; dQ
   *     is written to (FIRST) or added into (NEXT) dq_acc; dq is not written.
   *   OOMB_SEG_LAST (3): the call covers the listed past pages (the list may be
   *     empty) and the chunk itself, merges into o_acc / lse and writes o and
   *     the final lse (forward), adds into dq_acc and writes dq (backward).
   * Segments of one chunk: every forward segment (FIRST, NEXT..., LAST), then
   * the backward segments in any order that starts with FIRST and ends with
   * LAST (the backward needs the final o and lse).  Per-query-tile lists
   * cannot be combined with segments. */
  int32_t segment;
  float* o_acc;   /* device fp32 [chunk_len][num_q_heads][head_dim]: running O  */
  float* dq_acc;  /* device fp32, layout of o_acc: running dQ (backward)         */
  const uint8_t* past_masks;  /* lists_per_qtile == 2 only (else ignored), see above */
  /* Optional forward workspace (device fp32, oomb_chunk_attn_fwd_workspace_size()
   * bytes, 16-byte aligned; NULL: none).  The forward runs one CTA per (128-row
   * query tile, query head) and one CTA per SM; when the number of such units is
   * not a multiple of the SM count, the units of the last, partial wave are split
   * along their key tiles over the free SMs, each part writes a normalised
   * partial O and its LSE here, and a second launch merges them (LSE = ln sum_k
   * e^LSE_k, O = sum_k e^(LSE_k - LSE) O_k) and, for a segmented call, merges
   * that with the running o_acc / lse as a whole unit would.  Without it the
   * last wave runs its few units alone.  The backward ignores it.  Calls sharing
   * a workspace must be ordered (one stream). */
  float* fwd_ws;
} oomb_attn_args;

enum { OOMB_SEG_WHOLE = 0, OOMB_SEG_FIRST = 1, OOMB_SEG_NEXT = 2, OOMB_SEG_LAST = 3 };

/* Forward with online softmax; writes o and lse (one launch, or two with a
 * split last wave, see fwd_ws). */
oomb_status oomb_chunk_attn_fwd(oomb_pool* pool, const oomb_attn_args* args, void* stream);
/* Bytes of the optional forward workspace for head_dim (64 or 128); 0 otherwise. */
size_t oomb_chunk_attn_fwd_workspace_size(int32_t head_dim);

/* Backward of sum(O * dO): writes dq and ADDS dK, dV into the pool's gradient
 * blocks of every page read (fp32 atomic adds, in place; [it] §2B).  Needs o
 * and lse from the forward of the same chunk, and delta_ws as workspace. */
oomb_status oomb_chunk_attn_bwd(oomb_pool* pool, const oomb_attn_args* args, void* stream);

/* The backward's three launches, for timing them separately; running
 * PREPROCESS, DKDV and DQ in this order equals oomb_chunk_attn_bwd. */
typedef enum oomb_bwd_step {
  OOMB_BWD_PREPROCESS = 0, /* delta_ws = rowsum(dO * O)                          */
  OOMB_BWD_DKDV = 1,       /* grad pool += dK, dV (needs delta_ws)                */
  OOMB_BWD_DQ = 2          /* dq (needs delta_ws)                                 */
} oomb_bwd_step;
oomb_status oomb_chunk_attn_bwd_step(oomb_pool* pool, const oomb_attn_args* args, int32_t step,
                                     void* stream);

/* ---------------------------------------------------------------- projection
 * Q/K/V projection of one chunk with a paged epilogue ([pt] §2D: the pages a
 * sparse chunk needs are known once its queries exist, so their transfer can
 * overlap the rest of its work — here the K/V projection; [es] §2B).
 *   Y = X W^T, X = d_x [chunk_len][hidden] bf16 (token-major), W = d_w
 *   [(num_q_heads + 2 num_kv_heads) head_dim][hidden] bf16 with rows: the Q
 *   heads, then the K heads, then the V heads; fp32 accumulation, outputs
 *   rounded to bf16 (tcgen05 GEMM, 128 x 256 tiles, TMA, 4 stages).
 *   part OOMB_PROJ_Q: writes d_q [chunk_len][num_q_heads][head_dim] (if not
 *     NULL) and, if d_qsum is not NULL, sets d_qsum [num_kv_heads][head_dim]
 *     fp32 to the sum of the rounded Q over the chunk's rows and each group's
 *     G heads (q_bar = qsum / (chunk_len G), the Top-K query side).
 *   part OOMB_PROJ_KV: writes token t's K and V into page d_page_ids[t /
 *     page_size] of the pool (as oomb_kv_append does), sets those pages' fp32
 *     mean keys and zero-fills their gradient blocks.
 *   part OOMB_PROJ_QKV: both in one launch.
 * Requires a device pool, hidden a multiple of 64, chunk_len a multiple of
 * page_size, 16-byte aligned X, W and Q.  Page ids out of the pool are
 * skipped and set bit 0 of the device status word. */
enum { OOMB_PROJ_Q = 0, OOMB_PROJ_KV = 1, OOMB_PROJ_QKV = 2 };
oomb_status oomb_qkv_project(oomb_pool* pool, const void* d_x, const void* d_w, int32_t chunk_len,
                             int32_t hidden, int32_t num_q_heads, int32_t part, void* d_q,
                             float* d_qsum, const int32_t* d_page_ids, void* stream);

/* ---------------------------------------------------------------- Top-K
 * Page-level selection for one chunk ([pt] §2C, [es] §2B, [it] §2D):
 *   q_bar_g   = fp32 mean of the chunk's rows over the G query heads of group g
 *   score_p,g = q_bar_g . (summary of page p, KV head g)          (fp32)
 * Candidates are logical pages [0, n_past - n_recent); the top_k highest
 * scores are kept (ties: lower logical id first), together with the n_recent
 * most recent pages [n_past - n_recent, n_past).  Output per group: the kept
 * logical ids in ascending order, their physical ids, and the count
 * min(top_k, n_past - n_recent) + min(n_recent, n_past).
 *   d_q              device bf16 [chunk_len][num_q_heads][head_dim]
 *   d_page_table     device int32 [n_past]: logical -> physical page id
 *   d_out_logical    device int32 [num_kv_heads][top_k + n_recent]
 *   d_out_physical   device int32 [num_kv_heads][top_k + n_recent] (may be NULL)
 *   d_out_count      device int32 [num_kv_heads]
 *   d_out_scores     device fp32 [num_kv_heads][n_past] (may be NULL)
 *   d_workspace      device memory of oomb_page_topk_workspace_size() bytes
 * The pool may be a device pool or a pinned-host pool (its summaries are on
 * the device).  Limits: n_past <= 65536; 1 <= top_k + n_recent <= 4096. */
size_t oomb_page_topk_workspace_size(int32_t chunk_len, int32_t num_q_heads, int32_t num_kv_heads,
                                     int32_t head_dim, int32_t n_past);
oomb_status oomb_page_topk(const oomb_pool* pool, const void* d_q, int32_t chunk_len,
                           int32_t num_q_heads, const int32_t* d_page_table, int32_t n_past,
                           int32_t top_k, int32_t n_recent, int32_t* d_out_logical,
                           int32_t* d_out_physical, int32_t* d_out_count, float* d_out_scores,
                           void* d_workspace, size_t workspace_bytes, void* stream);

/* Per-query-page lists for the attention ([pt] §2C: the key pages relevant to
 * each query page).  Input: one selection per query page of a chunk, as
 * oomb_page_topk_batched returns them with one problem per query page (rows
 * b page_size .. b page_size + page_size - 1): d_sel_logical and
 * d_sel_physical [n_qpages][num_kv_heads][max_sel] (ascending logical ids),
 * d_sel_count [n_qpages][num_kv_heads], n_qpages = chunk_len / page_size.
 * Output per 128-row query tile t and group g: the union of the selections
 * of the tile's query pages in ascending logical order, as physical ids
 * d_out_pages [n_qtiles][num_kv_heads][max_union], the membership bits
 * d_out_masks (uint8, same layout; bit b: in the list of the tile's query
 * page b) and d_out_count [n_qtiles][num_kv_heads] — the past_pages,
 * past_masks and past_counts of oomb_attn_args with lists_per_qtile = 2.
 * max_union must be at least min(128 / page_size, n_qpages) * max_sel.
 * One launch on `stream`; a count outside [0, max_sel] is clamped and sets
 * bit 2 of the pool's device status word. */
oomb_status oomb_qpage_lists(oomb_pool* pool, const int32_t* d_sel_logical,
                             const int32_t* d_sel_physical, const int32_t* d_sel_count,
                             int32_t chunk_len, int32_t max_sel, int32_t* d_out_pages,
                             uint8_t* d_out_masks, int32_t* d_out_count, int32_t max_union,
                             void* stream);

/* oomb_page_topk from per-group sums of Q instead of Q: the query mean is
 * left to the kernel that produces Q (oomb_qkv_project's d_qsum, written by
 * its GEMM epilogue), so the selection is one launch that reads only the
 * page summaries ([pt] §2D: the pages a chunk needs are known once its
 * queries exist).
 *   d_qsum           device fp32 [num_kv_heads][head_dim]: per group g the
 *                    sum of Q over the chunk's chunk_len rows and the G =
 *                    num_q_heads / num_kv_heads heads of g; q_bar_g =
 *                    d_qsum[g] / (chunk_len G)
 *   d_workspace      device memory of oomb_page_topk_qsum_workspace_size()
 *                    bytes, 16-byte aligned.  Its first num_kv_heads words
 *                    are counters that must be zero before the first call on
 *                    a workspace (e.g. cudaMemsetAsync once); every completed
 *                    call leaves them at zero, so later calls need no clear.
 *                    Calls sharing a workspace must be ordered (one stream).
 * Everything else (outputs, limits, tie rule, pool locations) as
 * oomb_page_topk.  Scores use the fp32 q_bar of the given sums, so where
 * those sums differ in rounding from oomb_page_topk's own query mean (a
 * different summation order) pages whose scores tie within that rounding
 * may be exchanged. */
size_t oomb_page_topk_qsum_workspace_size(int32_t num_kv_heads, int32_t n_past);
oomb_status oomb_page_topk_qsum(const oomb_pool* pool, const float* d_qsum, int32_t chunk_len,
                                int32_t num_q_heads, const int32_t* d_page_table, int32_t n_past,
                                int32_t top_k, int32_t n_recent, int32_t* d_out_logical,
                                int32_t* d_out_physical, int32_t* d_out_count,
                                float* d_out_scores, void* d_workspace, size_t workspace_bytes,
                                void* stream);

/* Allocation-free variant of oomb_page_topk (this one has no counterpart in
 * the paper; it exists for callers that cannot allocate device memory, e.g.
 * code running under a host framework that owns every device allocation, or a
 * latency-critical loop that must not call cudaMalloc, which can synchronise
 * the device).  Same arguments and results as oomb_page_topk minus the
 * workspace: the scratch is a static device array of
 * OOMB_TOPK_STATIC_SCRATCH_BYTES inside the library, held on every GPU that
 * loads it until the process exits.  Returns OOMB_ERR_UNSUPPORTED when
 * oomb_page_topk_workspace_size() of the call exceeds that size (e.g. with
 * Hkv = 4 and d = 128, n_past up to 24,512 pages fits).  It allocates nothing.
 * The first call on a device looks up the array's device address (with that
 * device current); make that first call before any stream capture.  All calls
 * share the one array: calls that overlap on the GPU (different streams) race
 * on it and must be ordered by the caller.  The caller clears nothing: each
 * call writes every scratch word it reads, and its first launch zeroes the
 * counters its second launch counts on.  The looked-up address is kept per device
 * ordinal for the life of the process, so resetting a device
 * (cudaDeviceReset, or tearing down and re-creating its primary context)
 * while this library is loaded is not supported for this entry point. */
#define OOMB_TOPK_STATIC_SCRATCH_BYTES (1u << 20)
oomb_status oomb_page_topk_static(const oomb_pool* pool, const void* d_q, int32_t chunk_len,
                                  int32_t num_q_heads, const int32_t* d_page_table,
                                  int32_t n_past, int32_t top_k, int32_t n_recent,
                                  int32_t* d_out_logical, int32_t* d_out_physical,
                                  int32_t* d_out_count, float* d_out_scores, void* stream);

/* Batched Top-K: n_problems independent selections in one set of launches
 * (four dependent kernels for the whole batch: query means, their per-problem
 * sums, scores, select).  Problem b takes the query rows
 * [d_row_start[b], d_row_start[b+1]) of d_q ([num_rows][num_q_heads][d]
 * bf16) and the candidates among logical pages [0, d_n_past[b]) of the one
 * page table d_page_table (length >= max_past); each problem is exactly one
 * oomb_page_topk call on those rows.  Uses: the selections of many chunks at
 * once, and one selection per query page of a chunk ([pt] §2C speaks of the
 * pages relevant to each query page).
 *   d_row_start [n_problems + 1], d_n_past [n_problems]: device int32; values
 *     outside [0, num_rows] / [0, max_past] are clamped and set bit 2 of the
 *     device status word.
 *   max_rows: the largest row count of a problem (host-known bound, picks the
 *     slice count of the query mean; 1 <= max_rows <= num_rows).
 *   Outputs [n_problems][Hkv][top_k + n_recent] (ids), [n_problems][Hkv]
 *     (counts), optional scores [n_problems][Hkv][max_past].
 *   Workspace: oomb_page_topk_batched_workspace_size(n_problems, Hkv, d,
 *     max_past) bytes, 16-byte aligned; n_problems <= 65535. */
size_t oomb_page_topk_batched_workspace_size(int32_t n_problems, int32_t num_kv_heads,
                                             int32_t head_dim, int32_t max_past);
oomb_status oomb_page_topk_batched(const oomb_pool* pool, const void* d_q, int32_t num_rows,
                                   int32_t num_q_heads, int32_t n_problems,
                                   const int32_t* d_row_start, int32_t max_rows,
                                   const int32_t* d_n_past, int32_t max_past,
                                   const int32_t* d_page_table, int32_t top_k, int32_t n_recent,
                                   int32_t* d_out_logical, int32_t* d_out_physical,
                                   int32_t* d_out_count, float* d_out_scores, void* d_workspace,
                                   size_t workspace_bytes, void* stream);

/* Recent-only page lists ([it] §2D: layers that are sparse by construction
 * keep the most recent pages): for every KV-head group, the last `window` of
 * the first n_past logical pages of d_page_table, ascending, as physical ids
 * — the past-page arguments of oomb_chunk_attn_fwd / _bwd for attention over
 * a sliding window of pages plus the chunk itself (causal).
 *   d_page_table [>= n_past] device int32, logical -> physical page of `pool`
 *   d_out_pages  [num_kv_heads][window] device int32 (row stride = window;
 *                entries past the count are 0)
 *   d_out_count  [num_kv_heads] device int32: min(window, n_past)
 * window >= 1.  Ids outside the pool are written as 0 and set bit 0 of the
 * device status word. */
oomb_status oomb_local_pages(const oomb_pool* pool, const int32_t* d_page_table, int32_t n_past,
                             int32_t window, int32_t* d_out_pages, int32_t* d_out_count,
                             void* stream);

/* ---------------------------------------------------------------- offload
 * A block is the K and V of one page and one KV head: block id = page *
 * num_kv_heads + head, contiguous in both pools ([pt] §2D, [it] §2C: KV and
 * its gradients move between pinned host memory and the GPU on dedicated
 * streams, overlapped with compute).
 *
 * oomb_page_prefetch: copies KV blocks from src_pool to dst_pool, one
 * cudaMemcpyAsync per run of blocks consecutive in both pools, on `stream`,
 * then records `done_event` (a cudaEvent_t given as void*, may be NULL).
 * Pinned host -> device is the prefetch of selected pages; device -> pinned
 * host stores freshly appended pages, and then also copies each block's page
 * representative into the host pool's (device-resident) summaries.  The pools
 * must share page_size, num_kv_heads and head_dim; OOMB_LOC_HOST pools are
 * not accepted; block ids are checked on the host (OOMB_ERR_BAD_PAGE). */
oomb_status oomb_page_prefetch(const oomb_pool* src_pool, oomb_pool* dst_pool,
                               const int32_t* h_src_blocks, const int32_t* h_dst_blocks,
                               int32_t n_blocks, void* stream, void* done_event);

/* oomb_grad_writeback: adds the device pool's gradient blocks h_src_blocks
 * into the pinned host pool's gradient blocks h_dst_blocks (same order), then
 * zero-fills the device blocks.  On `stream` the blocks are copied device ->
 * host into one of two pinned staging slots owned by the device pool (one
 * cudaMemcpyAsync per run of consecutive source blocks) and the device blocks
 * are zero-filled; a library worker thread then adds the slot into the host
 * pool with up to 16 CPU threads, in submission order, without holding up the
 * stream.  The call itself blocks only while both slots are still being
 * added (OOMB_ERR_TIMEOUT after 120 s).  Destination blocks must be distinct
 * within one call: a repeated destination returns OOMB_ERR_INVALID_ARG (an id
 * outside its pool OOMB_ERR_BAD_PAGE) before any CUDA call.  The host
 * gradients include a call's blocks once oomb_grad_writeback_sync() has
 * returned OOMB_OK.
 * Failures: if a device -> host copy cannot be queued, the call returns
 * OOMB_ERR_CUDA, adds nothing, and leaves every device block as it was (the
 * zero-fills are queued only after all copies were); the staging slot is
 * reused only once copies already queued into it have finished.  If a copy
 * fails on the device, the worker skips that call's additions and the next
 * oomb_grad_writeback_sync() returns OOMB_ERR_CUDA.  If a zero-fill cannot be
 * queued, the additions still happen but some device blocks may keep their
 * values (OOMB_ERR_CUDA). */
oomb_status oomb_grad_writeback(oomb_pool* device_pool, oomb_pool* host_pool,
                                const int32_t* h_src_blocks, const int32_t* h_dst_blocks,
                                int32_t n_blocks, void* stream);
/* Waits until every gradient addition queued by oomb_grad_writeback for this
 * device pool has been applied to the host pool (OOMB_ERR_TIMEOUT after
 * timeout_us microseconds).  OOMB_ERR_CUDA: the copy of some call since the
 * previous sync failed and that call's blocks were not added (the report is
 * cleared by this call). */
oomb_status oomb_grad_writeback_sync(oomb_pool* device_pool, int64_t timeout_us);

/* ---------------------------------------------------------------- block moves with device lists
 * The same moves as above, but driven by block lists that live in DEVICE
 * memory (int32, caller-owned) and executed by one kernel launch each, so
 * that lists computed on the GPU (a Top-K selection) never travel to the host
 * ([pt] §2D: for sparse attention the page ids are known ahead of the
 * compute, which lets the transfer overlap it).  Pinned-host pools are read
 * and written in place over the host link (mapped memory); between two
 * device pools the moves are HBM gathers and scatter-adds.
 * Common rules: entry i moves src block d_src_blocks[i] to dst block
 * d_dst_blocks[i]; an entry with a negative id is padding and is skipped; an
 * id beyond its pool is skipped and sets bit 0 of dst_pool's device status
 * word; the pools must share page_size, num_kv_heads and head_dim and may not
 * be OOMB_LOC_HOST; n_blocks == 0 is a no-op; all work is on `stream`.
 *
 * oomb_block_copy: dst.kv[dst_i] = src.kv[src_i] and
 * dst.summary[dst_i] = src.summary[src_i] (the page representative travels
 * with its block).  Destination ids must be distinct within a call. */
oomb_status oomb_block_copy(const oomb_pool* src_pool, oomb_pool* dst_pool,
                            const int32_t* d_src_blocks, const int32_t* d_dst_blocks,
                            int32_t n_blocks, void* stream);
/* oomb_grad_block_add: dst.grad[dst_i] += src.grad[src_i] in fp32, then, if
 * zero_src != 0, src.grad[src_i] = 0.  src_pool must be a device pool; both
 * pools need gradients.  A device dst_pool is added with vector atomics (a
 * destination may repeat); a pinned-host dst_pool gets a plain
 * read-modify-write over the host link, so its destinations must be distinct
 * within a call.  With zero_src, source ids must be distinct too. */
oomb_status oomb_grad_block_add(oomb_pool* src_pool, oomb_pool* dst_pool,
                                const int32_t* d_src_blocks, const int32_t* d_dst_blocks,
                                int32_t n_blocks, int32_t zero_src, void* stream);
/* oomb_prefetch_lists: turns a Top-K selection into the lists that move the
 * selected blocks of src_pool into staging slots of dst_pool.
 *   d_sel_logical [Hkv][max_sel], d_sel_count [Hkv]: as written by
 *     oomb_page_topk (logical page ids, ascending, count per group);
 *   d_page_table [table_len]: logical -> physical page of src_pool;
 *   d_slot_pages [max_sel]: staging pages of dst_pool; slot i holds the i-th
 *     selected page of every group (one block per group).
 * Writes, for entry e = i * Hkv + g (slot-major, max_sel * Hkv entries):
 *   d_src_blocks[e] = table[sel[g][i]] * Hkv + g, d_dst_blocks[e] =
 *   slot_pages[i] * Hkv + g when i < count[g], else -1 (padding);
 *   d_past_pages[g][i] = slot_pages[i] (0 past the count): the past page list
 *   of the staging pool for oomb_chunk_attn_fwd / _bwd, with d_sel_count as
 *   its counts.
 * Ids out of range set bit 0 (a count out of [0, max_sel] bit 2) of
 * dst_pool's device status word and give padding entries. */
oomb_status oomb_prefetch_lists(const oomb_pool* src_pool, oomb_pool* dst_pool,
                                const int32_t* d_sel_logical, const int32_t* d_sel_count,
                                int32_t max_sel, const int32_t* d_page_table, int32_t table_len,
                                const int32_t* d_slot_pages, int32_t* d_src_blocks,
                                int32_t* d_dst_blocks, int32_t* d_past_pages, void* stream);

/* ---------------------------------------------------------------- status
 * Waits for a cudaEvent_t (given as void*) by polling, for at most timeout_us
 * microseconds; OOMB_ERR_TIMEOUT instead of blocking forever. */
oomb_status oomb_wait(void* event, int64_t timeout_us);
/* Synchronises with the pool's device, reads and clears its device status
 * word: OOMB_OK, or OOMB_ERR_DEVICE_CHECK if a kernel recorded a failure.
 * *out_word (may be NULL) receives the raw bits:
 *   bit 0 invalid page id, bit 1 wait limit reached, bit 2 bad count. */
oomb_status oomb_get_device_status(oomb_pool* pool, uint32_t* out_word);
const char* oomb_status_string(oomb_status status);
/* Self-test of the kernels' bounded waits (no counterpart in the paper): one
 * thread waits on an mbarrier that nothing arrives at; after the wait limit
 * (about a second) it gives up and sets bit 1 of the pool's device status
 * word, exactly as a kernel whose arrival was lost would.  Device or
 * pinned-host pools only. */
oomb_status oomb_selftest_wait_limit(oomb_pool* pool, void* stream);
/* Self-test of the gradient write-back worker (no counterpart in the paper;
 * host only, makes no CUDA call): a staging slot of n_blocks blocks of
 * block_floats floats, all 1.0, goes through the worker into host_grad
 * blocks 0 .. n_blocks-1, its copy reported as completed (fail_copy == 0) or
 * as failed (fail_copy != 0).  Returns what oomb_grad_writeback_sync would:
 * OOMB_OK with host_grad incremented by 1.0, or OOMB_ERR_CUDA with host_grad
 * untouched. */
oomb_status oomb_selftest_writeback_copy(float* host_grad, int32_t n_blocks,
                                         int32_t block_floats, int32_t fail_copy);
/* Library version as major*10000 + minor*100 + patch. */
int32_t oomb_version(void);

#ifdef __cplusplus
}
#endif
#endif /* OOMB_H */
