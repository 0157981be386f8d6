// fa_api.cu -- host side of the C ABI declared in include/fadecode.h:
// planner, argument validation, tensor-map construction, launches, and the
// standalone merge-states kernel.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <new>
#include <vector>

#include "../../include/fadecode.h"
#include "fa_kernel.cuh"
#include "fa_registry.h"

using fa::KernelEntry;

// ------------------------------------------------------------ registry
namespace {

constexpr int kMaxEntries = 64;
KernelEntry g_entries[kMaxEntries];
int g_num_entries = 0;
std::once_flag g_registry_once;

void build_registry() {
  int n = 0;
  n += fa::register_d64(g_entries + n, kMaxEntries - n);
  n += fa::register_d128(g_entries + n, kMaxEntries - n);
  n += fa::register_d256(g_entries + n, kMaxEntries - n);
  n += fa::register_tc(g_entries + n, kMaxEntries - n);
  g_num_entries = n;
}

// A paged tile is filled one page per box (pages shorter than the tile) or
// from one page (pages at least as long): the page size and the tile length
// must divide one another, or a tile would get too few copies, or a box
// would run past its page into an unrelated one.
bool tile_fits_pages(int tile_tokens, int page_size) {
  if (page_size <= 0) return true;  // contiguous
  return page_size < tile_tokens ? tile_tokens % page_size == 0 : page_size % tile_tokens == 0;
}

// The first variant (registry order) for the shape whose tiles fit the pages.
const KernelEntry* find_entry(int head_dim, int group, int kv_kind, int path, int page_size) {
  std::call_once(g_registry_once, build_registry);
  for (int i = 0; i < g_num_entries; ++i) {
    const KernelEntry& e = g_entries[i];
    if (e.head_dim != head_dim || e.kv_kind != kv_kind || e.path != path || e.heads_per_tile != 1)
      continue;
    if (!tile_fits_pages(e.tile_tokens, page_size)) continue;
    if (e.group != 0 ? e.group == group : group <= e.max_group) return &e;
  }
  return nullptr;
}

// The tensor-core variant whose tiles hold `ht` adjacent kv heads.
const KernelEntry* find_head_entry(int head_dim, int kv_kind, int ht) {
  std::call_once(g_registry_once, build_registry);
  for (int i = 0; i < g_num_entries; ++i) {
    const KernelEntry& e = g_entries[i];
    if (e.head_dim == head_dim && e.kv_kind == kv_kind && e.path == fa::kPathMma &&
        e.heads_per_tile == ht)
      return &e;
  }
  return nullptr;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Text of the last CUDA failure seen by a call on this thread.
thread_local char g_last_error[256] = "";

fa_status cuda_failure(const char* where, cudaError_t e) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(e),
           static_cast<int>(e));
  cudaGetLastError();  // clear a non-sticky error so the caller can continue
  return FA_ERR_CUDA;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

// ------------------------------------------------------------- the plan
struct fa_plan {
  fa_decode_desc desc;
  const KernelEntry* kernel;
  int32_t group;           // rows of a segment (group * q_len * heads_per_tile)
  int32_t heads_per_tile;  // kv heads of a segment (> 1: head-team variant)
  int32_t num_ctas;
  int32_t box_t;
  int32_t swz;
  int32_t page_shift;
  int32_t seg_parts;  // > 0: every segment cut into this many runs, one block each
  int32_t piece_cost; // equal runs: tiles charged per segment ahead of its own
  int64_t total_tiles;
  int64_t max_partials;
  size_t ws_bytes;
  size_t off_records, off_part_o, off_part_lse;
  size_t smem;
};

namespace {

int ilog2_exact(int x) {
  int s = 0;
  while ((1 << s) < x) ++s;
  return (1 << s) == x ? s : -1;
}

int64_t host_num_tiles(int32_t L, int32_t window, int32_t T) {
  if (L <= 0) return 0;
  const int32_t lo = (window > 0 && L > window) ? L - window : 0;
  return (L + T - 1) / T - lo / T;
}

fa_status validate_desc(const fa_decode_desc* d) {
  if (d->batch < 1 || d->qo_heads < 1 || d->kv_heads < 1 || d->head_dim < 1)
    return FA_ERR_INVALID_ARG;
  if (d->qo_heads % d->kv_heads != 0) return FA_ERR_INVALID_ARG;
  if (d->kv_dtype != FA_KV_BF16 && d->kv_dtype != FA_KV_FP8_E4M3 && d->kv_dtype != FA_KV_INT4)
    return FA_ERR_INVALID_ARG;
  if (d->kv_dtype == FA_KV_INT4 && d->head_dim % 2 != 0) return FA_ERR_INVALID_ARG;
  if (d->paged != 0 && d->paged != 1) return FA_ERR_INVALID_ARG;
  if (d->paged && (d->page_size < 1 || d->page_size > 256 || ilog2_exact(d->page_size) < 0))
    return FA_ERR_INVALID_ARG;
  if (!isfinite(d->sm_scale)) return FA_ERR_INVALID_ARG;
  if (d->path < FA_PATH_AUTO || d->path > FA_PATH_TC) return FA_ERR_INVALID_ARG;
  if (d->num_ctas < 0) return FA_ERR_INVALID_ARG;
  if (d->q_len < 0 || d->q_len > 64) return FA_ERR_INVALID_ARG;
  if (!(d->logit_cap >= 0.f) || !isfinite(d->logit_cap)) return FA_ERR_INVALID_ARG;
  if (d->unified_max != 0 && d->unified_max != 1) return FA_ERR_INVALID_ARG;
  if (d->unified_max && !isfinite(d->softmax_phi)) return FA_ERR_INVALID_ARG;
  if (d->piece_cost > 4096) return FA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(d->batch) * d->kv_heads > (1 << 30)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

int32_t q_len_of(const fa_decode_desc* d) { return d->q_len > 1 ? d->q_len : 1; }

// Bytes of one token's K (or V) row of one kv head.
int64_t row_bytes_of(const fa_decode_desc* d) {
  const int64_t D = d->head_dim;
  return d->kv_dtype == FA_KV_BF16 ? 2 * D : (d->kv_dtype == FA_KV_FP8_E4M3 ? D : D / 2);
}

// Keys that some query token of a request sees: the last token's window and
// the q_len - 1 keys before it (<= 0: all keys).
int32_t union_window(const fa_decode_desc* d) {
  return d->window > 0 ? d->window + q_len_of(d) - 1 : d->window;
}

// ------------------------------------------------------------ measured choice
// The dataflow-choice table ("FlashDecoding++" explainer, section
// "Hardware-aware heuristic dataflow"): rows measured on the GPU, first match
// wins.  Starts as the built-in table; fa_set_tuning replaces it.
#define FA_TUNING_ROW(d, dt, r0, r1, b0, b1, path, pieces) {d, dt, r0, r1, b0, b1, path, pieces},
const fa_tuning_entry kBuiltinTuning[] = {
#include "fa_tuning_b200.inc"
    {0, 0, 0, 0, 0, 0, 0, 0}};  // end mark
#undef FA_TUNING_ROW

std::vector<fa_tuning_entry> builtin_tuning() {
  std::vector<fa_tuning_entry> t;
  for (const fa_tuning_entry& e : kBuiltinTuning)
    if (e.head_dim != 0) t.push_back(e);
  return t;
}

std::vector<fa_tuning_entry>& tuning_table() {
  static std::vector<fa_tuning_entry> t = builtin_tuning();
  return t;
}

bool valid_tuning_row(const fa_tuning_entry& e) {
  return e.head_dim > 0 &&
         (e.kv_dtype == FA_KV_BF16 || e.kv_dtype == FA_KV_FP8_E4M3 || e.kv_dtype == FA_KV_INT4) &&
         e.rows_min >= 1 && e.rows_min <= e.rows_max && e.bytes_min >= 0 &&
         e.bytes_min <= e.bytes_max &&
         (e.path == FA_PATH_SIMT || e.path == FA_PATH_MMA || e.path == FA_PATH_TC) &&
         e.max_pieces >= 0 && e.max_pieces <= 1024;
}

// Visible K/V bytes of a decode: the keys some query token of each request
// sees, times kv heads, K and V, and the row size.
int64_t visible_kv_bytes(const fa_decode_desc* d, const int32_t* indptr) {
  const int32_t wu = union_window(d);
  int64_t toks = 0;
  for (int b = 0; b < d->batch; ++b) {
    const int64_t L = indptr[b + 1] - indptr[b];
    toks += (wu > 0 && L > wu) ? wu : L;
  }
  return toks * d->kv_heads * 2 * row_bytes_of(d);
}

}  // namespace

extern "C" fa_status fa_set_tuning(const fa_tuning_entry* entries, int32_t n) {
  if (n < 0 || n > 4096 || (entries == nullptr && n > 0)) return FA_ERR_INVALID_ARG;
  if (entries == nullptr) {
    tuning_table() = builtin_tuning();
    return FA_OK;
  }
  for (int32_t i = 0; i < n; ++i)
    if (!valid_tuning_row(entries[i])) return FA_ERR_INVALID_ARG;
  tuning_table().assign(entries, entries + n);
  return FA_OK;
}

extern "C" fa_status fa_get_tuning(fa_tuning_entry* out, int32_t cap, int32_t* n) {
  if (n == nullptr || cap < 0 || (out == nullptr && cap > 0)) return FA_ERR_INVALID_ARG;
  const std::vector<fa_tuning_entry>& t = tuning_table();
  *n = static_cast<int32_t>(t.size());
  for (int32_t i = 0; i < cap && i < *n; ++i) out[i] = t[static_cast<size_t>(i)];
  return FA_OK;
}

extern "C" fa_status fa_decode_plan(const fa_decode_desc* desc, const int32_t* kv_indptr_host,
                                    int32_t num_sms, fa_plan** plan, size_t* workspace_bytes) {
  if (desc == nullptr || kv_indptr_host == nullptr || plan == nullptr) return FA_ERR_INVALID_ARG;
  *plan = nullptr;
  fa_status st = validate_desc(desc);
  if (st != FA_OK) return st;
  if (kv_indptr_host[0] != 0) return FA_ERR_INVALID_ARG;
  for (int b = 0; b < desc->batch; ++b)
    if (kv_indptr_host[b + 1] < kv_indptr_host[b]) return FA_ERR_INVALID_ARG;
  if (num_sms < 0) return FA_ERR_INVALID_ARG;
  if (num_sms == 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_failure("fa_decode_plan: SM count", e);
  }
  // rows of a segment: the group's query heads for every query token
  const int group = desc->qo_heads / desc->kv_heads * q_len_of(desc);
  const int kind = desc->kv_dtype;  // registry kinds follow fa_kv_dtype
  const int pages = desc->paged ? desc->page_size : 0;

  // Dataflow choice.  Asked for: that dataflow.  Otherwise the first row of
  // the measured table that covers the shape (when the grid is not forced),
  // else the fixed rule: the tensor-core (MMA) path whenever a kernel exists
  // for the shape, the SIMT path otherwise.
  const KernelEntry* k = nullptr;
  int64_t max_pieces = 64;  // average blocks per segment, at most
  bool table_cap = false;   // max_pieces came from the measured table
  // the tcgen05 dataflow: bf16 K/V, head_dim 128, 9 to 32 rows, copies of
  // 8 tokens (pages of at least 8), the plain running max
  auto tc_entry = [&]() -> const KernelEntry* {
    // 9-32 rows by default; fewer (padded to 16) only when asked for
    if (desc->unified_max || (group <= 8 && desc->path != FA_PATH_TC) || (pages != 0 && pages < 8))
      return nullptr;
    const KernelEntry* e = find_entry(desc->head_dim, group, kind, fa::kPathTc, pages);
    // its rings leave room for the schedule arrays of a few hundred requests
    if (e != nullptr && e->smem_bytes(desc->batch, group) > 232448) return nullptr;
    return e;
  };
  auto path_entry = [&](int path) -> const KernelEntry* {
    return path == FA_PATH_SIMT ? find_entry(desc->head_dim, group, kind, fa::kPathSimt, pages)
           : path == FA_PATH_TC ? tc_entry()
                                : find_entry(desc->head_dim, group, kind, fa::kPathMma, pages);
  };
  if (desc->path != FA_PATH_AUTO) {
    k = path_entry(desc->path);
  } else {
    if (desc->num_ctas == 0) {
      const int64_t bytes = visible_kv_bytes(desc, kv_indptr_host);
      for (const fa_tuning_entry& e : tuning_table()) {
        if (e.head_dim != desc->head_dim || e.kv_dtype != desc->kv_dtype || group < e.rows_min ||
            group > e.rows_max || bytes < e.bytes_min || bytes > e.bytes_max)
          continue;
        k = path_entry(e.path);
        if (k == nullptr) continue;
        if (e.max_pieces > 0) {
          max_pieces = e.max_pieces;
          table_cap = true;
        }
        break;
      }
    }
    // fixed rule: the tcgen05 dataflow where it applies, then the
    // warp-level tensor-core one, then CUDA cores
    if (k == nullptr) k = tc_entry();
    if (k == nullptr) k = find_entry(desc->head_dim, group, kind, fa::kPathMma, pages);
    if (k == nullptr) k = find_entry(desc->head_dim, group, kind, fa::kPathSimt, pages);
  }
  if (k == nullptr) return FA_ERR_UNSUPPORTED;

  // INT4 on the tensor-core dataflow: a tile of 256 / row-bytes adjacent kv
  // heads per token, one row team per head.  A one-head int4 tile of 64
  // tokens is 4 KB, so the per-tile work around the math (waits, releases,
  // the softmax bookkeeping) outweighed its bytes: measured 2x faster on the
  // batch-64 paged shape, 7% on the long-context one.  (The same tiles for
  // fp8 and bf16 with 128-byte rows measured slower or equal: those passes
  // stream at full rate and lose only a fixed start-up and merge time.)
  // One query token, at most 8 rows per head.
  int32_t ht = 1;
  {
    const int64_t rb = row_bytes_of(desc);
    if (desc->kv_dtype == FA_KV_INT4 && k->path == fa::kPathMma && k->heads_per_tile == 1 &&
        q_len_of(desc) == 1 && group <= 8 &&
        rb < 256 && 256 % rb == 0 && desc->kv_heads % (256 / rb) == 0) {
      const KernelEntry* kh = find_head_entry(desc->head_dim, kind, static_cast<int>(256 / rb));
      if (kh != nullptr && tile_fits_pages(kh->tile_tokens, pages)) {
        k = kh;
        ht = static_cast<int32_t>(256 / rb);
      }
    }
  }
  if (!tile_fits_pages(k->tile_tokens, pages)) return FA_ERR_UNSUPPORTED;
  const int64_t seg_heads = desc->kv_heads / ht;  // segments per request
  const int seg_rows = group * ht;                // rows of a segment

  const int T = k->tile_tokens;
  int64_t tiles = 0;
  int64_t seg_tiles = -1;  // tiles of every segment when all are equal, else -1
  int64_t max_seg_bytes = 0;  // visible K/V bytes of the largest segment
  for (int b = 0; b < desc->batch; ++b) {
    const int32_t L = kv_indptr_host[b + 1] - kv_indptr_host[b];
    const int64_t n = host_num_tiles(L, union_window(desc), T);
    tiles += n;
    seg_tiles = b == 0 ? n : (seg_tiles == n ? n : -1);
    const int32_t wu = union_window(desc);
    const int64_t vis = (wu > 0 && L > wu) ? wu : L;
    const int64_t sb = vis * 2 * row_bytes_of(desc) * ht;
    if (sb > max_seg_bytes) max_seg_bytes = sb;
  }
  tiles *= seg_heads;

  int64_t P;
  int32_t seg_parts = 0;
  if (desc->num_ctas > 0) {
    P = desc->num_ctas;
  } else {
    // One block per SM (each holds a ~170 KB tile ring).  A problem with
    // fewer tiles than SMs gets one tile per block (the fixed cost of a
    // block is small next to a KV tile's load latency, and the tiles load in
    // parallel); a segment is cut into at most max_pieces runs on average,
    // so that merging its partial states stays short (64 unless the
    // measured table says otherwise), except where the K/V give every SM at
    // least 256 KB: then the streaming outweighs the merge.  Measured on B200
    // (one segment, device time per pass, 32 / 64 / 148 blocks): 8.4 MB
    // 21.5 / 19.5 / 21.5 us, 16.8 MB 23.5 / 19.5 / 21.5 us, 67 MB
    // 44.1 / 31.7 / 29.7 us; passes of 4 or more segments reach all SMs
    // either way.
    int64_t want = tiles;
    const int64_t seg_cap = max_pieces * desc->batch * desc->kv_heads;  // per kv head
    const bool wide = !table_cap && visible_kv_bytes(desc, kv_indptr_host) >=
                                        static_cast<int64_t>(num_sms) * (256 << 10);
    if (want > seg_cap && !wide) want = seg_cap;
    P = want < num_sms ? want : num_sms;
    if (P < 1) P = 1;
    // Segments of equal length and rows of at most 128 bytes: cut every
    // segment into the same number of runs, one block each, so no run
    // crosses a segment boundary, as long as that keeps 85% of the SMs busy.
    // The blocks that read the kv heads of the same tokens then advance in
    // step, so a DRAM row holding one token's heads is read while it is
    // open, instead of once per head at different times.  Measured on fp8
    // head_dim 128 (8 segments): 10% faster than equal runs over all tiles;
    // with 256-byte rows it made no difference.
    const int64_t segs = static_cast<int64_t>(desc->batch) * seg_heads;
    if (seg_tiles > 0 && k->row_bytes <= 128 && P == num_sms && segs <= num_sms) {
      int64_t parts = num_sms / segs;
      if (parts > seg_tiles) parts = seg_tiles;  // every run gets a tile
      if (parts * segs * 100 >= 85LL * num_sms) {
        P = parts * segs;
        seg_parts = static_cast<int32_t>(parts);
      }
    }
    // One whole segment per block: no segment is ever split, whatever the
    // lengths on the device, so the merge launch is not needed.  Taken when
    // the measured table caps the blocks per segment at one, and by default
    // when every segment is small enough that splitting it cannot pay for
    // the merge launch: a block streams a 128 KB segment in about the time
    // the second launch costs (measured on B200: 2 segments of 128 KB,
    // 15.4 us split over 8 blocks, 12.3 us whole; one 512 KB segment, 15.4
    // us split, 22.7 us whole), and as long as the segments fit one wave.
    const bool small_segs = max_seg_bytes <= (128 << 10) && segs <= num_sms;
    if ((max_pieces == 1 || (small_segs && !table_cap)) && P > 1 && segs <= (1 << 20)) {
      P = segs;
      seg_parts = 1;
    }
  }
  if (P > (1 << 20)) return FA_ERR_UNSUPPORTED;

  fa_plan* p = new (std::nothrow) fa_plan();
  if (p == nullptr) return FA_ERR_INVALID_ARG;
  p->desc = *desc;
  p->kernel = k;
  p->group = seg_rows;
  p->heads_per_tile = ht;
  p->num_ctas = static_cast<int32_t>(P);
  p->seg_parts = seg_parts;
  // The fixed cost of a segment piece in tile units.  Per-block timers on
  // a B200 put it near 2 us against 0.76 us of block time a tile with 8 rows,
  // and 5.6 against 0.8 with 16 rows (parking and merging two row blocks'
  // states); a sweep of the charge then measured the best values: 2 tiles
  // up to 8 rows (batch-64 paged, 1%; MHA 32k, 2%), 8 with 16 or 32 rows
  // (batch-16 paged with 4 query tokens, 22%; GQA-16, 8%), 4 for int4
  // head tiles (5%), 3 of the 128-token tiles of the tcgen05 dataflow (a
  // device timeline put a piece boundary near 3.5 us against 1.25 us a
  // tile; against 2 tiles, 32 rows 392.2 -> 390.0 us, GQA-16 60.3 -> 59.7
  // us back to back).  Only equal runs of several tiles per block are cut
  // by cost.
  p->piece_cost = 0;
  if (seg_parts == 0 && P > 1 && tiles > P && desc->piece_cost >= 0)
    p->piece_cost = desc->piece_cost > 0 ? desc->piece_cost
                    : k->path == fa::kPathTc ? 3
                    : (ht > 1 ? 4 : seg_rows <= 8 ? 2 : 8);
  p->total_tiles = tiles;
  const int segs = desc->batch * static_cast<int>(seg_heads);
  p->max_partials = P + segs;
  p->page_shift = desc->paged ? ilog2_exact(desc->page_size) : 0;
  p->box_t = desc->paged ? (desc->page_size < T ? desc->page_size : T) : T;
  // A tile is filled box by box (one box per page when pages are shorter
  // than a tile) and a bulk tensor copy must land on a 128-byte boundary of
  // shared memory: rows narrower than 128 bytes (int4 at head_dim 128) need
  // pages of at least 128 / row-bytes tokens.
  if ((static_cast<int64_t>(p->box_t) * k->row_bytes * ht) % 128 != 0) {
    delete p;
    return FA_ERR_UNSUPPORTED;
  }
  // 128B swizzle needs every copy to start on a 1024-byte boundary of the
  // tile: whole 8-line groups of 128-byte lines per copy.
  {
    const int lines_per_copy =
        k->token_major ? p->box_t * (k->row_bytes / k->plane_bytes) * ht : p->box_t;
    p->swz = (k->plane_bytes == 128 && lines_per_copy % 8 == 0) ? 1 : 0;
  }
  size_t off = 256;  // header: device-check word, timeout record
  p->off_records = off;
  off = align_up(off + sizeof(int32_t) * 4 * static_cast<size_t>(P), 256);
  p->off_part_o = off;
  off = align_up(off + sizeof(float) * static_cast<size_t>(p->max_partials) * seg_rows * desc->head_dim,
                 256);
  p->off_part_lse = off;
  off = align_up(off + sizeof(float) * static_cast<size_t>(p->max_partials) * seg_rows, 256);
  p->ws_bytes = off;
  p->smem = k->smem_bytes(desc->batch, seg_rows);
  if (p->smem > 232448) {
    delete p;
    return FA_ERR_UNSUPPORTED;  // batch too large for the per-block schedule arrays
  }
  *plan = p;
  if (workspace_bytes != nullptr) *workspace_bytes = p->ws_bytes;
  return FA_OK;
}

extern "C" fa_status fa_plan_get_info(const fa_plan* plan, fa_plan_info_t* info) {
  if (plan == nullptr || info == nullptr) return FA_ERR_INVALID_ARG;
  info->path = plan->kernel->path == fa::kPathMma ? FA_PATH_MMA
               : plan->kernel->path == fa::kPathTc ? FA_PATH_TC
                                                  : FA_PATH_SIMT;
  info->num_ctas = plan->num_ctas;
  info->tile_tokens = plan->kernel->tile_tokens;
  info->stages = plan->kernel->stages;
  info->v_stages = plan->kernel->v_stages;
  info->total_tiles = static_cast<int32_t>(plan->total_tiles > INT32_MAX ? INT32_MAX : plan->total_tiles);
  info->max_partials = static_cast<int32_t>(plan->max_partials);
  info->workspace_bytes = plan->ws_bytes;
  info->smem_bytes = plan->smem;
  info->heads_per_tile = plan->heads_per_tile;
  info->piece_cost = plan->piece_cost;
  info->launches = (plan->num_ctas > 1 && plan->seg_parts != 1) ? 2 : 1;
  return FA_OK;
}

extern "C" void fa_plan_destroy(fa_plan* plan) { delete plan; }

namespace fa {
// Bytes at the start of a plan's workspace that must be zero before a run
// (the device-check header); the boundary records and partial states after
// it are always written by a pass before that pass reads them.
size_t plan_zero_prefix_bytes(const fa_plan* plan) { return plan->off_records; }
// Sets the text returned by fa_last_error on this thread.
void set_last_error(const char* text) { snprintf(g_last_error, sizeof(g_last_error), "%s", text); }
}  // namespace fa

namespace {

fa_status make_kv_map(const fa_plan* p, const void* base, int64_t kv_rows, CUtensorMap* map) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
    return FA_ERR_CUDA;
  }
  const fa_decode_desc& d = p->desc;
  const KernelEntry* k = p->kernel;
  const int es = d.kv_dtype == FA_KV_BF16 ? 2 : 1;  // int4: bytes of two codes
  const cuuint64_t row = static_cast<cuuint64_t>(row_bytes_of(&d));
  const cuuint64_t cb = static_cast<cuuint64_t>(k->plane_bytes);
  const cuuint64_t np = row / cb;
  const CUtensorMapDataType dt = es == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
  const CUtensorMapSwizzle sw = p->swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  const cuuint32_t inner = static_cast<cuuint32_t>(cb / es);
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  // L2 fills no wider than a token row: a 256-byte fill of a 128-byte row
  // would pull in the next kv head's row, which another block reads much
  // later (measured 1.48x DRAM traffic on 128-byte fp8 rows).
  const cuuint64_t span = row * static_cast<cuuint64_t>(p->heads_per_tile);  // contiguous bytes a token
  const CUtensorMapL2promotion promo = span >= 256   ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B
                                      : span >= 128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                                                    : CU_TENSOR_MAP_L2_PROMOTION_NONE;
  CUresult r;
  if (k->tc_copies && !d.paged) {
    // tcgen05 dataflow, contiguous rows: copies of 8 token rows of one kv
    // head, landing as [plane][8 rows][128 bytes] (the 8-row groups the
    // tensor core reads with the 128-byte swizzle)
    const cuuint64_t dims[4] = {inner, static_cast<cuuint64_t>(kv_rows), np,
                                static_cast<cuuint64_t>(d.kv_heads)};
    const cuuint64_t strides[3] = {row * d.kv_heads, cb, row};
    const cuuint32_t box[4] = {inner, 8, static_cast<cuuint32_t>(np), 1};
    r = enc(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, promo,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else if (k->tc_copies) {
    // tcgen05 dataflow, paged pool: the pool's token rows (a page holds
    // page_size consecutive rows of [kv_heads][head_dim]) as groups of 8, so
    // one copy moves a whole page (or a 128-token slice of a longer one) and
    // lands as [group][plane][8 rows][128 bytes]
    const cuuint64_t groups = static_cast<cuuint64_t>(kv_rows) * d.page_size / 8;
    const cuuint64_t dims[5] = {inner, 8, np, static_cast<cuuint64_t>(d.kv_heads), groups};
    const cuuint64_t strides[4] = {row * d.kv_heads, cb, row, 8 * row * d.kv_heads};
    const int per_copy = d.page_size < k->tile_tokens ? d.page_size : k->tile_tokens;
    const cuuint32_t box[5] = {inner, 8, static_cast<cuuint32_t>(np), 1,
                               static_cast<cuuint32_t>(per_copy / 8)};
    r = enc(map, dt, 5, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, promo,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else if (k->token_major) {
    // [.. rows][kv_heads][planes][plane elements]: one copy carries whole rows
    if (!d.paged) {
      const cuuint64_t dims[4] = {inner, np, static_cast<cuuint64_t>(d.kv_heads),
                                  static_cast<cuuint64_t>(kv_rows)};
      const cuuint64_t strides[3] = {cb, row, row * d.kv_heads};
      const cuuint32_t box[4] = {inner, static_cast<cuuint32_t>(np),
                                 static_cast<cuuint32_t>(p->heads_per_tile),
                                 static_cast<cuuint32_t>(k->tile_tokens)};
      r = enc(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, promo,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
      const cuuint64_t dims[5] = {inner, np, static_cast<cuuint64_t>(d.kv_heads),
                                  static_cast<cuuint64_t>(d.page_size),
                                  static_cast<cuuint64_t>(kv_rows)};
      const cuuint64_t strides[4] = {cb, row, row * d.kv_heads, row * d.kv_heads * d.page_size};
      const cuuint32_t box[5] = {inner, static_cast<cuuint32_t>(np),
                                 static_cast<cuuint32_t>(p->heads_per_tile),
                                 static_cast<cuuint32_t>(p->box_t), 1};
      r = enc(map, dt, 5, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, promo,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
  } else if (!d.paged) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d.head_dim),
                                static_cast<cuuint64_t>(d.kv_heads),
                                static_cast<cuuint64_t>(kv_rows)};
    const cuuint64_t strides[2] = {row, row * d.kv_heads};
    const cuuint32_t box[3] = {inner, 1, static_cast<cuuint32_t>(k->tile_tokens)};
    r = enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, promo,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d.head_dim),
                                static_cast<cuuint64_t>(d.kv_heads),
                                static_cast<cuuint64_t>(d.page_size),
                                static_cast<cuuint64_t>(kv_rows)};
    const cuuint64_t strides[3] = {row, row * d.kv_heads, row * d.kv_heads * d.page_size};
    const cuuint32_t box[4] = {inner, 1, static_cast<cuuint32_t>(p->box_t), 1};
    r = enc(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, promo,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed (%d)",
             static_cast<int>(r));
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

// The query rows of the tcgen05 dataflow: [batch * q_len * qo_heads rows]
// of head_dim bf16, copied as (group) rows x one 128-byte plane with the
// 128-byte swizzle.
fa_status make_q_map(const fa_plan* p, const void* q, CUtensorMap* map) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled unavailable");
    return FA_ERR_CUDA;
  }
  const fa_decode_desc& d = p->desc;
  const cuuint64_t rows = static_cast<cuuint64_t>(d.batch) * q_len_of(&d) * d.qo_heads;
  const cuuint64_t dims[3] = {64, rows, static_cast<cuuint64_t>(d.head_dim / 64)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d.head_dim) * 2, 128};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(d.qo_heads / d.kv_heads), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(q), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled (q) failed (%d)",
             static_cast<int>(r));
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_decode_run(const fa_plan* plan, const void* q, const void* k,
                                   const void* v, int64_t kv_rows, const int32_t* page_table,
                                   int32_t page_table_stride, const int32_t* kv_indptr,
                                   const float* k_scale, const float* v_scale, void* out,
                                   float* lse, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  if (plan == nullptr || q == nullptr || k == nullptr || v == nullptr || kv_indptr == nullptr ||
      out == nullptr || workspace == nullptr)
    return FA_ERR_INVALID_ARG;
  const fa_decode_desc& d = plan->desc;
  const bool quant = d.kv_dtype != FA_KV_BF16;  // fp8 / int4 codes with per-head scales
  if (d.paged && (page_table == nullptr || page_table_stride < 1)) return FA_ERR_INVALID_ARG;
  if (quant && (k_scale == nullptr || v_scale == nullptr)) return FA_ERR_INVALID_ARG;
  if (kv_rows < 1 || kv_rows > INT32_MAX) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(workspace, 256) || !aligned(kv_indptr, 4) || (lse && !aligned(lse, 4)) ||
      (page_table && !aligned(page_table, 4)) || (k_scale && !aligned(k_scale, 4)) ||
      (v_scale && !aligned(v_scale, 4)))
    return FA_ERR_MISALIGNED;
  if (workspace_bytes < plan->ws_bytes) return FA_ERR_WORKSPACE_TOO_SMALL;

  const bool tc = plan->kernel->tc_copies != 0;
  // the tcgen05 dataflow addresses paged pools by token row (an int32)
  if (tc && d.paged && kv_rows * d.page_size > INT32_MAX) return FA_ERR_UNSUPPORTED;

  fa::KernelArgs a;
  memset(&a, 0, sizeof(a));
  fa_status st = make_kv_map(plan, k, kv_rows, &a.kmap);
  if (st == FA_OK) st = make_kv_map(plan, v, kv_rows, &a.vmap);
  if (st == FA_OK && tc) st = make_q_map(plan, q, &a.qmap);
  if (st != FA_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.q = static_cast<const uint16_t*>(q);
  a.kv_indptr = kv_indptr;
  a.page_table = d.paged ? page_table : nullptr;
  a.k_scale = quant ? k_scale : nullptr;
  a.v_scale = quant ? v_scale : nullptr;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.records = reinterpret_cast<int4*>(ws + plan->off_records);
  a.part_o = reinterpret_cast<float*>(ws + plan->off_part_o);
  a.part_lse = reinterpret_cast<float*>(ws + plan->off_part_lse);
  a.kv_rows = kv_rows;
  a.max_partials = static_cast<int>(plan->max_partials);
  a.batch = d.batch;
  a.qo_heads = d.qo_heads;
  // a segment covers heads_per_tile kv heads: seen by the kernel as one kv
  // head whose group holds all their query heads
  a.kv_heads = d.kv_heads / plan->heads_per_tile;
  a.group = d.qo_heads / d.kv_heads * plan->heads_per_tile;
  a.q_len = q_len_of(&d);
  a.window_u = d.window > 0 ? union_window(&d) : -1;
  a.window = d.window > 0 ? d.window : -1;
  a.paged = d.paged;
  a.page_shift = plan->page_shift;
  a.seg_parts = plan->seg_parts;
  a.piece_cost = plan->piece_cost;
  a.pt_stride = d.paged ? page_table_stride : 0;
  a.box_t = plan->box_t;
  a.swz = plan->swz;
  a.score_scale = d.sm_scale * 1.4426950408889634f;
  a.cap_l2 = d.logit_cap > 0.f ? d.logit_cap * 1.4426950408889634f : 0.f;
  a.m_init = d.unified_max ? d.softmax_phi * 1.4426950408889634f : -INFINITY;

  cudaError_t e = plan->kernel->launch(a, plan->num_ctas, plan->smem,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_failure("fa_decode_run: launch", e);
  fa::SplitMergeArgs m;
  m.records = a.records;
  m.part_o = a.part_o;
  m.part_lse = a.part_lse;
  m.out = a.out;
  m.lse = a.lse;
  m.num_records = plan->num_ctas;
  m.group = plan->group;
  m.kv_group = d.qo_heads / d.kv_heads * plan->heads_per_tile;
  m.q_len = q_len_of(&d);
  m.kv_heads = d.kv_heads / plan->heads_per_tile;
  m.qo_heads = d.qo_heads;
  m.batch = d.batch;
  m.max_partials = plan->max_partials;
  // one whole segment per block: nothing is split, nothing to merge
  if (plan->seg_parts == 1) return FA_OK;
  e = fa::launch_split_merge(m, d.head_dim, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_failure("fa_decode_run: merge launch", e);
  return FA_OK;
}

extern "C" fa_status fa_decode_status(void* workspace, size_t workspace_bytes, uint32_t* flags,
                                      void* stream) {
  if (workspace == nullptr || flags == nullptr || workspace_bytes < 256) return FA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_failure("fa_decode_status: read", e);
  *flags = h;
  if (h != 0) {
    // the whole header: the check word and the records of the first failed
    // check and the first wait that gave up (a record is written only into
    // a cleared slot, so a stale one would hide the next failure)
    e = cudaMemsetAsync(workspace, 0, 256, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_failure("fa_decode_status: clear", e);
    return FA_ERR_DEVICE_CHECK;
  }
  return FA_OK;
}

// ------------------------------------------------------- bounded-wait test
namespace {

// One thread waits on a fresh mbarrier with the kernels' bounded wait.  With
// `arrive` the thread arrives first, so the wait succeeds at once; without
// it nothing ever arrives, the wait gives up after limit_ns and records the
// timeout (site kSelftestSite, block 0, warp 0) as a pipeline wait would.
constexpr uint32_t kSelftestSite = 99;

__global__ void fa_wait_selftest_kernel(uint32_t* status, unsigned long long limit_ns, int arrive) {
  __shared__ alignas(8) unsigned long long bar;
  const uint32_t b = fa::smem_addr(&bar);
  if (threadIdx.x == 0) {
    fa::mbar_init(b, 1);
    fa::fence_mbar_init();
    if (arrive) fa::mbar_arrive(b);
    if (!fa::mbar_wait(b, 0, limit_ns)) fa::record_timeout(status, kSelftestSite, 0, 0, 0, b);
  }
}

}  // namespace

extern "C" fa_status fa_selftest_wait(void* workspace, size_t workspace_bytes, int64_t limit_ns,
                                      int32_t arrive, void* stream) {
  if (workspace == nullptr || workspace_bytes < 256 || limit_ns < 1 || limit_ns > 1000000000LL)
    return FA_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return FA_ERR_MISALIGNED;
  fa_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint32_t*>(workspace), static_cast<unsigned long long>(limit_ns), arrive ? 1 : 0);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_failure("fa_selftest_wait: launch", e);
  return FA_OK;
}

// ------------------------------------------------------------ merge states
namespace {

// One warp per (row, head): lse = M + ln sum exp(lse_c - M); out = sum
// exp(lse_c - lse) o_c.  States with lse = -inf carry no weight.
__global__ void fa_merge_states_kernel(const float* __restrict__ o_parts,
                                       const float* __restrict__ lse_parts, int n, long long rh_count,
                                       int d, uint16_t* __restrict__ out, float* __restrict__ lse_out) {
  const long long rh = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (rh >= rh_count) return;
  float M = -CUDART_INF_F;
  for (int c = lane; c < n; c += 32) M = fmaxf(M, lse_parts[c * rh_count + rh]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (M == -CUDART_INF_F) {
    for (int x = lane * 4; x < d; x += 128)
      *reinterpret_cast<uint2*>(out + rh * d + x) = make_uint2(0u, 0u);
    if (lane == 0 && lse_out != nullptr) lse_out[rh] = -CUDART_INF_F;
    return;
  }
  float Z = 0.f;
  for (int c = lane; c < n; c += 32) {
    const float l = lse_parts[c * rh_count + rh];
    if (l != -CUDART_INF_F) Z += exp2f((l - M) * fa::kLog2e);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, off);
  const float L = M + logf(Z);
  for (int x = lane * 4; x < d; x += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < n; ++c) {
      const float l = lse_parts[c * rh_count + rh];
      if (l == -CUDART_INF_F) continue;
      const float w = exp2f((l - L) * fa::kLog2e);
      const float4 v = *reinterpret_cast<const float4*>(o_parts + (c * rh_count + rh) * d + x);
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(acc.x)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(acc.y))) << 16);
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(acc.z)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(acc.w))) << 16);
    *reinterpret_cast<uint2*>(out + rh * d + x) = make_uint2(lo, hi);
  }
  if (lane == 0 && lse_out != nullptr) lse_out[rh] = L;
}

}  // namespace

extern "C" fa_status fa_merge_states(const float* o_parts, const float* lse_parts, int32_t n,
                                     int32_t rows, int32_t heads, int32_t head_dim, void* out,
                                     float* lse_out, void* stream) {
  if (o_parts == nullptr || lse_parts == nullptr || out == nullptr) return FA_ERR_INVALID_ARG;
  if (n < 1 || rows < 1 || heads < 1 || head_dim < 4 || head_dim % 4 != 0 || head_dim > 1024)
    return FA_ERR_INVALID_ARG;
  if (!aligned(o_parts, 16) || !aligned(out, 16) || !aligned(lse_parts, 4) ||
      (lse_out && !aligned(lse_out, 4)))
    return FA_ERR_MISALIGNED;
  const long long rh = static_cast<long long>(rows) * heads;
  const int threads = 256;
  const long long blocks = (rh * 32 + threads - 1) / threads;
  if (blocks > INT32_MAX) return FA_ERR_INVALID_ARG;
  fa_merge_states_kernel<<<static_cast<unsigned>(blocks), threads, 0,
                           static_cast<cudaStream_t>(stream)>>>(
      o_parts, lse_parts, n, rh, head_dim, static_cast<uint16_t*>(out), lse_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_failure("fa_merge_states: launch", e);
  return FA_OK;
}

extern "C" const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported shape or option";
    case FA_ERR_WORKSPACE_TOO_SMALL: return "workspace smaller than the plan requires";
    case FA_ERR_MISALIGNED: return "pointer below its required alignment";
    case FA_ERR_CUDA: return "CUDA call failed";
    case FA_ERR_DEVICE_CHECK: return "device-side check recorded an error";
  }
  return "unknown status";
}

extern "C" int32_t fa_version(void) { return FA_VERSION; }

extern "C" const char* fa_last_error(void) { return g_last_error; }
