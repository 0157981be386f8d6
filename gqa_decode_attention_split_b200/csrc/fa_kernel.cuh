// fa_kernel.cuh -- split-KV GQA decode attention for sm_100a.
//
// A pass is one launch of fa_decode_kernel plus, when a segment is split
// across blocks, one launch of fa_split_merge_kernel:
//  1. schedule: every (request, kv head) is a segment of KV tiles; segments
//     are laid end to end and cut into gridDim.x equal runs, one per thread
//     block, so every SM streams the same number of bytes whatever the
//     length mix ("FlashDecoding++" explainer, section "Hardware-aware
//     heuristic dataflow": the split is chosen from batch, lengths and GPU).
//     Each block derives its runs from kv_indptr in shared memory; nothing
//     is uploaded from the host.
//  2. load: a producer warp streams K and V tiles HBM -> shared memory with
//     bulk tensor copies (TMA) into a ring of mbarrier-guarded stages, so the
//     next tiles are in flight while the current ones are consumed ("Beyond
//     the Memory Wall", section on FlashAttention-3: the next tile is
//     prefetched while the current one is computed).
//  3. math: consumer warps take whole tiles round-robin.  Each keeps a
//     running (max, sum, acc) per query head and rescales when the max grows
//     ("Forcing Flash Attention onto a TPU", section "Flash Attention in
//     JAX").  Two dataflows: SIMT (per-lane fp32 FMAs, warp-shuffle
//     reductions) and MMA (the two skinny products on mma.sync with fp32
//     accumulation).
//  4. merge: warps of a block merge their states in shared memory; a
//     segment that lies whole in one block is written out directly.  A
//     segment cut across blocks writes one (o, lse) partial per block, and
//     a second, small kernel (fa_split_merge_kernel, launched as a
//     programmatic dependent of this one) merges them exactly through
//     log-sum-exp ("FlashDecoding++" explainer, section "Asynchronous softmax
//     and unified max value": partial softmax per tile, combined afterwards;
//     "Flashlight", section "Method": exp(x - y) = exp(x) / exp(y)).  The
//     merge runs on every SM at once: a single block merging a segment's
//     partials is bound by L2 round trips (one block keeps too few bytes in
//     flight), which on B200 cost about a microsecond each.
#pragma once

#include <math_constants.h>

#include "fa_device.cuh"

namespace fa {

// Tuning knobs (compile-time).  Defaults are the settings measured best on
// B200 for each dataflow: the tensor-core path wants large tiles (few bulk
// copies and barrier round trips per byte) and five consumer warps; the
// instruction-heavier SIMT and fp8 paths want more warps.  Every knob can be
// overridden with -D for tuning sweeps.
#ifndef FA_MMA_TILE_BYTES
#define FA_MMA_TILE_BYTES 16384      // bytes of K (and of V) per stage, bf16 MMA path
#endif
#ifndef FA_MMA_CONSUMER_WARPS
#define FA_MMA_CONSUMER_WARPS 5
#endif
#ifndef FA_FP8_MMA_TILE_BYTES
#define FA_FP8_MMA_TILE_BYTES 8192
#endif
#ifndef FA_FP8_MMA_CONSUMER_WARPS
#define FA_FP8_MMA_CONSUMER_WARPS 7
#endif
#ifndef FA_NB2_TOKENS
#define FA_NB2_TOKENS 64     // tile tokens, bf16 MMA with one team of two row blocks
#endif
#ifndef FA_NB2_WARPS
#define FA_NB2_WARPS 3       // its consumer warps
#endif
#ifndef FA_SIMT_TILE_BYTES
#define FA_SIMT_TILE_BYTES 8192
#endif
#ifndef FA_SIMT_CONSUMER_WARPS
#define FA_SIMT_CONSUMER_WARPS 6
#endif
#ifndef FA_MAX_STAGES_PER_WARP
#define FA_MAX_STAGES_PER_WARP 3
#endif
#ifndef FA_PLANE_COPIES
#define FA_PLANE_COPIES 0    // 0: one bulk copy per box, planes a tensor-map dimension
#endif
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait, then give up
constexpr float kRescaleSlack = 8.0f;               // log2 units
// Unified max: a row whose first finite scores sit more than this far (log2
// units) below phi starts from its own maximum instead; nothing has
// accumulated yet, so the switch is exact.  With the slack above, a row's
// largest weight stays in [2^-8, 2^8], inside the range of the f16
// probabilities of the fp8 / int4 tensor-core products (a weight of 2^-43
// against a phi far above the scores flushed to zero there).
constexpr float kPhiDrop = kRescaleSlack;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Device-check bits (same values as the public FA_DEVICE_* constants).
constexpr uint32_t kFlagBadPage = 1u;
constexpr uint32_t kFlagTimeout = 2u;
constexpr uint32_t kFlagBadIndptr = 4u;

struct KernelArgs {
  CUtensorMap kmap;
  CUtensorMap vmap;
  CUtensorMap qmap;   // tcgen05 dataflow only: the query rows, 128-byte swizzled planes
  const uint16_t* q;
  const int32_t* kv_indptr;
  const int32_t* page_table;
  const float* k_scale;
  const float* v_scale;
  uint16_t* out;
  float* lse;
  uint32_t* status;
  int4* records;     // [gridDim.x]: split segment whose first cut is at block c
  float* part_o;
  float* part_lse;
  long long kv_rows;
  int max_partials;
  int batch, qo_heads, kv_heads, group;   // group: query heads per kv head
  int q_len;          // query tokens per request (rows of a segment: group * q_len)
  int window_u;       // keys any query token of a request sees: window + q_len - 1 (<= 0: all)
  int window;
  int paged, page_shift, pt_stride, box_t, swz;
  int seg_parts;      // 0: equal runs of all tiles; k > 0: k runs per segment
  int piece_cost;     // equal runs: tile units charged to every segment ahead of its tiles
  float score_scale;  // sm_scale * log2(e)
  float cap_l2;       // > 0: logit soft-cap in log2 units (cap * log2(e)); 0: none
  float m_init;       // start of every running max: -inf, or the unified max phi (log2 units)
};

constexpr int kSmemPerBlock = 232448;  // 227 KB of shared memory per block (sm_100)
constexpr int kSchedReserve = 8192;    // schedule arrays for up to 682 requests
constexpr int kScaleCap = 128;         // fp8 per-kv-head scales kept in shared memory

// Shared-memory tile geometry for one head_dim / element type.  A token row
// is cut into NP planes of CB = min(128, row bytes) bytes (the widest box row
// the 128-byte swizzle allows).  Default (token-major) layout of a K or V
// tile: [T][NP][CB], written by ONE bulk copy per box whose tensor map has
// the plane as a dimension; the 16-byte chunks of 128-byte line l of the tile
// are XOR-swizzled by (l & 7) (TMA 128B swizzle).  With FA_PLANE_COPIES the
// layout is plane-major, [NP][T][CB], one copy per plane.
// A tile holds TILE_BYTES_TARGET / row bytes tokens (16 to 128).  K and V
// tiles live in two rings that take what is left of the block's shared
// memory after the merge area: KSTAGES K slots and VSTAGES V slots.  The NW
// consumer warps form R row teams of NT = NW / R warps: a tile is consumed
// by one warp of every team (warp u of each team takes tiles i with
// i % NT == u, the team's own GW query rows of the segment), so a tile
// carries up to GW * R rows.  Both slot counts are multiples of NT and tile
// i uses K slot i % KSTAGES and V slot i % VSTAGES: every slot belongs to
// exactly one tile lane u, whose R warps wait on it round after round.  (A
// slot shared by two tile lanes would let one wait for round r+1 while round
// r is still pending; an mbarrier parity wait cannot tell the two apart and
// would pass early.)  A consumer that frees its K slot as soon as the scores
// are taken (EARLY_K) holds V longer than K, so the V ring gets the extra
// slots: a slot is refilled only after its warps release it, and a slot
// held through the tile's math is a slot with no copy in flight.
// KV element kinds: bf16, fp8 e4m3, int4 (two codes per byte).
enum : int { kKvBf16 = 0, kKvFp8 = 1, kKvInt4 = 2 };

template <int D, int KIND, int GW, int R, int TILE_BYTES_TARGET, int NWARPS, bool EARLY_K,
          int HT_ = 1>
struct TileCfg {
  static constexpr int DIM = D;
  // kv heads per tile: a tile holds the rows of HT adjacent kv heads for each
  // of its tokens ([T][HT][row], one box), so a copy moves HT * ROWB
  // contiguous bytes per token
  static constexpr int HT = HT_;
  static constexpr bool QUANT = KIND != kKvBf16;  // codes with per-kv-head scales
  static constexpr int ES = KIND == kKvBf16 ? 2 : 1;  // bytes per tensor-map element
  static constexpr int ROWB = KIND == kKvBf16 ? 2 * D : (KIND == kKvFp8 ? D : D / 2);
  static constexpr int CB = ROWB < 128 ? ROWB : 128;
  static constexpr int NP = ROWB / CB;
  static constexpr int TOKB = HT * ROWB;  // tile bytes per token
  static constexpr int T_RAW = TILE_BYTES_TARGET / TOKB;
  static constexpr int T = T_RAW < 16 ? 16 : (T_RAW > 128 ? 128 : T_RAW);
  static constexpr int TILE_BYTES = T * TOKB;
  static constexpr int NW = NWARPS;
  static constexpr int TEAMS = R;       // row teams
  static constexpr int NT = NW / R;     // tile lanes (warps per team)
  static_assert(NW % R == 0, "every row team has the same warps");
  static constexpr int GMAX = GW * R;   // rows of a segment
  // merge area: one (m, l, acc[D]) state per tile lane and row
  static constexpr int MERGE_BYTES = NT * GMAX * (D + 2) * 4;
  // q area: four mbarriers, then (STAGE_Q) two slots of a piece's GMAX query
  // rows (bf16) that the producer stages, then (fp8) the k / v scale tables.
  // Query rows are staged only where the slots cost no ring stage; otherwise
  // consumers read them from global memory.
  static constexpr int QSLOT_BYTES = GMAX * D * 2;
  static constexpr int SCALE_BYTES = QUANT ? 2 * kScaleCap * 4 : 0;
  // (1024: base alignment; 272: merge counter, merge mbarrier, 64 page ids)
  static constexpr int BASE_BUDGET = kSmemPerBlock - 1024 - kSchedReserve - 272 - MERGE_BYTES - 32 - SCALE_BYTES;
  // K + V tiles per tile lane that fit (a tile slot costs its bytes plus two
  // 8-byte mbarriers)
  static constexpr int kLaneCap = 2 * FA_MAX_STAGES_PER_WARP * R;
  static constexpr int tiles_per_warp(int budget) {
    return budget / (TILE_BYTES + 16) / NT > kLaneCap ? kLaneCap : budget / (TILE_BYTES + 16) / NT;
  }
  static constexpr bool STAGE_Q = tiles_per_warp(BASE_BUDGET - 2 * QSLOT_BYTES) == tiles_per_warp(BASE_BUDGET);
  static constexpr int QAREA_BYTES = 32 + (STAGE_Q ? 2 * QSLOT_BYTES : 0) + SCALE_BYTES;
  static constexpr int RING_BUDGET = BASE_BUDGET + 32 + SCALE_BYTES - QAREA_BYTES;
  static constexpr int TPW = tiles_per_warp(RING_BUDGET);
  static constexpr int KPW = EARLY_K ? (TPW / 3 > 1 ? TPW / 3 : 1) : TPW / 2;
  static constexpr int VPW = EARLY_K ? TPW - KPW : KPW;
  static_assert(KPW >= 1 && VPW >= 1, "every tile lane needs a K and a V slot");
  static constexpr int KSTAGES = NT * KPW;
  static constexpr int VSTAGES = NT * VPW;
  static constexpr int RING_BYTES = (KSTAGES + VSTAGES) * TILE_BYTES;
  static constexpr int THREADS = (NW + 1) * 32;
  static constexpr bool TOKEN_MAJOR = FA_PLANE_COPIES == 0;
  static_assert(ROWB % 16 == 0, "rows must be whole 16-byte chunks");
  static_assert(HT == 1 || TOKEN_MAJOR, "tiles of several heads are token-major");
};

__device__ __forceinline__ uint32_t swz_off(int row, int chunk, int swz) {
  return static_cast<uint32_t>(((chunk ^ (swz ? (row & 7) : 0)) << 4));
}

// Shared-memory address of 16-byte chunk `chunk` of plane `plane` of token
// row `row` in a tile.
template <class C>
__device__ __forceinline__ uint32_t tile_addr(uint32_t tile, int row, int plane, int chunk, int swz) {
  if constexpr (C::TOKEN_MAJOR) {
    const int line = row * C::NP + plane;
    return tile + line * C::CB + swz_off(line, chunk, swz);
  } else {
    return tile + plane * (C::T * C::CB) + row * C::CB + swz_off(row, chunk, swz);
  }
}

// A wait that gives up records where (first one wins) in words 8..15 of the
// workspace header: site (1 producer/empty, 2 producer drain/full,
// 3 consumer/full), block, warp, block-sequence tile index, stage, parity and
// the barrier's raw 64-bit state.
__device__ __noinline__ static void record_timeout(uint32_t* status, uint32_t site, int tile, int stage,
                                                   uint32_t parity, uint32_t bar) {
  atomicOr(status, kFlagTimeout);
  if (atomicCAS(status + 8, 0u, site) == 0u) {
    const uint64_t raw = mbar_raw_state(bar);
    status[9] = blockIdx.x;
    status[10] = threadIdx.x >> 5;
    status[11] = static_cast<uint32_t>(tile);
    status[12] = static_cast<uint32_t>(stage);
    status[13] = parity;
    status[14] = static_cast<uint32_t>(raw);
    status[15] = static_cast<uint32_t>(raw >> 32);
  }
}

// ------------------------------------------------------- debug checks
// Built with -DFA_CHECKS, every shared-memory read, bulk-copy destination and
// global write is range- and alignment-checked; a violation sets
// kFlagCheck in the status word, records (code, block, thread, value) in the
// next four words of the workspace header (first violation wins) and the
// access is skipped.  Without FA_CHECKS the checks compile to nothing.
constexpr uint32_t kFlagCheck = 8u;
#ifdef FA_CHECKS
static __device__ __noinline__ void check_fail(uint32_t* status, uint32_t code, long long value) {
  atomicOr(status, kFlagCheck);
  if (atomicCAS(status + 1, 0u, code) == 0u) {
    status[2] = blockIdx.x;
    status[3] = threadIdx.x;
    status[4] = static_cast<uint32_t>(value);
    status[5] = static_cast<uint32_t>(value >> 32);
  }
}
#define FA_CHECK(status, cond, code, value) \
  ((cond) ? true : (::fa::check_fail((status), (code), static_cast<long long>(value)), false))
#else
#define FA_CHECK(status, cond, code, value) true
#endif
// Shared-memory 16-byte load that stays inside [tile, tile + bytes).
// Row address for a warp-collective ldmatrix: a bad address is replaced by
// the tile base (the instruction must still be executed by every lane).
__device__ __forceinline__ uint32_t ldsm_addr_in(uint32_t* status, uint32_t addr, uint32_t tile,
                                                 uint32_t bytes, uint32_t code) {
  return FA_CHECK(status, addr >= tile && addr + 16 <= tile + bytes && (addr & 15u) == 0, code,
                  static_cast<long long>(addr) - tile)
             ? addr
             : tile;
}
__device__ __forceinline__ uint4 lds128_in(uint32_t* status, uint32_t addr, uint32_t tile,
                                           uint32_t bytes, uint32_t code) {
  if (!FA_CHECK(status, addr >= tile && addr + 16 <= tile + bytes && (addr & 15u) == 0, code,
                static_cast<long long>(addr) - tile))
    return make_uint4(0, 0, 0, 0);
  return lds128(addr);
}

// Shared-memory 8-byte load that stays inside [tile, tile + bytes).
__device__ __forceinline__ uint2 lds64_in(uint32_t* status, uint32_t addr, uint32_t tile,
                                          uint32_t bytes, uint32_t code) {
  if (!FA_CHECK(status, addr >= tile && addr + 8 <= tile + bytes && (addr & 7u) == 0, code,
                static_cast<long long>(addr) - tile))
    return make_uint2(0, 0);
  return lds64(addr);
}

// ------------------------------------------------------------ schedule
// a / b for non-negative a, positive b: 32-bit division when both
// fit (the schedule's tile counts do, short of 2^31 tiles), else 64-bit.  A
// 64-bit division is a long software routine, and a block's schedule takes
// several before its first copy goes out.
__device__ __forceinline__ long long div_fast(long long a, long long b) {
  if (((a | b) >> 31) == 0) return static_cast<long long>(static_cast<uint32_t>(a) / static_cast<uint32_t>(b));
  return a / b;
}

struct Piece {
  int b, h;          // request, kv head
  int t0, t1;        // request-local tile indices [t0, t1)
  int seg;           // b * kv_heads + h
  int n_pieces;      // blocks sharing this segment
  int c_first;       // first block of the segment
};

// The block's run is units [u, u1) of the segments laid end to end.  Either
// all runs have `per` units (parts == 0), or every segment is cut into
// `parts` runs, block c taking run c % parts of segment c / parts (units are
// tiles).  With equal runs every segment spans `cost` units ahead of its
// tiles: the fixed cost of a piece (parking and merging its state, its
// ragged last tile) in tile units, so a block whose run starts more
// segments gets fewer tiles.  A run may end inside those units; units that
// hold no tile are skipped.
struct PieceIter {
  long long u, u1, per;
  int parts;
  int cost;
};

__device__ __forceinline__ int first_tile(int L, int window, int T) {
  int lo = (window > 0 && L > window) ? L - window : 0;
  return lo / T;
}
__device__ __forceinline__ int num_tiles(int L, int window, int T) {
  if (L <= 0) return 0;
  return (L + T - 1) / T - first_tile(L, window, T);
}

__device__ __forceinline__ bool next_piece(PieceIter& it, Piece& pc, const int* s_pre,
                                           const int* s_len, int B, int H, int window, int T) {
  const long long K = it.cost;
  while (it.u < it.u1) {
    // request b: H*(pre[b] + K*b) <= u < H*(pre[b+1] + K*(b+1))
    int lo = 0, hi = B;
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (static_cast<long long>(H) * (s_pre[mid] + K * mid) <= it.u)
        lo = mid;
      else
        hi = mid;
    }
    const int b = lo;
    const int n = s_pre[b + 1] - s_pre[b];
    const long long span = n + K;  // units of each of the request's segments
    const long long base = static_cast<long long>(H) * (s_pre[b] + K * b);
    const int h = static_cast<int>(div_fast(it.u - base, span));
    const long long first = base + static_cast<long long>(h) * span + K;  // unit of tile 0
    const long long seg_end = first + n;
    if (n == 0) {  // no tile: skip the segment (reached only with K > 0)
      it.u = seg_end;
      continue;
    }
    if (it.u < first) it.u = first;
    if (it.u >= it.u1) return false;  // the run ends among the segment's charge
    const int tin = static_cast<int>(it.u - first);
    long long len = n - tin;
    if (it.u1 - it.u < len) len = it.u1 - it.u;
    const int ft = first_tile(s_len[b], window, T);
    pc.b = b;
    pc.h = h;
    pc.t0 = ft + tin;
    pc.t1 = pc.t0 + static_cast<int>(len);
    pc.seg = b * H + h;
    if (it.parts > 0) {
      pc.c_first = pc.seg * it.parts;
      pc.n_pieces = it.parts;
    } else {
      pc.c_first = static_cast<int>(div_fast(first, it.per));
      pc.n_pieces = static_cast<int>(div_fast(seg_end - 1, it.per)) - pc.c_first + 1;
    }
    it.u += len;
    return true;
  }
  return false;
}

// ------------------------------------------------------ pass set-up
// Every kernel of a pass starts the same way: validated request lengths,
// the tile prefix over requests, and the block's run of the schedule.

// s_start[b], s_len[b] from the device kv_indptr (all threads of the block).
// A decreasing indptr or one past the K/V extent (or the page table) sets
// FA_DEVICE_BAD_INDPTR; such a request is read as empty or clipped.
__device__ __forceinline__ void load_lengths(const KernelArgs& a, int* s_start, int* s_len) {
  const int ps = a.paged ? (1 << a.page_shift) : 0;
  for (int b = threadIdx.x; b < a.batch; b += blockDim.x) {
    const int st = __ldg(a.kv_indptr + b), en = __ldg(a.kv_indptr + b + 1);
    int L = en - st;
    bool bad = false;
    if (st < 0 || L < 0) {
      L = 0;
      bad = true;
    } else if (!a.paged && static_cast<long long>(en) > a.kv_rows) {
      bad = true;  // rows past the extent read as zeros
    } else if (a.paged && L > 0 && ((L + ps - 1) >> a.page_shift) > a.pt_stride) {
      L = a.pt_stride << a.page_shift;
      bad = true;
    }
    s_start[b] = st;
    s_len[b] = L;
    if (bad) atomicOr(a.status, kFlagBadIndptr);
  }
}

// s_pre[b] = tiles of requests before b, s_pre[batch] = all tiles (one warp).
__device__ __forceinline__ void tile_prefix(const KernelArgs& a, const int* s_len, int* s_pre, int T,
                                            int lane) {
  const int B = a.batch;
  int carry = 0;
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int b = b0 + lane;
    const int n = b < B ? num_tiles(s_len[b], a.window_u, T) : 0;
    int incl = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (b < B) s_pre[b] = carry + incl - n;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) s_pre[B] = carry;
}

// Block c's run of the schedule: equal runs of all segments' tiles (plus the
// per-segment charge), or run c % k of segment c / k.
__device__ __forceinline__ PieceIter block_run(const KernelArgs& a, const int* s_pre, int P, int c) {
  const int B = a.batch, H = a.kv_heads;
  PieceIter it;
  it.cost = a.seg_parts > 0 ? 0 : a.piece_cost;
  const long long N = static_cast<long long>(H) * (s_pre[B] + static_cast<long long>(it.cost) * B);
  it.per = N > 0 ? div_fast(N + P - 1, P) : 1;
  it.parts = 0;
  it.u = static_cast<long long>(c) * it.per;
  it.u1 = it.u + it.per < N ? it.u + it.per : N;
  if (a.seg_parts > 0) {
    // run c % k of segment c / k (runs differ by at most one tile; the
    // planner gives every run at least one tile)
    const int k = a.seg_parts;
    const int seg = c / k, part = c - seg * k;
    it.parts = k;
    it.u = it.u1 = 0;
    if (seg < B * H) {
      const int b = seg / H, h = seg - b * H;
      const long long n = s_pre[b + 1] - s_pre[b];
      const long long base = static_cast<long long>(H) * s_pre[b] + static_cast<long long>(h) * n;
      it.u = base + div_fast(part * n, k);
      it.u1 = base + div_fast((part + 1) * n, k);
    }
  }
  return it;
}

// Boundary record (one thread): block c's run starts at tile c * per.  If
// that cut lies inside a segment that began in block c - 1's run, it is the
// segment's first cut and block c names the segment for the merge kernel;
// every other block writes "none", so no record survives from an earlier
// pass.
__device__ __forceinline__ void write_boundary_record(const KernelArgs& a, const PieceIter& it,
                                                      const int* s_pre, const int* s_len, int T,
                                                      int c) {
  if (c == 0) return;
  PieceIter i0 = it;
  Piece p0;
  int4 rec = make_int4(-1, 0, 0, 0);
  if (next_piece(i0, p0, s_pre, s_len, a.batch, a.kv_heads, a.window_u, T) && p0.c_first == c - 1)
    rec = make_int4(p0.seg, p0.c_first, p0.n_pieces, 0);
  a.records[c] = rec;
}

// Results no piece writes (threads ctid < nct of the block): a run of a split
// segment that holds no tile (only if the device indptr is not the plan's)
// gets an empty partial state, so the merge gives it no weight; requests
// without keys get out = 0, lse = -inf (spread over blocks).
__device__ __forceinline__ void write_empty_results(const KernelArgs& a, const PieceIter& it,
                                                    const int* s_len, int G, int D, int c, int P,
                                                    int ctid, int nct) {
  const int B = a.batch, H = a.kv_heads, Q = a.q_len;
  if (it.parts > 1 && it.u >= it.u1 && c / it.parts < B * H) {
    const size_t slot = static_cast<size_t>(c) + c / it.parts;
    for (int x = ctid; x < G * D; x += nct) {
      a.part_o[slot * G * D + x] = 0.f;
      if (x < G) a.part_lse[slot * G + x] = -CUDART_INF_F;
    }
  }
  for (int b = c; b < B; b += P) {
    if (s_len[b] != 0) continue;
    const int nq = Q * a.qo_heads * D;  // every query token's rows
    for (int x = ctid; x < nq; x += nct) {
      a.out[static_cast<size_t>(b) * nq + x] = 0;
      if (a.lse != nullptr && (x % D) == 0)
        a.lse[static_cast<size_t>(b) * Q * a.qo_heads + x / D] = -CUDART_INF_F;
    }
  }
}

// ------------------------------------------------------ SIMT dataflow
// Lanes are grouped LPT per token; a lane owns CPL 16-byte chunks of every
// row (E elements), holds q for those elements for all G heads and an fp32
// accumulator for the same.  q.k partial sums are all-reduced over the LPT
// lanes with xor shuffles; each group of lanes ("slot") keeps its own
// running softmax state, merged across slots at the end of a segment piece.
template <int D, int G, bool FP8>
struct SimtConsumer {
  // fp8 with 8 rows at head_dim 128 takes a seventh consumer warp (one K and
  // one V slot each instead of two): measured 11% faster on the fp8
  // long-context decode, while bf16 with 4 rows ran 12% slower that way
  static constexpr int kWarps = (FP8 && G >= 8 && D == 128) ? FA_SIMT_CONSUMER_WARPS + 1
                                                             : FA_SIMT_CONSUMER_WARPS;
  using C = TileCfg<D, FP8 ? kKvFp8 : kKvBf16, G, 1, FA_SIMT_TILE_BYTES, kWarps, false>;
  __host__ __device__ static constexpr int team_head(int) { return 0; }  // one kv head per tile
  // bytes of a lane's chunk: 16, or 8 for fp8 with 8 rows, whose 16-element
  // chunks would hold q and acc for 8 x 16 elements per lane (256 registers)
  static constexpr int CHB = (FP8 && G >= 8) ? 8 : 16;
  static constexpr int EPC = CHB / C::ES;
  static constexpr int NCH = C::ROWB / CHB;
  static constexpr int E_TARGET = 64 / G;
  static constexpr int CPL_RAW = E_TARGET / EPC;
  static constexpr int CPL = CPL_RAW < 1 ? 1 : (CPL_RAW > NCH ? NCH : CPL_RAW);
  static constexpr int E = CPL * EPC;
  static constexpr int LPT = NCH / CPL;
  static constexpr int SLOTS = 32 / LPT;
  static constexpr int TPS = C::T / SLOTS;
  static constexpr int NCP = C::CB / CHB;
  static_assert(LPT >= 1 && LPT <= 32 && (NCH % CPL) == 0, "lane mapping");
  static_assert(TPS >= 1 && (C::T % SLOTS) == 0, "tokens per slot");

  // q and the accumulators in element pairs: both products run on the
  // packed fp32 FMA (two lanes of fp32 per instruction on sm_100)
  float2 q[G][E / 2];
  float2 acc[G][E / 2];
  float m[G], l[G];
  // the lane's chunk offsets within a tile row, when the swizzle phase of a
  // row depends only on the lane's slot (rows of one lane step by SLOTS)
  static constexpr bool kFixedSwizzle = C::TOKEN_MAJOR && (SLOTS * C::NP) % 8 == 0;
  uint32_t koff[CPL];
  uint32_t fresh;  // unified max: bit h set while row h has seen no finite score
  int slot, j;

  __device__ __forceinline__ int chunk_plane(int k) const { return (j + LPT * k) / NCP; }
  __device__ __forceinline__ int chunk_in_plane(int k) const { return (j + LPT * k) % NCP; }
  __device__ __forceinline__ int dim_of(int k, int e) const {
    return chunk_plane(k) * (C::CB / C::ES) + chunk_in_plane(k) * EPC + e;
  }

  // The lane's chunk k of tile row r, widened to fp32 (site: the debug
  // build's check code).
  __device__ __forceinline__ void load(const KernelArgs& a, uint32_t tile, int r, int k,
                                       uint32_t site, float (&x)[EPC]) const {
    constexpr int W = CHB / 4;
    uint32_t u[W];
    const uint32_t ad = addr(tile, r, k, a.swz);
    if constexpr (CHB == 16) {
      const uint4 w = lds128_in(a.status, ad, tile, C::TILE_BYTES, site);
      u[0] = w.x;
      u[1] = w.y;
      u[2] = w.z;
      u[3] = w.w;
    } else {
      const uint2 w = lds64_in(a.status, ad, tile, C::TILE_BYTES, site);
      u[0] = w.x;
      u[1] = w.y;
    }
    if constexpr (!FP8) {
#pragma unroll
      for (int i = 0; i < W; ++i) {
        x[2 * i] = bf16lo(u[i]);
        x[2 * i + 1] = bf16hi(u[i]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < W; ++i) {
        float2 lo2 = f16x2_to_float2(e4m3x2_to_f16x2(static_cast<uint16_t>(u[i] & 0xFFFFu)));
        float2 hi2 = f16x2_to_float2(e4m3x2_to_f16x2(static_cast<uint16_t>(u[i] >> 16)));
        x[4 * i] = lo2.x;
        x[4 * i + 1] = lo2.y;
        x[4 * i + 2] = hi2.x;
        x[4 * i + 3] = hi2.y;
      }
    }
  }

  // Shared address of the lane's chunk k of tile row r (8-byte chunks: the
  // 16-byte chunk that holds it, plus the half).
  __device__ __forceinline__ uint32_t addr(uint32_t tile, int r, int k, int swz) const {
    if constexpr (kFixedSwizzle) {
      return tile + static_cast<uint32_t>(r * C::NP * C::CB) + koff[k];
    } else {
      const int cip = chunk_in_plane(k);
      return tile_addr<C>(tile, r, chunk_plane(k), cip * CHB / 16, swz) + (cip * CHB) % 16;
    }
  }

  // qs: the piece's query rows (staged in shared memory, or in global
  // memory where the tile geometry leaves no room): row r (token r / group,
  // head r % group) at qs + (r / group) * qstride + (r % group) * D; kscale:
  // the fp8 K scale of the piece's kv head (1 for bf16).
  __device__ __forceinline__ void begin_piece(const KernelArgs& a, const uint16_t* qs, int qstride,
                                              float kscale, int lane, int /*team: one team*/) {
    slot = lane / LPT;
    j = lane % LPT;
    if constexpr (kFixedSwizzle) {
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
        const int cip = chunk_in_plane(k), p = chunk_plane(k);
        koff[k] = tile_addr<C>(0u, slot, p, cip * CHB / 16, a.swz) - slot * C::NP * C::CB +
                  (cip * CHB) % 16;
      }
    }
    float scale = a.score_scale;
    if constexpr (FP8) scale *= kscale;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const uint16_t* qrow = qs + (h / a.group) * qstride + (h % a.group) * D;
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
#pragma unroll
        for (int e = 0; e < EPC; e += 8) {
          const uint4 w = *reinterpret_cast<const uint4*>(qrow + dim_of(k, e));
          const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            q[h][(k * EPC + e) / 2 + i] = make_float2(bf16lo(u[i]) * scale, bf16hi(u[i]) * scale);
          }
        }
#pragma unroll
        for (int e = 0; e < EPC / 2; ++e) acc[h][k * EPC / 2 + e] = make_float2(0.f, 0.f);
      }
      m[h] = a.m_init;
      l[h] = 0.f;
    }
    fresh = a.m_init > -CUDART_INF_F ? (1u << G) - 1u : 0u;
  }

  // A tile is processed in sub-steps of TPSC tokens per slot (bounded
  // register use); each sub-step updates the slot's running softmax once.
  static constexpr int TPSC = TPS < 4 ? TPS : 4;
  static constexpr int NSUB = TPS / TPSC;
  static_assert(TPS % TPSC == 0, "sub-steps");

  // K and V rows are read together sub-step by sub-step, so K is released
  // at the end (release_k as for the MMA dataflow).  [lo, hi) is the union
  // of the rows' key ranges (hi: the request's length); with several query
  // tokens, row h (token h / group) sees one key fewer per token before the
  // last, within its own window.
  __device__ __forceinline__ bool row_sees(const KernelArgs& a, int h, int pos, int hi) const {
    const int rhi = hi - (a.q_len - 1 - h / a.group);
    const int rlo = (a.window > 0 && rhi > a.window) ? rhi - a.window : 0;
    return pos >= rlo && pos < rhi;
  }
  template <class ReleaseK>
  __device__ __forceinline__ void tile(const KernelArgs& a, uint32_t kt, uint32_t vt, int pos0,
                                       int lo, int hi, int lane, ReleaseK&& release_k) {
    const bool multi = a.q_len > 1;
#pragma unroll 1
    for (int si = 0; si < NSUB; ++si) {
      float s[TPSC][G];
#pragma unroll
      for (int tt = 0; tt < TPSC; ++tt) {
        const int r = (si * TPSC + tt) * SLOTS + slot;
        float2 part2[G];
#pragma unroll
        for (int h = 0; h < G; ++h) part2[h] = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
          float x[EPC];
          load(a, kt, r, k, 101, x);
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < EPC; e += 2)
              part2[h] = __ffma2_rn(q[h][(k * EPC + e) / 2], make_float2(x[e], x[e + 1]), part2[h]);
        }
        float part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) part[h] = part2[h].x + part2[h].y;
#pragma unroll
        for (int off = 1; off < LPT; off <<= 1)
#pragma unroll
          for (int h = 0; h < G; ++h) part[h] += __shfl_xor_sync(0xffffffffu, part[h], off);
#pragma unroll
        for (int h = 0; h < G; ++h) s[tt][h] = part[h];
      }
      // soft-cap and masking once per sub-step, behind uniform branches, so
      // the score products above schedule as one straight block
      if (a.cap_l2 > 0.f) {  // c tanh(s / c), log2 units
#pragma unroll
        for (int tt = 0; tt < TPSC; ++tt)
#pragma unroll
          for (int h = 0; h < G; ++h) s[tt][h] = a.cap_l2 * tanhf(s[tt][h] / a.cap_l2);
      }
      if (multi) {
#pragma unroll
        for (int tt = 0; tt < TPSC; ++tt) {
          const int pos = pos0 + (si * TPSC + tt) * SLOTS + slot;
#pragma unroll
          for (int h = 0; h < G; ++h)
            if (!row_sees(a, h, pos, hi)) s[tt][h] = -CUDART_INF_F;
        }
      } else {
#pragma unroll
        for (int tt = 0; tt < TPSC; ++tt) {
          const int pos = pos0 + (si * TPSC + tt) * SLOTS + slot;
          if (pos < lo || pos >= hi) {
#pragma unroll
            for (int h = 0; h < G; ++h) s[tt][h] = -CUDART_INF_F;
          }
        }
      }
      // running max with slack: rescale only when the max grows by more than kRescaleSlack
      bool need = false;
      float tmax[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        tmax[h] = s[0][h];
#pragma unroll
        for (int tt = 1; tt < TPSC; ++tt) tmax[h] = fmaxf(tmax[h], s[tt][h]);
      }
      if (fresh != 0u) {  // unified max: a row's first finite scores
#pragma unroll
        for (int h = 0; h < G; ++h)
          if (((fresh >> h) & 1u) && tmax[h] > -CUDART_INF_F) {
            if (tmax[h] < m[h] - kPhiDrop) m[h] = tmax[h];
            fresh &= ~(1u << h);
          }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) need |= tmax[h] > m[h] + kRescaleSlack;
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          if (tmax[h] > m[h] + kRescaleSlack) {
            const float alpha = exp2_approx(m[h] - tmax[h]);  // m = -inf -> 0
            l[h] *= alpha;
#pragma unroll
            for (int e = 0; e < E / 2; ++e) {
              acc[h][e].x *= alpha;
              acc[h][e].y *= alpha;
            }
            m[h] = tmax[h];
          }
        }
      }
#pragma unroll
      for (int tt = 0; tt < TPSC; ++tt)
#pragma unroll
        for (int h = 0; h < G; ++h) {
          s[tt][h] = (m[h] == -CUDART_INF_F) ? 0.f : exp2_approx(s[tt][h] - m[h]);
          l[h] += s[tt][h];
        }
#pragma unroll
      for (int tt = 0; tt < TPSC; ++tt) {
        const int r = (si * TPSC + tt) * SLOTS + slot;
        const int pos = pos0 + r;
        if (pos >= lo && pos < hi) {  // masked rows may hold anything: never read them as values
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            float x[EPC];
            load(a, vt, r, k, 102, x);
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
              for (int e = 0; e < EPC; e += 2)
                acc[h][(k * EPC) / 2 + e / 2] = __ffma2_rn(make_float2(s[tt][h], s[tt][h]),
                                                           make_float2(x[e], x[e + 1]),
                                                           acc[h][(k * EPC) / 2 + e / 2]);
          }
        }
      }
    }
    release_k();
  }

  // Merge the slots' states and publish the warp's state.
  __device__ __forceinline__ void end_piece(float* m_area, float* l_area, float* acc_area, int w,
                                            int lane, int /*group*/) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      // a state that saw no finite score holds nothing: its max is -inf (with
      // the unified max it would otherwise report phi)
      const float mh = ((fresh >> h) & 1u) ? -CUDART_INF_F : m[h];
      float M = mh;
#pragma unroll
      for (int off = LPT; off < 32; off <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
      const float sc = (mh == -CUDART_INF_F) ? 0.f : exp2_approx(mh - M);
      float lh = l[h] * sc;
#pragma unroll
      for (int off = LPT; off < 32; off <<= 1) lh += __shfl_xor_sync(0xffffffffu, lh, off);
#pragma unroll
      for (int e = 0; e < E / 2; ++e) {
        float v0 = acc[h][e].x * sc, v1 = acc[h][e].y * sc;
#pragma unroll
        for (int off = LPT; off < 32; off <<= 1) {
          v0 += __shfl_xor_sync(0xffffffffu, v0, off);
          v1 += __shfl_xor_sync(0xffffffffu, v1, off);
        }
        acc[h][e] = make_float2(v0, v1);
      }
      if (lane == 0) {
        m_area[w * G + h] = M;
        l_area[w * G + h] = lh;
      }
      if (slot == 0) {
#pragma unroll
        for (int k = 0; k < CPL; ++k)
#pragma unroll
          for (int e = 0; e < EPC; e += 2) {
            const float2 v = acc[h][(k * EPC + e) / 2];
            acc_area[(w * G + h) * D + dim_of(k, e)] = v.x;
            acc_area[(w * G + h) * D + dim_of(k, e + 1)] = v.y;
          }
      }
    }
  }
};

// ------------------------------------------------------- MMA dataflow
// Scores S^T = K . Q^T on mma.m16n8k16 (16 tokens x 8 query rows x 16 dims
// per instruction, fp32 accumulate); probabilities are transposed in
// registers (movmatrix) into the B operand of O^T += V^T . P^T, with O^T
// (dims x rows) accumulated in fp32 registers.  A block of 8 query rows per
// product; missing rows are zero columns.  bf16 K/V use bf16 operands.  fp8
// and int4 K/V are widened exactly to f16, and q is held in f16 times a
// power of two per row, undone on the fp32 scores.
// R row teams of 8 * NB query rows each (a segment of up to 8 * NB * R rows:
// the query heads of a kv head times the query tokens).  A team's warp
// computes its rows of every tile it takes, in NB blocks of 8 that share
// each K / V fragment (one shared-memory read or conversion feeds NB
// products).  Several teams use 32-token tiles, so that the fewer tile
// lanes keep a deep ring.
// KIND: bf16 (tiles through ldmatrix), fp8 e4m3 or int4 (bytes loaded per
// lane and widened to f16; the query is held as f16 times a power of two).
// HEADS: the R teams are R adjacent kv heads of one segment instead of R
// blocks of rows of one kv head: team t computes the (at most 8) query rows
// of kv head t of the tile, whose rows sit at token * R + t.
template <int D, int KIND, int R = 1, bool HEADS = false, int NB = 1, int TOK = 0>
struct MmaConsumer {
  static constexpr int HT = HEADS ? R : 1;  // kv heads per tile
  static constexpr bool FP8 = KIND == kKvFp8;
  static constexpr bool I4 = KIND == kKvInt4;
  static constexpr bool BF16 = KIND == kKvBf16;
  static_assert(NB == 1 || NB == 2, "one or two row blocks per warp");
  static_assert(!HEADS || NB == 1, "head teams hold one row block");
  static constexpr int ROWB_K = BF16 ? 2 * D : (FP8 ? D : D / 2);  // bytes of one head's row
  // Two row blocks: 64-token tiles with one team (a few spilled registers,
  // measured 5% faster than 32 tokens at 16 rows); with two teams TOK
  // tokens (48 leaves two K and two V slots per tile lane: 7.5% faster than
  // 32 at 32 rows; 32 serves pages that 48 does not divide).
  static_assert(TOK == 0 || TOK % 16 == 0, "tiles are whole 16-token subtiles");
  static constexpr int kTileBytes = HEADS ? 16384
                                    : TOK > 0 ? TOK * ROWB_K
                                    : NB > 1 ? (R == 1 ? (BF16 ? FA_NB2_TOKENS : 64) : 32) * ROWB_K
                                    : FP8 ? FA_FP8_MMA_TILE_BYTES
                                    : I4  ? FA_FP8_MMA_TILE_BYTES / 2
                                          : (R == 1 ? FA_MMA_TILE_BYTES : FA_MMA_TILE_BYTES / 2);
  // Consumer warps: two teams of 3, or four of 2 (a 9-warp block, whose
  // registers are capped at 168 per thread); fp8 rows of 256 dims need more
  // registers than that and take four teams of one warp.  bf16 with two row
  // blocks and one team: 3 warps, so that each tile lane owns two K and two V
  // slots of 64 tokens (the next tile lands while the current one is
  // computed; measured 5% faster than 5 warps with one slot each, while the
  // compute-bound fp8 / int4 variants keep their 7 warps: int4 was 75%
  // slower with 3).
  static constexpr int kWarps = (R == 1 && NB == 2 && BF16) ? FA_NB2_WARPS
                                : R == 1   ? (!BF16 ? FA_FP8_MMA_CONSUMER_WARPS : FA_MMA_CONSUMER_WARPS)
                                : R == 2 ? 6
                                         : (!BF16 && D >= 256 ? 4 : 8);
  // V held longer than K (EARLY_K: one K slot per two V slots) pays where
  // the V half of a tile is the longer one, fp8 with one team of 8 rows;
  // elsewhere equal rings keep the most tiles in flight.
  using C = TileCfg<D, KIND, 8 * NB, R, kTileBytes, kWarps, !BF16 && R == 1 && NB == 1, HT>;
  static constexpr int KS = D / 16;     // k-steps of the score product = m-tiles of O^T
  static constexpr int SUB = C::T / 16;  // 16-token subtiles per tile
  static constexpr int BPT = D / 4;      // fp8 / int4 K: elements of a row owned by one lane
  static constexpr int VBT = D / 8;      // fp8 / int4 V: elements of a row owned by one lane
  static constexpr int KB = I4 ? BPT / 2 : BPT;  // their bytes
  static constexpr int VB = I4 ? VBT / 2 : VBT;
  // Unified max: how far below phi a row's first scores may sit and keep
  // phi.  The fp8 / int4 products carry the probabilities in f16, whose
  // subnormals (below 2^-14) hold them to 2^-24 absolute: with the row's
  // largest weight below 1 that costs up to 2^-8 of relative precision
  // (measured: 1.6% error on a small output), so there a row keeps phi
  // only when its first scores reach it; bf16 probabilities keep 8 exponent
  // bits and allow the full drop.
  static constexpr float kDrop = BF16 ? kPhiDrop : 0.f;
  static_assert(D % 16 == 0 && C::T % 16 == 0, "mma tiling");
  static_assert(!FP8 || C::CB == 128, "fp8 mma path needs 128-byte planes");
  static_assert(!I4 || ((D == 128 || D == 256) && KB % 16 == 0 && (VB == 8 || VB == 16)),
                "int4 mma path: 64- or 128-byte rows");

  uint32_t qb[NB][KS][2];
  float o[NB][KS][4];
  float m[NB][2], l[NB][2];
  uint32_t fresh;  // unified max: bit 2 nb + j set while row 8 nb + 2t + j has seen no finite score
  float sscale[NB][2];
  int g, t;
  int rbase;  // first segment row of this warp's team
  int tr;     // rows of the team (8 NB; with HEADS the group of one kv head)
  int hrow;   // with HEADS: the team's kv head within the tile, else 0

  // Tile row (in units of one head's row) of token r for this team.
  __device__ __forceinline__ int srow(int r) const { return r * HT + hrow; }
  // First kv head of a team relative to its segment's first kv head.
  __host__ __device__ static constexpr int team_head(int team) { return HEADS ? team : 0; }

  // qs: the piece's query rows (staged in shared memory, or in global
  // memory where the tile geometry leaves no room): row r (token r / group,
  // head r % group) at qs + (r / group) * qstride + (r % group) * D; kscale:
  // the fp8 K scale of the piece's kv head (1 for bf16); team: this warp's
  // row team (rows 8 NB team .. 8 NB team + 8 NB - 1).
  __device__ __forceinline__ void begin_piece(const KernelArgs& a, const uint16_t* qs, int qstride,
                                              float kscale, int lane, int team) {
    g = lane >> 2;
    t = lane & 3;
    const int G = a.group * a.q_len;
    tr = HEADS ? a.group / HT : 8 * NB;  // with HEADS: one query token, group rows per head
    rbase = tr * team;
    hrow = HEADS ? team : 0;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const bool real = 8 * nb + g < tr && rbase + 8 * nb + g < G;
      const int r = real ? rbase + 8 * nb + g : 0;
      const uint16_t* qrow = qs + (r / a.group) * qstride + (r % a.group) * D;
      if constexpr (BF16) {
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          qb[nb][kk][0] = real ? *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * t) : 0u;
          qb[nb][kk][1] = real ? *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * t + 8) : 0u;
        }
        sscale[nb][0] = sscale[nb][1] = a.score_scale;
      } else {
        // this lane's q elements: [BPT*t, BPT*t + BPT)
        float mx = 0.f;
        uint32_t qw[BPT / 2];
#pragma unroll
        for (int i = 0; i < BPT / 8; ++i) {
          const uint4 w = real ? *reinterpret_cast<const uint4*>(qrow + BPT * t + 8 * i)
                               : make_uint4(0, 0, 0, 0);
          qw[4 * i] = w.x;
          qw[4 * i + 1] = w.y;
          qw[4 * i + 2] = w.z;
          qw[4 * i + 3] = w.w;
        }
#pragma unroll
        for (int i = 0; i < BPT / 2; ++i)
          mx = fmaxf(mx, fmaxf(fabsf(bf16lo(qw[i])), fabsf(bf16hi(qw[i]))));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        int ex = 0;
        frexpf(mx, &ex);
        const int sh = (mx > 0.f && isfinite(mx)) ? 15 - ex : 0;  // |q| * 2^sh < 2^15
        const float mul = ldexpf(1.f, sh);
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          if constexpr (FP8) {
            // logical k-columns 2t,2t+1 / 2t+8,2t+9 of step kk <-> bytes BPT*t + 4kk + {0,1} / {2,3}
            const uint32_t w0 = qw[2 * kk], w1 = qw[2 * kk + 1];
            qb[nb][kk][0] = pack_f16x2(bf16lo(w0) * mul, bf16hi(w0) * mul);
            qb[nb][kk][1] = pack_f16x2(bf16lo(w1) * mul, bf16hi(w1) * mul);
          } else {
            // int4: logical k-columns 2t,2t+1 / 2t+8,2t+9 of step kk <-> the
            // lane's elements (8j + 2c, 8j + 2c + 4) / (8j + 2c + 1, 8j + 2c + 5),
            // j = kk / 2, c = kk % 2: the nibble pairs one shift and one mask
            // take out of K's 32-bit word j.  The second pair is widened to
            // 16 times its codes, so its q values carry 1/16 (exact: a power
            // of two, with max |q| scaled to [2^10, 2^11) here)
            const int e = 8 * (kk >> 1) + 2 * (kk & 1);
            const float mul16 = mul * 0.0625f;
            auto qe = [&](int i) { return (i & 1) ? bf16hi(qw[i >> 1]) : bf16lo(qw[i >> 1]); };
            qb[nb][kk][0] = pack_f16x2(qe(e) * mul, qe(e + 4) * mul);
            qb[nb][kk][1] = pack_f16x2(qe(e + 1) * mul16, qe(e + 5) * mul16);
          }
        }
        const int sh0 = __shfl_sync(0xffffffffu, sh, (2 * t) * 4);
        const int sh1 = __shfl_sync(0xffffffffu, sh, (2 * t + 1) * 4);
        const float base = a.score_scale * kscale;
        sscale[nb][0] = base * ldexpf(1.f, -sh0);
        sscale[nb][1] = base * ldexpf(1.f, -sh1);
      }
#pragma unroll
      for (int mt = 0; mt < KS; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[nb][mt][i] = 0.f;
      m[nb][0] = m[nb][1] = a.m_init;
      l[nb][0] = l[nb][1] = 0.f;
    }
    fresh = a.m_init > -CUDART_INF_F ? (1u << (2 * NB)) - 1u : 0u;
  }

  __device__ __forceinline__ uint32_t chunk_addr(uint32_t tile, int row, int chunk, int swz) const {
    return tile_addr<C>(tile, row, chunk >> 3, chunk & 7, swz);
  }
  // Shared address of byte `off` of tile row `row` (a srow() index):
  // swizzled 128-byte planes, or one unswizzled plane for rows narrower than
  // 128 bytes.
  __device__ __forceinline__ uint32_t byte_addr(uint32_t tile, int row, int off, int swz) const {
    if constexpr (C::CB == 128)
      return chunk_addr(tile, row, off >> 4, swz) + (off & 15);
    else
      return tile + row * C::ROWB + off;
  }

  // One subtile's scores for every row block: each K fragment is read (or
  // widened) once and feeds NB products.  Two accumulators per block (even /
  // odd k-steps) halve the dependent chain of mma.
  __device__ __forceinline__ void scores(const KernelArgs& a, uint32_t kt, int sub, int lane,
                                         float (&c)[NB][4]) const {
    const int swz = a.swz;
    float c2[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int i = 0; i < 4; ++i) c[nb][i] = c2[nb][i] = 0.f;
    if constexpr (BF16) {
      const int row = sub * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        uint32_t af[4];
        const int ch = kk * 2 + (lane >> 4);
        if constexpr (C::CB == 128)
          ldsm_x4(ldsm_addr_in(a.status, chunk_addr(kt, srow(row), ch, swz), kt, C::TILE_BYTES, 201), af);
        else  // 64-element rows: one plane of CB bytes, no swizzle
          ldsm_x4(ldsm_addr_in(a.status, kt + srow(row) * C::CB + ch * 16, kt, C::TILE_BYTES, 202), af);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          if (kk & 1)
            mma_bf16(c2[nb], af, qb[nb][kk][0], qb[nb][kk][1]);
          else
            mma_bf16(c[nb], af, qb[nb][kk][0], qb[nb][kk][1]);
        }
      }
    } else {
      const int r0 = sub * 16 + g, r1 = r0 + 8;
      uint32_t w0[KB / 4], w1[KB / 4];
#pragma unroll
      for (int i = 0; i < KB / 16; ++i) {
        const int off = KB * t + 16 * i;
        const uint4 x0 = lds128_in(a.status, byte_addr(kt, srow(r0), off, swz), kt, C::TILE_BYTES, 203);
        const uint4 x1 = lds128_in(a.status, byte_addr(kt, srow(r1), off, swz), kt, C::TILE_BYTES, 204);
        w0[4 * i] = x0.x; w0[4 * i + 1] = x0.y; w0[4 * i + 2] = x0.z; w0[4 * i + 3] = x0.w;
        w1[4 * i] = x1.x; w1[4 * i + 1] = x1.y; w1[4 * i + 2] = x1.z; w1[4 * i + 3] = x1.w;
      }
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        uint32_t af[4];
        if constexpr (I4) {
          // word kk / 2 of each row, shifted down by 8c bits (c = kk % 2):
          // its bits 0-3 / 16-19 and 4-7 / 20-23 are the nibble pairs of
          // the lane's elements listed in begin_piece; the second pair
          // widens to 16 times its codes, and begin_piece gives the q
          // values it meets a factor 1/16
          const int sh = 8 * (kk & 1);
          const uint32_t x0 = w0[kk >> 1] >> sh, x1 = w1[kk >> 1] >> sh;
          af[0] = int4_lo_to_f16x2(x0, kInt4Bias);
          af[1] = int4_lo_to_f16x2(x1, kInt4Bias);
          af[2] = int4_hi_to_f16x2(x0, kInt4Bias);
          af[3] = int4_hi_to_f16x2(x1, kInt4Bias);
        } else {
          af[0] = e4m3x2_to_f16x2(static_cast<uint16_t>(w0[kk] & 0xFFFFu));
          af[1] = e4m3x2_to_f16x2(static_cast<uint16_t>(w1[kk] & 0xFFFFu));
          af[2] = e4m3x2_to_f16x2(static_cast<uint16_t>(w0[kk] >> 16));
          af[3] = e4m3x2_to_f16x2(static_cast<uint16_t>(w1[kk] >> 16));
        }
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          if (kk & 1)
            mma_f16(c2[nb], af, qb[nb][kk][0], qb[nb][kk][1]);
          else
            mma_f16(c[nb], af, qb[nb][kk][0], qb[nb][kk][1]);
        }
      }
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int i = 0; i < 4; ++i) c[nb][i] += c2[nb][i];
  }

  // One tile: the scores of all SUB subtiles first (independent mma chains),
  // one softmax update for the whole tile, then O^T += V^T P^T per subtile.
  // release_k() is called as soon as the K tile is no longer read.
  template <class ReleaseK>
  __device__ __forceinline__ void tile(const KernelArgs& a, uint32_t kt, uint32_t vt, int pos0,
                                       int lo, int hi, int lane, ReleaseK&& release_k) {
    float sc[SUB][NB][4];
#pragma unroll
    for (int sub = 0; sub < SUB; ++sub) scores(a, kt, sub, lane, sc[sub]);
    release_k();
    float mx[NB][2];
    bool up = false;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      // key range of this lane's two columns (rows 8 nb + 2t, + 1: query
      // token row / group sees one key fewer per token before the last,
      // within its own window); [lo, hi) is the union, and padding columns
      // keep it
      const int rr = rbase + 8 * nb + 2 * t;
      int chi0 = hi - (a.q_len - 1 - rr / a.group);
      int chi1 = hi - (a.q_len - 1 - (rr + 1) / a.group);
      chi0 = chi0 < hi ? chi0 : hi;
      chi1 = chi1 < hi ? chi1 : hi;
      const int clo0 = (a.window > 0 && chi0 > a.window) ? chi0 - a.window : 0;
      const int clo1 = (a.window > 0 && chi1 > a.window) ? chi1 - a.window : 0;
      float mx0 = -CUDART_INF_F, mx1 = -CUDART_INF_F;
#pragma unroll
      for (int sub = 0; sub < SUB; ++sub) {
        float* s = sc[sub][nb];
        const int pr = pos0 + sub * 16 + g;
        const bool v00 = pr >= clo0 && pr < chi0, v01 = pr >= clo1 && pr < chi1;
        const bool v80 = pr + 8 >= clo0 && pr + 8 < chi0, v81 = pr + 8 >= clo1 && pr + 8 < chi1;
        s[0] *= sscale[nb][0];
        s[1] *= sscale[nb][1];
        s[2] *= sscale[nb][0];
        s[3] *= sscale[nb][1];
        if (a.cap_l2 > 0.f) {  // soft-cap: c tanh(s / c) (log2 units), before the masks
#pragma unroll
          for (int e = 0; e < 4; ++e) s[e] = a.cap_l2 * tanhf(s[e] / a.cap_l2);
        }
        // a masked key has weight zero: -inf, never the cap's floor -c
        s[0] = v00 ? s[0] : -CUDART_INF_F;
        s[1] = v01 ? s[1] : -CUDART_INF_F;
        s[2] = v80 ? s[2] : -CUDART_INF_F;
        s[3] = v81 ? s[3] : -CUDART_INF_F;
        mx0 = fmaxf(mx0, fmaxf(s[0], s[2]));
        mx1 = fmaxf(mx1, fmaxf(s[1], s[3]));
      }
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      if (fresh != 0u) {  // unified max: the rows' first finite scores (row-uniform: mx is reduced)
        const uint32_t b0 = 1u << (2 * nb), b1 = b0 << 1;
        if ((fresh & b0) && mx0 > -CUDART_INF_F) {
          if (mx0 < m[nb][0] - kDrop) m[nb][0] = mx0;
          fresh &= ~b0;
        }
        if ((fresh & b1) && mx1 > -CUDART_INF_F) {
          if (mx1 < m[nb][1] - kDrop) m[nb][1] = mx1;
          fresh &= ~b1;
        }
      }
      mx[nb][0] = mx0;
      mx[nb][1] = mx1;
      up |= mx0 > m[nb][0] + kRescaleSlack || mx1 > m[nb][1] + kRescaleSlack;
    }
    if (__any_sync(0xffffffffu, up)) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const bool up0 = mx[nb][0] > m[nb][0] + kRescaleSlack, up1 = mx[nb][1] > m[nb][1] + kRescaleSlack;
        const float a0 = up0 ? exp2_approx(m[nb][0] - mx[nb][0]) : 1.f;
        const float a1 = up1 ? exp2_approx(m[nb][1] - mx[nb][1]) : 1.f;
        if (up0) m[nb][0] = mx[nb][0];
        if (up1) m[nb][1] = mx[nb][1];
        l[nb][0] *= a0;
        l[nb][1] *= a1;
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          o[nb][mt][0] *= a0;
          o[nb][mt][1] *= a1;
          o[nb][mt][2] *= a0;
          o[nb][mt][3] *= a1;
        }
      }
    }
    // P enters the tensor core as hi + lo 16-bit parts (two products), so the
    // weights keep ~16 significant bits instead of 8 (bf16) or 11 (f16).
    uint32_t pb[SUB][NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const bool dead0 = m[nb][0] == -CUDART_INF_F, dead1 = m[nb][1] == -CUDART_INF_F;
#pragma unroll
      for (int sub = 0; sub < SUB; ++sub) {
        const float* s = sc[sub][nb];
        const float p0 = dead0 ? 0.f : exp2_approx(s[0] - m[nb][0]);
        const float p1 = dead1 ? 0.f : exp2_approx(s[1] - m[nb][1]);
        const float p2 = dead0 ? 0.f : exp2_approx(s[2] - m[nb][0]);
        const float p3 = dead1 ? 0.f : exp2_approx(s[3] - m[nb][1]);
        l[nb][0] += p0 + p2;
        l[nb][1] += p1 + p3;
        uint32_t x0, x1, y0, y1;
        if constexpr (!BF16) {  // the f16 product of the fp8 / int4 dataflow
          x0 = pack_f16x2(p0, p1);
          x1 = pack_f16x2(p2, p3);
          const float2 h0 = f16x2_to_float2(x0), h1 = f16x2_to_float2(x1);
          y0 = pack_f16x2(p0 - h0.x, p1 - h0.y);
          y1 = pack_f16x2(p2 - h1.x, p3 - h1.y);
        } else {
          x0 = pack_bf16x2(p0, p1);
          x1 = pack_bf16x2(p2, p3);
          y0 = pack_bf16x2(p0 - bf16lo(x0), p1 - bf16hi(x0));
          y1 = pack_bf16x2(p2 - bf16lo(x1), p3 - bf16hi(x1));
        }
        pb[sub][nb][0] = movmatrix_trans(x0);  // P[row g][tokens 2t, 2t+1]
        pb[sub][nb][1] = movmatrix_trans(x1);  // P[row g][tokens 2t+8, 2t+9]
        pb[sub][nb][2] = movmatrix_trans(y0);
        pb[sub][nb][3] = movmatrix_trans(y1);
      }
    }
#pragma unroll
    for (int sub = 0; sub < SUB; ++sub) {
      // rows that are not visible may hold anything (NaN included): zero them in V
      const int pt = pos0 + sub * 16 + 2 * t;
      const bool e0 = pt >= lo && pt < hi, e1 = pt + 1 >= lo && pt + 1 < hi;
      const bool e8 = pt + 8 >= lo && pt + 8 < hi, e9 = pt + 9 >= lo && pt + 9 < hi;
      const bool edge = __any_sync(0xffffffffu, !(e0 && e1 && e8 && e9));
      const uint32_t mk01 = (e0 ? 0x0000FFFFu : 0u) | (e1 ? 0xFFFF0000u : 0u);
      const uint32_t mk89 = (e8 ? 0x0000FFFFu : 0u) | (e9 ? 0xFFFF0000u : 0u);
      if constexpr (BF16) {
        const int vrow = sub * 16 + (lane & 7) + (lane >> 4) * 8;
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          uint32_t af[4];
          const int ch = mt * 2 + ((lane >> 3) & 1);
          if constexpr (C::CB == 128)
            ldsm_x4_trans(ldsm_addr_in(a.status, chunk_addr(vt, srow(vrow), ch, a.swz), vt, C::TILE_BYTES, 205), af);
          else
            ldsm_x4_trans(ldsm_addr_in(a.status, vt + srow(vrow) * C::CB + ch * 16, vt, C::TILE_BYTES, 206), af);
          if (edge) {
            af[0] &= mk01;
            af[1] &= mk01;
            af[2] &= mk89;
            af[3] &= mk89;
          }
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            mma_bf16(o[nb][mt], af, pb[sub][nb][0], pb[sub][nb][1]);
            mma_bf16(o[nb][mt], af, pb[sub][nb][2], pb[sub][nb][3]);
          }
        }
      } else if constexpr (I4) {
        // lane owns dims [VBT*g, VBT*g + VBT) (VB bytes) of tokens 2t, 2t+1,
        // 2t+8, 2t+9.  Byte b = 2u + s of two tokens' chunks, permuted into
        // bytes 0 and 2 of one word, holds the f16 pairs (tok0, tok1) of
        // dims 2b (low nibbles) and 2b + 1 (high nibbles, widened to 16
        // times their codes): m-tile b takes dims 4u + 2s (row g) and
        // 4u + 2s + 1 (row g + 8), as out_dim states, and end_piece takes
        // the factor 16 off the row g + 8 accumulators.
        const int rb = sub * 16 + 2 * t;
        const int rows[4] = {rb, rb + 1, rb + 8, rb + 9};
        uint32_t vw[4][VB / 4];
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          if constexpr (VB == 8) {
            const uint2 x = lds64_in(a.status, byte_addr(vt, srow(rows[rr]), VB * g, a.swz), vt, C::TILE_BYTES, 208);
            vw[rr][0] = x.x;
            vw[rr][1] = x.y;
          } else {
            const uint4 x = lds128_in(a.status, byte_addr(vt, srow(rows[rr]), VB * g, a.swz), vt, C::TILE_BYTES, 209);
            vw[rr][0] = x.x;
            vw[rr][1] = x.y;
            vw[rr][2] = x.z;
            vw[rr][3] = x.w;
          }
        }
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          const int u = mt >> 1;
          const uint32_t byt = mt & 3;  // byte of the tokens' word u / 2
          const uint32_t sel = byt | ((4u + byt) << 8);  // -> bytes 0 and 2
          const uint32_t z01 = prmt(vw[0][u >> 1], vw[1][u >> 1], sel);
          const uint32_t z89 = prmt(vw[2][u >> 1], vw[3][u >> 1], sel);
          uint32_t af[4];
          af[0] = int4_lo_to_f16x2(z01, kInt4Bias);
          af[1] = int4_hi_to_f16x2(z01, kInt4Bias);
          af[2] = int4_lo_to_f16x2(z89, kInt4Bias);
          af[3] = int4_hi_to_f16x2(z89, kInt4Bias);
          if (edge) {
            af[0] &= mk01;
            af[1] &= mk01;
            af[2] &= mk89;
            af[3] &= mk89;
          }
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            mma_f16(o[nb][mt], af, pb[sub][nb][0], pb[sub][nb][1]);
            mma_f16(o[nb][mt], af, pb[sub][nb][2], pb[sub][nb][3]);
          }
        }
      } else {
        // lane owns dims [VBT*g, VBT*g + VBT) of tokens 2t, 2t+1, 2t+8, 2t+9
        const int rb = sub * 16 + 2 * t;
        const int rows[4] = {rb, rb + 1, rb + 8, rb + 9};
        uint32_t vw[4][VBT / 4];
#pragma unroll
        for (int rr = 0; rr < 4; ++rr)
#pragma unroll
          for (int i = 0; i < VBT / 16; ++i) {
            const uint4 x = lds128_in(a.status, chunk_addr(vt, srow(rows[rr]), (VBT * g) / 16 + i, a.swz), vt,
                                      C::TILE_BYTES, 207);
            vw[rr][4 * i] = x.x;
            vw[rr][4 * i + 1] = x.y;
            vw[rr][4 * i + 2] = x.z;
            vw[rr][4 * i + 3] = x.w;
          }
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
          const uint32_t x01 = prmt(vw[0][mt >> 1], vw[1][mt >> 1], sel);
          const uint32_t x89 = prmt(vw[2][mt >> 1], vw[3][mt >> 1], sel);
          uint32_t af[4];
          af[0] = e4m3x2_to_f16x2(static_cast<uint16_t>(x01 & 0xFFFFu));
          af[1] = e4m3x2_to_f16x2(static_cast<uint16_t>(x01 >> 16));
          af[2] = e4m3x2_to_f16x2(static_cast<uint16_t>(x89 & 0xFFFFu));
          af[3] = e4m3x2_to_f16x2(static_cast<uint16_t>(x89 >> 16));
          if (edge) {
            af[0] &= mk01;
            af[1] &= mk01;
            af[2] &= mk89;
            af[3] &= mk89;
          }
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            mma_f16(o[nb][mt], af, pb[sub][nb][0], pb[sub][nb][1]);
            mma_f16(o[nb][mt], af, pb[sub][nb][2], pb[sub][nb][3]);
          }
        }
      }
    }
  }

  __device__ __forceinline__ int out_dim(int mt, int half) const {
    if constexpr (!BF16)
      return VBT * g + 2 * mt + half;
    else
      return mt * 16 + g + 8 * half;
  }

  // Park this warp's state for its team's rows as tile lane w's state.
  __device__ __forceinline__ void end_piece(float* m_area, float* l_area, float* acc_area, int w,
                                            int lane, int G) {
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      float l0 = l[nb][0], l1 = l[nb][1];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
      }
      const int lr = 8 * nb + 2 * t;  // team-local row of column 0
      const int h0 = rbase + lr, h1 = h0 + 1;
      const bool r0 = lr < tr && h0 < G, r1 = lr + 1 < tr && h1 < G;
      const uint32_t b0 = 1u << (2 * nb), b1 = b0 << 1;
      if (g == 0) {  // a row that saw no finite score holds nothing: max -inf (not phi)
        if (r0) m_area[w * G + h0] = (fresh & b0) ? -CUDART_INF_F : m[nb][0];
        if (r1) m_area[w * G + h1] = (fresh & b1) ? -CUDART_INF_F : m[nb][1];
        if (r0) l_area[w * G + h0] = l0;
        if (r1) l_area[w * G + h1] = l1;
      }
      // int4: the odd dims were summed from values 16 times the codes
      constexpr float kOdd = I4 ? 0.0625f : 1.f;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        if (r0) {
          acc_area[(w * G + h0) * D + out_dim(mt, 0)] = o[nb][mt][0];
          acc_area[(w * G + h0) * D + out_dim(mt, 1)] = o[nb][mt][2] * kOdd;
        }
        if (r1) {
          acc_area[(w * G + h1) * D + out_dim(mt, 0)] = o[nb][mt][1];
          acc_area[(w * G + h1) * D + out_dim(mt, 1)] = o[nb][mt][3] * kOdd;
        }
      }
    }
  }
};

// ------------------------------------------------------------- kernel
// Block shared memory, from a 1024-aligned base:
//   K ring [KSTAGES][tile] | V ring [VSTAGES][tile] |
//   fullK[KSTAGES], emptyK[KSTAGES], fullV[VSTAGES], emptyV[VSTAGES] mbarriers |
//   m[NT][G], l[NT][G] | acc[NT][G][D] | merge counter, merge mbarrier |
//   pages[64] | q mbarriers, q slots, scales | start[B], len[B], pre[B+1]
template <class Cons>
struct SmemLayout {
  using C = typename Cons::C;
  static constexpr int D = C::DIM;
  static constexpr int kBars = C::RING_BYTES;
  static constexpr int kMerge = kBars + 2 * (C::KSTAGES + C::VSTAGES) * 8;
  __host__ __device__ static constexpr int acc_off(int G) {
    return kMerge + ((C::NT * G * 2 * 4 + 15) / 16) * 16;
  }
  __host__ __device__ static constexpr int misc_off(int G) { return acc_off(G) + C::NT * G * D * 4; }
  // misc: merge counter (4 B), pad, merge-free mbarrier (8 B), then 64
  // staged page ids (256 B)
  // q area: qfull[2], qempty[2] mbarriers (32 B) | q slots [2][QSLOT_BYTES]
  // (if STAGE_Q) | fp8: k scales [kScaleCap], v scales [kScaleCap]
  __host__ __device__ static constexpr int q_off(int G) { return misc_off(G) + 16 + 256; }
  __host__ __device__ static constexpr int sched_off(int G) { return q_off(G) + C::QAREA_BYTES; }
  static constexpr size_t bytes(int batch, int G) {
    return 1024 + static_cast<size_t>(sched_off(G)) + static_cast<size_t>(3 * batch + 1) * 4;
  }
};

// Registers per thread: each of an SM's four sub-partitions holds 16384, and
// a block's warps are spread over them, so a block of 9 to 12 warps (3 on
// some sub-partition) may use at most 168 per thread; up to 8 warps, 224.
template <class Cons>
__host__ __device__ constexpr int max_regs() {
  return Cons::C::THREADS > 8 * 32 ? 168 : 224;
}

template <class Cons>
__global__ void __maxnreg__(max_regs<Cons>())
    fa_decode_kernel(const __grid_constant__ KernelArgs a) {
  using C = typename Cons::C;
  using S = SmemLayout<Cons>;
  constexpr int D = C::DIM;
  constexpr int T = C::T;
  constexpr int NW = C::NW;
  constexpr int NT = C::NT;  // tile lanes (NW / row teams)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (sbase - raw);
  const uint32_t ring = sbase;
  const uint32_t full0 = sbase + S::kBars;
  const uint32_t empty0 = full0 + C::KSTAGES * 8;    // K slots: full0[s], empty0[s]
  const uint32_t vfull0 = empty0 + C::KSTAGES * 8;   // V slots: vfull0[s], vempty0[s]
  const uint32_t vempty0 = vfull0 + C::VSTAGES * 8;
  const uint32_t vring = ring + C::KSTAGES * C::TILE_BYTES;
  // Separate K and V barriers only where the rings differ in depth.  With
  // equal depths a tile's K and V copies complete on its K slot's barriers
  // and are released together: a second wait and a second release per tile
  // measured slower in the paged producer loop (one copy per page, so the
  // loop's length bounds how fast copies go out), for no gain.
  constexpr bool kSplitKV = C::KSTAGES != C::VSTAGES;
  // A segment's rows are its group's query heads for each of the request's
  // query tokens: row r is token r / GK, head r % GK of the group.
  const int GK = a.group, Q = a.q_len;
  const int G = GK * Q;
  float* m_area = reinterpret_cast<float*>(base + S::kMerge);
  float* l_area = m_area + NT * G;
  float* acc_area = reinterpret_cast<float*>(base + S::acc_off(G));
  int* s_mcnt = reinterpret_cast<int*>(base + S::misc_off(G));  // warps done with the open piece
  const uint32_t mfree = sbase + S::misc_off(G) + 8;              // completes when a piece is merged
  int* s_pages = reinterpret_cast<int*>(base + S::misc_off(G)) + 4;
  const uint32_t qfull0 = sbase + S::q_off(G), qempty0 = qfull0 + 16;  // [2] each
  uint16_t* q_slots = reinterpret_cast<uint16_t*>(base + S::q_off(G) + 32);
  float* s_kscale = reinterpret_cast<float*>(base + S::q_off(G) + 32 + (C::STAGE_Q ? 2 * C::QSLOT_BYTES : 0));
  float* s_vscale = s_kscale + kScaleCap;
  int* s_start = reinterpret_cast<int*>(base + S::sched_off(G));
  const int B = a.batch, H = a.kv_heads;
  int* s_len = s_start + B;
  int* s_pre = s_len + B;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ps = a.paged ? (1 << a.page_shift) : 0;
  if (tid == 0) {  // kernel parameters: safe to touch before the wait below
    prefetch_tensormap(&a.kmap);
    prefetch_tensormap(&a.vmap);
  }
  // Nothing in global memory is read or written before the work that
  // precedes this launch on the stream has finished (this kernel may be
  // placed early as a programmatic dependent of it).
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- setup: request lengths (validated), barriers, tile prefix sums
  load_lengths(a, s_start, s_len);
  const int HK = H * C::HT;  // kv heads (a segment covers HT of them)
  const bool scales_in_smem = HK <= kScaleCap;
  if (C::QUANT && scales_in_smem) {
    for (int i = tid; i < HK; i += blockDim.x) {
      s_kscale[i] = __ldg(a.k_scale + i);
      s_vscale[i] = __ldg(a.v_scale + i);
    }
  }
  if (tid == 32) {
    // a slot is free again once every row team's warp has released it
    for (int s = 0; s < C::KSTAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, C::TEAMS);
    }
    for (int s = 0; s < C::VSTAGES; ++s) {
      mbar_init(vfull0 + 8 * s, 1);
      mbar_init(vempty0 + 8 * s, C::TEAMS);
    }
    mbar_init(mfree, 1);
    *s_mcnt = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(qfull0 + 8 * s, 1);
      mbar_init(qempty0 + 8 * s, NW);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) tile_prefix(a, s_len, s_pre, T, lane);
  __syncthreads();

  const int P = gridDim.x, c = blockIdx.x;
  PieceIter it = block_run(a, s_pre, P, c);

  // The merge kernel may be scheduled now (it waits for this grid to finish
  // before it reads anything this grid writes).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // a consumer thread: the producer lane goes straight to its copies
  if (tid == 32) write_boundary_record(a, it, s_pre, s_len, T, c);

  if (warp == 0) {
    // ================= producer
    // Lane 0 walks the block's tiles in order and, per tile, waits for its
    // ring stage to be free, arms the stage's barrier with the tile's bytes
    // and issues the bulk tensor copies.  Tiles go out in windows.  For paged
    // KV the page ids of the current window sit in shared memory (read from
    // the page table by the whole warp, coalesced), so lane 0's loop has no
    // global loads and no warp-wide operations; the next window's ids are
    // loaded into registers before lane 0 issues the current window and
    // stored after it, so the page-table round trip overlaps the copies.
    const uint64_t pol = l2_evict_first_policy();
    const int NB = T / a.box_t;  // boxes per tile (paged: one page each, contiguous: 1)
    // tiles per window of 64 page ids (a window that starts inside a page may
    // touch one page more than its token count suggests)
    const int win_paged = !a.paged ? 1 : (ps >= T ? 63 * (ps / T) : (64 * ps) / T);
    int ks = 0, vs = 0;          // lane 0's ring positions (K slot, V slot)
    uint32_t kph = 0, vph = 0;   // and their wrap parities
    int issued = 0;              // tiles whose K and V copies were issued
    int pq = 0;                  // pieces whose query rows were staged
    bool ok = true;
    // this lane's two page ids of the window starting at tile w of piece p
    auto load_ids = [&](const Piece& p, int w, int (&v)[2], bool (&in)[2]) {
      const int np = (s_len[p.b] + ps - 1) >> a.page_shift;
      const int pb = (w * T) >> a.page_shift;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int e = pb + half * 32 + lane;
        in[half] = e < np;
        v[half] = in[half] ? __ldg(a.page_table + static_cast<long long>(p.b) * a.pt_stride + e) : -1;
      }
    };
    auto store_ids = [&](const int (&v)[2], const bool (&in)[2]) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        int x = v[half];
        if (in[half] && (x < 0 || static_cast<long long>(x) >= a.kv_rows)) {
          atomicOr(a.status, kFlagBadPage);
          x = -1;  // the copy reads out of range: zeros, no memory access
        }
        s_pages[half * 32 + lane] = in[half] ? x : -1;
      }
    };
    Piece pc;
    bool have = next_piece(it, pc, s_pre, s_len, B, H, a.window_u, T);
    int w0 = have ? pc.t0 : 0;
    if (have && a.paged) {
      int v[2];
      bool in[2];
      load_ids(pc, w0, v, in);
      store_ids(v, in);
      __syncwarp();
    }
    while (ok && have) {
      const int L = s_len[pc.b];
      if (w0 == pc.t0) {
        // stage the piece's G query rows (contiguous in q) in q slot pq % 2
        // once the consumers have read what the slot held two pieces ago
        if (C::STAGE_Q && lane == 0) {
          const int qs = pq & 1;
          const uint32_t qpar = ((pq >> 1) & 1) ^ 1u;
          if (!mbar_wait(qempty0 + 8 * qs, qpar, kWaitLimitNs)) {
            record_timeout(a.status, 5, pq, qs, qpar, qempty0 + 8 * qs);
            ok = false;
          } else {
            // one copy per query token: its GK rows are contiguous in q
            const uint32_t tbytes = static_cast<uint32_t>(GK * D * 2);
            const uint32_t qbytes = tbytes * static_cast<uint32_t>(Q);
            if (FA_CHECK(a.status, qbytes <= static_cast<uint32_t>(C::QSLOT_BYTES), 304, qbytes)) {
              mbar_arrive_expect_tx(qfull0 + 8 * qs, qbytes);
              for (int i = 0; i < Q; ++i)
                bulk_load(smem_addr(q_slots) + qs * C::QSLOT_BYTES + i * tbytes,
                          a.q + ((static_cast<size_t>(pc.b) * Q + i) * a.qo_heads +
                                 static_cast<size_t>(pc.h) * GK) * D,
                          tbytes, qfull0 + 8 * qs);
            }
          }
        }
        ++pq;
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      const int w1 = a.paged && w0 + win_paged < pc.t1 ? w0 + win_paged : pc.t1;
      // the window after this one: the rest of this piece, else the next piece
      PieceIter itn = it;
      Piece pn = pc;
      int nw0 = w1;
      bool nhave = true;
      if (w1 >= pc.t1) {
        nhave = next_piece(itn, pn, s_pre, s_len, B, H, a.window_u, T);
        nw0 = nhave ? pn.t0 : 0;
      }
      int nv[2] = {-1, -1};
      bool nin[2] = {false, false};
      if (a.paged && nhave) load_ids(pn, nw0, nv, nin);  // in flight during the issue loop
      const int npages = a.paged ? (L + ps - 1) >> a.page_shift : 0;
      const int pbase = a.paged ? (w0 * T) >> a.page_shift : 0;
      if (lane == 0) {
        for (int tt = w0; tt < w1; ++tt) {
          // both slots first, then the K and V copies of each box back to back
          // (one pass over the boxes keeps lane 0's issue loop as short as a
          // single ring's: paged tiles take one copy per page and the loop's
          // length bounds how fast copies go out).  V is waited for first: a
          // warp frees its V slot after its K slot, so the K wait then passes
          // without a second suspension.
          if (kSplitKV && !mbar_wait(vempty0 + 8 * vs, vph ^ 1u, kWaitLimitNs)) {
            record_timeout(a.status, 8, issued, vs, vph ^ 1u, vempty0 + 8 * vs);
            ok = false;
            break;
          }
          if (!mbar_wait(empty0 + 8 * ks, kph ^ 1u, kWaitLimitNs)) {
            record_timeout(a.status, 1, issued, ks, kph ^ 1u, empty0 + 8 * ks);
            ok = false;
            break;
          }
          const uint32_t kfb = full0 + 8 * ks, vfb = kSplitKV ? vfull0 + 8 * vs : kfb;
          const uint32_t kdst = ring + ks * C::TILE_BYTES, vdst = vring + vs * C::TILE_BYTES;
          if constexpr (kSplitKV) {
            mbar_arrive_expect_tx(kfb, C::TILE_BYTES);
            mbar_arrive_expect_tx(vfb, C::TILE_BYTES);
          } else {
            mbar_arrive_expect_tx(kfb, 2 * C::TILE_BYTES);
          }
          if (!a.paged) {
            const int row = s_start[pc.b] + tt * T;
            if constexpr (C::TOKEN_MAJOR) {
              tma_load_4d(kdst, &a.kmap, kfb, 0, 0, pc.h * C::HT, row, pol);
              tma_load_4d(vdst, &a.vmap, vfb, 0, 0, pc.h * C::HT, row, pol);
            } else {
#pragma unroll
              for (int p = 0; p < C::NP; ++p) {
                const uint32_t off = p * (T * C::CB);
                if (FA_CHECK(a.status, off + T * C::CB <= C::TILE_BYTES && (off & 127u) == 0, 301, off)) {
                  tma_load_3d(kdst + off, &a.kmap, kfb, p * (C::CB / C::ES), pc.h, row, pol);
                  tma_load_3d(vdst + off, &a.vmap, vfb, p * (C::CB / C::ES), pc.h, row, pol);
                }
              }
            }
          } else if constexpr (C::TOKEN_MAJOR) {
            for (int jb = 0; jb < NB; ++jb) {
              const int tok = tt * T + jb * a.box_t;
              const int pidx = tok >> a.page_shift;
              const int page = (pidx < npages && pidx - pbase < 64) ? s_pages[pidx - pbase] : -1;
              const int slot0 = tok & (ps - 1);
              const uint32_t off = jb * a.box_t * C::TOKB;
              if (FA_CHECK(a.status, off + a.box_t * C::TOKB <= C::TILE_BYTES && (off & 127u) == 0 &&
                                         pidx - pbase >= 0 && pidx - pbase < 64,
                           303, off)) {
                tma_load_5d(kdst + off, &a.kmap, kfb, 0, 0, pc.h * C::HT, slot0, page, pol);
                tma_load_5d(vdst + off, &a.vmap, vfb, 0, 0, pc.h * C::HT, slot0, page, pol);
              }
            }
          } else {
            for (int jb = 0; jb < NB; ++jb) {
              const int tok = tt * T + jb * a.box_t;
              const int pidx = tok >> a.page_shift;
              const int page = (pidx < npages && pidx - pbase < 64) ? s_pages[pidx - pbase] : -1;
              const int slot0 = tok & (ps - 1);
#pragma unroll
              for (int p = 0; p < C::NP; ++p) {
                const uint32_t off = p * (T * C::CB) + jb * a.box_t * C::CB;
                if (FA_CHECK(a.status, off + a.box_t * C::CB <= C::TILE_BYTES && (off & 127u) == 0 &&
                                           pidx - pbase >= 0 && pidx - pbase < 64,
                             302, off)) {
                  tma_load_4d(kdst + off, &a.kmap, kfb, p * (C::CB / C::ES), pc.h, slot0, page, pol);
                  tma_load_4d(vdst + off, &a.vmap, vfb, p * (C::CB / C::ES), pc.h, slot0, page, pol);
                }
              }
            }
          }
          ++issued;
          if (++ks == C::KSTAGES) {
            ks = 0;
            kph ^= 1u;
          }
          if (++vs == C::VSTAGES) {
            vs = 0;
            vph ^= 1u;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      __syncwarp();
      if (a.paged && nhave) store_ids(nv, nin);
      __syncwarp();
      if (w1 >= pc.t1) {
        have = nhave;
        pc = pn;
        it = itn;
        w0 = nw0;
      } else {
        w0 = w1;
      }
    }
    // drain: every issued copy has landed before the block may exit
    if (lane == 0) {
      for (int j = issued - C::KSTAGES < 0 ? 0 : issued - C::KSTAGES; j < issued; ++j) {
        const int st = j % C::KSTAGES;
        const uint32_t par = (j / C::KSTAGES) & 1;
        if (!mbar_wait(full0 + 8 * st, par, kWaitLimitNs)) {
          record_timeout(a.status, 2, j, st, par, full0 + 8 * st);
          break;
        }
      }
      for (int j = !kSplitKV ? issued : (issued - C::VSTAGES < 0 ? 0 : issued - C::VSTAGES); j < issued; ++j) {
        const int st = j % C::VSTAGES;
        const uint32_t par = (j / C::VSTAGES) & 1;
        if (!mbar_wait(vfull0 + 8 * st, par, kWaitLimitNs)) {
          record_timeout(a.status, 9, j, st, par, vfull0 + 8 * st);
          break;
        }
      }
      // and the last staged query rows (each slot's latest copy)
      for (int k = !C::STAGE_Q ? pq : (pq - 2 < 0 ? 0 : pq - 2); k < pq; ++k) {
        if (!mbar_wait(qfull0 + 8 * (k & 1), (k >> 1) & 1, kWaitLimitNs)) {
          record_timeout(a.status, 7, k, k & 1, (k >> 1) & 1, qfull0 + 8 * (k & 1));
          break;
        }
      }
    }
    return;
  }

  // ================= consumers
  const int w = warp - 1;
  const int ctid = tid - 32;
  constexpr int NCT = NW * 32;

  write_empty_results(a, it, s_len, G, D, c, P, ctid, NCT);

  // Tile i of the block's sequence lives in K slot i % KSTAGES and V slot
  // i % VSTAGES and is consumed by tile lane i % NT, one warp per row team
  // (both slot counts are multiples of NT, so each slot has one owner lane
  // whose warps wait on it in order); each warp tracks its next tile and
  // that tile's slots.
  const int u = w % NT;     // this warp's tile lane
  const int team = w / NT;  // and row team
  Cons cons;
  int next = u;          // next tile index (block sequence) of this warp
  int kslot = u;         // its K slot (KSTAGES >= NT)
  int vslot = u;         // its V slot (VSTAGES >= NT)
  uint32_t kph = 0;      // wrap parities of those slots
  uint32_t vph = 0;
  int base_i = 0;        // block-sequence index of the current piece's first tile
  bool alive = true;
  int piece = 0;         // pieces this block has finished (merge-area uses)
  Piece pc;
  while (next_piece(it, pc, s_pre, s_len, B, H, a.window_u, T)) {
    const int L = s_len[pc.b];
    const int lo = (a.window_u > 0 && L > a.window_u) ? L - a.window_u : 0;  // union of the rows' ranges
    const int n = pc.t1 - pc.t0;
    if constexpr (C::STAGE_Q) {
      const int qs = piece & 1;
      if (alive) {
        const bool ok = __all_sync(0xffffffffu, mbar_wait(qfull0 + 8 * qs, (piece >> 1) & 1, kWaitLimitNs));
        if (!ok) {
          if (lane == 0) record_timeout(a.status, 6, piece, qs, (piece >> 1) & 1, qfull0 + 8 * qs);
          alive = false;
        }
      }
      const int kh = pc.h * C::HT + Cons::team_head(team);  // this team's kv head
      const float ks = C::QUANT ? (scales_in_smem ? s_kscale[kh] : __ldg(a.k_scale + kh)) : 1.f;
      cons.begin_piece(a, q_slots + qs * (C::QSLOT_BYTES / 2), GK * D, ks, lane, team);
      __syncwarp();
      if (lane == 0) mbar_arrive(qempty0 + 8 * qs);
    } else {
      const int kh = pc.h * C::HT + Cons::team_head(team);  // this team's kv head
      const float ks = C::QUANT ? (scales_in_smem ? s_kscale[kh] : __ldg(a.k_scale + kh)) : 1.f;
      cons.begin_piece(a,
                       a.q + (static_cast<size_t>(pc.b) * Q * a.qo_heads + static_cast<size_t>(pc.h) * GK) * D,
                       a.qo_heads * D, ks, lane, team);
    }
    for (; next < base_i + n; next += NT) {
      // both halves of the tile are waited for up front (a second wait in
      // the middle of the tile's math measured slower than it saves); V
      // first, as its last copy is issued after K's
      if (kSplitKV && alive) {
        const bool ok = __all_sync(0xffffffffu, mbar_wait(vfull0 + 8 * vslot, vph, kWaitLimitNs));
        if (!ok) {
          if (lane == 0) record_timeout(a.status, 10, next, vslot, vph, vfull0 + 8 * vslot);
          alive = false;
        }
      }
      if (alive) {
        const bool ok = __all_sync(0xffffffffu, mbar_wait(full0 + 8 * kslot, kph, kWaitLimitNs));
        if (!ok) {
          if (lane == 0) record_timeout(a.status, 3, next, kslot, kph, full0 + 8 * kslot);
          alive = false;
        }
      }
      if (alive) {
        const uint32_t kempty = empty0 + 8 * kslot;
        cons.tile(a, ring + kslot * C::TILE_BYTES, vring + vslot * C::TILE_BYTES,
                  (pc.t0 + next - base_i) * T, lo, L, lane, [&] {
                    if constexpr (kSplitKV) {  // K slot free: the scores are taken
                      __syncwarp();
                      if (lane == 0) mbar_arrive(kempty);
                    }
                  });
        __syncwarp();
        if (lane == 0) mbar_arrive(kSplitKV ? vempty0 + 8 * vslot : kempty);
      }
      kslot += NT;
      if (kslot >= C::KSTAGES) {
        kslot -= C::KSTAGES;
        kph ^= 1u;
      }
      vslot += NT;
      if (vslot >= C::VSTAGES) {
        vslot -= C::VSTAGES;
        vph ^= 1u;
      }
    }
    base_i += n;
    // ---- merge the warps' states of this piece, without a block barrier:
    // each warp parks its state in the merge area and goes on to its tiles
    // of the next piece; the last warp to park merges the NW states, writes
    // the result (or the partial) and frees the area.  A warp waits only if
    // it finishes its share of the next piece before that merge is done.
    // V scale of row h's kv head (tiles of several heads: GK / HT rows per head)
    auto vscale_of = [&](int h) {
      const int vh = pc.h * C::HT + (C::HT > 1 ? h / (GK / C::HT) : 0);
      return C::QUANT ? (scales_in_smem ? s_vscale[vh] : __ldg(a.v_scale + vh)) : 1.f;
    };
    if (piece > 0 && alive) {
      const bool ok = __all_sync(0xffffffffu, mbar_wait(mfree, (piece - 1) & 1, kWaitLimitNs));
      if (!ok) {
        if (lane == 0) record_timeout(a.status, 4, piece, 0, (piece - 1) & 1, mfree);
        alive = false;
      }
    }
    cons.end_piece(m_area, l_area, acc_area, u, lane, G);
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      __threadfence_block();  // this warp's state is visible before it is counted
      last = atomicAdd(s_mcnt, 1) == NW - 1;
      __threadfence_block();  // and the other warps' states before they are read
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      __syncwarp();
      const bool whole = pc.n_pieces == 1;
      const int slot_idx = c + pc.seg;
      // 1) lane h < G: the row's max over the tile lanes' states, each
      //    lane's weight exp(m_u - M) / L (times the fp8 V scale) written
      //    over m_u, and the row's lse.  end_piece writes every lane's
      //    accumulator (zeros for a lane without tiles), so a zero weight is
      //    exact.
      if (lane < G) {
        const int h = lane;
        float M = -CUDART_INF_F;
#pragma unroll
        for (int ww = 0; ww < NT; ++ww) M = fmaxf(M, m_area[ww * G + h]);
        float scw[NT];
        float Ls = 0.f;
#pragma unroll
        for (int ww = 0; ww < NT; ++ww) {
          const float mw = m_area[ww * G + h];
          scw[ww] = (M == -CUDART_INF_F || mw == -CUDART_INF_F) ? 0.f : exp2_approx(mw - M);
          Ls = fmaf(l_area[ww * G + h], scw[ww], Ls);
        }
        const bool empty = !(Ls > 0.f);
        const float f = empty ? 0.f : vscale_of(h) / Ls;
#pragma unroll
        for (int ww = 0; ww < NT; ++ww) m_area[ww * G + h] = scw[ww] * f;
        const float lv = empty ? -CUDART_INF_F : (M + __log2f(Ls)) * kLn2;
        const size_t row = (static_cast<size_t>(pc.b) * Q + h / GK) * a.qo_heads +
                           static_cast<size_t>(pc.h) * GK + h % GK;
        if (whole) {
          if (a.lse != nullptr && FA_CHECK(a.status, row < static_cast<size_t>(B) * Q * a.qo_heads, 401, row))
            a.lse[row] = lv;
        } else if (FA_CHECK(a.status, slot_idx < a.max_partials, 402, slot_idx)) {
          a.part_lse[static_cast<size_t>(slot_idx) * G + h] = lv;
        }
      }
      __syncwarp();
      // 2) four dims per lane: out = sum_u weight_u * acc_u, branch-free
      //    float4 reads, one 16-byte partial store (or bf16x4 output store)
      constexpr int D4 = D / 4;
      // unrolled up to 16 rows: the loop is latency-bound (shared-memory
      // reads, then the store) and sits on the block's critical path once
      // per piece (measured 1.2-1.4% faster at 16 rows); the 32-row and
      // int4 head-tile variants spill more registers with it and measured
      // slower
      constexpr int kMergeUnroll = C::GMAX <= 16 && C::HT == 1 ? 4 : 1;
#pragma unroll kMergeUnroll
      for (int x4 = lane; x4 < G * D4; x4 += 32) {
        const int h = x4 / D4, dim = (x4 - h * D4) * 4;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int ww = 0; ww < NT; ++ww) {
          const float f = m_area[ww * G + h];
          const float4 av = *reinterpret_cast<const float4*>(acc_area + (ww * G + h) * D + dim);
          O.x = fmaf(av.x, f, O.x);
          O.y = fmaf(av.y, f, O.y);
          O.z = fmaf(av.z, f, O.z);
          O.w = fmaf(av.w, f, O.w);
        }
        const size_t row = (static_cast<size_t>(pc.b) * Q + h / GK) * a.qo_heads +
                           static_cast<size_t>(pc.h) * GK + h % GK;
        if (whole) {
          if (FA_CHECK(a.status, row < static_cast<size_t>(B) * Q * a.qo_heads, 401, row)) {
            uint2 packed;
            packed.x = pack_bf16x2(O.x, O.y);
            packed.y = pack_bf16x2(O.z, O.w);
            *reinterpret_cast<uint2*>(a.out + row * D + dim) = packed;
          }
        } else if (FA_CHECK(a.status, slot_idx < a.max_partials, 402, slot_idx)) {
          *reinterpret_cast<float4*>(a.part_o + (static_cast<size_t>(slot_idx) * G + h) * D + dim) = O;
        }
      }
      __syncwarp();
      if (lane == 0) {
        *s_mcnt = 0;
        mbar_arrive(mfree);
      }
    }
    ++piece;
  }
}

}  // namespace fa
