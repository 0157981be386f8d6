/*
 * fadecode.h -- C ABI of the split-KV GQA decode-attention library for
 * NVIDIA B200 (sm_100a).
 *
 * The operation (one new query token per request, attending over that
 * request's KV cache):
 *
 *   for request b, query head h, kv head g = h / (qo_heads / kv_heads),
 *   visible keys J_b = [max(0, L_b - window), L_b)   (all keys if window <= 0)
 *     s_j   = sm_scale * <q[b,h,:], K_b[j,g,:]>
 *     out   = sum_j softmax(s)_j * V_b[j,g,:]          (bf16, round-to-nearest)
 *     lse   = ln sum_j exp(s_j)                         (fp32, natural log)
 *
 * Sources: "Forcing Flash Attention onto a TPU" (LLM internals part 5),
 * sections "Standard causal attention" (the definition) and "Flash Attention
 * in JAX" (tiles with a running max, running sum and accumulator);
 * "FlashInfer x JAX via jax-tvm-ffi", section on single_decode (GQA decode of
 * one request over its KV cache, a caller-provided scratch buffer, sentinel
 * values for optional arguments) and section "Applying it to Gemma 3"
 * (local sliding-window layers); "Beyond the Memory Wall", section
 * "2. FlashInfer" (paged KV, FP8 KV); "FlashDecoding++" explainer, sections
 * "Asynchronous softmax and unified max value" (partial softmax per KV tile,
 * merged afterwards) and "Hardware-aware heuristic dataflow" (the path is
 * chosen from the shape and the GPU).
 *
 * Conventions shared by every entry point:
 *  - Every buffer is owned by the caller.  The library never allocates or
 *    frees device memory.  A plan is a small host object owned by the
 *    caller and released with fa_plan_destroy.
 *  - Device pointers are plain CUDA device addresses on the current device.
 *    `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream); work is enqueued on it and the call returns without waiting,
 *    except where a function says it synchronises.
 *  - Errors are returned as fa_status; nothing aborts or traps.  Argument
 *    errors are detected on the host before any work is enqueued.
 *  - bf16 tensors are raw IEEE bfloat16 bit patterns (uint16); fp8 tensors
 *    are e4m3 "fn" codes (uint8: bias 7, no infinities); int4 tensors are
 *    two's-complement 4-bit codes in [-8, 7], two per byte, the even element
 *    of a row in the low nibble (a row of head_dim codes is head_dim / 2
 *    bytes).  INT4 KV quantisation is named on "Beyond the Memory Wall",
 *    section "2. FlashInfer", without a layout; this is the plainest one.
 */
#ifndef FADECODE_H_
#define FADECODE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,         /* null pointer, bad shape, bad sentinel   */
  FA_ERR_UNSUPPORTED = 2,         /* valid, but no kernel for this shape    */
  FA_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes below the plan's need  */
  FA_ERR_MISALIGNED = 4,          /* a pointer below its required alignment */
  FA_ERR_CUDA = 5,                /* a CUDA runtime/driver call failed      */
  FA_ERR_DEVICE_CHECK = 6         /* a kernel recorded a device-side check  */
} fa_status;

/* K/V element type.  FP8 and INT4 codes carry one fp32 scale per kv head
 * for K and one for V (k_scale, v_scale): element = code * scale. */
typedef enum { FA_KV_BF16 = 0, FA_KV_FP8_E4M3 = 1, FA_KV_INT4 = 2 } fa_kv_dtype;

/* Dataflow for the KV-tile math.  SIMT computes q.k with per-lane fp32 FMAs
 * and warp-shuffle reductions (a GEMV per head); MMA runs the two skinny
 * products (scores and probabilities times V) on the warp-level tensor-core
 * instruction with fp32 accumulation, which keeps the instruction count per
 * KV byte low when several query heads share a kv head.  TC runs the same
 * two products on the 5th-generation tensor cores (tcgen05, accumulators in
 * tensor memory) with 128-token tiles as the large dimension; it covers bf16
 * K/V with head_dim 128, 9 to 32 rows per segment (query heads per kv head
 * times query tokens; 1 to 8 rows too when TC is asked for, padded to 16,
 * where MMA measured faster), contiguous K/V or pages of at least 8 tokens,
 * and the plain running max (not unified_max).  AUTO lets the planner choose
 * from the shape (see fa_plan_info): TC where it applies, else MMA, else
 * SIMT, unless the measured table (fa_set_tuning) says otherwise. */
typedef enum { FA_PATH_AUTO = 0, FA_PATH_SIMT = 1, FA_PATH_MMA = 2, FA_PATH_TC = 3 } fa_path;

/* Device-side check bits, reported by fa_decode_status. */
enum {
  FA_DEVICE_BAD_PAGE = 1u,   /* a page_table entry outside [0, num_pages)     */
  FA_DEVICE_TIMEOUT = 2u,    /* a pipeline wait exceeded its time limit       */
  FA_DEVICE_BAD_INDPTR = 4u  /* kv_indptr decreasing or past the K/V extent   */
};

typedef struct {
  int32_t batch;      /* requests, >= 1                                       */
  int32_t qo_heads;   /* query heads per request                              */
  int32_t kv_heads;   /* kv heads; qo_heads % kv_heads == 0                   */
  int32_t head_dim;   /* 64, 128 or 256 (fp8, int4: 128 or 256)               */
  int32_t kv_dtype;   /* fa_kv_dtype                                          */
  int32_t paged;      /* 0: contiguous (ragged) rows, 1: paged pool           */
  int32_t page_size;  /* paged only: tokens per page, a power of two <= 256  */
  int32_t window;     /* sentinel -1 (or any value <= 0): attend to all keys; */
                      /* w > 0: attend to the last w keys only               */
  float sm_scale;     /* multiplies q.k before the softmax; must be finite   */
  int32_t path;       /* fa_path                                             */
  int32_t num_ctas;   /* 0: planner's choice.  n > 0 forces n thread blocks, */
                      /* i.e. the KV split granularity (used to test that    */
                      /* split-then-merge equals the unsplit result)         */
  int32_t q_len;      /* query tokens per request, 0 or 1: one.  q_len > 1   */
                      /* (speculative or chunked decode, the small-M case of */
                      /* the "FlashDecoding++" explainer, section "Flat GEMM */
                      /* optimization"): the request's q_len newest keys are */
                      /* its query tokens, and token i (position            */
                      /* L - q_len + i) sees the keys up to and including    */
                      /* itself, or the last `window` of them.  The rows of  */
                      /* a (request, kv head) segment, (qo_heads / kv_heads) */
                      /* * q_len, must be <= 32 on the MMA dataflow (SIMT:   */
                      /* exactly 1, 2, 4 or 8; int4 runs on the tensor-core  */
                      /* dataflows only; TC: 9 to 32, see fa_path).          */
  float logit_cap;    /* 0: none.  c > 0: logit soft-capping, each scaled    */
                      /* score s becomes c * tanh(s / c) before the softmax  */
                      /* (Gemma 2's soft-cap, named on "FlashInfer x JAX via */
                      /* jax-tvm-ffi", section "Applying it to Gemma 3").    */
                      /* Must be finite and >= 0.                            */
  int32_t unified_max; /* 0: off.  1: unified max ("FlashDecoding++"         */
                      /* explainer, section "Asynchronous softmax and        */
                      /* unified max value"): every running max starts at   */
                      /* softmax_phi instead of -inf, so partial states     */
                      /* share one max and are not rescaled while the       */
                      /* scores stay below it.  Exact for any phi: a score  */
                      /* more than 8 log2-units above phi falls back to the */
                      /* exact rescale, and a row whose first scores sit     */
                      /* more than 8 log2-units below phi (for fp8 / int4   */
                      /* K/V on the MMA dataflow: below phi at all) starts  */
                      /* from its own maximum instead.                      */
  float softmax_phi;  /* unified_max only: phi, in natural-log units of the */
                      /* scaled (and soft-capped) score; must be finite.    */
  int32_t piece_cost; /* Cost model of the split.  A thread block pays a    */
                      /* fixed cost per segment piece it takes (parking and */
                      /* merging the piece's softmax state, its ragged last */
                      /* tile).  With piece_cost c > 0 every segment is     */
                      /* charged c tiles ahead of its own when the segments */
                      /* are cut into equal runs, so a block that starts    */
                      /* more segments gets fewer tiles.  0: planner's      */
                      /* choice; c < 0: equal tiles, no charge; at most    */
                      /* 4096.                                              */
} fa_decode_desc;

typedef struct fa_plan fa_plan;

/* What the planner chose (read-only view of a plan). */
typedef struct {
  int32_t path;             /* FA_PATH_SIMT, FA_PATH_MMA or FA_PATH_TC        */
  int32_t num_ctas;         /* thread blocks launched by fa_decode_run        */
  int32_t tile_tokens;      /* tokens per KV tile moved by one TMA transaction */
  int32_t stages;           /* K tile slots of the shared-memory ring         */
  int32_t total_tiles;      /* KV tiles over all (request, kv head) segments  */
  int32_t max_partials;     /* partial-state slots reserved in the workspace  */
  size_t workspace_bytes;   /* minimum workspace size for fa_decode_run       */
  size_t smem_bytes;        /* dynamic shared memory per thread block         */
  int32_t v_stages;         /* V tile slots (at least stages: V is held longer) */
  int32_t heads_per_tile;   /* kv heads whose rows one tile holds per token:   */
                            /* > 1 for int4 (256 contiguous bytes a token)     */
  int32_t piece_cost;       /* tiles charged per segment in the split (0: none) */
  int32_t launches;         /* kernel launches of one fa_decode_run: 1 (no     */
                            /* segment is ever split: one block, or one whole  */
                            /* segment per block) or 2 (with the split merge)  */
} fa_plan_info_t;

/*
 * fa_decode_plan -- host only; touches no device memory and enqueues nothing.
 *
 * Decides the split of the KV sequence into tiles and of the tiles over
 * thread blocks ("FlashDecoding++", section "Hardware-aware heuristic
 * dataflow": the dataflow is chosen from batch, lengths and the GPU).
 * Every (request, kv head) is a segment of KV tiles; the segments are laid
 * end to end and cut into num_ctas equal runs, so every SM streams about the
 * same number of bytes whatever the length mix.  Each segment is counted as
 * its tiles plus piece_cost tiles for the fixed cost of a segment piece, so
 * a block that starts more segments takes fewer tiles (see
 * fa_decode_desc.piece_cost).  A segment cut into several runs yields
 * partial softmax states that fa_decode_run merges exactly.
 *
 *  desc            shapes and options (copied into the plan).
 *  kv_indptr_host  int32[batch + 1], host memory: cumulative token counts;
 *                  kv_indptr_host[0] == 0, non-decreasing.  Only used to size
 *                  the split; fa_decode_run reads the device copy.
 *  num_sms         SM count of the target device (0: query the current
 *                  device; on a host without a GPU pass it explicitly).
 *  plan            receives the new plan (caller frees: fa_plan_destroy).
 *  workspace_bytes receives the minimum workspace size.
 * Errors: FA_ERR_INVALID_ARG (null pointer, non-positive shape, qo_heads not
 * a multiple of kv_heads, bad indptr, non-finite sm_scale, bad page_size,
 * q_len < 0 or > 64, negative or non-finite logit_cap), FA_ERR_UNSUPPORTED (head_dim / group * q_len / dtype /
 * path combination without a kernel), FA_ERR_CUDA (num_sms == 0 and no
 * device could be queried).
 */
FA_API fa_status fa_decode_plan(const fa_decode_desc* desc, const int32_t* kv_indptr_host,
                         int32_t num_sms, fa_plan** plan, size_t* workspace_bytes);

/* Fills *info from a plan.  FA_ERR_INVALID_ARG on null pointers. */
FA_API fa_status fa_plan_get_info(const fa_plan* plan, fa_plan_info_t* info);

/* Releases a plan (NULL is a no-op). */
FA_API void fa_plan_destroy(fa_plan* plan);

/*
 * Measured dataflow choice ("FlashDecoding++" explainer, section
 * "Hardware-aware heuristic dataflow": which implementation runs a shape is
 * decided from measurements of the shapes on the GPU, not from a fixed
 * rule).  A table row covers decodes with the given head_dim and kv dtype
 * whose rows per (request, kv head) segment, (qo_heads / kv_heads) * q_len,
 * lie in [rows_min, rows_max] and whose visible K/V bytes (keys each query
 * token sees, at most window + q_len - 1 per request, x kv_heads x 2 x
 * head_dim x element size) lie in [bytes_min, bytes_max].  It names the
 * dataflow and the largest average number of thread blocks per segment
 * (max_pieces; 0: the planner's default of 32), which bounds the split of
 * short problems.
 */
typedef struct {
  int32_t head_dim;
  int32_t kv_dtype;      /* fa_kv_dtype                                     */
  int32_t rows_min, rows_max;
  int64_t bytes_min, bytes_max;
  int32_t path;          /* FA_PATH_SIMT or FA_PATH_MMA                     */
  int32_t max_pieces;    /* 0, or 1 .. 1024                                 */
} fa_tuning_entry;

/*
 * fa_set_tuning -- install the table fa_decode_plan consults when
 * desc->path is FA_PATH_AUTO and desc->num_ctas is 0.  The first matching
 * row wins; a row whose dataflow has no kernel for the shape is passed
 * over; a decode no row matches gets the fixed rule (MMA where a kernel
 * exists, else SIMT; up to 32 blocks per segment).  The rows are copied.
 * entries == NULL (with n == 0) restores the built-in table, which was
 * measured on a B200 by the package's tuning script; n == 0 with a non-NULL
 * pointer installs an empty table (fixed rule only).  Not safe to call while
 * another thread is planning.
 * Errors: FA_ERR_INVALID_ARG (n < 0 or > 4096, NULL with n > 0, a row with
 * rows_min > rows_max, bytes_min > bytes_max, rows_min < 1, an unknown path
 * or dtype, max_pieces outside 0 .. 1024).
 */
FA_API fa_status fa_set_tuning(const fa_tuning_entry* entries, int32_t n);

/*
 * fa_get_tuning -- copy the active table: *n receives its row count and the
 * first min(cap, *n) rows go to out (out may be NULL when cap == 0).
 * Errors: FA_ERR_INVALID_ARG (n NULL, cap < 0, out NULL with cap > 0).
 */
FA_API fa_status fa_get_tuning(fa_tuning_entry* out, int32_t cap, int32_t* n);

/*
 * fa_decode_run -- enqueue one decode-attention pass on `stream`.
 *
 * What it computes is the formula at the top of this header ("Forcing Flash
 * Attention onto a TPU", section "Standard causal attention"), reached as the
 * pages describe: the KV sequence is cut into tiles, each run of tiles is
 * reduced to a partial softmax state (running max, running sum,
 * accumulator; same page, section "Flash Attention in JAX"), and the states
 * of a split request are merged exactly through log-sum-exp
 * ("FlashDecoding++" explainer, section "Asynchronous softmax and unified max
 * value").  The call shape is the single-request GQA decode with a scratch
 * buffer of "FlashInfer x JAX via jax-tvm-ffi" (section on single_decode),
 * extended to a batch over contiguous or paged KV ("Beyond the Memory Wall",
 * section "2. FlashInfer").
 *
 * Layouts (row-major, all device memory):
 *  q           bf16 [batch, q_len, qo_heads, head_dim] (q_len = 1:
 *              [batch, qo_heads, head_dim]), 16-byte aligned.
 *  k, v        contiguous: [kv_rows, kv_heads, head_dim]; request b owns rows
 *              [kv_indptr[b], kv_indptr[b+1]) (batch 1: rows 0..kv_len-1).
 *              paged: pools [kv_rows, page_size, kv_heads, head_dim] where
 *              kv_rows is the number of pages.  Element type per desc
 *              (bf16, e4m3, or int4 with head_dim / 2 bytes per row),
 *              16-byte aligned.
 *  kv_rows     contiguous: number of rows of k and v; paged: number of pages
 *              in each pool.  Reads never leave [0, kv_rows).
 *  page_table  paged only (else NULL): int32 [batch, page_table_stride];
 *              token t of request b lives in page page_table[b][t/page_size],
 *              slot t % page_size.  Only entries of pages holding visible
 *              tokens are read.  An entry outside [0, kv_rows) reads zeros
 *              and sets FA_DEVICE_BAD_PAGE.
 *  kv_indptr   int32 [batch + 1], device copy of the plan's indptr.
 *  k_scale,    fp8 and int4 only (else NULL): fp32 [kv_heads]; a stored
 *  v_scale     code c of kv head g means e4m3(c) * scale[g] (fp8) or
 *              c * scale[g] (int4).
 *  out         bf16 [batch, q_len, qo_heads, head_dim], 16-byte aligned.
 *  lse         fp32 [batch, q_len, qo_heads], natural log; NULL = do not
 *              write.  A query token with no visible key (a request shorter
 *              than q_len) gets out = 0, lse = -inf.
 *              A request with no visible key gets out = 0, lse = -inf.
 *  workspace   device scratch of >= the plan's workspace_bytes, 256-byte
 *              aligned, zero-filled once before its first use (and again
 *              after FA_ERR_DEVICE_CHECK).  Apart from its check word every
 *              byte is written by a pass before that pass reads it, so one
 *              workspace serves any number of calls in stream order.  Two
 *              calls that share a workspace must not overlap on the GPU.
 * A pass is one kernel launch, plus a second small one when some segment is
 * cut across thread blocks: it merges those segments' partial states and is
 * enqueued as a programmatic dependent launch of the first (it is scheduled
 * early and waits on the device for the first to finish).
 * No allocation, no synchronisation, no host<->device copies.  Errors:
 * FA_ERR_INVALID_ARG, FA_ERR_MISALIGNED, FA_ERR_WORKSPACE_TOO_SMALL,
 * FA_ERR_CUDA (launch failure).  Device-side checks are reported later by
 * fa_decode_status.
 * CUDA graphs: a pass can be recorded by stream capture, once the plan's
 * kernel has run on the device outside a capture (its first launch sets the
 * kernel's shared-memory limit).  A replay reads q, K/V, page_table and
 * kv_indptr where they were at capture.  Their contents may change between
 * replays, requests' lengths included, as long as the extents passed at
 * capture (kv_rows, page_table_stride) still hold.
 */
FA_API fa_status fa_decode_run(const fa_plan* plan, const void* q, const void* k, const void* v,
                        int64_t kv_rows, const int32_t* page_table, int32_t page_table_stride,
                        const int32_t* kv_indptr, const float* k_scale, const float* v_scale,
                        void* out, float* lse, void* workspace, size_t workspace_bytes,
                        void* stream);

/* Size of the fixed scratch behind fa_decode_run_static: 4 MiB. */
#define FA_STATIC_WORKSPACE_BYTES (4u << 20)

/*
 * fa_decode_run_static -- fa_decode_run for callers that cannot allocate.
 * (An addition of this library; the pages have no counterpart.)
 *
 * Some callers cannot call cudaMalloc or any other allocating routine where
 * they run attention: a runtime that hands out all device memory itself, a
 * plugin that receives only input and output buffers, or a path that must
 * not synchronise the device (cudaMalloc and cudaFree may).  This entry point
 * takes the same arguments as fa_decode_run minus the workspace, and
 * allocates nothing: its scratch is a fixed array of
 * FA_STATIC_WORKSPACE_BYTES in the library's device memory, which every GPU
 * that loads the library holds until the process exits.
 *  - The first call on a device looks up that array's device address (once
 *    per device, on the current device); make that first call before any
 *    stream capture.
 *  - Every call on a device shares the one array, which keeps what the
 *    previous call left.  Each call clears the part that must start at zero
 *    (the check word) in stream order before its kernel.  Calls
 *    that overlap on the GPU (other streams, other host threads) race on the
 *    array and must be avoided.
 *  - A plan whose workspace_bytes exceeds FA_STATIC_WORKSPACE_BYTES is
 *    rejected with FA_ERR_WORKSPACE_TOO_SMALL (fa_last_error says how much
 *    it needed).  Other errors as fa_decode_run.
 *  - Device-side checks (bad page ids, a bad kv_indptr, a wait that gave
 *    up) land in the scratch's check word; read them with
 *    fa_decode_status_static before the next static call clears it.
 *  - The scratch address is kept for the life of the process, so the
 *    static entry points are not supported after cudaDeviceReset.
 */
FA_API fa_status fa_decode_run_static(const fa_plan* plan, const void* q, const void* k,
                                      const void* v, int64_t kv_rows, const int32_t* page_table,
                                      int32_t page_table_stride, const int32_t* kv_indptr,
                                      const float* k_scale, const float* v_scale, void* out,
                                      float* lse, void* stream);

/*
 * fa_decode_status_static -- fa_decode_status for the fixed scratch behind
 * fa_decode_run_static.  (An addition of this library; the pages have no
 * counterpart.)
 *
 * A caller without a workspace has no address to pass to fa_decode_status,
 * so this call reads the static scratch of the current device instead: it
 * SYNCHRONISES `stream`, copies the device-check word into *flags
 * (FA_DEVICE_* bits: a page id outside the pool, a kv_indptr that decreases
 * or runs past the extent, a wait that gave up) and, when a bit was set,
 * clears the 256-byte header (word and records).  Every fa_decode_run_static
 * call clears the word before its kernel, so read the status of a call
 * before the next static call is enqueued.  Like every static call, it
 * allocates nothing; it needs one small device-to-host copy.
 * Returns FA_ERR_DEVICE_CHECK when any bit was set, FA_ERR_INVALID_ARG for
 * a NULL flags, FA_ERR_CUDA when the copy failed, else FA_OK.
 */
FA_API fa_status fa_decode_status_static(uint32_t* flags, void* stream);

/*
 * fa_decode_status -- SYNCHRONISES `stream`, then reads the device-side check
 * word of `workspace` into *flags (FA_DEVICE_* bits, 0 = clean).  When a bit
 * was set it clears the workspace's 256-byte header: the word and the records
 * of the first failed check and the first wait that gave up.  Returns
 * FA_ERR_DEVICE_CHECK when any bit was set, FA_ERR_CUDA when the copy failed,
 * else FA_OK.
 */
FA_API fa_status fa_decode_status(void* workspace, size_t workspace_bytes, uint32_t* flags,
                           void* stream);

/*
 * fa_selftest_wait -- a check of the failure path, not part of a pass.
 * Enqueues on `stream` a one-thread kernel that waits on an mbarrier with
 * the same bounded wait every pipeline wait of the decode kernels uses.
 * With arrive != 0 the thread arrives first and the wait succeeds at once;
 * with arrive == 0 nothing arrives, so the wait gives up after limit_ns
 * (1 .. 10^9 ns) and records itself as a pipeline wait that timed out:
 * FA_DEVICE_TIMEOUT in the check word of `workspace` and the wait's record
 * (site 99, block 0, warp 0) in its header, which fa_decode_status then
 * reports and clears.  The GPU context stays usable.  workspace: >= 256
 * bytes, 256-byte aligned, its header zero-filled.  Returns
 * FA_ERR_INVALID_ARG, FA_ERR_MISALIGNED, FA_ERR_CUDA (launch) or FA_OK.
 */
FA_API fa_status fa_selftest_wait(void* workspace, size_t workspace_bytes, int64_t limit_ns,
                                  int32_t arrive, void* stream);

/*
 * fa_merge_states -- exact merge of n partial attention states per
 * (row, head) ("FlashDecoding++" explainer, partial softmax per tile combined
 * afterwards; "Flashlight", section "Method": exp(x - y) = exp(x) / exp(y)
 * makes the combination exact):
 *   lse = M + ln sum_c exp(lse_c - M),  M = max_c lse_c
 *   out = sum_c exp(lse_c - lse) * o_c
 * States with lse_c = -inf carry no weight; all -inf gives out = 0,
 * lse = -inf.
 *  o_parts   fp32 [n, rows, heads, head_dim] (each o_c already normalised)
 *  lse_parts fp32 [n, rows, heads], natural log
 *  out       bf16 [rows, heads, head_dim]; lse_out fp32 [rows, heads] or NULL
 * head_dim must be a multiple of 4 and <= 1024; o_parts, out 16-byte aligned.
 * Errors: FA_ERR_INVALID_ARG, FA_ERR_MISALIGNED, FA_ERR_CUDA.
 */
FA_API fa_status fa_merge_states(const float* o_parts, const float* lse_parts, int32_t n, int32_t rows,
                          int32_t heads, int32_t head_dim, void* out, float* lse_out,
                          void* stream);

/* Static description of a status code (never NULL). */
FA_API const char* fa_status_string(fa_status status);

/* Text of the most recent CUDA failure (FA_ERR_CUDA) returned to the calling
 * thread, or "" if there was none.  The buffer is thread-local and is
 * overwritten by the next failure. */
FA_API const char* fa_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch.  The structures of
 * this header are those of FA_VERSION (0.2.0 added fa_decode_desc.piece_cost
 * and fa_plan_info_t.piece_cost; 0.3.0 added FA_PATH_TC and
 * fa_plan_info_t.launches; 0.3.1 added fa_selftest_wait, no structure
 * changed); a caller built against it should check that
 * fa_version() / 100 == FA_VERSION / 100. */
#define FA_VERSION 301
FA_API int32_t fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FADECODE_H_ */
