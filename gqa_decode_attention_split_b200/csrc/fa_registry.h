// fa_registry.h -- compiled decode-kernel variants and how to launch them.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace fa {

struct KernelArgs;

enum : int { kPathSimt = 1, kPathMma = 2, kPathTc = 3 };

struct KernelEntry {
  int head_dim;
  int group;        // SIMT: exact group size; MMA: 0 (any group <= max_group)
  int max_group;
  int kv_kind;      // fa_kv_dtype: bf16, fp8 e4m3, int4
  int path;
  int tile_tokens;  // T
  int stages;       // K tile slots
  int v_stages;     // V tile slots
  int threads;
  int row_bytes;    // head_dim * element size
  int plane_bytes;  // min(128, row_bytes)
  int token_major;  // 1: one copy per box with planes as a tensor-map dimension
  int heads_per_tile;  // kv heads per tile (> 1: head teams, one segment per head block)
  int tc_copies;    // tcgen05 dataflow: 8-token copies landing as [group][plane][8][128]
  size_t (*smem_bytes)(int batch, int group);
  cudaError_t (*launch)(const KernelArgs& args, int grid, size_t smem, cudaStream_t stream);
};

// Arguments of the split-segment merge kernel (fa_split_merge.cu).
struct SplitMergeArgs {
  const int4* records;    // [num_records]: (segment, first block, pieces) or segment -1
  const float* part_o;    // [max_partials][group][head_dim], each o_k normalised
  const float* part_lse;  // [max_partials][group], natural log
  uint16_t* out;          // bf16 [batch][qo_heads][head_dim]
  float* lse;             // [batch][qo_heads] or null
  int num_records;        // blocks of the main launch
  int group;              // rows of a segment: kv_group * q_len
  int kv_group, q_len;    // query heads per kv head, query tokens per request
  int kv_heads, qo_heads, batch;
  long long max_partials;
};

// Enqueues the merge behind the main kernel on `stream` as a programmatic
// dependent launch; nothing is launched for a single-block pass.
cudaError_t launch_split_merge(const SplitMergeArgs& args, int head_dim, cudaStream_t stream);

// Each instantiation unit appends its variants; returns how many it wrote.
int register_d64(KernelEntry* out, int cap);
int register_d128(KernelEntry* out, int cap);
int register_d256(KernelEntry* out, int cap);
int register_tc(KernelEntry* out, int cap);

}  // namespace fa
