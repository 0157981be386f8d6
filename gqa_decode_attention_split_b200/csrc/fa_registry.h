// fa_registry.h -- compiled decode-kernel variants and how to launch them.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace fa {

struct KernelArgs;

enum : int { kPathSimt = 1, kPathMma = 2 };

struct KernelEntry {
  int head_dim;
  int group;        // SIMT: exact group size; MMA: 0 (any group <= max_group)
  int max_group;
  int fp8;
  int path;
  int tile_tokens;  // T
  int stages;
  int threads;
  int row_bytes;    // head_dim * element size
  int plane_bytes;  // min(128, row_bytes)
  int token_major;  // 1: one copy per box with planes as a tensor-map dimension
  size_t (*smem_bytes)(int batch, int group);
  cudaError_t (*launch)(const KernelArgs& args, int grid, size_t smem, cudaStream_t stream);
};

// Each instantiation unit appends its variants; returns how many it wrote.
int register_d64(KernelEntry* out, int cap);
int register_d128(KernelEntry* out, int cap);
int register_d256(KernelEntry* out, int cap);

}  // namespace fa
