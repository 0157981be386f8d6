// fa_instantiate.cuh -- helpers that turn a consumer type into a registry
// entry (included by the per-head_dim instantiation units only).
#pragma once

#include <atomic>

#include "fa_kernel.cuh"
#include "fa_registry.h"

namespace fa {

constexpr int kMaxDynamicSmem = 232448;  // 227 KB per block on sm_100

template <class Cons>
cudaError_t launch_decode(const KernelArgs& args, int grid, size_t smem, cudaStream_t stream) {
  static std::atomic<unsigned long long> configured{0};  // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(fa_decode_kernel<Cons>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kMaxDynamicSmem);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  // Launched as a programmatic dependent of whatever precedes it on the
  // stream: its blocks may be placed while that work drains (they wait in
  // griddepcontrol.wait before touching global memory), which hides the
  // launch between back-to-back passes.  The split-merge kernel that ends a
  // pass does not signal early, so the next pass's blocks are placed only
  // once it has finished.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(Cons::C::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fa_decode_kernel<Cons>, args);
}

template <class Cons>
size_t smem_bytes_for(int batch, int group) {
  return SmemLayout<Cons>::bytes(batch, group);
}

template <class Cons>
KernelEntry make_entry(int path, int group, int max_group, int kv_kind) {
  using C = typename Cons::C;
  KernelEntry e;
  e.head_dim = C::DIM;
  e.group = group;
  e.max_group = max_group;
  e.kv_kind = kv_kind;
  e.path = path;
  e.tile_tokens = C::T;
  e.stages = C::KSTAGES;
  e.v_stages = C::VSTAGES;
  e.threads = C::THREADS;
  e.row_bytes = C::ROWB;
  e.plane_bytes = C::CB;
  e.token_major = C::TOKEN_MAJOR ? 1 : 0;
  e.heads_per_tile = C::HT;
  e.tc_copies = 0;
  e.smem_bytes = &smem_bytes_for<Cons>;
  e.launch = &launch_decode<Cons>;
  return e;
}

template <int D>
int register_variants(KernelEntry* out, int cap, bool with_quant) {
  int n = 0;
  auto add = [&](const KernelEntry& e) {
    if (n < cap) out[n++] = e;
  };
  // tensor-core variants in order of rows (the planner takes the first that
  // holds a segment's rows): 8 rows; 16 and 32 rows as one and two teams of
  // warps with two row blocks of 8 each (head_dim <= 128; measured 13%
  // faster than four one-block teams at 32 rows), or as two and four teams
  // of one block (head_dim 256, whose two-block accumulators do not fit the
  // registers)
  add(make_entry<MmaConsumer<D, kKvBf16, 1>>(kPathMma, 0, 8, kKvBf16));
  if constexpr (D <= 128) {
    add(make_entry<MmaConsumer<D, kKvBf16, 1, false, 2>>(kPathMma, 0, 16, kKvBf16));
    add(make_entry<MmaConsumer<D, kKvBf16, 2, false, 2, 48>>(kPathMma, 0, 32, kKvBf16));
    add(make_entry<MmaConsumer<D, kKvBf16, 2, false, 2>>(kPathMma, 0, 32, kKvBf16));
  } else {
    add(make_entry<MmaConsumer<D, kKvBf16, 2>>(kPathMma, 0, 16, kKvBf16));
    add(make_entry<MmaConsumer<D, kKvBf16, 4>>(kPathMma, 0, 32, kKvBf16));
  }
  add(make_entry<SimtConsumer<D, 1, false>>(kPathSimt, 1, 1, kKvBf16));
  add(make_entry<SimtConsumer<D, 2, false>>(kPathSimt, 2, 2, kKvBf16));
  add(make_entry<SimtConsumer<D, 4, false>>(kPathSimt, 4, 4, kKvBf16));
  add(make_entry<SimtConsumer<D, 8, false>>(kPathSimt, 8, 8, kKvBf16));
  if constexpr (D >= 128) {
    if (with_quant) {
      add(make_entry<MmaConsumer<D, kKvFp8, 1>>(kPathMma, 0, 8, kKvFp8));
      if constexpr (D <= 128) {
        add(make_entry<MmaConsumer<D, kKvFp8, 1, false, 2>>(kPathMma, 0, 16, kKvFp8));
        add(make_entry<MmaConsumer<D, kKvFp8, 2, false, 2, 48>>(kPathMma, 0, 32, kKvFp8));
        add(make_entry<MmaConsumer<D, kKvFp8, 2, false, 2>>(kPathMma, 0, 32, kKvFp8));
      } else {
        add(make_entry<MmaConsumer<D, kKvFp8, 2>>(kPathMma, 0, 16, kKvFp8));
        add(make_entry<MmaConsumer<D, kKvFp8, 4>>(kPathMma, 0, 32, kKvFp8));
      }
      add(make_entry<SimtConsumer<D, 1, true>>(kPathSimt, 1, 1, kKvFp8));
      add(make_entry<SimtConsumer<D, 2, true>>(kPathSimt, 2, 2, kKvFp8));
      add(make_entry<SimtConsumer<D, 4, true>>(kPathSimt, 4, 4, kKvFp8));
      add(make_entry<SimtConsumer<D, 8, true>>(kPathSimt, 8, 8, kKvFp8));
      // int4 KV: tensor-core dataflow only
      add(make_entry<MmaConsumer<D, kKvInt4, 1>>(kPathMma, 0, 8, kKvInt4));
      if constexpr (D <= 128) {
        add(make_entry<MmaConsumer<D, kKvInt4, 1, false, 2>>(kPathMma, 0, 16, kKvInt4));
        add(make_entry<MmaConsumer<D, kKvInt4, 2, false, 2, 48>>(kPathMma, 0, 32, kKvInt4));
        add(make_entry<MmaConsumer<D, kKvInt4, 2, false, 2>>(kPathMma, 0, 32, kKvInt4));
      } else {
        add(make_entry<MmaConsumer<D, kKvInt4, 2>>(kPathMma, 0, 16, kKvInt4));
        add(make_entry<MmaConsumer<D, kKvInt4, 4>>(kPathMma, 0, 32, kKvInt4));
      }
      // int4: tiles of 256 / row-bytes adjacent kv heads (one row team per
      // head), so one tile's bookkeeping serves several heads' 4 KB
      if constexpr (D == 128)
        add(make_entry<MmaConsumer<D, kKvInt4, 4, true>>(kPathMma, 0, 8, kKvInt4));
      else
        add(make_entry<MmaConsumer<D, kKvInt4, 2, true>>(kPathMma, 0, 8, kKvInt4));
    }
  }
  return n;
}

}  // namespace fa
