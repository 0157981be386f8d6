// fa_split_merge.cu -- second kernel of a decode pass: exact merge of the
// partial softmax states of every segment that the main kernel cut across
// thread blocks ("FlashDecoding++" explainer, section "Asynchronous softmax
// and unified max value": partial softmax per tile, combined afterwards;
// "Flashlight", section "Method": exp(x - y) = exp(x) / exp(y) makes the
// combination exact):
//   lse = M + ln sum_k exp(lse_k - M),   M = max_k lse_k
//   out = sum_k exp(lse_k - lse) * o_k
//
// It is launched right behind fa_decode_kernel as a programmatic dependent:
// its blocks may be scheduled while the main grid still runs (the main
// kernel signals that early), and each one waits in griddepcontrol.wait
// until the main grid has finished and its writes are visible.  One block
// merges one (split segment, query head) row; the split segments are named
// by the main kernel's boundary records, so this kernel needs no schedule of
// its own.
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "fa_device.cuh"
#include "fa_registry.h"

namespace fa {

namespace {

constexpr float kLog2eM = 1.4426950408889634f;
constexpr int kMergeWarps = 4;
constexpr int kMergeThreads = 32 * kMergeWarps;

// One block per (boundary, query head).  The boundary record names the
// segment whose first cut lies there (other blocks leave at once).  The four
// warps take pieces k = w, w + 4, ... and load a batch of them at once (o_k
// and lse_k for U pieces: one round trip; on B200 a dependent global round
// trip costs about a microsecond, so the merge is built to need two: the
// record, then the data).  Each warp keeps an online (max, sum, acc) state
// over its pieces; the four states are combined in shared memory.
template <int D>
__global__ void __launch_bounds__(kMergeThreads)
    fa_split_merge_kernel(const __grid_constant__ SplitMergeArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int D4 = D / 4;
  constexpr int J = (D4 + 31) / 32;   // float4 columns per lane
  constexpr int U = J >= 8 ? 1 : 8 / J;  // pieces per load batch
  __shared__ float4 s_acc[kMergeWarps][D4];
  __shared__ float s_m[kMergeWarps], s_z[kMergeWarps];

  const int G = a.group;
  const long long cb = 1 + static_cast<long long>(blockIdx.x) / G;  // boundary this block serves
  const int h = static_cast<int>(blockIdx.x % G);
  if (cb >= a.num_records) return;
  const int4 rec = __ldcg(a.records + cb);
  if (rec.x < 0) return;  // the cut at this boundary is not a segment's first
  const int seg = rec.x, c_first = rec.y, n = rec.z;
  if (seg >= a.batch * a.kv_heads || n < 2 || c_first < 0 ||
      static_cast<long long>(c_first) + n - 1 + seg >= a.max_partials)
    return;  // cannot come from the main kernel's schedule
  const int b = seg / a.kv_heads, hk = seg - b * a.kv_heads;
  const size_t slot0 = static_cast<size_t>(c_first) + seg;  // piece k lives in slot slot0 + k
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t kstep = static_cast<size_t>(G) * D4;  // float4s per slot
  const float4* src = reinterpret_cast<const float4*>(a.part_o) + (slot0 * G + h) * D4;

  float m = -CUDART_INF_F, z = 0.f;
  float4 acc[J];
#pragma unroll
  for (int j = 0; j < J; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k0 = w; k0 < n; k0 += kMergeWarps * U) {
    float4 v[U][J];
    float lw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + u * kMergeWarps;
      lw[u] = k < n ? __ldcg(a.part_lse + (slot0 + k) * G + h) : -CUDART_INF_F;
#pragma unroll
      for (int j = 0; j < J; ++j) {
        const int col = lane + 32 * j;
        v[u][j] = (k < n && col < D4) ? __ldcg(src + k * kstep + col) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float mb = m;
#pragma unroll
    for (int u = 0; u < U; ++u) mb = fmaxf(mb, lw[u]);
    if (mb == -CUDART_INF_F) continue;  // nothing but empty pieces so far
    const float sc = m == -CUDART_INF_F ? 0.f : exp2_approx((m - mb) * kLog2eM);
    z *= sc;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      acc[j].x *= sc;
      acc[j].y *= sc;
      acc[j].z *= sc;
      acc[j].w *= sc;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float wk = lw[u] == -CUDART_INF_F ? 0.f : exp2_approx((lw[u] - mb) * kLog2eM);
      z += wk;
#pragma unroll
      for (int j = 0; j < J; ++j) {
        acc[j].x = fmaf(wk, v[u][j].x, acc[j].x);
        acc[j].y = fmaf(wk, v[u][j].y, acc[j].y);
        acc[j].z = fmaf(wk, v[u][j].z, acc[j].z);
        acc[j].w = fmaf(wk, v[u][j].w, acc[j].w);
      }
    }
    m = mb;
  }
  if (lane == 0) {
    s_m[w] = m;
    s_z[w] = z;
  }
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int col = lane + 32 * j;
    if (col < D4) s_acc[w][col] = acc[j];
  }
  __syncthreads();

  float M = -CUDART_INF_F;
#pragma unroll
  for (int i = 0; i < kMergeWarps; ++i) M = fmaxf(M, s_m[i]);
  float sw[kMergeWarps];
  float Z = 0.f;
#pragma unroll
  for (int i = 0; i < kMergeWarps; ++i) {
    sw[i] = (M == -CUDART_INF_F || s_m[i] == -CUDART_INF_F) ? 0.f : exp2_approx((s_m[i] - M) * kLog2eM);
    Z = fmaf(s_z[i], sw[i], Z);
  }
  const bool none = !(Z > 0.f);
  const float inv = none ? 0.f : 1.f / Z;
  // row h of the segment: query token h / kv_group, head h % kv_group
  const size_t row = (static_cast<size_t>(b) * a.q_len + h / a.kv_group) * a.qo_heads +
                     static_cast<size_t>(hk) * a.kv_group + h % a.kv_group;
  for (int col = threadIdx.x; col < D4; col += kMergeThreads) {
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kMergeWarps; ++i) {
      const float4 x = s_acc[i][col];
      o.x = fmaf(sw[i], x.x, o.x);
      o.y = fmaf(sw[i], x.y, o.y);
      o.z = fmaf(sw[i], x.z, o.z);
      o.w = fmaf(sw[i], x.w, o.w);
    }
    uint2 packed;
    packed.x = pack_bf16x2(o.x * inv, o.y * inv);
    packed.y = pack_bf16x2(o.z * inv, o.w * inv);
    *reinterpret_cast<uint2*>(a.out + row * D + col * 4) = packed;
  }
  if (threadIdx.x == 0 && a.lse != nullptr) a.lse[row] = none ? -CUDART_INF_F : M + __logf(Z);
}

template <int D>
cudaError_t launch_for(const SplitMergeArgs& args, cudaStream_t stream) {
  const long long blocks = static_cast<long long>(args.num_records - 1) * args.group;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fa_split_merge_kernel<D>, args);
}

}  // namespace

cudaError_t launch_split_merge(const SplitMergeArgs& args, int head_dim, cudaStream_t stream) {
  if (args.num_records < 2) return cudaSuccess;  // one block: nothing is split
  switch (head_dim) {
    case 64: return launch_for<64>(args, stream);
    case 128: return launch_for<128>(args, stream);
    case 256: return launch_for<256>(args, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fa
