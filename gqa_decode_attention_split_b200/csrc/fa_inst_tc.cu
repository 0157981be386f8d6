// Decode-kernel variants of the tcgen05 dataflow (bf16 K/V, head_dim 128,
// 16 or 32 query rows per segment after padding).
#include <atomic>

#include "fa_registry.h"
#include "fa_tc.cuh"

namespace fa {
namespace {

constexpr int kMaxDynamicSmemTc = 232448;  // 227 KB per block on sm_100

template <int NR>
cudaError_t launch_tc(const KernelArgs& args, int grid, size_t smem, cudaStream_t stream) {
  static std::atomic<unsigned long long> configured{0};  // one bit per device ordinal
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(fa_decode_tc_kernel<NR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kMaxDynamicSmemTc);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  // a programmatic dependent of the work before it, as the other variants
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(TcCfg<NR>::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fa_decode_tc_kernel<NR>, args);
}

template <int NR>
size_t smem_tc(int batch, int /*group*/) {
  return TcCfg<NR>::bytes(batch);
}

template <int NR>
KernelEntry make_tc_entry() {
  using C = TcCfg<NR>;
  KernelEntry e;
  e.head_dim = C::D;
  e.group = 0;
  e.max_group = NR;
  e.kv_kind = kKvBf16;
  e.path = kPathTc;
  e.tile_tokens = C::T;
  e.stages = C::KSTAGES;
  e.v_stages = C::VSTAGES;
  e.threads = C::THREADS;
  e.row_bytes = C::ROWB;
  e.plane_bytes = 128;
  e.token_major = 0;
  e.heads_per_tile = 1;
  e.tc_copies = 1;
  e.smem_bytes = &smem_tc<NR>;
  e.launch = &launch_tc<NR>;
  return e;
}

}  // namespace

int register_tc(KernelEntry* out, int cap) {
  int n = 0;
  if (n < cap) out[n++] = make_tc_entry<16>();
  if (n < cap) out[n++] = make_tc_entry<32>();
  return n;
}

}  // namespace fa
