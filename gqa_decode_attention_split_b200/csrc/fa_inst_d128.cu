// Decode-kernel variants for head_dim 128.
#include "fa_instantiate.cuh"

namespace fa {
int register_d128(KernelEntry* out, int cap) { return register_variants<128>(out, cap, true); }
}  // namespace fa
