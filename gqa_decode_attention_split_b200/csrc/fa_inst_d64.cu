// Decode-kernel variants for head_dim 64.
#include "fa_instantiate.cuh"

namespace fa {
int register_d64(KernelEntry* out, int cap) { return register_variants<64>(out, cap, true); }
}  // namespace fa
