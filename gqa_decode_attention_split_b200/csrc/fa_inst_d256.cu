// Decode-kernel variants for head_dim 256.
#include "fa_instantiate.cuh"

namespace fa {
int register_d256(KernelEntry* out, int cap) { return register_variants<256>(out, cap, true); }
}  // namespace fa
