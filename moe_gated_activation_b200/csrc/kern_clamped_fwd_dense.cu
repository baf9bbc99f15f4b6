// Instantiates every dense fused forward kernel of ClampedSwiGLU (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_fwd_clamped_dense(FwdVariant* t) { fill_fwd<kClamped, false, false>(t); }
}  // namespace moeact
