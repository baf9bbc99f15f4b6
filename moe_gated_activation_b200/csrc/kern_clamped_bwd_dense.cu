// Instantiates every dense fused backward kernel of ClampedSwiGLU (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_bwd_clamped_dense(BwdVariant* t) { fill_bwd<kClamped, false>(t); }
}  // namespace moeact
