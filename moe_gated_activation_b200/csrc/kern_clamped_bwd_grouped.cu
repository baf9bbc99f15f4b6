// Instantiates every grouped fused backward kernel of ClampedSwiGLU (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_bwd_clamped_grouped(BwdVariant* t) { fill_bwd<kClamped, true>(t); }
}  // namespace moeact
