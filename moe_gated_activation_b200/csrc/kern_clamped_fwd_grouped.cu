// Instantiates every grouped fused forward kernel of ClampedSwiGLU (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_fwd_clamped_grouped(FwdVariant* t) { fill_fwd<kClamped, false, true>(t); }
}  // namespace moeact
