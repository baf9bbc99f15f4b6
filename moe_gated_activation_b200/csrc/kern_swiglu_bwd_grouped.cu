// Instantiates every grouped fused backward kernel of SwiGLU (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_bwd_swiglu_grouped(BwdVariant* t) { fill_bwd<kSwiGLU, true>(t); }
}  // namespace moeact
