// Instantiates every grouped fused forward kernel of SwiGLU (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_fwd_swiglu_grouped(FwdVariant* t) { fill_fwd<kSwiGLU, true, true>(t); }
}  // namespace moeact
