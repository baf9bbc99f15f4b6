// Instantiates every dense fused backward kernel of SwiGLU (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_bwd_swiglu_dense(BwdVariant* t) { fill_bwd<kSwiGLU, false>(t); }
}  // namespace moeact
