// Instantiates every dense fused forward kernel of SwiGLU (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_fwd_swiglu_dense(FwdVariant* t) { fill_fwd<kSwiGLU, true, false>(t); }
}  // namespace moeact
