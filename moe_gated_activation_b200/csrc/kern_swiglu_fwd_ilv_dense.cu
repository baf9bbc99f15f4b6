// Instantiates every dense fused forward kernel of SwiGLU for an input whose
// gate and up columns are interleaved in blocks (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_fwd_swiglu_ilv_dense(FwdVariant* t) { fill_fwd<kSwiGLU, true, false, true>(t); }
}  // namespace moeact
