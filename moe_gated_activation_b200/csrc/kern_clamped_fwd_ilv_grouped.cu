// Instantiates every grouped fused forward kernel of ClampedSwiGLU for an input whose
// gate and up columns are interleaved in blocks (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_fwd_clamped_ilv_grouped(FwdVariant* t) { fill_fwd<kClamped, false, true, true>(t); }
}  // namespace moeact
