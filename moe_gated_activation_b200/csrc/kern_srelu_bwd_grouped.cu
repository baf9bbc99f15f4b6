// Instantiates every grouped fused backward kernel of SReLU (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_bwd_srelu_grouped(BwdVariant* t) { fill_bwd<kSReLU, true>(t); }
}  // namespace moeact
