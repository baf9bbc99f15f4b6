// Instantiates every grouped fused forward kernel of SReLU (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_fwd_srelu_grouped(FwdVariant* t) { fill_fwd<kSReLU, false, true>(t); }
}  // namespace moeact
