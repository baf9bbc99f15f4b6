// Instantiates every dense fused backward kernel of SReLU (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_bwd_srelu_dense(BwdVariant* t) { fill_bwd<kSReLU, false>(t); }
}  // namespace moeact
