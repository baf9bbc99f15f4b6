// Instantiates every dense fused forward kernel of SReLU (see variants.cuh).
#include "variants.cuh"

namespace moeact {
void fill_fwd_srelu_dense(FwdVariant* t) { fill_fwd<kSReLU, false, false>(t); }
}  // namespace moeact
