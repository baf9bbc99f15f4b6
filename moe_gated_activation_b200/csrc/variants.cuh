// The instantiated fused kernels, one table per activation and direction of
// the pass, each filled in its own translation unit (kern_*.cu) so that the
// kernels compile in parallel; capi.cu picks an entry per call.
#pragma once

#include "kernels.cuh"

namespace moeact {

using FwdFn = void (*)(const CUtensorMap, const Params);
using BwdFn = void (*)(const CUtensorMap, const CUtensorMap, const Params);
// smem_fixed: shared memory without group offsets; sig: the kernel carries the
// sigmoid table, whose gap holds the group offsets (so they add nothing)
struct FwdVariant { FwdFn fn; int threads; int smem_fixed; bool sig; };
struct BwdVariant { BwdFn fn; int threads; int smem_fixed; bool sig; };

// Table slots: forward by (grouped, staged, dirs | layout | interleave),
// backward by (grouped, dX re-read, dirs | layout); kdirs = ROWWISE/COLWISE
// bits | kGemm (| kIlv, forward only).
constexpr int kFwdSlots = 64;
constexpr int kBwdSlots = 32;
inline int fwd_slot(bool grouped, bool staged, int kdirs) {
  return ((grouped ? 2 : 0) + (staged ? 1 : 0)) * 16 + kdirs;
}
inline int bwd_slot(bool grouped, bool reread, int kdirs) {
  return ((grouped ? 2 : 0) + (reread ? 1 : 0)) * 8 + kdirs;
}

template <int ACT, int DIRS, bool STAGED, bool GROUPED>
void put_fwd(FwdVariant* t) {
  t[fwd_slot(GROUPED, STAGED, DIRS)] = {act_fwd_kernel<ACT, DIRS, STAGED, GROUPED>,
                                        Cfg<ACT, false>::kThreads,
                                        smem_bytes<ACT, false>(false, 0), Cfg<ACT, false>::kSig};
}

template <int ACT, int DIRS, bool GROUPED, bool REREAD>
void put_bwd(BwdVariant* t) {
  t[bwd_slot(GROUPED, REREAD, DIRS)] = {act_bwd_kernel<ACT, DIRS, GROUPED, REREAD>,
                                        Cfg<ACT, true>::kThreads,
                                        smem_bytes<ACT, true>(false, 0), Cfg<ACT, true>::kSig};
}

// Every forward variant of one activation, dense or grouped (STAGED: also
// the staged-rounding ones; ILV: the interleaved gate / up input's).
template <int ACT, bool STAGED, bool GROUPED, bool ILV = false>
void fill_fwd(FwdVariant* t) {
  constexpr int I = ILV ? kIlv : 0;
#define MOEACT_FWD_DIRS(ST, G)                              \
  put_fwd<ACT, I | kRow, ST, G>(t);                         \
  put_fwd<ACT, I | kCol, ST, G>(t);                         \
  put_fwd<ACT, I | kRow | kCol, ST, G>(t);                  \
  put_fwd<ACT, I | kRow | kGemm, ST, G>(t);                 \
  put_fwd<ACT, I | kCol | kGemm, ST, G>(t);                 \
  put_fwd<ACT, I | kRow | kCol | kGemm, ST, G>(t);
  MOEACT_FWD_DIRS(false, GROUPED)
  if constexpr (STAGED) {
    MOEACT_FWD_DIRS(true, GROUPED)
  }
#undef MOEACT_FWD_DIRS
}

// Every backward variant of one activation, dense or grouped.
template <int ACT, bool GROUPED>
void fill_bwd(BwdVariant* t) {
#define MOEACT_BWD_DIRS(G, RR)                              \
  put_bwd<ACT, 0, G, RR>(t);                                \
  put_bwd<ACT, kRow, G, RR>(t);                             \
  put_bwd<ACT, kCol, G, RR>(t);                             \
  put_bwd<ACT, kRow | kCol, G, RR>(t);                      \
  put_bwd<ACT, kRow | kGemm, G, RR>(t);                     \
  put_bwd<ACT, kCol | kGemm, G, RR>(t);                     \
  put_bwd<ACT, kRow | kCol | kGemm, G, RR>(t);
  MOEACT_BWD_DIRS(GROUPED, false)
  MOEACT_BWD_DIRS(GROUPED, true)
#undef MOEACT_BWD_DIRS
}

// Defined in kern_<activation>_<pass>[_ilv]_<dense|grouped>.cu; each fills
// its entries of a kFwdSlots / kBwdSlots table (unused slots stay zero).
void fill_fwd_swiglu_dense(FwdVariant* t);
void fill_fwd_swiglu_grouped(FwdVariant* t);
void fill_fwd_swiglu_ilv_dense(FwdVariant* t);
void fill_fwd_swiglu_ilv_grouped(FwdVariant* t);
void fill_fwd_clamped_ilv_dense(FwdVariant* t);
void fill_fwd_clamped_ilv_grouped(FwdVariant* t);
void fill_bwd_swiglu_dense(BwdVariant* t);
void fill_bwd_swiglu_grouped(BwdVariant* t);
void fill_fwd_srelu_dense(FwdVariant* t);
void fill_fwd_srelu_grouped(FwdVariant* t);
void fill_bwd_srelu_dense(BwdVariant* t);
void fill_bwd_srelu_grouped(BwdVariant* t);
void fill_fwd_clamped_dense(FwdVariant* t);
void fill_fwd_clamped_grouped(FwdVariant* t);
void fill_bwd_clamped_dense(BwdVariant* t);
void fill_bwd_clamped_grouped(BwdVariant* t);

}  // namespace moeact
