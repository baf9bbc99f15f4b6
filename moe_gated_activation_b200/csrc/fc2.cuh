// The activation -> MXFP8 -> expert FC2 GEMM, fused on the tensor cores
// (kern_fc2.cu): the host side's view (parameters, shared-memory size,
// launcher).
//
// TransformerEngine PR #3238 (Greptile summary, sequence diagram): the
// grouped scaled activation hands its quantized grouped tensor straight to the
// grouped linear that follows it (ForwardScaledActivationGroupedLinear).  Here
// the two are one kernel: each CTA computes the rowwise MXFP8 of the scaled
// SwiGLU for one 128-row block of one expert into shared memory and
// multiplies it with that expert's MXFP8 FC2 weight on the tensor cores
// (tcgen05.mma kind::mxf8f6f4, block-scaled), so the quantized activation
// never goes to HBM.
#pragma once

#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

namespace moeact {

struct Fc2Params {
  const float* s;             // fp32 [M] row scales
  int64_t M;
  int N;                      // activation width = the GEMM's K (multiple of 128, <= 768)
  int H;                      // FC2 output width (multiple of 128)
  const int64_t* row_offs;    // [E + 1]
  int E;
  int32_t* status;
  const uint8_t* w_codes;     // E4M3, per expert H/128 x N/128 operand tiles of 16 KiB
  const uint8_t* w_scales;    // E8M0, per expert the [H, N/32] matrix in 128 x 4 tiles
  uint16_t* out;              // bf16 [M, ldo]
  int64_t ldo;
  const float* sig_src;       // the sigmoid table (device memory, shared-memory layout)
  const int32_t* noop;        // nullable
  uint32_t* err;              // device error word
  int n_sms;                  // SMs of the device (the last wave's blocks are split to fill them)
};

constexpr int kFc2MaxN = 768;
constexpr int kFc2Threads = 320;   // 8 math warps, a TMA warp, an MMA warp
constexpr int kFc2XBoxRows = 8;    // rows of X per tensor-map box (a prologue sub-slot)

// Dynamic shared memory of a launch with activation width N.
int fc2_smem_bytes(int N);
// Sets the kernels' shared-memory limit (once per device).
cudaError_t fc2_prepare();
// Launches the fused kernel: one CTA per 128-row block of an expert, or per
// part of one when the last wave of blocks is split over several CTAs
// (`grid` = ceil(M/128) + E + n_sms covers every split and every tail); tm_x
// is the bf16 [M, 2N] input in 128 x kFc2XBoxRows boxes.
cudaError_t fc2_launch(const Fc2Params& p, const CUtensorMap& tm_x, int staged, unsigned grid,
                       cudaStream_t stream);

}  // namespace moeact
