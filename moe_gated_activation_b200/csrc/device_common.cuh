// Device helpers shared by the kernels of libmoeact: bf16 unpacking, the
// sigmoid table lookup, the RCEIL E8M0 exponent and E4M3 packing.
//
// Numerics follow pytorch/ao PR #4743 "[mxfp8 training] Add a fused
// gated-activation (SwiGLU) + MXFP8 quantization kernel" (Summary: RCEIL
// MXFP8 cast of the SwiGLU output, 1x32 / 32x1 blocks) with the readings stated
// in include/moeact.h.  Every fp32 step is an explicit round-to-nearest
// intrinsic so that no multiply-add contraction can change a rounding.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace moeact {

constexpr unsigned kFull = 0xFFFFFFFFu;

// ---------------------------------------------------------------- sigmoid
// The table holds the correctly rounded fp32 sigma(g) for every bf16 g with
// |g| in [2^-25, 128] (bit patterns 0x3300..0x4300), positive then negative.
// Outside that range sigma rounds to 0.5 (|g| < 2^-24), 1 (g > 17.33) or +0
// (g < -103.97), so clamping the magnitude to the range end gives the right
// value; NaN inputs are caught by silu = g * sigma, which is NaN.
constexpr uint32_t kSigLo = 0x3300u;
constexpr uint32_t kSigHi = 0x4300u;
constexpr uint32_t kSigPerSign = kSigHi - kSigLo + 1;   // 4097
constexpr int kSigEntries = 2 * kSigPerSign;            // 8194 (global copy: +, then -)
constexpr int kSigEntriesPadded = 8196;                 // whole float4s

// Shared-memory copy: positive gates at float index m, negative gates at
// 8192 + m (m = clamped magnitude - 0x3300), so that the sign bit of the bf16
// (0x8000) is itself the byte offset 32768 between the two halves.
constexpr int kSigNegOffset = 8192;
constexpr int kSigBytes = (kSigNegOffset + kSigPerSign + 3) / 4 * 16;   // 49168
constexpr int kSigHalfBytes = (kSigPerSign + 3) / 4 * 16;                 // 16400

// sigma of both bf16 values of a packed pair: both byte offsets are computed
// at once in 16-bit lanes (clamp of the magnitude, minus the range start,
// times 4, plus the sign bit as the 32 KiB offset of the negative half).
__device__ __forceinline__ void sigma_pair(const float* tab, uint32_t G, float& s_lo,
                                           float& s_hi) {
  const uint32_t lo2 = kSigLo * 0x10001u, hi2 = kSigHi * 0x10001u;
  const uint32_t c = __vimin3_u16x2(__vimax3_u16x2(G & 0x7FFF7FFFu, lo2, lo2), hi2, hi2);
  const uint32_t off = (c - lo2) * 4u + (G & 0x80008000u);
  const unsigned char* tb = reinterpret_cast<const unsigned char*>(tab);
  s_lo = *reinterpret_cast<const float*>(tb + (off & 0xFFFFu));
  s_hi = *reinterpret_cast<const float*>(tb + (off >> 16));
}

// The same pair lookup on a table in shared memory whose highest address is
// below 64 KiB, with the table's address folded into one constant, `key`
// (sigma_key): both 16-bit lanes of c * 4 + key + sign bits are then the two
// entries' shared-memory addresses.  The low lane's c * 4 + key always
// carries exactly one into the high lane (its low half of key is
// T - 4 lo + 2^16 for a table at T, and 4 c - 4 lo + T < 2^16), which the
// high half of key pre-subtracts; the sign bits add 32 KiB to a lane without
// a carry (T + 4 (hi - lo) + 32 KiB + 4 < 2^16 for T < 16 KiB).
__host__ __device__ constexpr uint32_t sigma_key(uint32_t T) {
  return ((T - 4u * kSigLo) & 0xFFFFu) | (((T - 4u * kSigLo - 1u) & 0xFFFFu) << 16);
}

// A plain (non-volatile) shared load: ordered after the table's copy only
// through its address, which the callers derive from data read after the
// copy's barrier.
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sigma_pair_s(uint32_t key, uint32_t G, float& s_lo,
                                             float& s_hi) {
  const uint32_t lo2 = kSigLo * 0x10001u, hi2 = kSigHi * 0x10001u;
  const uint32_t c = __vimin3_u16x2(__vimax3_u16x2(G & 0x7FFF7FFFu, lo2, lo2), hi2, hi2);
  const uint32_t a = c * 4u + key + (G & 0x80008000u);
  s_lo = lds_f32(a & 0xFFFFu);
  s_hi = lds_f32(a >> 16);
}

// ---------------------------------------------------------------- bf16
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// The same unpacking through a byte permute; used where a second pass over
// values that an earlier pass already unpacked must not share (and keep
// alive) the earlier pass's fp32 copies.
__device__ __forceinline__ float bf16_lo_p(uint32_t v) { return __uint_as_float(__byte_perm(v, 0u, 0x1044)); }
__device__ __forceinline__ float bf16_hi_p(uint32_t v) { return __uint_as_float(__byte_perm(v, 0u, 0x3244)); }

// Two fp32 values -> packed bf16x2 (a in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Per 16-bit lane of two packed bf16 pairs: 0xFFFF where a > b, else 0 (an
// ordered comparison: false when either value is NaN).
__device__ __forceinline__ uint32_t bf16x2_gt_mask(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("set.gt.u32.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Per 16-bit lane: 0xFFFF where a != b (ordered: false when either is NaN).
__device__ __forceinline__ uint32_t bf16x2_ne_mask(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("set.ne.u32.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// NaN-propagating minimum / maximum of two packed bf16 pairs (exact).
__device__ __forceinline__ uint32_t bf16x2_min_nan(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.NaN.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_max_nan(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// relu that keeps NaN (NaN in -> NaN out); negative and zero inputs give +0.
__device__ __forceinline__ float relu_keep_nan(float v) {
  return v > 0.0f ? v : (v != v ? v : 0.0f);
}

// ---------------------------------------------------------------- E8M0
// RCEIL shared exponent from the magnitude bits of the block amax (an fp32
// bit pattern with the sign cleared; NaN patterns compare above +Inf so an
// integer max over magnitudes is NaN-propagating).  b = 127 + e with e the
// smallest integer such that amax <= 448 * 2^e: for a normal amax with biased
// exponent E and mantissa m that is E - 8, plus one when m > 0x600000
// (amax above 1.75 * 2^(E-127)); adding 0x1FFFFF carries exactly then.
// Subnormal and zero amax clamp to 0; +Inf gives 254; NaN 255.
__device__ __forceinline__ uint32_t e8m0_from_amax(uint32_t amag) {
  if (amag >= 0x7F800000u) return amag == 0x7F800000u ? 254u : 255u;
  const int b = (int)((amag + 0x1FFFFFu) >> 23) - 8;
  return (uint32_t)max(b, 0);
}

constexpr uint32_t kNanScale = 0x7FC00000u;

// Bit pattern of the quantization multiplier 2^(127-b): 2^127 .. 2^-126 as a
// normal float, 2^-127 as the subnormal 0x00400000, and a NaN marker for the
// NaN scale 255 (whose block is all 0x7F codes).
__device__ __forceinline__ uint32_t scale_multiplier(uint32_t b) {
  return b < 254u ? (254u - b) << 23 : (b == 254u ? 0x00400000u : kNanScale);
}

// A copy of v the compiler cannot see through: used so that a later pass
// recomputes per-row addresses instead of keeping an earlier pass's live.
__device__ __forceinline__ int opaque(int v) {
  int r;
  asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(v));
  return r;
}

// ---------------------------------------------------------------- packed fp32
// sm_100 packed fp32 arithmetic: two independent IEEE operations (round to
// nearest even, subnormals kept) in one instruction.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 r;
  asm("{ .reg .b64 ra, rb, rd; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5}; "
      "mul.rn.f32x2 rd, ra, rb; mov.b64 {%0, %1}, rd; }"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{ .reg .b64 ra, rb, rc, rd; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5}; "
      "mov.b64 rc, {%6, %7}; fma.rn.f32x2 rd, ra, rb, rc; mov.b64 {%0, %1}, rd; }"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 r;
  asm("{ .reg .b64 ra, rb, rd; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5}; "
      "add.rn.f32x2 rd, ra, rb; mov.b64 {%0, %1}, rd; }"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 r;
  asm("{ .reg .b64 ra, rb, rd; mov.b64 ra, {%2, %3}; mov.b64 rb, {%4, %5}; "
      "sub.rn.f32x2 rd, ra, rb; mov.b64 {%0, %1}, rd; }"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t v) { return make_float2(bf16_lo(v), bf16_hi(v)); }
__device__ __forceinline__ float2 bf16x2_to_f2_p(uint32_t v) { return make_float2(bf16_lo_p(v), bf16_hi_p(v)); }

// Two E4M3 codes (low byte: v.x): nearest even of v.x * ma and v.y * mb
// (ma, mb the bit patterns of the multipliers 2^(127-b)), saturating, through
// one packed multiply.  For the NaN scale (b = 255) the multiplier is a NaN,
// the product is NaN and the conversion gives the E4M3 NaN code 0x7F.
__device__ __forceinline__ uint32_t e4m3x2_2(float2 v, uint32_t ma, uint32_t mb) {
  const float2 q = mul2(v, make_float2(__uint_as_float(ma), __uint_as_float(mb)));
  return (uint32_t)__nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);
}


// ---------------------------------------------------------------- TMA / mbarrier
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

// Nanoseconds of the GPU's global timer.
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Tests whether the phase of `bar` with the given parity has completed; a
// thread whose phase has not completed is suspended until it does or
// `hint_ns` nanoseconds pass (it takes no issue slots from the warps that are
// working meanwhile).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; "
               "selp.u32 %0, 1, 0, p; }"
               : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns) : "memory");
  return ok != 0;
}

// Waits for a phase of `bar` for at most `limit_ns` nanoseconds of wall time
// (the global timer is read every 4 polls); false on timeout.  Each poll
// may suspend the thread for up to 100 us -- it resumes as soon as the phase
// completes -- so that a warp waiting for its data takes no issue slots from
// the warps that compute (measured 1-2% faster on the Qwen3-MoE-shaped
// workload, neutral on the largest).  A copy of a few KiB lands in
// microseconds, so the kernels' limit, one second, is only ever reached by a
// copy that will never complete.
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr uint32_t kWaitHintNs = 100000;
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait_sleep(bar, parity, kWaitHintNs)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 4; ++i)
      if (mbar_try_wait_sleep(bar, parity, kWaitHintNs)) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  return mbar_wait_for(bar, parity, kWaitLimitNs);
}

// 1-D bulk copy (this CTA only) of `bytes` (a multiple of 16, both addresses
// 16-byte aligned) from global to shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// 2-D TMA tile load (this CTA only) of box {x .. x+bx, y .. y+by} into shared
// memory, completing on `bar`; rows and columns outside the tensor read zero.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y),
        "r"(smem_addr(bar))
      : "memory");
}

// 3-D box load: coordinates (x, z, y) of a [rows][2][width] view (z selects
// the gate or the up half of a SwiGLU input row).
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, int x, int z, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(z), "r"(y),
        "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const void* tmap, int x, int z, int w,
                                            int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5}], [%6];"
      ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(z), "r"(w),
        "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// ---------------------------------------------------------------- warp butterflies
// "Transposed" butterfly: each lane holds one value per row for 2*HALF rows;
// after the step it holds HALF partial reductions, over lanes {l, l ^ off},
// for the rows selected by bit `off` of the lane.  Chaining the steps for
// off = 8, 4, 2, 1 leaves lane l with rows 2(l & 15) and 2(l & 15) + 1 reduced
// over its 16-lane half; chaining off = 16 .. 1 leaves lane l with row l
// reduced over the warp.  The order of every reduction is fixed.
template <int HALF>
__device__ __forceinline__ void bfly_max_u32(uint32_t* a, int lane, int off) {
  const bool up = (lane & off) != 0;
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const uint32_t send = up ? a[i] : a[HALF + i];
    const uint32_t keep = a[i] ^ a[HALF + i] ^ send;
    a[i] = max(keep, __shfl_xor_sync(kFull, send, off));
  }
}

// Same on two packed 16-bit magnitudes per word.
template <int HALF>
__device__ __forceinline__ void bfly_max_u16x2(uint32_t* a, int lane, int off) {
  const bool up = (lane & off) != 0;
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const uint32_t send = up ? a[i] : a[HALF + i];
    const uint32_t keep = a[i] ^ a[HALF + i] ^ send;
    a[i] = __vmaxu2(keep, __shfl_xor_sync(kFull, send, off));
  }
}

template <int HALF>
__device__ __forceinline__ void bfly_sum_f32(float* a, int lane, int off) {
  const bool up = (lane & off) != 0;
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const float send = up ? a[i] : a[HALF + i];
    const float keep = __uint_as_float(__float_as_uint(a[i]) ^ __float_as_uint(a[HALF + i]) ^
                                       __float_as_uint(send));
    a[i] = __fadd_rn(keep, __shfl_xor_sync(kFull, send, off));
  }
}

}  // namespace moeact
