// The scaled SwiGLU + rowwise MXFP8 of an expert's rows fused with that
// expert's FC2 GEMM on the fifth-generation tensor cores (sm_100a).
//
// TransformerEngine PR #3238 (Greptile summary, sequence diagram): the
// grouped scaled activation emits quantized grouped storage that the grouped
// linear after it consumes (ForwardScaledActivationGroupedLinear).  Here both
// run in one kernel and the quantized activation stays on chip:
//
//   out[i, h] = sum_k A[i, k] * W_e[h, k]     (row i of expert e)
//
// A = rowwise MXFP8 (1 x 32 blocks along k, E8M0 RCEIL scales, E4M3 codes)
// of y = SwiGLU(x) * s, exactly as the stand-alone forward computes it;
// W_e = the expert's weight, MXFP8 with 1 x 32 blocks along k; the products
// of the block-scaled operands are summed by the tensor cores in fp32 and the
// result rounded to bf16.
//
// One CTA per (expert, 128-row block), or per range of its output tiles for
// the blocks of a last, partial wave (split so that the wave fills the SMs);
// 10 warps:
//   warps 0-7  prologue: stream the block's gate / up rows in by TMA (one
//              16-row half-tile slot per warp, as two 8-row sub-slots each
//              refilled as soon as it is read), compute y and its rowwise
//              MXFP8, write the codes into shared memory in the tensor
//              cores' K-major 128-byte-swizzled layout and the scales into
//              tensor memory; then, per 128-column output tile, drain the
//              accumulator (tcgen05.ld) into bf16 rows of `out`, warps 0-3
//              writing the weight scales of the tile two ahead into the
//              drained buffer's scale columns (tcgen05.st: a tcgen05.cp would
//              cost the tensor pipe time, measured 6% of the kernel);
//   warp 8     producer of the weight tiles (128 rows x 128 bytes of k,
//              stored pre-swizzled in the tensor cores' operand layout, so
//              each is one contiguous 16 KiB bulk copy), a 5-stage ring that
//              reuses the prologue's staging and sigmoid-table memory;
//   warp 9     allocates tensor memory and issues the MMAs (one thread):
//              tcgen05.mma.kind::mxf8f6f4.block_scale, M = N = 128, K = 32,
//              two accumulators in tensor memory so that one tile's drain
//              overlaps the next tile's MMAs.
// Every wait is bounded (one second); on a timeout the kernel records
// MOEACT_DEVERR_FC2_WAIT, lets its copies and MMAs in flight finish (bounded
// again), frees its tensor memory and returns.
#include "fc2.cuh"
#include "kernels.cuh"

namespace moeact {
namespace {

constexpr int kAtom = 16384;              // 128 rows x 128 bytes of k (one swizzle atom column)
constexpr int kEpiWarpBytes = 4096;       // the epilogue's per-warp staging: 32 rows x 128 B
constexpr int kEpiBytes = 8 * kEpiWarpBytes;
constexpr int kStageBytes = 16384;        // 128 weight rows x 128 bytes of k
constexpr int kXSlotBytes = 2 * kOpHalfBytes;   // gate + up of 16 rows x 128 columns
constexpr int kXBytes = 8 * kXSlotBytes;  // the prologue's slots (8 warps)
// A warp's slot as two sub-slots of kFc2XBoxRows rows (gate rows, then up
// rows), each refilled as soon as its rows are read.
constexpr int kXSub = 16 / kFc2XBoxRows;
constexpr int kXSubBytes = kXSlotBytes / kXSub;
constexpr int kXSubOpBytes = kXSubBytes / 2;
// The staging region: (prologue) the X slots and the sigmoid table after
// them; (GEMM) the weight ring and the epilogue's staging, as many ring stages
// as fit.
constexpr int kRBytes = (kXBytes + kSigBytes + 1023) / 1024 * 1024;
constexpr int kStages = (kRBytes - kEpiBytes) / kStageBytes;   // weight ring
constexpr int kMiscBytes = 2048;
constexpr int kSfSlotBytes = 512 * (kFc2MaxN / 128);   // a tile's weight scales (tiled layout)
constexpr int kSfSlots = 4;                               // loaded three tiles ahead
constexpr int kSfBytes = (kSfSlots * kSfSlotBytes + 1023) / 1024 * 1024;
constexpr int kSfaCol = 256;              // tensor-memory columns: accumulators [0, 256),
constexpr int kSfbCol = 288;              // A scales [256, 288), W scales [288, 352)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kErrFc2Wait = 0x20u;

constexpr int kXBars = 8 * kXSub;         // the prologue's sub-slot barriers
constexpr int kBarSlots = 64;             // mbarriers at the start of the misc region

// misc ints
constexpr int kMiscTmem = 0, kMiscAbort = 1, kMiscE = 2, kMiscBlk = 3, kMiscScan = 16;

// ------------------------------------------------------------ tcgen05 wrappers
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_addr(dst)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrives on `bar` once every tcgen05 operation this thread issued before has
// completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_addr(bar)) : "memory");
}
// D (+)= A x B^T with E8M0 block scales: A [128 x 32] and B [128 x 32] E4M3
// from shared-memory descriptors, scales from tensor memory.
__device__ __forceinline__ void tc_mma_mx(uint32_t d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                          uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p; }"
      ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
// Four 32-bit words into four consecutive columns of the warp's 32 lanes
// (thread t: lane t).
__device__ __forceinline__ void tc_st4(uint32_t taddr, uint32_t v0, uint32_t v1, uint32_t v2,
                                       uint32_t v3) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};"
               ::"r"(taddr), "r"(v0), "r"(v1), "r"(v2), "r"(v3) : "memory");
}
__device__ __forceinline__ void tc_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// 32 consecutive columns of the warp's 32 lanes (thread t: lane t).
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
        "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
        "=r"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Non-suspending test of a phase, and a spin on it bounded by the global
// timer: the single threads that feed the tensor cores (weight producer, MMA
// issuer) spin rather than suspend, as their wake-up latency is on the
// critical path (measured 2% faster than suspending waits).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{ .reg .pred p; mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2; "
               "selp.u32 %0, 1, 0, p; }"
               : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_spin(uint64_t* bar, uint32_t parity) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 64; ++i)
      if (mbar_test(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile in the 128-byte
// swizzled layout: rows of 128 bytes, 8-row groups 1024 bytes apart (the
// stride byte offset), 16-byte chunks of row r stored at chunk ^ (r mod 8);
// descriptor version 1 (sm_100).  `saddr` may sit 32, 64 or 96 bytes into a
// 1024-byte-aligned atom (the K steps of one atom).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::mxf8f6f4 with block scaling: E4M3 x E4M3,
// both K-major, N = 128 (bits 17-22: N / 8), E8M0 scales (bit 23), M = 128
// (bits 24-28: M / 16); the scale byte of each 32-bit tensor-memory word that
// this K step uses is `sf` for both operands (bits 4-5 and 29-30).
__device__ __forceinline__ uint32_t mx_idesc(uint32_t sf) {
  return (16u << 17) | (1u << 23) | (8u << 24) | (sf << 4) | (sf << 29);
}

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
  return p + ((1024u - (smem_addr(p) & 1023u)) & 1023u);
}

struct Fc2Smem {
  unsigned char* A;       // [N/128 atoms][128 rows][128 bytes], swizzled
  unsigned char* sf;      // [2 tiles][N/128 groups][512 bytes]: weight scales, tiled
  unsigned char* R;       // staging: weight ring / X slots + sigmoid table
  const float* sig;
  uint64_t* xbar;         // [8 * kXSub]: the prologue sub-slots, kXSub per warp
  uint64_t* sig_bar;
  uint64_t* pro_done;     // count 8: the block's A codes and scales are complete
  uint64_t* b_full;       // [kStages] a weight stage has landed
  uint64_t* b_empty;      // [kStages] ... and its MMAs are done
  uint64_t* sf_full;      // [kSfSlots] a tile's weight scales have landed in shared memory
  uint64_t* sf_empty;     // [kSfSlots] ... and have been copied to tensor memory (count 4)
  uint64_t* d_full;       // [2] an accumulator holds a finished tile
  uint64_t* d_empty;      // [2] count 8: an accumulator has been drained
  uint64_t* mma_done;
  int* misc;
};

__device__ __forceinline__ bool aborted(const Fc2Smem& m) {
  return *reinterpret_cast<volatile int*>(m.misc + kMiscAbort) != 0;
}
// The same verdict in every lane of the warp (the tcgen05 loads and stores
// that follow are warp-collective).
__device__ __forceinline__ bool warp_aborted(const Fc2Smem& m) {
  return __any_sync(kFull, aborted(m));
}
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  return __all_sync(kFull, mbar_wait(bar, parity));
}
__device__ __forceinline__ void set_abort(const Fc2Params& p, const Fc2Smem& m) {
  *reinterpret_cast<volatile int*>(m.misc + kMiscAbort) = 1;
  atomicOr(p.err, kErrFc2Wait);
}

// ------------------------------------------------------------ prologue
// One 16-row half of a warp-tile (32 rows of the block's quarter q x the 128
// columns of atom a): y = SwiGLU(g, u) * s, its rowwise E8M0 scales (returned
// packed as in fwd_tile: lane l holds blocks l >> 3 of rows 2 (l & 7) + {0,1})
// and its E4M3 codes, stored into the atom at the swizzled positions.
// The half's rows arrive in kXSub sub-slots: `wait(sub)` before a sub-slot's
// first row (false on a timeout: `ok` is cleared and nothing is written),
// `refill(sub)` once every lane has read its last row.
template <bool STAGED, typename Wait, typename Refill>
__device__ __forceinline__ uint32_t fc2_half(const Fc2Smem& m, const unsigned char* slot,
                                             int lane, int q, int a, int h, int nvq, float sv,
                                             Wait&& wait, Refill&& refill, bool& ok) {
  float Y[16][4];
  const unsigned char* sm = slot + 8 * lane;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int sub = i / kFc2XBoxRows, ri = i % kFc2XBoxRows;
    if (ri == 0 && !wait(sub)) {
      ok = false;
      return 0;
    }
    const uint2 G = *reinterpret_cast<const uint2*>(sm + sub * kXSubBytes + ri * kRowBytes);
    const uint2 U =
        *reinterpret_cast<const uint2*>(sm + sub * kXSubBytes + kXSubOpBytes + ri * kRowBytes);
    const float sr = __shfl_sync(kFull, sv, 16 * h + i);
    const float2 s2 = make_float2(sr, sr);
    float2 sg01, sg23;
    sigma_pair(m.sig, G.x, sg01.x, sg01.y);
    sigma_pair(m.sig, G.y, sg23.x, sg23.y);
    const float2 si01 = mul2(bf16x2_to_f2(G.x), sg01), si23 = mul2(bf16x2_to_f2(G.y), sg23);
    const float2 u01 = bf16x2_to_f2(U.x), u23 = bf16x2_to_f2(U.y);
    float2 h01, h23;
    if (STAGED) {
      const float2 a01 = bf16x2_to_f2(pack_bf16x2(si01.x, si01.y));
      const float2 a23 = bf16x2_to_f2(pack_bf16x2(si23.x, si23.y));
      const float2 p01 = mul2(a01, u01), p23 = mul2(a23, u23);
      h01 = bf16x2_to_f2(pack_bf16x2(p01.x, p01.y));
      h23 = bf16x2_to_f2(pack_bf16x2(p23.x, p23.y));
    } else {
      h01 = mul2(si01, u01);
      h23 = mul2(si23, u23);
    }
    const float2 y01 = mul2(h01, s2), y23 = mul2(h23, s2);
    const bool live = 16 * h + i < nvq;   // rows past the expert's end stay zero
    Y[i][0] = live ? y01.x : 0.0f;
    Y[i][1] = live ? y01.y : 0.0f;
    Y[i][2] = live ? y23.x : 0.0f;
    Y[i][3] = live ? y23.y : 0.0f;
    if (ri == kFc2XBoxRows - 1) {
      // every lane has read the sub-slot: its next copy overlaps the rest
      __syncwarp();
      refill(sub);
    }
  }
  uint32_t Am[16];
#pragma unroll
  for (int i = 0; i < 16; ++i)
    Am[i] = __float_as_uint(max_nan(max3_nan(fabsf(Y[i][0]), fabsf(Y[i][1]), fabsf(Y[i][2])),
                                    fabsf(Y[i][3])));
  bfly_max_u32<8>(Am, lane, 4);
  bfly_max_u32<4>(Am, lane, 2);
  bfly_max_u32<2>(Am, lane, 1);
  const uint32_t b0 = e8m0_from_amax(Am[0]), b1 = e8m0_from_amax(Am[1]);
  const uint32_t m0 = scale_multiplier(b0), m1 = scale_multiplier(b1);
  unsigned char* atom = m.A + a * kAtom;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t mm = __shfl_sync(kFull, (i & 1) ? m1 : m0, (lane & 24) | (i >> 1));
    const uint32_t code = e4m3x2_2(make_float2(Y[i][0], Y[i][1]), mm, mm) |
                          (e4m3x2_2(make_float2(Y[i][2], Y[i][3]), mm, mm) << 16);
    const int row = 32 * q + 16 * h + i;
    *reinterpret_cast<uint32_t*>(atom + row * 128 + ((((lane >> 2) ^ (row & 7))) << 4) +
                                 ((lane & 3) << 2)) = code;
  }
  return b0 | (b1 << 8);
}

// Warps 0-3 (warp q: lanes 32 q .. 32 q + 31): output tile t's weight scales
// from its shared-memory slot (N/128 groups of 512 bytes, row 32 c + l's four
// k-block scales at byte 16 l + 4 c) into the scale columns of accumulator
// buffer t & 1: lane l, column 4 g + c of every quarter holds row 32 c + l's
// word (the layout the MMA reads), written with tcgen05.st so that the
// tensor pipe spends no time on it.  The slot is released afterwards.
// Returns false on a timeout.
__device__ __forceinline__ bool fc2_put_w_scales(const Fc2Params& p, const Fc2Smem& m, int t,
                                                 int q, int lane, uint32_t tbase) {
  const int KA = p.N >> 7;
  if (!warp_wait(m.sf_full + t % kSfSlots, (uint32_t)(t / kSfSlots) & 1u)) return false;
  const unsigned char* src = m.sf + (t % kSfSlots) * kSfSlotBytes + 16 * lane;
  const uint32_t dst = tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)(kSfbCol + 32 * (t & 1));
  for (int g = 0; g < KA; ++g) {
    const uint4 w = *reinterpret_cast<const uint4*>(src + 512 * g);
    tc_st4(dst + 4 * g, w.x, w.y, w.z, w.w);
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(m.sf_empty + t % kSfSlots);
  tc_wait_st();
  return true;
}

template <bool STAGED>
__device__ void fc2_math(const CUtensorMap* tm_x, const Fc2Params& p, const Fc2Smem& m, int e,
                         int64_t row0, int mrows, uint32_t tbase, int t0, int T) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3, half_sel = warp >> 2;
  const int KA = p.N >> 7;
  const int nvq = max(0, min(32, mrows - 32 * q));   // rows of this quarter in the expert
  const int n_atoms = KA > half_sel ? (KA - half_sel + 1) / 2 : 0;
  const int Kw = 2 * n_atoms;                          // half-tiles of this warp
  unsigned char* slot = m.R + warp * kXSlotBytes;
  uint64_t* xb = m.xbar + kXSub * warp;
  // unit u: sub-slot u % kXSub of half-tile u / kXSub; sub-slot b's barrier
  // completes once per unit, parity (u / kXSub) & 1
  const int U = kXSub * Kw;
  auto issue = [&](int u) {
    const int j = u / kXSub, b = u % kXSub;
    const int a = half_sel + 2 * (j >> 1);
    const int y = (int)row0 + 32 * q + 16 * (j & 1) + kFc2XBoxRows * b;
    unsigned char* dst = slot + b * kXSubBytes;
    mbar_expect_tx(xb + b, kXSubBytes);
    tma_load_2d(dst, tm_x, 128 * a, y, xb + b);
    tma_load_2d(dst + kXSubOpBytes, tm_x, p.N + 128 * a, y, xb + b);
  };
  if (threadIdx.x == 0) {
    mbar_expect_tx(m.sig_bar, 2 * kSigHalfBytes);
    bulk_load(const_cast<float*>(m.sig), p.sig_src, kSigHalfBytes, m.sig_bar);
    bulk_load(const_cast<float*>(m.sig) + kSigNegOffset, p.sig_src + kSigNegOffset,
              kSigHalfBytes, m.sig_bar);
  }
  if (lane == 0)
    for (int u = 0; u < kXSub && u < U; ++u) issue(u);
  const float sv = lane < nvq ? __ldg(p.s + row0 + 32 * q + lane) : 0.0f;
  bool ok = warp_wait(m.sig_bar, 0u);
  int waited = 0;   // units whose copy this warp has seen land
  uint32_t bh0 = 0;
  for (int j = 0; ok && j < Kw; ++j) {
    const int a = half_sel + 2 * (j >> 1), h = j & 1;
    const uint32_t bh = fc2_half<STAGED>(
        m, slot, lane, q, a, h, nvq, sv,
        [&](int b) {
          const int u = kXSub * j + b;
          if (!warp_wait(xb + b, (uint32_t)(u / kXSub) & 1u)) return false;
          waited = u + 1;
          return true;
        },
        [&](int b) {
          const int u = kXSub * (j + 1) + b;
          if (lane == 0 && u < U) issue(u);
        },
        ok);
    if (!ok) break;
    if (h == 0) {
      bh0 = bh;
    } else {
      // lane l: the four block scales of row 32 q + l for atom a.  The MMA
      // reads the scale of its M-operand row 32 q + l from lane 32 q + l,
      // column q of the group (the layout fc2_put_w_scales writes the
      // weight's scales in, of which each quarter needs only its own
      // column); the word goes to all four.
      const uint32_t v = gather_row_scales(bh0, bh, lane, 0, 1);
      tc_st4(tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)(kSfaCol + 4 * a), v, v, v, v);
    }
  }
  if (!ok) {
    set_abort(p, m);
    // copies this warp issued that never landed: wait for them (bounded)
    if (lane == 0) {
      for (int u = waited; u < U && u < waited + kXSub; ++u)
        mbar_wait(xb + u % kXSub, (uint32_t)(u / kXSub) & 1u);
      mbar_wait(m.sig_bar, 0u);
    }
  }
  // the weight scales of the first two output tiles
  if (ok && half_sel == 0)
    for (int t = 0; t < 2 && t < T; ++t)
      if (!fc2_put_w_scales(p, m, t, q, lane, tbase)) {
        set_abort(p, m);
        break;
      }
  tc_wait_st();
  fence_proxy_async_smem();   // the codes written above are read by the tensor cores
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(m.pro_done);

  // ---- output tiles: drain each accumulator into bf16 rows
  for (int n = 0; n < T; ++n) {
    if (warp_aborted(m)) break;
    const int b = n & 1;
    if (!warp_wait(m.d_full + b, (uint32_t)(n >> 1) & 1u)) { set_abort(p, m); break; }
    tc_fence_after();
    uint32_t v[64];
    const uint32_t t = tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)(128 * b + 64 * half_sel);
    tc_ld32(t, v);
    tc_ld32(t + 32, v + 32);
    tc_wait_ld();
    // buffer b's scale columns are free (tile n's MMAs are done): tile n + 2's
    // go there before the buffer is released
    if (half_sel == 0 && n + 2 < T && !fc2_put_w_scales(p, m, n + 2, q, lane, tbase)) {
      set_abort(p, m);
      break;
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(m.d_empty + b);
    // through this warp's staging in shared memory (16-byte chunk c of row t
    // at chunk c ^ (a function of t), so that 8 consecutive threads or rows
    // touch 8 different bank groups), then several lanes per row: each store
    // instruction writes whole row segments
    unsigned char* stg = m.R + kStages * kStageBytes + warp * kEpiWarpBytes;
    constexpr int kChunks = kEpiWarpBytes / 32 / 16;      // 16-byte chunks of a staged row
    constexpr int kPasses = 8 / kChunks;
#pragma unroll
    for (int ps = 0; ps < kPasses; ++ps) {
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        const uint32_t* vv = v + 8 * (ps * kChunks + c);
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(vv[0]), __uint_as_float(vv[1]));
        w.y = pack_bf16x2(__uint_as_float(vv[2]), __uint_as_float(vv[3]));
        w.z = pack_bf16x2(__uint_as_float(vv[4]), __uint_as_float(vv[5]));
        w.w = pack_bf16x2(__uint_as_float(vv[6]), __uint_as_float(vv[7]));
        const int sw = kChunks == 8 ? (lane & 7) : ((lane >> 1) & 3);
        *reinterpret_cast<uint4*>(stg + lane * (16 * kChunks) + ((c ^ sw) << 4)) = w;
      }
      __syncwarp();
      const int cc = lane % kChunks;
#pragma unroll
      for (int k = 0; k < kChunks; ++k) {
        const int r = (32 / kChunks) * k + lane / kChunks;
        const int sw = kChunks == 8 ? (r & 7) : ((r >> 1) & 3);
        const uint4 w = *reinterpret_cast<const uint4*>(stg + r * (16 * kChunks) + ((cc ^ sw) << 4));
        if (32 * q + r < mrows)
          *reinterpret_cast<uint4*>(p.out + (row0 + 32 * q + r) * p.ldo + 128 * (t0 + n) +
                                    64 * half_sel + 8 * (ps * kChunks + cc)) = w;
      }
      __syncwarp();
    }
  }
}

// One lane of a converged warp (elect.sync), the same lane every call.
__device__ __forceinline__ bool elect_one() {
  uint32_t r;
  asm volatile("{ .reg .pred p; elect.sync _|p, 0xffffffff; selp.u32 %0, 1, 0, p; }" : "=r"(r));
  return r != 0;
}

// Warp 8, converged, one elected lane issuing (as the MMA warp, for the same
// reason): the weight tiles of every output tile, in k order (each a
// contiguous 16 KiB of the tiled weight: one bulk copy, which streams into an
// SM faster than a 2-D tensor copy of the same tile), and each output tile's
// weight scales (N/128 tiles of 512 bytes, contiguous in the tiled layout)
// kSfSlots - 1 output tiles ahead: the scales of tile n + 3 go out after the
// last weight tile of tile n, when the slot they reuse (tile n - 1's) is
// already free, and have two tiles of MMAs to land.
__device__ void fc2_producer(const Fc2Params& p, const Fc2Smem& m, int e, int t0, int T) {
  const int KA = p.N >> 7;
  const int64_t tile0 = (int64_t)e * (p.H >> 7) + t0;   // the expert's tile t0 in the tiled layout
  const bool leader = elect_one();
  int issued = 0, sf_issued = 0;
  auto issue_sf = [&](int n) {   // false on a timeout
    const int ss = n % kSfSlots;
    if (n >= kSfSlots &&
        !__all_sync(kFull, mbar_spin(m.sf_empty + ss, (uint32_t)(n / kSfSlots - 1) & 1u)))
      return false;
    if (leader) {
      mbar_expect_tx(m.sf_full + ss, 512 * KA);
      bulk_load(m.sf + ss * kSfSlotBytes, p.w_scales + (tile0 + n) * KA * 512, 512 * KA,
                m.sf_full + ss);
    }
    __syncwarp();
    sf_issued = n + 1;
    return true;
  };
  // the first scales do not wait for the prologue (their slots are not
  // shared with it); the weight tiles reuse the prologue's staging memory
  for (int n = 0; n < T && n < kSfSlots - 1; ++n) issue_sf(n);
  if (!__all_sync(kFull, mbar_wait(m.pro_done, 0u)) && leader) set_abort(p, m);
  const uint8_t* wsrc = p.w_codes + tile0 * KA * kStageBytes;
  for (int g = 0; g < T * KA && !warp_aborted(m); ++g) {
    const int n = g / KA, ks = g - n * KA, slot = g % kStages;
    if (g >= kStages &&
        !__all_sync(kFull, mbar_spin(m.b_empty + slot, (uint32_t)(g / kStages - 1) & 1u))) {
      if (leader) set_abort(p, m);
      break;
    }
    if (leader) {
      mbar_expect_tx(m.b_full + slot, kStageBytes);
      bulk_load(m.R + slot * kStageBytes, wsrc + (int64_t)g * kStageBytes, kStageBytes,
                m.b_full + slot);
    }
    __syncwarp();
    issued = g + 1;
    if (ks == KA - 1 && n + kSfSlots - 1 < T && !issue_sf(n + kSfSlots - 1)) {
      if (leader) set_abort(p, m);
      break;
    }
  }
  // every copy issued has landed before the CTA can exit (bounded)
  if (leader) {
    for (int g = max(0, issued - kStages); g < issued; ++g)
      mbar_wait(m.b_full + g % kStages, (uint32_t)(g / kStages) & 1u);
    for (int n = max(0, sf_issued - kSfSlots); n < sf_issued; ++n)
      mbar_wait(m.sf_full + n % kSfSlots, (uint32_t)(n / kSfSlots) & 1u);
  }
  __syncwarp();
}

// Warp 9, the whole warp converged, one elected lane issuing: the MMAs of
// every output tile.  The loop runs on all 32 lanes so that its operands
// (descriptors, tensor-memory addresses) are warp-uniform values the
// tcgen05 instructions take directly; issued from a single-thread branch
// they were rebuilt before every MMA, and the issue, not the tensor pipe,
// set the rate.  A K step of 32 bytes advances a descriptor's start-address
// field by 2 (16-byte units; shared-memory addresses stay below 2^18, so
// the field never carries).
__device__ void fc2_mma(const Fc2Params& p, const Fc2Smem& m, uint32_t tbase, int T) {
  const int KA = p.N >> 7;
  const bool leader = elect_one();
  bool ok = __all_sync(kFull, mbar_wait(m.pro_done, 0u)) && !warp_aborted(m);
  if (!ok && leader) set_abort(p, m);
  tc_fence_after();
  const uint64_t a_desc0 = umma_desc_sw128(smem_addr(m.A));
  const uint64_t b_desc0 = umma_desc_sw128(smem_addr(m.R));
  for (int n = 0; ok && n < T; ++n) {
    const int b = n & 1;
    // accumulator b is free, and holds tile n's weight scales, once tile
    // n - 2 has been drained (tiles 0 and 1: once the prologue is done)
    if (n >= 2 && !__all_sync(kFull, mbar_spin(m.d_empty + b, (uint32_t)((n >> 1) - 1) & 1u))) {
      ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t d = tbase + 128 * b;
    for (int ks = 0; ks < KA; ++ks) {
      const int g = n * KA + ks, slot = g % kStages;
      if (warp_aborted(m) ||
          !__all_sync(kFull, mbar_spin(m.b_full + slot, (uint32_t)(g / kStages) & 1u))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t ad = a_desc0 + (uint64_t)((ks * kAtom) >> 4);
      const uint64_t bd = b_desc0 + (uint64_t)((slot * kStageBytes) >> 4);
      const uint32_t sfa = tbase + kSfaCol + 4 * ks, sfb = tbase + kSfbCol + 32 * b + 4 * ks;
      if (leader) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tc_mma_mx(d, ad + 2 * j, bd + 2 * j, mx_idesc((uint32_t)j), sfa, sfb,
                    (ks | j) != 0 ? 1u : 0u);
        tc_commit(m.b_empty + slot);   // the stage is free once these MMAs are done
      }
      __syncwarp();
    }
    if (!ok) break;
    if (leader) tc_commit(m.d_full + b);
    __syncwarp();
  }
  if (!ok && leader) set_abort(p, m);
  // every MMA issued has completed before tensor memory is freed (bounded)
  if (leader) {
    tc_commit(m.mma_done);
    mbar_wait(m.mma_done, 0u);
  }
  __syncwarp();
}

template <bool STAGED>
__global__ void __launch_bounds__(kFc2Threads, 1)
    fc2_kernel(const __grid_constant__ CUtensorMap tm_x, const Fc2Params p) {
  if (p.noop != nullptr && *p.noop != 0) return;
  extern __shared__ __align__(1024) unsigned char fc2_smem[];
  unsigned char* base = align1024(fc2_smem);
  Fc2Smem m;
  const int KA = p.N >> 7;
  m.A = base;
  m.sf = base + KA * kAtom;
  m.R = m.sf + kSfBytes;
  m.sig = reinterpret_cast<const float*>(m.R + kXBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(m.R + kRBytes);
  m.xbar = bars;
  m.sig_bar = bars + kXBars;
  m.pro_done = bars + kXBars + 1;
  m.b_full = bars + kXBars + 2;
  m.b_empty = m.b_full + kStages;
  m.sf_full = m.b_empty + kStages;
  m.sf_empty = m.sf_full + kSfSlots;
  m.d_full = m.sf_empty + kSfSlots;
  m.d_empty = m.d_full + 2;
  m.mma_done = m.d_empty + 2;
  m.misc = reinterpret_cast<int*>(bars + kBarSlots);
  const int tid = threadIdx.x, warp = tid >> 5;

  // ---- this CTA's (expert, 128-row block); the offsets are validated first
  const int E = p.E;
  const int C = (E + kFc2Threads - 1) / kFc2Threads;
  const int e_lo = min(E, tid * C), e_hi = min(E, e_lo + C);
  int local = 0, bad = 0;
  for (int e = e_lo; e < e_hi; ++e) {
    const int64_t r0 = p.row_offs[e], r1 = p.row_offs[e + 1];
    if (r1 < r0 || r0 < 0 || r1 > p.M) bad = 1;
    else local += (int)((r1 - r0 + 127) >> 7);
  }
  if (tid == 0 && (p.row_offs[0] != 0 || p.row_offs[E] != p.M)) bad = 1;
  // exclusive prefix of the per-thread block counts: a shuffle scan inside
  // each warp, then the 10 warp totals
  const int lane0 = tid & 31;
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(kFull, incl, off);
    if (lane0 >= off) incl += v;
  }
  if (lane0 == 31) m.misc[kMiscScan + warp] = incl;
  const int any_bad = __syncthreads_or(bad);
  if (blockIdx.x == 0 && tid == 0) *p.status = any_bad ? 3 : 0;
  if (any_bad) return;
  int wbase = 0, total = 0;
  for (int w = 0; w < kFc2Threads / 32; ++w) {
    const int v = m.misc[kMiscScan + w];
    if (w < warp) wbase += v;
    total += v;
  }
  // this CTA's block and output tiles [t0, t0 + tn): blocks of the whole
  // waves take every tile; when the last wave holds r < n_sms blocks, each of
  // its blocks is split over k = min(n_sms / r, T) CTAs by output tiles (each
  // part repeats the block's prologue), so that the wave fills the SMs
  const int T = p.H >> 7;
  const int r_tail = total % p.n_sms;
  const int k_split = r_tail > 0 ? min(p.n_sms / r_tail, T) : 1;
  const int n_whole = total - (k_split > 1 ? r_tail : 0);
  int u = blockIdx.x, t0 = 0, tn = T;
  if (u >= n_whole) {
    const int v = u - n_whole;
    if (k_split == 1 || v >= r_tail * k_split) return;
    const int part = v % k_split;
    u = n_whole + v / k_split;
    t0 = part * T / k_split;
    tn = (part + 1) * T / k_split - t0;
  }
  {
    int acc = wbase + incl - local;
    if (u >= acc && u < acc + local) {
      for (int e = e_lo; e < e_hi; ++e) {
        const int nb = (int)((p.row_offs[e + 1] - p.row_offs[e] + 127) >> 7);
        if (u < acc + nb) {
          m.misc[kMiscE] = e;
          m.misc[kMiscBlk] = u - acc;
          break;
        }
        acc += nb;
      }
    }
  }
  __syncthreads();
  const int e = m.misc[kMiscE];
  const int64_t row0 = p.row_offs[e] + 128 * (int64_t)m.misc[kMiscBlk];
  const int mrows = (int)min((int64_t)128, p.row_offs[e + 1] - row0);

  // ---- barriers and tensor memory
  if (tid == 0) {
    for (int i = 0; i < kXBars; ++i) mbar_init(m.xbar + i, 1);
    mbar_init(m.sig_bar, 1);
    mbar_init(m.pro_done, 8);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(m.b_full + i, 1);
      mbar_init(m.b_empty + i, 1);
    }
    for (int i = 0; i < kSfSlots; ++i) {
      mbar_init(m.sf_full + i, 1);
      mbar_init(m.sf_empty + i, 4);   // warps 0-3 have copied the slot to tensor memory
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(m.d_full + i, 1);
      mbar_init(m.d_empty + i, 8);
    }
    mbar_init(m.mma_done, 1);
    m.misc[kMiscAbort] = 0;
    mbar_init_fence();
  }
  if (warp == 9) {
    tmem_alloc(reinterpret_cast<uint32_t*>(m.misc + kMiscTmem), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(m.misc + kMiscTmem);

  if (warp < 8) {
    fc2_math<STAGED>(&tm_x, p, m, e, row0, mrows, tbase, t0, tn);
  } else if (warp == 8) {
    fc2_producer(p, m, e, t0, tn);
  } else {
    fc2_mma(p, m, tbase, tn);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

}  // namespace

int fc2_smem_bytes(int N) { return 1024 + (N / 128) * kAtom + kSfBytes + kRBytes + kMiscBytes; }

cudaError_t fc2_prepare() {
  const int bytes = fc2_smem_bytes(kFc2MaxN);
  cudaError_t e = cudaFuncSetAttribute(fc2_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(fc2_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes);
  return e;
}

cudaError_t fc2_launch(const Fc2Params& p, const CUtensorMap& tm_x, int staged, unsigned grid,
                       cudaStream_t stream) {
  const int bytes = fc2_smem_bytes(p.N);
  if (staged)
    fc2_kernel<true><<<grid, kFc2Threads, bytes, stream>>>(tm_x, p);
  else
    fc2_kernel<false><<<grid, kFc2Threads, bytes, stream>>>(tm_x, p);
  return cudaGetLastError();
}

static_assert(kMiscScan * 4 + (kFc2Threads / 32) * 4 + kBarSlots * 8 <= kMiscBytes,
              "misc region too small");
static_assert(kXBars + 2 + 2 * kStages + 2 * kSfSlots + 5 <= kBarSlots,
              "barrier region too small");
static_assert(16 % kFc2XBoxRows == 0 && kXSubBytes % 128 == 0, "sub-slot geometry");
static_assert(kSfBytes % 1024 == 0, "the staging region must stay 1024-byte aligned");
static_assert(kXBytes + kSigBytes <= kRBytes, "staging region too small");
static_assert(kStages * kStageBytes + kEpiBytes <= kRBytes && kStages >= 4,
              "epilogue staging does not fit");
static_assert(kSfbCol + 64 <= (int)kTmemCols && kSfaCol + 32 <= kSfbCol,
              "tensor-memory columns overlap");

}  // namespace moeact
