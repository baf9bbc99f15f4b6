// Kernels of libmoeact (sm_100a).
//
// * sigma_table_init  -- builds the correctly rounded fp32 sigmoid table once
//                        per device (binary64 evaluation + rounding check).
// * splits_kernel     -- m_splits -> row / col-block offsets and a status
//                        (TransformerEngine PR #3238, Greptile summary:
//                        splits_to_offsets_multi computes all offsets once).
// * act_fwd_kernel    -- scaled SwiGLU / SReLU fused with the MXFP8 cast,
//                        rowwise 1x32 and/or colwise 32x1 from one read of the
//                        input (pytorch/ao PR #4743, Summary).
// * act_bwd_kernel    -- dgate / dup (bf16), per-row dscale and the MXFP8 of
//                        the gradient in one pass (TransformerEngine PR #3238,
//                        sequence diagram: grouped_dy quantized, dense_dy,
//                        grad_scales; pytorch/ao PR #4743, API).
//
// Work decomposition (both fused kernels).  A work item is one warp-tile:
// 32 rows (one colwise block, never crossing an expert boundary) x 64
// columns; lane l owns columns 2l and 2l+1 for all 32 rows, so the colwise
// amax is a per-lane loop over registers and the rowwise 1x32 amax is a
// 16-lane reduction.  The grid is persistent (one CTA per SM, the sigmoid
// table staged once per CTA in shared memory); warps walk the items
// slab-major so that neighbouring warps read neighbouring columns of the same
// rows.
//
// Data movement.  Each warp owns a ring of shared-memory slots, each holding
// one 16-row half of a warp-tile's inputs ([16 x 64] bf16 per operand), filled
// by TMA (cp.async.bulk.tensor, no multicast) and signalled through one
// mbarrier per slot.  Lane 0 keeps two half-tiles in flight ahead of the one
// being computed, so the warp never waits on global-memory latency and the
// inputs never occupy registers; rows and columns outside the tensor arrive
// as zeros.  Lanes read their two columns of each row from shared memory
// (conflict-free: a warp reads one 128-byte row).  Codes, scales and
// gradients are stored directly, 64 (codes) or 128 (bf16) contiguous bytes
// per warp per row; full tiles take a path without bounds predicates.
#pragma once

#include <cstdint>

#include <cuda.h>

#include "device_common.cuh"

namespace moeact {

enum Act : int { kSwiGLU = 0, kSReLU = 1 };
constexpr int kRow = 1;
constexpr int kCol = 2;
constexpr int kTileCols = 64;

// The table lives in device global memory of this module: one copy per
// device, written by sigma_table_init before any activation kernel reads it.
__device__ __align__(16) float g_sigma_table[kSigEntriesPadded];

// Builds the table.  For |g| < 2^-9, sigma(g) = 1/2 + g/4 - g^3/48 + O(g^5):
// hi = 1/2 + g/4 is exact in binary64 and the rest is far smaller than any
// distance from hi to an fp32 rounding boundary except when hi sits exactly on
// one (a midpoint), where binary64 cannot see the remainder; there the
// remainder's sign (that of -g) decides.  Elsewhere the table comes from
// binary64 exp and division (error < 2^-51 relative), and entries whose
// binary64 value lies within 2^-48 (relative) of a rounding boundary are
// counted as uncertain (none are expected: the closest true value stays
// 2^-37 away).
__global__ void sigma_table_init(int* uncertain) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= kSigEntriesPadded) return;
  if (i >= kSigEntries) { g_sigma_table[i] = 0.0f; return; }
  const uint32_t neg = i >= (int)kSigPerSign ? 1u : 0u;
  const uint32_t mag = (uint32_t)i - neg * kSigPerSign + kSigLo;
  const float g = __uint_as_float(((neg << 15) | mag) << 16);
  if (fabsf(g) < 0x1p-9f) {
    const double hi = 0.5 + 0.25 * (double)g;
    const float d = __double2float_rd(hi), u = __double2float_ru(hi);
    float f;
    if (d == u) {
      f = d;
    } else if (hi == 0.5 * ((double)d + (double)u)) {
      f = g > 0.0f ? d : u;
    } else {
      f = __double2float_rn(hi);
    }
    g_sigma_table[i] = f;
    return;
  }
  const double sd = 1.0 / (1.0 + exp(-(double)g));
  const float f = __double2float_rn(sd);
  const double up = 0.5 * ((double)f + (double)nextafterf(f, __int_as_float(0x7F800000)));
  const double dn = 0.5 * ((double)f + (double)nextafterf(f, __int_as_float(0xFF800000)));
  const double tol = fabs(sd) * 0x1p-48;
  if (!(fabs(sd - up) > tol && fabs(sd - dn) > tol)) atomicAdd(uncertain, 1);
  g_sigma_table[i] = f;
}

// Expands the table to all 65536 bf16 patterns (test hook), through the same
// shared-memory layout and pair lookup the fused kernels use: thread t looks
// up the packed pair (2t, 2t + 1).
__global__ void sigma_table_dump(float* out) {
  extern __shared__ __align__(16) float tab[];
  for (int i = threadIdx.x; i < kSigEntries; i += blockDim.x)
    tab[i < (int)kSigPerSign ? i : i - (int)kSigPerSign + kSigNegOffset] = g_sigma_table[i];
  __syncthreads();
  const uint32_t t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < 32768) {
    float a, b;
    sigma_pair(tab, (2 * t) | ((2 * t + 1) << 16), a, b);
    out[2 * t] = a;
    out[2 * t + 1] = b;
  }
}

// ---------------------------------------------------------------- offsets
// One CTA of 1024 threads; thread t owns a contiguous chunk of the groups.
__global__ void __launch_bounds__(1024) splits_kernel(const int64_t* __restrict__ m, int E,
                                                      int64_t M, int64_t* __restrict__ ro,
                                                      int64_t* __restrict__ cb,
                                                      int32_t* __restrict__ status) {
  __shared__ long long s_r[32], s_c[32];
  __shared__ int s_neg, s_big;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  if (t == 0) { s_neg = 0; s_big = 0; }
  __syncthreads();
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = min(E, t * per), e1 = min(E, e0 + per);
  long long r = 0, c = 0;
  int neg = 0, big = 0;
  for (int e = e0; e < e1; ++e) {
    const long long v = m[e];
    if (v < 0) neg = 1;
    else if (v > M) big = 1;
    else { r += v; c += (v + 31) / 32; }
  }
  if (neg) atomicOr(&s_neg, 1);
  if (big) atomicOr(&s_big, 1);
  // block-wide exclusive scan of (r, c)
  long long ir = r, ic = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long yr = __shfl_up_sync(kFull, ir, o), yc = __shfl_up_sync(kFull, ic, o);
    if (lane >= o) { ir += yr; ic += yc; }
  }
  if (lane == 31) { s_r[warp] = ir; s_c[warp] = ic; }
  __syncthreads();
  if (warp == 0) {
    long long wr = lane < (int)(blockDim.x >> 5) ? s_r[lane] : 0;
    long long wc = lane < (int)(blockDim.x >> 5) ? s_c[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long yr = __shfl_up_sync(kFull, wr, o), yc = __shfl_up_sync(kFull, wc, o);
      if (lane >= o) { wr += yr; wc += yc; }
    }
    s_r[lane] = wr; s_c[lane] = wc;   // inclusive over warps
  }
  __syncthreads();
  const long long total = s_r[(blockDim.x >> 5) - 1];
  int st = 0;
  if (s_neg) st = 1;
  else if (s_big || total != M) st = 2;
  if (t == 0) *status = st;
  if (st) return;
  long long base_r = (warp ? s_r[warp - 1] : 0) + ir - r;
  long long base_c = (warp ? s_c[warp - 1] : 0) + ic - c;
  for (int e = e0; e < e1; ++e) {
    ro[e] = base_r;
    if (cb) cb[e] = base_c;
    const long long v = m[e];
    base_r += v;
    base_c += (v + 31) / 32;
  }
  if (t == 0) { ro[E] = total; if (cb) cb[E] = s_c[(blockDim.x >> 5) - 1]; }
}

// ---------------------------------------------------------------- dscale sum
// dscale[row] = sum over tiles t = 0, 1, ... of part[t][row], in that order.
__global__ void __launch_bounds__(256) dscale_reduce_kernel(const float* __restrict__ part,
                                                            int n_tiles, int64_t M,
                                                            float* __restrict__ dscale) {
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= M) return;
  float acc = 0.0f;
#pragma unroll 8
  for (int t = 0; t < n_tiles; ++t) acc = __fadd_rn(acc, __ldcg(part + (int64_t)t * M + row));
  dscale[row] = acc;
}

// ---------------------------------------------------------------- fused kernels
struct Params {
  const uint16_t* x;
  int64_t ldx;
  const uint16_t* dy;
  int64_t lddy;
  const float* s;
  int64_t M;
  int N;   // activation width
  int W;   // width of the quantized tensor (N fwd; 2N or N bwd)
  uint8_t* rq;
  uint8_t* rs;
  uint8_t* cq;
  uint8_t* cs;
  uint16_t* dx;
  float* dscale;
  float* part;        // dscale partials [n_tiles][M] (tile-major)
  const int64_t* row_offs;
  const int64_t* cb_offs;
  int E;
  int32_t* status;
  int64_t dense_slabs;
  int n_tiles;
  uint32_t* err;      // device error word (timeouts), never expected to be set
};

constexpr int kSlots = 3;            // half-tile slots per warp
constexpr int kHalfRows = 16;
constexpr int kOperandHalfBytes = kHalfRows * kTileCols * 2;   // 2 KiB

// Threads per CTA: one CTA per SM; the shared memory of the warps' rings
// (slots x operands x 2 KiB) plus the sigmoid table bounds the warp count.
__host__ __device__ constexpr int fwd_warps(int act) { return act == 0 ? 12 : 12; }
__host__ __device__ constexpr int bwd_warps(int act) { return act == 0 ? 8 : 12; }
__host__ __device__ constexpr int fwd_threads(int act, int dirs) { return 32 * fwd_warps(act) + 0 * dirs; }
__host__ __device__ constexpr int bwd_threads(int act, int dirs) { return 32 * bwd_warps(act) + 0 * dirs; }
__host__ __device__ constexpr int fwd_operands(int act) { return act == 0 ? 2 : 1; }
__host__ __device__ constexpr int bwd_operands(int act) { return act == 0 ? 3 : 2; }
__host__ __device__ constexpr int ring_bytes(int warps, int operands) {
  return warps * kSlots * operands * kOperandHalfBytes;
}

// Shared-memory layout of a CTA: [rings][sigmoid table][col-block offsets][mbarriers]
// (E < 0: without the col-block offsets, which the launcher adds for grouped calls)
// (128 bytes of slack let the kernel align the base for the TMA destinations;
// a grouped call adds its row and col-block offsets as two int32 arrays)
__host__ __device__ constexpr int group_bytes(int E) { return 2 * ((E + 1 + 3) / 4) * 16; }
__host__ __device__ constexpr int smem_bytes(int warps, int operands, bool sig, int E) {
  return 128 + ring_bytes(warps, operands) + (sig ? kSigBytes : 0) +
         (E < 0 ? 0 : group_bytes(E)) + warps * kSlots * 8;
}

__device__ __forceinline__ unsigned char* align_smem(unsigned char* p) {
  return p + ((128u - (smem_addr(p) & 127u)) & 127u);
}

// Stages the sigmoid table (and, grouped, the row and col-block offsets as
// int32) in shared memory and validates grouped offsets.  Returns the slab
// count, or -1 if the offsets are not those of valid splits (every CTA reaches
// the same verdict; CTA 0 writes the status word).
template <bool NEED_SIG, bool GROUPED>
__device__ __forceinline__ int64_t stage_and_validate(const Params& p, float* sig_s, int* cb_s,
                                                      int* ro_s) {
  if (NEED_SIG) {
    for (int i = threadIdx.x; i < kSigEntries; i += blockDim.x)
      sig_s[i < (int)kSigPerSign ? i : i - (int)kSigPerSign + kSigNegOffset] = g_sigma_table[i];
  }
  int bad = 0;
  if (GROUPED) {
    for (int e = threadIdx.x; e <= p.E; e += blockDim.x) {
      const int64_t r = p.row_offs[e], c = p.cb_offs[e];
      bool ok;
      if (e == 0) {
        ok = (r == 0) && (c == 0);
      } else {
        const int64_t r0 = p.row_offs[e - 1], c0 = p.cb_offs[e - 1];
        const int64_t m = r - r0;
        ok = (m >= 0) && (r <= p.M) && (c - c0 == (m + 31) / 32);
      }
      if (e == p.E) ok = ok && (r == p.M);
      if (!ok) bad = 1;
      cb_s[e] = (int)c;
      ro_s[e] = (int)r;
    }
  }
  bad = __syncthreads_or(bad);
  if (!GROUPED) return p.dense_slabs;
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.status = bad ? 3 : 0;
  return bad ? -1 : (int64_t)cb_s[p.E];
}

// Rows of slab `slab`: first row and count (<= 32).  Grouped offsets come from
// shared memory (int32: rows are below 2^30).
template <bool GROUPED>
__device__ __forceinline__ void slab_rows(const Params& p, const int* cb_s, const int* ro_s,
                                          int64_t slab, int64_t& row0, int& nrows) {
  if (!GROUPED) {
    row0 = slab * 32;
    nrows = (int)min((int64_t)32, p.M - row0);
  } else {
    // largest e in [0, E-1] with cb[e] <= slab (empty groups are skipped)
    int lo = 0, hi = p.E - 1;
    const int sl = (int)slab;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cb_s[mid] <= sl) lo = mid; else hi = mid - 1;
    }
    const int r0 = ro_s[lo] + 32 * (sl - cb_s[lo]);
    row0 = r0;
    nrows = min(32, ro_s[lo + 1] - r0);
  }
}

// Stores the two E8M0 bytes (blocks 2*tile, 2*tile+1) of one row.  `blk1`
// exists only when the tile has a second 32-column block; the 16-bit store is
// used when the address is even.
__device__ __forceinline__ void store_row_scales(uint8_t* dst, uint32_t b0, uint32_t b1,
                                                 bool has1) {
  if (has1 && ((reinterpret_cast<uintptr_t>(dst) & 1u) == 0)) {
    __stcs(reinterpret_cast<unsigned short*>(dst), (unsigned short)(b0 | (b1 << 8)));
  } else {
    dst[0] = (uint8_t)b0;
    if (has1) dst[1] = (uint8_t)b1;
  }
}

// ------------------------------------------------------------- the warp's ring
// Half-tile k of a warp is half (k & 1) of its (k >> 1)-th work item; it lives
// in slot k % kSlots, whose mbarrier completes once per use (parity
// (k / kSlots) & 1).
struct Ring {
  unsigned char* slots;   // kSlots * OPS * 2 KiB
  uint64_t* bars;         // kSlots
  int ops;
};

template <bool GROUPED>
__device__ __forceinline__ void issue_half(const Params& p, const int* cb_s, const int* ro_s,
                                           const Ring& r,
                                           const void* tm_x, const void* tm_dy, int64_t item,
                                           int k, bool swiglu, bool with_dy) {
  const int64_t slab = item / p.n_tiles;
  const int tile = (int)(item - slab * p.n_tiles);
  int64_t row0;
  int nrows;
  slab_rows<GROUPED>(p, cb_s, ro_s, slab, row0, nrows);
  const int slot = k % kSlots;
  unsigned char* dst = r.slots + slot * r.ops * kOperandHalfBytes;
  uint64_t* bar = r.bars + slot;
  const int x = tile * kTileCols, y = (int)row0 + (k & 1) * kHalfRows;
  mbar_expect_tx(bar, r.ops * kOperandHalfBytes);
  int o = 0;
  if (with_dy) tma_load_2d(dst + (o++) * kOperandHalfBytes, tm_dy, x, y, bar);
  tma_load_2d(dst + (o++) * kOperandHalfBytes, tm_x, x, y, bar);
  if (swiglu) tma_load_2d(dst + (o++) * kOperandHalfBytes, tm_x, x + p.N, y, bar);
}

__device__ __forceinline__ void report_timeout(const Params& p, uint32_t code) {
  atomicOr(p.err, code);
}

// ------------------------------------------------------------- forward tile
// Rowwise work runs per 16-row half: after the 4-step butterfly (off = 8, 4,
// 2, 1) lane l holds the amax of row 16h + (l & 15) in block (l >> 4).
template <int ACT, int DIRS, bool STAGED, bool GROUPED, bool FULL>
__device__ __forceinline__ void fwd_tile(const Params& p, const float* sig, const Ring& ring,
                                         int k0, int64_t slab, int tile, int64_t row0, int nrows,
                                         int lane, const int* cb_s, const int* ro_s,
                                         const void* tm_x, int64_t next_item0,
                                         int64_t next_item1, int K, bool& ok_flag) {
  const int c0 = tile * kTileCols + 2 * lane;
  const bool colok = c0 < p.N;
  const int W = p.W;
  const int Wh = W >> 1;
  const float sv = lane < nrows ? __ldg(p.s + row0 + lane) : 0.0f;

  float Y0[32], Y1[32];
  uint32_t bh[2];
  unsigned short* rqb = reinterpret_cast<unsigned short*>(p.rq + row0 * (int64_t)W + c0);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int k = k0 + h;
    const int slot = k % kSlots;
    if (!mbar_wait(ring.bars + slot, (uint32_t)(k / kSlots) & 1u)) { ok_flag = false; return; }
    const unsigned char* sm = ring.slots + slot * ring.ops * kOperandHalfBytes + 4 * lane;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = 16 * h + i;
      const uint32_t G = *reinterpret_cast<const uint32_t*>(sm + i * 128);
      const float sr = __shfl_sync(kFull, sv, r);
      float h0, h1;
      if (ACT == kSwiGLU) {
        const uint32_t U = *reinterpret_cast<const uint32_t*>(sm + kOperandHalfBytes + i * 128);
        const float g0 = bf16_lo(G), g1 = bf16_hi(G);
        const float u0 = bf16_lo(U), u1 = bf16_hi(U);
        float sg0, sg1;
        sigma_pair(sig, G, sg0, sg1);
        const float si0 = __fmul_rn(g0, sg0);
        const float si1 = __fmul_rn(g1, sg1);
        if (STAGED) {
          h0 = bf16_round(__fmul_rn(bf16_round(si0), u0));
          h1 = bf16_round(__fmul_rn(bf16_round(si1), u1));
        } else {
          h0 = __fmul_rn(si0, u0);
          h1 = __fmul_rn(si1, u1);
        }
      } else {
        const float r0 = relu_keep_nan(bf16_lo(G)), r1 = relu_keep_nan(bf16_hi(G));
        h0 = __fmul_rn(r0, r0);
        h1 = __fmul_rn(r1, r1);
      }
      Y0[r] = __fmul_rn(h0, sr);
      Y1[r] = __fmul_rn(h1, sr);
      if (!FULL && r >= nrows) { Y0[r] = 0.0f; Y1[r] = 0.0f; }
    }
    // the slot is consumed: refill it with the half-tile kSlots ahead
    __syncwarp();
    if (lane == 0 && k + kSlots < K) {
      const int kn = k + kSlots;
      issue_half<GROUPED>(p, cb_s, ro_s, ring, tm_x, nullptr,
                          (kn >> 1) == (k0 >> 1) + 1 ? next_item0 : next_item1, kn,
                          ACT == kSwiGLU, false);
    }
    if (DIRS & kRow) {
      uint32_t A[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) A[i] = max(f32_mag(Y0[16 * h + i]), f32_mag(Y1[16 * h + i]));
      bfly_max_u32<8>(A, lane, 8);
      bfly_max_u32<4>(A, lane, 4);
      bfly_max_u32<2>(A, lane, 2);
      bfly_max_u32<1>(A, lane, 1);
      bh[h] = e8m0_from_amax(A[0]);
      const uint32_t mh = scale_multiplier(bh[h]);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * h + i;
        const uint32_t m = __shfl_sync(kFull, mh, (lane & 16) | i);
        const uint32_t q = e4m3x2(Y0[r], m, Y1[r], m);
        if (FULL || (colok && r < nrows)) __stcs(rqb + r * Wh, (unsigned short)q);
      }
    }
  }
  if (DIRS & kRow) {
    // lane l stores both blocks of row l
    const uint32_t mine = bh[0] | (bh[1] << 8);
    const uint32_t other = __shfl_xor_sync(kFull, mine, 16);
    if (lane < nrows) {
      const uint32_t blk0 = lane < 16 ? (mine & 0xFFu) : ((other >> 8) & 0xFFu);
      const uint32_t blk1 = lane < 16 ? (other & 0xFFu) : ((mine >> 8) & 0xFFu);
      const bool has1 = tile * kTileCols + 32 < p.N;
      store_row_scales(p.rs + (row0 + lane) * (int64_t)(W / 32) + 2 * tile, blk0, blk1, has1);
    }
  }
  if (DIRS & kCol) {
    uint32_t a0 = 0u, a1 = 0u;
#pragma unroll
    for (int r = 0; r < 32; r += 2) {
      a0 = __vimax3_u32(a0, f32_mag(Y0[r]), f32_mag(Y0[r + 1]));
      a1 = __vimax3_u32(a1, f32_mag(Y1[r]), f32_mag(Y1[r + 1]));
    }
    const uint32_t b0 = e8m0_from_amax(a0), b1 = e8m0_from_amax(a1);
    const uint32_t m0 = scale_multiplier(b0), m1 = scale_multiplier(b1);
    if (colok)
      __stcs(reinterpret_cast<unsigned short*>(p.cs + slab * (int64_t)W + c0),
             (unsigned short)(b0 | (b1 << 8)));
    unsigned short* qb = reinterpret_cast<unsigned short*>(p.cq + row0 * (int64_t)W + c0);
    const int Whc = opaque(Wh);
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const uint32_t q = e4m3x2(Y0[r], m0, Y1[r], m1);
      if (FULL || (colok && r < nrows)) __stcs(qb + r * Whc, (unsigned short)q);
    }
  }
}

// Sets up the warp's ring (barriers initialised by lane 0) and primes it.
template <bool GROUPED>
__device__ __forceinline__ void ring_prime(const Params& p, const int* cb_s, const int* ro_s,
                                           const Ring& ring,
                                           const void* tm_x, const void* tm_dy, int64_t first,
                                           int64_t stride, int K, int lane, bool swiglu,
                                           bool with_dy) {
  if (lane == 0) {
    for (int i = 0; i < kSlots; ++i) mbar_init(ring.bars + i, 1);
    mbar_init_fence();
    for (int k = 0; k < kSlots && k < K; ++k)
      issue_half<GROUPED>(p, cb_s, ro_s, ring, tm_x, tm_dy, first + (k >> 1) * stride, k, swiglu,
                          with_dy);
  }
  __syncwarp();
}

// After a timeout: bounded waits for the copies still in flight into this
// warp's slots, so that none lands after the CTA has exited.
__device__ __forceinline__ void ring_drain(const Ring& ring, int k_next, int K) {
  for (int k = k_next; k < K && k < k_next + kSlots; ++k)
    mbar_wait(ring.bars + (k % kSlots), (uint32_t)(k / kSlots) & 1u);
}

template <int ACT, int DIRS, bool STAGED, bool GROUPED>
__global__ void __launch_bounds__(fwd_threads(ACT, DIRS), 1)
    act_fwd_kernel(const __grid_constant__ CUtensorMap tm_x, const Params p) {
  constexpr int kWarps = fwd_warps(ACT);
  constexpr int kOps = fwd_operands(ACT);
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* smem = align_smem(smem_raw);
  float* sig_s = reinterpret_cast<float*>(smem + ring_bytes(kWarps, kOps));
  int* cb_s = reinterpret_cast<int*>(smem + ring_bytes(kWarps, kOps) +
                                     (ACT == kSwiGLU ? kSigBytes : 0));
  int* ro_s = cb_s + (GROUPED ? ((p.E + 1 + 3) / 4) * 4 : 0);
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      smem + ring_bytes(kWarps, kOps) + (ACT == kSwiGLU ? kSigBytes : 0) +
      (GROUPED ? group_bytes(p.E) : 0));
  const int64_t n_slabs = stage_and_validate<ACT == kSwiGLU, GROUPED>(p, sig_s, cb_s, ro_s);
  if (n_slabs < 0) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t n_items = n_slabs * p.n_tiles;
  const int64_t first = (int64_t)blockIdx.x * kWarps + warp;
  const int64_t stride = (int64_t)gridDim.x * kWarps;
  const int count = first < n_items ? (int)((n_items - 1 - first) / stride + 1) : 0;
  const int K = 2 * count;
  Ring ring{smem + warp * kSlots * kOps * kOperandHalfBytes, bars + warp * kSlots, kOps};
  ring_prime<GROUPED>(p, cb_s, ro_s, ring, &tm_x, nullptr, first, stride, K, lane, ACT == kSwiGLU,
                      false);
  bool ok = true;
  for (int j = 0; j < count; ++j) {
    const int64_t it = first + j * stride;
    const int64_t slab = it / p.n_tiles;
    const int tile = (int)(it - slab * p.n_tiles);
    int64_t row0;
    int nrows;
    slab_rows<GROUPED>(p, cb_s, ro_s, slab, row0, nrows);
    const bool full = nrows == 32 && (tile + 1) * kTileCols <= p.N;
    const int64_t n1 = it + stride, n2 = it + 2 * stride;
    if (full)
      fwd_tile<ACT, DIRS, STAGED, GROUPED, true>(p, sig_s, ring, 2 * j, slab, tile, row0, nrows, lane,
                                        cb_s, ro_s, &tm_x, n1, n2, K, ok);
    else
      fwd_tile<ACT, DIRS, STAGED, GROUPED, false>(p, sig_s, ring, 2 * j, slab, tile, row0, nrows, lane,
                                         cb_s, ro_s, &tm_x, n1, n2, K, ok);
    if (!ok) {
      if (lane == 0) {
        report_timeout(p, 1u);
        ring_drain(ring, 2 * j, K);
      }
      return;
    }
  }
}

// ------------------------------------------------------------- backward tile
// dscale: each warp reduces its 32 rows x 64 columns to one partial per row
// and stores it, lane = row, into the workspace at [tile][row] -- plain
// stores, no fences or counters.  dscale_reduce_kernel, launched right after
// on the same stream, sums each row's partials in tile order (a fixed order,
// so dscale is deterministic).

// Row-direction work (dx stores, dscale partials, rowwise MXFP8) runs per
// 16-row half as the half arrives; the packed bf16 gradients of all 32 rows
// stay in registers for the colwise pass.
template <int ACT, int DIRS, bool GROUPED, bool FULL>
__device__ __forceinline__ void bwd_tile(const Params& p, const float* sig, const Ring& ring,
                                         int k0, int64_t slab, int tile, int64_t row0, int nrows,
                                         int lane, const int* cb_s, const int* ro_s,
                                         const void* tm_x, const void* tm_dy,
                                         int64_t next_item0, int64_t next_item1, int K,
                                         bool& ok_flag) {
  const int N = p.N, W = p.W;
  const int Wh = W >> 1;
  const int c0 = tile * kTileCols + 2 * lane;
  const bool colok = c0 < N;
  const float sv = lane < nrows ? __ldg(p.s + row0 + lane) : 0.0f;

  uint32_t DG[32], DU[32];
  float ph[2];
  uint32_t bh[2];
  unsigned short* rqb = reinterpret_cast<unsigned short*>(p.rq + row0 * (int64_t)W + c0);
  uint32_t* dxb = reinterpret_cast<uint32_t*>(p.dx + row0 * (int64_t)W + c0);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int k = k0 + h;
    const int slot = k % kSlots;
    if (!mbar_wait(ring.bars + slot, (uint32_t)(k / kSlots) & 1u)) { ok_flag = false; return; }
    const unsigned char* sm = ring.slots + slot * ring.ops * kOperandHalfBytes + 4 * lane;
    float P[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = 16 * h + i;
      const uint32_t D = *reinterpret_cast<const uint32_t*>(sm + i * 128);
      const uint32_t G = *reinterpret_cast<const uint32_t*>(sm + kOperandHalfBytes + i * 128);
      const float sr = __shfl_sync(kFull, sv, r);
      const float d0 = bf16_lo(D), d1 = bf16_hi(D);
      const float p0 = __fmul_rn(d0, sr), p1 = __fmul_rn(d1, sr);
      float h0, h1;
      if (ACT == kSwiGLU) {
        const uint32_t U =
            *reinterpret_cast<const uint32_t*>(sm + 2 * kOperandHalfBytes + i * 128);
        const float g0 = bf16_lo(G), g1 = bf16_hi(G);
        const float u0 = bf16_lo(U), u1 = bf16_hi(U);
        float s0, s1;
        sigma_pair(sig, G, s0, s1);
        const float si0 = __fmul_rn(g0, s0), si1 = __fmul_rn(g1, s1);
        const float ds0 = __fmaf_rn(si0, __fsub_rn(1.0f, s0), s0);
        const float ds1 = __fmaf_rn(si1, __fsub_rn(1.0f, s1), s1);
        DG[r] = pack_bf16x2(__fmul_rn(__fmul_rn(p0, u0), ds0), __fmul_rn(__fmul_rn(p1, u1), ds1));
        DU[r] = pack_bf16x2(__fmul_rn(p0, si0), __fmul_rn(p1, si1));
        h0 = __fmul_rn(si0, u0);
        h1 = __fmul_rn(si1, u1);
      } else {
        const float r0 = relu_keep_nan(bf16_lo(G)), r1 = relu_keep_nan(bf16_hi(G));
        DG[r] = pack_bf16x2(__fmul_rn(p0, __fmul_rn(2.0f, r0)), __fmul_rn(p1, __fmul_rn(2.0f, r1)));
        DU[r] = 0u;
        h0 = __fmul_rn(r0, r0);
        h1 = __fmul_rn(r1, r1);
      }
      P[i] = __fmaf_rn(d1, h1, __fmul_rn(d0, h0));
      if (!FULL && r >= nrows) { DG[r] = 0u; DU[r] = 0u; P[i] = 0.0f; }
      if (p.dx != nullptr && (FULL || (colok && r < nrows))) {
        __stcs(dxb + r * Wh, DG[r]);
        if (ACT == kSwiGLU) __stcs(dxb + r * Wh + (N >> 1), DU[r]);
      }
    }
    __syncwarp();
    if (lane == 0 && k + kSlots < K) {
      const int kn = k + kSlots;
      issue_half<GROUPED>(p, cb_s, ro_s, ring, tm_x, tm_dy,
                          (kn >> 1) == (k0 >> 1) + 1 ? next_item0 : next_item1, kn,
                          ACT == kSwiGLU, true);
    }
    if (p.dscale != nullptr) {
      // lane l ends with the warp sum of row 16h + (l >> 1)
      bfly_sum_f32<8>(P, lane, 16);
      bfly_sum_f32<4>(P, lane, 8);
      bfly_sum_f32<2>(P, lane, 4);
      bfly_sum_f32<1>(P, lane, 2);
      ph[h] = __fadd_rn(P[0], __shfl_xor_sync(kFull, P[0], 1));
    }
    if (DIRS & kRow) {
      // packed per-row block maxima: low half dgate, high half dup
      uint32_t A[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t ag = DG[16 * h + i] & 0x7FFF7FFFu, au = DU[16 * h + i] & 0x7FFF7FFFu;
        A[i] = __vmaxu2(__byte_perm(ag, au, 0x5410), __byte_perm(ag, au, 0x7632));
      }
      bfly_max_u16x2<8>(A, lane, 8);
      bfly_max_u16x2<4>(A, lane, 4);
      bfly_max_u16x2<2>(A, lane, 2);
      bfly_max_u16x2<1>(A, lane, 1);
      // lane l: row 16h + (l & 15), block (l >> 4)
      const uint32_t bg = e8m0_from_amax(A[0] << 16), bu = e8m0_from_amax(A[0] & 0xFFFF0000u);
      bh[h] = bg | (bu << 8);
      const uint32_t mgh = scale_multiplier(bg), muh = scale_multiplier(bu);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * h + i;
        const int src = (lane & 16) | i;
        const uint32_t mg = __shfl_sync(kFull, mgh, src);
        const uint32_t qg = e4m3x2(bf16_lo(DG[r]), mg, bf16_hi(DG[r]), mg);
        uint32_t qu = 0;
        if (ACT == kSwiGLU) {
          const uint32_t mu = __shfl_sync(kFull, muh, src);
          qu = e4m3x2(bf16_lo(DU[r]), mu, bf16_hi(DU[r]), mu);
        }
        if (FULL || (colok && r < nrows)) {
          __stcs(rqb + r * Wh, (unsigned short)qg);
          if (ACT == kSwiGLU) __stcs(rqb + r * Wh + (N >> 1), (unsigned short)qu);
        }
      }
    }
  }
  if (p.dscale != nullptr) {
    const int src = 2 * (lane & 15);
    const float v0 = __shfl_sync(kFull, ph[0], src), v1 = __shfl_sync(kFull, ph[1], src);
    if (lane < nrows) __stcg(p.part + (int64_t)tile * p.M + row0 + lane, lane < 16 ? v0 : v1);
  }
  if (DIRS & kRow) {
    // lane l stores the four blocks (dgate 0/1, dup 0/1) of row l
    const uint32_t mine = bh[0] | (bh[1] << 16);   // bytes: g(h0) u(h0) g(h1) u(h1)
    const uint32_t other = __shfl_xor_sync(kFull, mine, 16);
    if (lane < nrows) {
      const int sh = lane < 16 ? 0 : 16;
      const uint32_t lo = lane < 16 ? mine : other, hi = lane < 16 ? other : mine;
      const bool has1 = tile * kTileCols + 32 < N;
      uint8_t* rsr = p.rs + (row0 + lane) * (int64_t)(W / 32) + 2 * tile;
      store_row_scales(rsr, (lo >> sh) & 0xFFu, (hi >> sh) & 0xFFu, has1);
      if (ACT == kSwiGLU)
        store_row_scales(rsr + N / 32, (lo >> (sh + 8)) & 0xFFu, (hi >> (sh + 8)) & 0xFFu, has1);
    }
  }
  if (DIRS & kCol) {
    uint32_t ag = 0u, au = 0u;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      ag = __vmaxu2(ag, DG[r] & 0x7FFF7FFFu);
      au = __vmaxu2(au, DU[r] & 0x7FFF7FFFu);
    }
    const uint32_t bg0 = e8m0_from_amax(ag << 16), bg1 = e8m0_from_amax(ag & 0xFFFF0000u);
    const uint32_t bu0 = e8m0_from_amax(au << 16), bu1 = e8m0_from_amax(au & 0xFFFF0000u);
    const uint32_t mg0 = scale_multiplier(bg0), mg1 = scale_multiplier(bg1);
    const uint32_t mu0 = scale_multiplier(bu0), mu1 = scale_multiplier(bu1);
    if (colok) {
      uint8_t* csr = p.cs + slab * (int64_t)W + c0;
      __stcs(reinterpret_cast<unsigned short*>(csr), (unsigned short)(bg0 | (bg1 << 8)));
      if (ACT == kSwiGLU)
        __stcs(reinterpret_cast<unsigned short*>(csr + N), (unsigned short)(bu0 | (bu1 << 8)));
    }
    unsigned short* qb = reinterpret_cast<unsigned short*>(p.cq + row0 * (int64_t)W + c0);
    const int Whc = opaque(Wh);
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const uint32_t qg = e4m3x2(bf16_lo_p(DG[r]), mg0, bf16_hi_p(DG[r]), mg1);
      if (FULL || (colok && r < nrows)) {
        __stcs(qb + r * Whc, (unsigned short)qg);
        if (ACT == kSwiGLU) {
          const uint32_t qu = e4m3x2(bf16_lo_p(DU[r]), mu0, bf16_hi_p(DU[r]), mu1);
          __stcs(qb + r * Whc + (N >> 1), (unsigned short)qu);
        }
      }
    }
  }
}

template <int ACT, int DIRS, bool GROUPED>
__global__ void __launch_bounds__(bwd_threads(ACT, DIRS), 1)
    act_bwd_kernel(const __grid_constant__ CUtensorMap tm_x,
                   const __grid_constant__ CUtensorMap tm_dy, const Params p) {
  constexpr int kWarps = bwd_warps(ACT);
  constexpr int kOps = bwd_operands(ACT);
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* smem = align_smem(smem_raw);
  float* sig_s = reinterpret_cast<float*>(smem + ring_bytes(kWarps, kOps));
  int* cb_s = reinterpret_cast<int*>(smem + ring_bytes(kWarps, kOps) +
                                     (ACT == kSwiGLU ? kSigBytes : 0));
  int* ro_s = cb_s + (GROUPED ? ((p.E + 1 + 3) / 4) * 4 : 0);
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      smem + ring_bytes(kWarps, kOps) + (ACT == kSwiGLU ? kSigBytes : 0) +
      (GROUPED ? group_bytes(p.E) : 0));
  const int64_t n_slabs = stage_and_validate<ACT == kSwiGLU, GROUPED>(p, sig_s, cb_s, ro_s);
  if (n_slabs < 0) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t n_items = n_slabs * p.n_tiles;
  const int64_t first = (int64_t)blockIdx.x * kWarps + warp;
  const int64_t stride = (int64_t)gridDim.x * kWarps;
  const int count = first < n_items ? (int)((n_items - 1 - first) / stride + 1) : 0;
  const int K = 2 * count;
  Ring ring{smem + warp * kSlots * kOps * kOperandHalfBytes, bars + warp * kSlots, kOps};
  ring_prime<GROUPED>(p, cb_s, ro_s, ring, &tm_x, &tm_dy, first, stride, K, lane, ACT == kSwiGLU,
                      true);
  bool ok = true;
  for (int j = 0; j < count; ++j) {
    const int64_t it = first + j * stride;
    const int64_t slab = it / p.n_tiles;
    const int tile = (int)(it - slab * p.n_tiles);
    int64_t row0;
    int nrows;
    slab_rows<GROUPED>(p, cb_s, ro_s, slab, row0, nrows);
    const bool full = nrows == 32 && (tile + 1) * kTileCols <= p.N;
    const int64_t n1 = it + stride, n2 = it + 2 * stride;
    if (full)
      bwd_tile<ACT, DIRS, GROUPED, true>(p, sig_s, ring, 2 * j, slab, tile, row0, nrows, lane,
                                         cb_s, ro_s, &tm_x, &tm_dy, n1, n2, K, ok);
    else
      bwd_tile<ACT, DIRS, GROUPED, false>(p, sig_s, ring, 2 * j, slab, tile, row0, nrows, lane,
                                          cb_s, ro_s, &tm_x, &tm_dy, n1, n2, K, ok);
    if (!ok) {
      if (lane == 0) {
        report_timeout(p, 2u);
        ring_drain(ring, 2 * j, K);
      }
      return;
    }
  }
}
}  // namespace moeact
