// Kernels of libmoeact (sm_100a).
//
// (The sigmoid tables and their set-up kernel are in sigma.cuh.)
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
// 32 rows (one colwise block, never crossing an expert boundary) x 128
// columns; lane l owns columns 4l .. 4l+3 for all 32 rows, so the colwise
// amax is a per-lane loop over registers and the rowwise 1x32 amax is an
// 8-lane reduction.  The grid is persistent (one CTA per SM, the sigmoid
// table staged once per CTA in shared memory).
//
// Data movement.  Each warp owns a ring of shared-memory slots, each holding
// one 16-row half of a warp-tile's inputs ([16 x 128] bf16 per operand),
// filled by TMA (cp.async.bulk.tensor, this CTA only) and signalled through
// one mbarrier per slot; lane 0 refills a slot as soon as it is consumed, so
// the loads of the next half-tiles overlap the math of the current one, and
// rows and columns outside the tensor arrive as zeros.  Lanes read their four
// columns of each row from shared memory (a warp reads one 256-byte row).
// Codes, scales and gradients are stored directly, 128 (codes) or 256 (bf16)
// contiguous bytes per warp per row; full tiles take a path without bounds
// predicates.
#pragma once

#include <cstdint>

#include <cuda.h>

#include "device_common.cuh"

namespace moeact {

enum Act : int { kSwiGLU = 0, kSReLU = 1, kClamped = 2 };   // kClamped: ClampedSwiGLU
constexpr int kRow = 1;
constexpr int kCol = 2;
// Kernel template flag carried in the DIRS bits: scales in the GEMM-ready
// tiled layout (a compile-time choice, so the row-major kernels carry none of
// its code).
constexpr int kGemm = 4;
// Forward template flag in the DIRS bits: gate and up interleaved in blocks
// (loads through a 4-D map), so the halves layout's forward keeps its own
// instantiation, untouched by the interleaved load code.
constexpr int kIlv = 8;
constexpr int kTileCols = 128;   // columns of a warp-tile (4 per lane)

__host__ __device__ constexpr int sig_slot(int i) {
  return i < (int)kSigPerSign ? i : i - (int)kSigPerSign + kSigNegOffset;
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
  int gemm_scales;    // scales in the GEMM-ready tiled layout (see gemm_row_scales_off)
  const float* sig_src;   // the sigmoid table to stage (device memory, shared-memory layout)
  // ClampedSwiGLU: gate and up limit L and slope alpha.  Both are folded
  // into sig_src, which holds sigma(RN(alpha * g)) for g <= L and
  // sigma(RN(alpha * L)) for every gate above L.  clamp_Lb2: the largest
  // bf16 not above L, in both halves (a bf16 value is above L exactly when it
  // is above that).
  float clamp_L;
  float clamp_alpha;
  uint32_t clamp_Lb2;
  int clamp_bf16;     // L is itself a bf16 value (then clamp_Lb2 is L, both halves)
  const int32_t* noop;   // nullable: a non-zero flag makes the call write nothing
  // Gated layouts of x and dX (width 2N): ilv == 0 is [gate | up] halves;
  // ilv = G > 0 is G gate columns, then the G matching up columns, repeated.
  // up = the stored distance from a gate column to its up column (N or G).
  int ilv;
  int up;
  uint32_t* err;      // device error word (timeouts), never expected to be set
};

constexpr int kHalfRows = 16;
constexpr int kOpHalfBytes = kHalfRows * kTileCols * 2;   // one operand's half-tile: 4 KiB
constexpr int kRowBytes = kTileCols * 2;                   // 256 B of a bf16 tile row

// Per-kernel configuration: warps per CTA (one CTA per SM) and ring slots per
// warp, chosen so that rings + sigmoid table fit the 227 KiB of shared memory.
template <int ACT, bool BWD>
struct Cfg {
  static constexpr bool kSig = ACT != kSReLU;   // gated: sigmoid table, gate + up
  // the table first in shared memory, looked up by 16-bit addresses
  // (sigma_pair_s): the gated forwards, where it measured faster
  static constexpr bool kSigFront = !BWD && (ACT == kSwiGLU || ACT == kClamped);
  static constexpr int kOps = BWD ? (kSig ? 3 : 2) : (kSig ? 2 : 1);
  static constexpr int kWarps = BWD ? (kSig ? 7 : 8) : 8;
  static constexpr int kSlots = (!BWD && !kSig) ? 3 : 2;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kRing = kWarps * kSlots * kOps * kOpHalfBytes;
  static constexpr int kBars = kWarps * kSlots + 1;
};

// Grouped offsets (int32 copies of row_offs and colblk_offs): with the
// sigmoid table they live in its unused gap (float indices 4100.. and 6144..,
// room for MOEACT_MAX_GROUPS + 1 entries each); without it, after the ring.
constexpr int kGapCb = 4100;
constexpr int kGapRo = 6144;
__host__ __device__ constexpr int group_bytes(int E) { return 2 * ((E + 1 + 3) / 4) * 16; }

// Shared memory of a CTA: 128 B of alignment slack, then the sigmoid table
// (padded to 1 KiB) and the ring (Cfg::kSigFront: the gated forwards), or the
// ring and the table (the gated backwards), or the ring and the group offsets
// (SReLU); then the mbarriers.  A table in front has shared-memory addresses
// that fit in 16 bits (see sigma_pair_s); the backwards measured slower with
// that order, and look their table up through its pointer.
constexpr int kSigRegion = (kSigBytes + 1023) / 1024 * 1024;
template <int ACT, bool BWD>
__host__ __device__ constexpr int smem_bytes(bool grouped, int E) {
  using C = Cfg<ACT, BWD>;
  return 128 + C::kRing +
         (C::kSig ? (C::kSigFront ? kSigRegion : kSigBytes) : (grouped ? group_bytes(E) : 0)) +
         C::kBars * 8;
}

__device__ __forceinline__ unsigned char* align_smem(unsigned char* p) {
  return p + ((128u - (smem_addr(p) & 127u)) & 127u);
}

struct Smem {
  unsigned char* ring;
  float* sig;
  uint32_t sig_key;   // kSigFront: sigma_pair_s's constant for this table's address
  int* cb;
  int* ro;
  uint64_t* bars;
};

template <int ACT, bool BWD>
__device__ __forceinline__ Smem carve(unsigned char* raw, int E) {
  using C = Cfg<ACT, BWD>;
  Smem m;
  unsigned char* base = align_smem(raw);
  unsigned char* after;
  if (C::kSigFront) {
    m.sig = reinterpret_cast<float*>(base);
    m.sig_key = sigma_key(smem_addr(base));
    m.cb = reinterpret_cast<int*>(m.sig + kGapCb);
    m.ro = reinterpret_cast<int*>(m.sig + kGapRo);
    m.ring = base + kSigRegion;
    after = m.ring + C::kRing;
  } else if (C::kSig) {
    m.ring = base;
    m.sig = reinterpret_cast<float*>(base + C::kRing);
    m.sig_key = 0;
    m.cb = reinterpret_cast<int*>(m.sig + kGapCb);
    m.ro = reinterpret_cast<int*>(m.sig + kGapRo);
    after = base + C::kRing + kSigBytes;
  } else {
    m.ring = base;
    after = base + C::kRing;
    m.sig = nullptr;
    m.sig_key = 0;
    m.cb = reinterpret_cast<int*>(after);
    m.ro = m.cb + ((E + 1 + 3) / 4) * 4;
    after += group_bytes(E);
  }
  m.bars = reinterpret_cast<uint64_t*>(after);
  return m;
}

// Starts the bulk copy of the sigmoid table (thread 0) and validates grouped
// offsets while staging them as int32.  Returns the slab count, or -1 if the
// offsets are not those of valid splits (every CTA reaches the same verdict;
// CTA 0 writes the status word).  The table copy completes on sig_bar.
template <bool SIG, bool GROUPED>
__device__ __forceinline__ int64_t stage_and_validate(const Params& p, const Smem& m,
                                                      uint64_t* sig_bar) {
  if (SIG && threadIdx.x == 0) {
    // the two halves of the table; the gap between them is not copied
    mbar_init(sig_bar, 1);
    mbar_init_fence();
    mbar_expect_tx(sig_bar, 2 * kSigHalfBytes);
    bulk_load(m.sig, p.sig_src, kSigHalfBytes, sig_bar);
    bulk_load(m.sig + kSigNegOffset, p.sig_src + kSigNegOffset, kSigHalfBytes, sig_bar);
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
        const int64_t mm = r - r0;
        ok = (mm >= 0) && (r <= p.M) && (c - c0 == (mm + 31) / 32);
      }
      if (e == p.E) ok = ok && (r == p.M);
      if (!ok) bad |= 1;
      if (p.gemm_scales && (r & 127)) bad |= 2;
      m.cb[e] = (int)c;
      m.ro[e] = (int)r;
    }
  }
  const int bad_offsets = __syncthreads_or(bad & 1);
  const int unaligned = __syncthreads_or(bad & 2);
  if (!GROUPED) return p.dense_slabs;
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.status = bad_offsets ? 3 : (unaligned ? 4 : 0);
  return (bad_offsets || unaligned) ? -1 : (int64_t)m.cb[p.E];
}

// Rows of slab `slab`: first row and count (<= 32).
template <bool GROUPED>
__device__ __forceinline__ void slab_rows(const Params& p, const Smem& m, int64_t slab,
                                          int64_t& row0, int& nrows) {
  if (!GROUPED) {
    row0 = slab * 32;
    nrows = (int)min((int64_t)32, p.M - row0);
  } else {
    // largest e in [0, E-1] with cb[e] <= slab (empty groups are skipped)
    int lo = 0, hi = p.E - 1;
    const int sl = (int)slab;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (m.cb[mid] <= sl) lo = mid; else hi = mid - 1;
    }
    const int r0 = m.ro[lo] + 32 * (sl - m.cb[lo]);
    row0 = r0;
    nrows = min(32, m.ro[lo + 1] - r0);
  }
}

// Walks a warp's work items (item j = first + j * stride) as (slab, tile)
// without dividing per item.
struct Cursor {
  int64_t slab;
  int tile;
  int64_t dslab;
  int dtile;
  int n_tiles;
  __device__ __forceinline__ void init(int64_t first, int64_t stride, int nt) {
    n_tiles = nt;
    slab = first / nt;
    tile = (int)(first - slab * nt);
    dslab = stride / nt;
    dtile = (int)(stride - dslab * nt);
  }
  __device__ __forceinline__ void next() {
    slab += dslab;
    tile += dtile;
    if (tile >= n_tiles) { tile -= n_tiles; ++slab; }
  }
};

// The first item of this warp; the warp then takes every
// (gridDim.x * warps)-th item.  With few items per warp (up to 16), item i
// goes to warp i / gridDim.x of CTA i % gridDim.x, so that consecutive items
// spread over the SMs first and every SM gets the same number within one
// (measured: -4% on a 2-tile-per-warp forward); with more, CTA b takes items
// b * warps + w, the neighbouring tiles of one slab (measured faster there).
__device__ __forceinline__ int64_t first_item(int64_t n_items, int warps, int warp) {
  const int64_t total = (int64_t)gridDim.x * warps;
  return n_items <= 16 * total ? (int64_t)warp * gridDim.x + blockIdx.x
                               : (int64_t)blockIdx.x * warps + warp;
}

// The warp's ring: half-tile k (half k & 1 of the warp's item k >> 1) lives in
// slot k % SLOTS, whose mbarrier completes once per use (parity
// (k / SLOTS) & 1).  Lane 0 issues the loads, walking its own cursor.
template <int OPS, int SLOTS>
struct Ring {
  unsigned char* slots;
  uint64_t* bars;
  Cursor cur;        // item of the next half-tile to issue (lane 0)
  int64_t row0;      // its first row
  int k_issue;       // next half-tile to issue
};

// Issues the boxes of one half-tile at column x, row y into shared memory
// (dst, completing on bar).
template <int OPS, bool FWD_ILV>
__device__ __forceinline__ void ring_boxes(const Params& p, unsigned char* dst, uint64_t* bar,
                                           const void* tm_x, const void* tm_dy, int x, int y) {
  if (OPS == 3 || (OPS == 2 && tm_dy != nullptr)) {
    // backward: dY, then x (gate), then up (SwiGLU).  A SwiGLU input has a 3-D
    // map whose middle coordinate picks gate (0) or up (1), so that columns
    // past N read as zero in both halves: the dscale sum runs across all the
    // lanes of a tile, including those past N.  SReLU's map is 2-D, [rows][N].
    tma_load_2d(dst, tm_dy, x, y, bar);
    if (OPS == 3) {
      if (p.ilv) {
        tma_load_4d(dst + kOpHalfBytes, tm_x, x % p.ilv, 0, x / p.ilv, y, bar);
        tma_load_4d(dst + 2 * kOpHalfBytes, tm_x, x % p.ilv, 1, x / p.ilv, y, bar);
      } else {
        tma_load_3d(dst + kOpHalfBytes, tm_x, x, 0, y, bar);
        tma_load_3d(dst + 2 * kOpHalfBytes, tm_x, x, 1, y, bar);
      }
    } else {
      tma_load_2d(dst + kOpHalfBytes, tm_x, x, y, bar);
    }
  } else if (FWD_ILV) {
    // forward, interleaved gate / up blocks: a 4-D map [rows][N/G][2][G]
    // whose box gathers the tile's 128 gate (then up) columns into the same
    // dense [16][128] half-tile as the 2-D case
    tma_load_4d(dst, tm_x, x % p.ilv, 0, x / p.ilv, y, bar);
    tma_load_4d(dst + kOpHalfBytes, tm_x, x % p.ilv, 1, x / p.ilv, y, bar);
  } else {
    // forward: gate, then up (SwiGLU) from a 2-D [rows][width] map, width 2N
    // for SwiGLU (measured faster than the 3-D map).  In a ragged last column
    // tile the gate box reaches into the up half; the lanes past N compute on
    // those values, but nothing they produce crosses into a column below N
    // (rowwise blocks are 8-lane aligned) or is stored.
    tma_load_2d(dst, tm_x, x, y, bar);
    if (OPS == 2) tma_load_2d(dst + kOpHalfBytes, tm_x, x + p.N, y, bar);
  }
}

// FWD_ILV: a forward whose input interleaves gate and up in blocks (kIlv).
template <int OPS, int SLOTS, bool GROUPED, bool FWD_ILV = false>
__device__ __forceinline__ void ring_issue(const Params& p, const Smem& m,
                                           Ring<OPS, SLOTS>& r, const void* tm_x,
                                           const void* tm_dy) {
  const int k = r.k_issue;
  const int half = k & 1;
  if (half == 0) {
    int nrows;
    slab_rows<GROUPED>(p, m, r.cur.slab, r.row0, nrows);
  }
  const int slot = k % SLOTS;
  unsigned char* dst = r.slots + slot * OPS * kOpHalfBytes;
  uint64_t* bar = r.bars + slot;
  const int x = r.cur.tile * kTileCols, y = (int)r.row0 + half * kHalfRows;
  mbar_expect_tx(bar, OPS * kOpHalfBytes);
  ring_boxes<OPS, FWD_ILV>(p, dst, bar, tm_x, tm_dy, x, y);
  r.k_issue = k + 1;
  if (half == 1) r.cur.next();
}

// Bits of the device error word (the same values as MOEACT_DEVERR_* in
// include/moeact.h, checked there by capi.cu).
constexpr uint32_t kErrFwdWait = 0x1u;     // a forward gave up waiting for its copies
constexpr uint32_t kErrBwdWait = 0x2u;     // a backward gave up waiting for its copies
constexpr uint32_t kErrTableWait = 0x4u;   // the sigmoid table's copy never landed
constexpr uint32_t kErrTableAddr = 0x8u;   // the table lies outside 16-bit addresses

__device__ __forceinline__ void report_timeout(const Params& p, uint32_t code) {
  atomicOr(p.err, code);
}

// The sigmoid lookups address the table with 16-bit shared-memory addresses
// (sigma_pair_s); a CTA whose table would end above 64 KiB (not expected:
// the table starts the dynamic shared memory) records error bit 3 and does
// nothing, before any copy is issued.
template <bool FRONT>
__device__ __forceinline__ bool sig_table_addressable(const Params& p, const Smem& m) {
  if (!FRONT || smem_addr(m.sig) + kSigBytes <= 0x10000u) return true;
  if (threadIdx.x == 0) report_timeout(p, kErrTableAddr);
  return false;
}

// After a timeout: bounded waits for the copies still in flight into the
// warp's slots, so that none lands after the CTA has exited.
template <int OPS, int SLOTS>
__device__ __forceinline__ void ring_drain(const Ring<OPS, SLOTS>& r, int k_next) {
  for (int k = k_next; k < r.k_issue; ++k)
    mbar_wait(r.bars + (k % SLOTS), (uint32_t)(k / SLOTS) & 1u);
}


// Stores the E8M0 bytes of one row's blocks [4*tile, 4*tile + nb) (packed in
// v, block 0 in the low byte): one 32-bit store when all four exist and the
// address is aligned, bytes otherwise.
__device__ __forceinline__ void store_scales4(uint8_t* dst, uint32_t v, int nb) {
  if (nb == 4 && ((reinterpret_cast<uintptr_t>(dst) & 3u) == 0)) {
    __stcs(reinterpret_cast<unsigned int*>(dst), v);
  } else {
    for (int b = 0; b < nb; ++b) dst[b] = (uint8_t)(v >> (8 * b));
  }
}

// GEMM-ready scale layout: the E8M0 matrix cut into tiles of 128 rows x 4
// scale columns (512 bytes), tiles in row-major order, element (r, c) of a
// tile at byte (r % 32) * 16 + (r / 32) * 4 + c.  Used only when M, every
// group's rows and N are multiples of 128, so that no tile is partial.
// Byte offset of the four row scales of row r in scale columns 4t .. 4t+3
// (tile column t) of a matrix with `nct` tile columns:
__device__ __forceinline__ int64_t gemm_row_scales_off(int64_t r, int t, int nct) {
  return ((((r >> 7) * nct + t)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2);
}

// Colwise scales in the GEMM layout: a group's colwise data is read by the
// GEMM transposed ([W] rows, K = the group's rows), so its scales form the
// [W][m_e / 32] matrix of the same tiled layout; groups follow one another,
// group e's tiles starting at byte base = row_offs[e] / 32 * W (the same
// place its row-major colwise scales start).  Byte offset of the scale of
// column w, K block j (of the group), with kt = m_e / 128 tile columns:
__device__ __forceinline__ int64_t gemm_col_scale_off(int64_t base, int w, int j, int kt) {
  return base + ((int64_t)((w >> 7) * kt + (j >> 2)) << 9) + ((w & 31) << 4) +
         (((w >> 5) & 3) << 2) + (j & 3);
}

// The group geometry of slab `slab` for gemm_col_scale_off: base, the slab's
// K block j within its group, and the group's tile columns kt.
template <bool GROUPED>
__device__ __forceinline__ void gemm_col_geom(const Params& p, const Smem& m, int64_t slab,
                                              int64_t& base, int& j, int& kt) {
  if (!GROUPED) {
    base = 0;
    j = (int)slab;
    kt = (int)(p.M >> 7);
    return;
  }
  int lo = 0, hi = p.E - 1;
  const int sl = (int)slab;
  while (lo < hi) {   // largest e with cb[e] <= slab (as slab_rows)
    const int mid = (lo + hi + 1) >> 1;
    if (m.cb[mid] <= sl) lo = mid; else hi = mid - 1;
  }
  base = (int64_t)(m.ro[lo] >> 5) * p.W;
  j = sl - m.cb[lo];
  kt = (m.ro[lo + 1] - m.ro[lo]) >> 7;
}

// Gathers, for row `lane` of the tile, the four blocks' E8M0 bytes from the
// lanes that reduced them: bytes `byte_lo` (rows 0-15) / `byte_hi` (rows
// 16-31) of w[h] in lanes 8k + ((row & 15) >> 1).
__device__ __forceinline__ uint32_t gather_row_scales(uint32_t w0, uint32_t w1, int lane,
                                                      int byte_even, int byte_odd) {
  const int j = lane & 15;
  const int sh = 8 * ((j & 1) ? byte_odd : byte_even);
  uint32_t v = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int src = 8 * k + (j >> 1);
    const uint32_t a = __shfl_sync(kFull, w0, src), b = __shfl_sync(kFull, w1, src);
    v |= (((lane < 16 ? a : b) >> sh) & 0xFFu) << (8 * k);
  }
  return v;
}

// Stored column, in a gated tensor of width 2N (x, dX and the MXFP8 of dX),
// of gate column c; its up column is `p.up` further on.  [gate | up] halves
// (ilv == 0) keep c; interleaved blocks of G put it at (c / G) 2G + c % G.
__device__ __forceinline__ int glu_col(const Params& p, int c) {
  return p.ilv ? (c / p.ilv) * 2 * p.ilv + c % p.ilv : c;
}

// Row scales of row `row` of a backward tile: vg / vu hold the E8M0 bytes of
// the tile's four dgate / dup blocks (block 0 in the low byte), nb of which
// exist.  With [gate | up] halves or an interleave of 128 columns or more,
// each set of four stays adjacent (dup's `p.up` columns after dgate's); an
// interleave of 32 or 64 columns alternates them within the 8 adjacent scale
// bytes of the tile's 256 stored columns.
template <int ACT, int DIRS>
__device__ __forceinline__ void store_bwd_row_scales(const Params& p, int64_t row, int tile,
                                                     uint32_t vg, uint32_t vu, int nb) {
  const int W = p.W;
  if (ACT == kSReLU || p.ilv == 0 || p.ilv >= kTileCols) {
    const int sc = glu_col(p, tile * kTileCols);   // stored column of the tile's dgate
    if (DIRS & kGemm) {
      const int nct = W >> 7;
      __stcs(reinterpret_cast<unsigned int*>(p.rs + gemm_row_scales_off(row, sc >> 7, nct)), vg);
      if (ACT != kSReLU)
        __stcs(reinterpret_cast<unsigned int*>(
                   p.rs + gemm_row_scales_off(row, (sc + p.up) >> 7, nct)), vu);
    } else {
      uint8_t* rsr = p.rs + row * (int64_t)(W / 32) + sc / 32;
      store_scales4(rsr, vg, nb);
      if (ACT != kSReLU) store_scales4(rsr + p.up / 32, vu, nb);
    }
  } else {
    // G = 32: g0 u0 g1 u1 | g2 u2 g3 u3;  G = 64: g0 g1 u0 u1 | g2 g3 u2 u3
    const bool g32 = p.ilv == 32;
    const uint32_t w0 = __byte_perm(vg, vu, g32 ? 0x5140 : 0x5410);
    const uint32_t w1 = __byte_perm(vg, vu, g32 ? 0x7362 : 0x7632);
    if (DIRS & kGemm) {
      const int nct = W >> 7;
      __stcs(reinterpret_cast<unsigned int*>(p.rs + gemm_row_scales_off(row, 2 * tile, nct)), w0);
      __stcs(reinterpret_cast<unsigned int*>(p.rs + gemm_row_scales_off(row, 2 * tile + 1, nct)),
             w1);
    } else {
      uint8_t* rsr = p.rs + row * (int64_t)(W / 32) + 8 * tile;
      store_scales4(rsr, w0, min(4, 2 * nb));
      if (nb > 2) store_scales4(rsr + 4, w1, 2 * nb - 4);
    }
  }
}

// ------------------------------------------------------------- ClampedSwiGLU
// NaN-propagating min / max (one instruction each).
__device__ __forceinline__ float min_nan(float a, float b) {
  float r;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// Three-input form (sm_100): NaN if any input is NaN, else the largest.
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float r;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// A pair of gates clamped at L (NaN passes through).  Their sigmoids need no
// clamp: the table of a ClampedSwiGLU call holds sigma(RN(alpha * L)) for
// every gate above L.
__device__ __forceinline__ float2 clamp_gate_pair(float2 g, float L) {
  return make_float2(min_nan(g.x, L), min_nan(g.y, L));
}

// clamp(u, -L, L) + 1 for a pair of ups (NaN passes through).
__device__ __forceinline__ float2 clamped_up_plus_one(float2 u, float L) {
  return add2(make_float2(max_nan(min_nan(u.x, L), -L), max_nan(min_nan(u.y, L), -L)),
              make_float2(1.0f, 1.0f));
}

// Backward of ClampedSwiGLU for the four columns of a lane in one row (p =
// dY * s), as packed bf16 pairs: the SwiGLU form with slope alpha, dsilu =
// fma(RN(alpha * silu), 1 - sig, sig).  A gate above L or an up outside
// [-L, L] gets a +0 gradient: its half of the packed pair is cleared, so that
// a NaN or Inf in dY does not reach it.  The comparisons take the bf16 inputs
// as they are (NaN compares false).
// LB: L is a bf16 value, so both clamps are exact packed bf16 min / max on
// the inputs (one instruction per pair instead of one or two per value) and
// an up is clamped exactly when its clamp differs from it.
template <bool LB>
__device__ __forceinline__ void clamped_bwd_math(const Params& p, const float* sig, uint2 G,
                                                 uint2 U, float2 p01, float2 p23, uint32_t& dg0,
                                                 uint32_t& dg1, uint32_t& du0, uint32_t& du1,
                                                 float2& h01, float2& h23) {
  const float L = p.clamp_L;
  const uint32_t Lb2 = p.clamp_Lb2;
  float2 sg01, sg23;
  sigma_pair(sig, G.x, sg01.x, sg01.y);
  sigma_pair(sig, G.y, sg23.x, sg23.y);
  float2 si01, si23, v01, v23;
  uint2 UC = make_uint2(0u, 0u);
  if (LB) {
    const uint32_t nL2 = Lb2 ^ 0x80008000u;
    UC = make_uint2(bf16x2_min_nan(bf16x2_max_nan(U.x, nL2), Lb2),
                    bf16x2_min_nan(bf16x2_max_nan(U.y, nL2), Lb2));
    si01 = mul2(bf16x2_to_f2(bf16x2_min_nan(G.x, Lb2)), sg01);
    si23 = mul2(bf16x2_to_f2(bf16x2_min_nan(G.y, Lb2)), sg23);
    const float2 one = make_float2(1.0f, 1.0f);
    v01 = add2(bf16x2_to_f2(UC.x), one);
    v23 = add2(bf16x2_to_f2(UC.y), one);
  } else {
    si01 = mul2(clamp_gate_pair(bf16x2_to_f2(G.x), L), sg01);
    si23 = mul2(clamp_gate_pair(bf16x2_to_f2(G.y), L), sg23);
    v01 = clamped_up_plus_one(bf16x2_to_f2(U.x), L);
    v23 = clamped_up_plus_one(bf16x2_to_f2(U.y), L);
  }
  const float2 one = make_float2(1.0f, 1.0f), a2 = make_float2(p.clamp_alpha, p.clamp_alpha);
  const float2 ds01 = fma2(mul2(a2, si01), sub2(one, sg01), sg01);
  const float2 ds23 = fma2(mul2(a2, si23), sub2(one, sg23), sg23);
  const float2 dga = mul2(mul2(p01, v01), ds01), dgb = mul2(mul2(p23, v23), ds23);
  const float2 dua = mul2(p01, si01), dub = mul2(p23, si23);
  dg0 = pack_bf16x2(dga.x, dga.y) & ~bf16x2_gt_mask(G.x, Lb2);
  dg1 = pack_bf16x2(dgb.x, dgb.y) & ~bf16x2_gt_mask(G.y, Lb2);
  if (LB) {
    du0 = pack_bf16x2(dua.x, dua.y) & ~bf16x2_ne_mask(UC.x, U.x);
    du1 = pack_bf16x2(dub.x, dub.y) & ~bf16x2_ne_mask(UC.y, U.y);
  } else {
    du0 = pack_bf16x2(dua.x, dua.y) & ~bf16x2_gt_mask(U.x & 0x7FFF7FFFu, Lb2);
    du1 = pack_bf16x2(dub.x, dub.y) & ~bf16x2_gt_mask(U.y & 0x7FFF7FFFu, Lb2);
  }
  h01 = mul2(si01, v01);
  h23 = mul2(si23, v23);
}

// ------------------------------------------------------------- forward tile
// Lane l owns columns 4l .. 4l+3 of a 32 x 128 warp-tile; a rowwise block is
// 8 lanes.  Rowwise work runs per 16-row half: after the 3-step butterfly
// (off = 4, 2, 1) lane l holds the amax of rows 16h + 2(l & 7) + {0, 1} of
// block l >> 3.
template <int ACT, int DIRS, bool STAGED, bool GROUPED, bool FULL, bool LB, int OPS, int SLOTS>
__device__ __forceinline__ void fwd_tile(const Params& p, const Smem& m, Ring<OPS, SLOTS>& ring,
                                         int k0, int K, int64_t slab, int tile, int64_t row0,
                                         int nrows, float sv, int lane, const void* tm_x,
                                         bool& ok_flag) {
  const int c0 = tile * kTileCols + 4 * lane;
  const bool colok = c0 < p.N;
  const int W = p.W;
  const int Wq = W >> 2;   // row stride of the code arrays in 32-bit words

  float Y[32][4];
  uint32_t bh[2];
  unsigned int* rqb = reinterpret_cast<unsigned int*>(p.rq + row0 * (int64_t)W + c0);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int k = k0 + h;
    const int slot = k % SLOTS;
    if (!mbar_wait(ring.bars + slot, (uint32_t)(k / SLOTS) & 1u)) { ok_flag = false; return; }
    const unsigned char* sm = ring.slots + slot * OPS * kOpHalfBytes + 8 * lane;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = 16 * h + i;
      const uint2 G = *reinterpret_cast<const uint2*>(sm + i * kRowBytes);
      const float sr = __shfl_sync(kFull, sv, r);
      const float2 s2 = make_float2(sr, sr);
      float2 h01, h23;
      if (ACT == kClamped) {
        const uint2 U = *reinterpret_cast<const uint2*>(sm + kOpHalfBytes + i * kRowBytes);
        float2 sg01, sg23;
        sigma_pair_s(m.sig_key, G.x, sg01.x, sg01.y);
        sigma_pair_s(m.sig_key, G.y, sg23.x, sg23.y);
        if (LB) {
          // L is a bf16 value: both clamps as packed bf16 min / max (exact)
          const uint32_t L2 = p.clamp_Lb2, nL2 = L2 ^ 0x80008000u;
          const float2 one = make_float2(1.0f, 1.0f);
          const float2 si01 = mul2(bf16x2_to_f2(bf16x2_min_nan(G.x, L2)), sg01);
          const float2 si23 = mul2(bf16x2_to_f2(bf16x2_min_nan(G.y, L2)), sg23);
          h01 = mul2(si01, add2(bf16x2_to_f2(bf16x2_min_nan(bf16x2_max_nan(U.x, nL2), L2)), one));
          h23 = mul2(si23, add2(bf16x2_to_f2(bf16x2_min_nan(bf16x2_max_nan(U.y, nL2), L2)), one));
        } else {
          const float2 si01 = mul2(clamp_gate_pair(bf16x2_to_f2(G.x), p.clamp_L), sg01);
          const float2 si23 = mul2(clamp_gate_pair(bf16x2_to_f2(G.y), p.clamp_L), sg23);
          h01 = mul2(si01, clamped_up_plus_one(bf16x2_to_f2(U.x), p.clamp_L));
          h23 = mul2(si23, clamped_up_plus_one(bf16x2_to_f2(U.y), p.clamp_L));
        }
      } else if (ACT == kSwiGLU) {
        const uint2 U = *reinterpret_cast<const uint2*>(sm + kOpHalfBytes + i * kRowBytes);
        float2 sg01, sg23;
        sigma_pair_s(m.sig_key, G.x, sg01.x, sg01.y);
        sigma_pair_s(m.sig_key, G.y, sg23.x, sg23.y);
        const float2 si01 = mul2(bf16x2_to_f2(G.x), sg01), si23 = mul2(bf16x2_to_f2(G.y), sg23);
        const float2 u01 = bf16x2_to_f2(U.x), u23 = bf16x2_to_f2(U.y);
        if (STAGED) {
          // a = bf16(silu), h = bf16(a * u) (the product is exact in fp32),
          // each pair rounded by one packed conversion
          const float2 a01 = bf16x2_to_f2(pack_bf16x2(si01.x, si01.y));
          const float2 a23 = bf16x2_to_f2(pack_bf16x2(si23.x, si23.y));
          const float2 p01 = mul2(a01, u01), p23 = mul2(a23, u23);
          h01 = bf16x2_to_f2(pack_bf16x2(p01.x, p01.y));
          h23 = bf16x2_to_f2(pack_bf16x2(p23.x, p23.y));
        } else {
          h01 = mul2(si01, u01);
          h23 = mul2(si23, u23);
        }
      } else {
        const float r0 = relu_keep_nan(bf16_lo(G.x)), r1 = relu_keep_nan(bf16_hi(G.x));
        const float r2 = relu_keep_nan(bf16_lo(G.y)), r3 = relu_keep_nan(bf16_hi(G.y));
        h01 = mul2(make_float2(r0, r1), make_float2(r0, r1));
        h23 = mul2(make_float2(r2, r3), make_float2(r2, r3));
      }
      const float2 y01 = mul2(h01, s2), y23 = mul2(h23, s2);
      const bool live = FULL || r < nrows;
      Y[r][0] = live ? y01.x : 0.0f;
      Y[r][1] = live ? y01.y : 0.0f;
      Y[r][2] = live ? y23.x : 0.0f;
      Y[r][3] = live ? y23.y : 0.0f;
    }
    // the slot is consumed: refill it with the half-tile SLOTS ahead
    __syncwarp();
    if (lane == 0 && ring.k_issue < K)
      ring_issue<OPS, SLOTS, GROUPED, (DIRS & kIlv) != 0>(p, m, ring, tm_x, nullptr);
    if (DIRS & kRow) {
      // per-row amax of the lane's 4 values as the bits of a non-negative
      // float (NaN above +Inf), so the butterfly can take integer maxima
      uint32_t A[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * h + i;
        A[i] = __float_as_uint(max_nan(max3_nan(fabsf(Y[r][0]), fabsf(Y[r][1]), fabsf(Y[r][2])),
                                       fabsf(Y[r][3])));
      }
      bfly_max_u32<8>(A, lane, 4);
      bfly_max_u32<4>(A, lane, 2);
      bfly_max_u32<2>(A, lane, 1);
      const uint32_t b0 = e8m0_from_amax(A[0]), b1 = e8m0_from_amax(A[1]);
      bh[h] = b0 | (b1 << 8);
      const uint32_t m0 = scale_multiplier(b0), m1 = scale_multiplier(b1);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * h + i;
        const uint32_t mm = __shfl_sync(kFull, (i & 1) ? m1 : m0, (lane & 24) | (i >> 1));
        const uint32_t q = e4m3x2_2(make_float2(Y[r][0], Y[r][1]), mm, mm) |
                           (e4m3x2_2(make_float2(Y[r][2], Y[r][3]), mm, mm) << 16);
        if (FULL || (colok && r < nrows)) __stcs(rqb + r * Wq, q);
      }
    }
  }
  if (DIRS & kRow) {
    // lane l stores the four block scales of row l
    const uint32_t v = gather_row_scales(bh[0], bh[1], lane, 0, 1);
    if (lane < nrows) {
      const int nb = min(4, (p.N - tile * kTileCols) / 32);
      if (DIRS & kGemm)
        __stcs(reinterpret_cast<unsigned int*>(
                   p.rs + gemm_row_scales_off(row0 + lane, tile, p.n_tiles)), v);
      else
        store_scales4(p.rs + (row0 + lane) * (int64_t)(W / 32) + 4 * tile, v, nb);
    }
  }
  if (DIRS & kCol) {
    float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int r = 0; r < 32; r += 2)
#pragma unroll
      for (int c = 0; c < 4; ++c) a[c] = max3_nan(a[c], fabsf(Y[r][c]), fabsf(Y[r + 1][c]));
    uint32_t b[4], mu[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      b[c] = e8m0_from_amax(__float_as_uint(a[c]));
      mu[c] = scale_multiplier(b[c]);
    }
    if (colok) {
      if (DIRS & kGemm) {
        int64_t base;
        int j, kt;
        gemm_col_geom<GROUPED>(p, m, slab, base, j, kt);
#pragma unroll
        for (int c = 0; c < 4; ++c) p.cs[gemm_col_scale_off(base, c0 + c, j, kt)] = (uint8_t)b[c];
      } else {
        __stcs(reinterpret_cast<unsigned int*>(p.cs + slab * (int64_t)W + c0),
               b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24));
      }
    }
    unsigned int* qb = reinterpret_cast<unsigned int*>(p.cq + row0 * (int64_t)W + c0);
    const int Wqc = opaque(Wq);
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const uint32_t q = e4m3x2_2(make_float2(Y[r][0], Y[r][1]), mu[0], mu[1]) |
                         (e4m3x2_2(make_float2(Y[r][2], Y[r][3]), mu[2], mu[3]) << 16);
      if (FULL || (colok && r < nrows)) __stcs(qb + r * Wqc, q);
    }
  }
}

// Sets up the warp's ring (barriers initialised by lane 0) and primes it.
template <int OPS, int SLOTS, bool GROUPED, bool FWD_ILV = false>
__device__ __forceinline__ void ring_prime(const Params& p, const Smem& m, Ring<OPS, SLOTS>& r,
                                           const void* tm_x, const void* tm_dy, int K,
                                           int lane) {
  if (lane == 0) {
    for (int i = 0; i < SLOTS; ++i) mbar_init(r.bars + i, 1);
    mbar_init_fence();
    while (r.k_issue < K && r.k_issue < SLOTS)
      ring_issue<OPS, SLOTS, GROUPED, FWD_ILV>(p, m, r, tm_x, tm_dy);
  }
  __syncwarp();
}

template <int ACT, int DIRS, bool STAGED, bool GROUPED>
__global__ void __launch_bounds__(Cfg<ACT, false>::kThreads, 1)
    act_fwd_kernel(const __grid_constant__ CUtensorMap tm_x, const Params p) {
  using C = Cfg<ACT, false>;
  if (p.noop != nullptr && *p.noop != 0) return;   // a skipped replay: nothing issued yet
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const Smem m = carve<ACT, false>(smem_raw, GROUPED ? p.E : 0);
  if (!sig_table_addressable<C::kSigFront>(p, m)) return;
  uint64_t* sig_bar = m.bars + C::kWarps * C::kSlots;
  const int64_t n_slabs = stage_and_validate<C::kSig, GROUPED>(p, m, sig_bar);
  if (n_slabs < 0) {
    // bad offsets: nothing to do, but the table copy must land before exit
    if (C::kSig && threadIdx.x == 0) mbar_wait(sig_bar, 0u);
    return;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t n_items = n_slabs * p.n_tiles;
  const int64_t first = first_item(n_items, C::kWarps, warp);
  const int64_t stride = (int64_t)gridDim.x * C::kWarps;
  const int count = first < n_items ? (int)((n_items - 1 - first) / stride + 1) : 0;
  const int K = 2 * count;
  Ring<C::kOps, C::kSlots> ring;
  ring.slots = m.ring + warp * C::kSlots * C::kOps * kOpHalfBytes;
  ring.bars = m.bars + warp * C::kSlots;
  ring.k_issue = 0;
  ring.row0 = 0;
  if (count > 0) ring.cur.init(first, stride, p.n_tiles);
  ring_prime<C::kOps, C::kSlots, GROUPED, (DIRS & kIlv) != 0>(p, m, ring, &tm_x, nullptr, K, lane);
  if (C::kSig && !mbar_wait(sig_bar, 0u)) {
    if (lane == 0) {
      report_timeout(p, kErrTableWait);
      ring_drain(ring, 0);
    }
    return;
  }
  // the row scales of each item are loaded one item ahead
  Cursor cur;
  int64_t row0 = 0;
  int nrows = 0;
  float sv = 0.0f;
  if (count > 0) {
    cur.init(first, stride, p.n_tiles);
    slab_rows<GROUPED>(p, m, cur.slab, row0, nrows);
    sv = lane < nrows ? __ldg(p.s + row0 + lane) : 0.0f;
  }
  bool ok = true;
  for (int j = 0; j < count; ++j) {
    Cursor nx = cur;
    nx.next();
    int64_t row0n = 0;
    int nrowsn = 0;
    float svn = 0.0f;
    if (j + 1 < count) {
      slab_rows<GROUPED>(p, m, nx.slab, row0n, nrowsn);
      svn = lane < nrowsn ? __ldg(p.s + row0n + lane) : 0.0f;
    }
    const bool full = nrows == 32 && (cur.tile + 1) * kTileCols <= p.N;
    // (ClampedSwiGLU with a bf16 limit: the packed-clamp form of the tile)
    if (ACT == kClamped && p.clamp_bf16) {
      if (full)
        fwd_tile<ACT, DIRS, STAGED, GROUPED, true, ACT == kClamped>(
            p, m, ring, 2 * j, K, cur.slab, cur.tile, row0, nrows, sv, lane, &tm_x, ok);
      else
        fwd_tile<ACT, DIRS, STAGED, GROUPED, false, ACT == kClamped>(
            p, m, ring, 2 * j, K, cur.slab, cur.tile, row0, nrows, sv, lane, &tm_x, ok);
    } else if (full) {
      fwd_tile<ACT, DIRS, STAGED, GROUPED, true, false>(p, m, ring, 2 * j, K, cur.slab, cur.tile,
                                                        row0, nrows, sv, lane, &tm_x, ok);
    } else {
      fwd_tile<ACT, DIRS, STAGED, GROUPED, false, false>(p, m, ring, 2 * j, K, cur.slab,
                                                         cur.tile, row0, nrows, sv, lane, &tm_x,
                                                         ok);
    }
    cur = nx;
    row0 = row0n;
    nrows = nrowsn;
    sv = svn;
    if (!ok) {
      if (lane == 0) {
        report_timeout(p, kErrFwdWait);
        ring_drain(ring, 2 * j);
      }
      return;
    }
  }
}

// ------------------------------------------------------------- backward row
// The backward of one row's four columns (a lane's share): packed bf16
// dgate/dup pairs and the row's dscale partial sum_c dY*h.
template <int ACT, bool LB>
__device__ __forceinline__ void bwd_row(const Params& p, const float* sig, uint2 D, uint2 G,
                                        uint2 U, float sr, uint32_t& dg0, uint32_t& dg1,
                                        uint32_t& du0, uint32_t& du1, float& part) {
  const float2 s2 = make_float2(sr, sr);
  const float2 d01 = bf16x2_to_f2(D.x), d23 = bf16x2_to_f2(D.y);
  const float2 p01 = mul2(d01, s2), p23 = mul2(d23, s2);
  float2 h01, h23;
  if (ACT == kClamped) {
    clamped_bwd_math<LB>(p, sig, G, U, p01, p23, dg0, dg1, du0, du1, h01, h23);
  } else if (ACT == kSwiGLU) {
    const float2 u01 = bf16x2_to_f2(U.x), u23 = bf16x2_to_f2(U.y);
    float2 sg01, sg23;
    sigma_pair(sig, G.x, sg01.x, sg01.y);
    sigma_pair(sig, G.y, sg23.x, sg23.y);
    const float2 si01 = mul2(bf16x2_to_f2(G.x), sg01), si23 = mul2(bf16x2_to_f2(G.y), sg23);
    const float2 one = make_float2(1.0f, 1.0f);
    const float2 ds01 = fma2(si01, sub2(one, sg01), sg01);
    const float2 ds23 = fma2(si23, sub2(one, sg23), sg23);
    const float2 dga = mul2(mul2(p01, u01), ds01), dgb = mul2(mul2(p23, u23), ds23);
    const float2 dua = mul2(p01, si01), dub = mul2(p23, si23);
    dg0 = pack_bf16x2(dga.x, dga.y);
    dg1 = pack_bf16x2(dgb.x, dgb.y);
    du0 = pack_bf16x2(dua.x, dua.y);
    du1 = pack_bf16x2(dub.x, dub.y);
    h01 = mul2(si01, u01);
    h23 = mul2(si23, u23);
  } else {
    const float2 r01 = make_float2(relu_keep_nan(bf16_lo(G.x)), relu_keep_nan(bf16_hi(G.x)));
    const float2 r23 = make_float2(relu_keep_nan(bf16_lo(G.y)), relu_keep_nan(bf16_hi(G.y)));
    const float2 two = make_float2(2.0f, 2.0f);
    const float2 dga = mul2(p01, mul2(two, r01)), dgb = mul2(p23, mul2(two, r23));
    dg0 = pack_bf16x2(dga.x, dga.y);
    dg1 = pack_bf16x2(dgb.x, dgb.y);
    du0 = du1 = 0u;
    h01 = mul2(r01, r01);
    h23 = mul2(r23, r23);
  }
  part = __fmaf_rn(d23.y, h23.y, __fmaf_rn(d23.x, h23.x, __fmaf_rn(d01.y, h01.y,
                                                                    __fmul_rn(d01.x, h01.x))));
}

// ------------------------------------------------------------- backward tile
// dscale: each warp reduces its 32 rows x 128 columns to one partial per row
// and stores it, lane = row, into the workspace at [tile][row] (plain stores,
// no fences or counters); dscale_reduce_kernel, launched next on the same
// stream, sums each row's partials in tile order (a fixed order, so dscale is
// deterministic).  Row-direction work runs per 16-row half as the half
// arrives; the packed bf16 gradients of all 32 rows stay in registers for the
// colwise pass.
// (`full`: all 32 rows and 128 columns exist; a runtime flag, so that the
// large unrolled body exists once)
template <int ACT, int DIRS, bool GROUPED, int OPS, int SLOTS>
__device__ __forceinline__ void bwd_tile(const Params& p, const Smem& m, Ring<OPS, SLOTS>& ring,
                                         int k0, int K, int64_t slab, int tile, int64_t row0,
                                         int nrows, bool FULL, float sv, int lane,
                                         const void* tm_x, const void* tm_dy, bool& ok_flag) {
  const int N = p.N, W = p.W;
  const int Wq = W >> 2;   // code row stride in 32-bit words
  const int c0 = tile * kTileCols + 4 * lane;
  const bool colok = c0 < N;
  const int cs0 = glu_col(p, c0), Uq = p.up >> 2;   // stored column; up offset in words

  uint32_t DG[32][2], DU[32][2];
  float ph[2];
  uint32_t bh[2];
  unsigned int* rqb = reinterpret_cast<unsigned int*>(p.rq + row0 * (int64_t)W + cs0);
  uint2* dxb = reinterpret_cast<uint2*>(p.dx + row0 * (int64_t)W + cs0);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int k = k0 + h;
    const int slot = k % SLOTS;
    if (!mbar_wait(ring.bars + slot, (uint32_t)(k / SLOTS) & 1u)) { ok_flag = false; return; }
    const unsigned char* sm = ring.slots + slot * OPS * kOpHalfBytes + 8 * lane;
    float P[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = 16 * h + i;
      const uint2 D = *reinterpret_cast<const uint2*>(sm + i * kRowBytes);
      const uint2 G = *reinterpret_cast<const uint2*>(sm + kOpHalfBytes + i * kRowBytes);
      const float sr = __shfl_sync(kFull, sv, r);
      const float2 s2 = make_float2(sr, sr);
      const float2 d01 = bf16x2_to_f2(D.x), d23 = bf16x2_to_f2(D.y);
      const float2 p01 = mul2(d01, s2), p23 = mul2(d23, s2);
      float2 dg01, dg23, du01, du23, h01, h23;
      uint32_t qg0, qg1, qu0, qu1;   // the packed bf16 gradients
      if (ACT == kClamped) {
        const uint2 U = *reinterpret_cast<const uint2*>(sm + 2 * kOpHalfBytes + i * kRowBytes);
        clamped_bwd_math<false>(p, m.sig, G, U, p01, p23, qg0, qg1, qu0, qu1, h01, h23);
      } else if (ACT == kSwiGLU) {
        const uint2 U = *reinterpret_cast<const uint2*>(sm + 2 * kOpHalfBytes + i * kRowBytes);
        const float2 u01 = bf16x2_to_f2(U.x), u23 = bf16x2_to_f2(U.y);
        float2 sg01, sg23;
        sigma_pair(m.sig, G.x, sg01.x, sg01.y);
        sigma_pair(m.sig, G.y, sg23.x, sg23.y);
        const float2 si01 = mul2(bf16x2_to_f2(G.x), sg01), si23 = mul2(bf16x2_to_f2(G.y), sg23);
        const float2 one = make_float2(1.0f, 1.0f);
        const float2 ds01 = fma2(si01, sub2(one, sg01), sg01);
        const float2 ds23 = fma2(si23, sub2(one, sg23), sg23);
        dg01 = mul2(mul2(p01, u01), ds01);
        dg23 = mul2(mul2(p23, u23), ds23);
        du01 = mul2(p01, si01);
        du23 = mul2(p23, si23);
        h01 = mul2(si01, u01);
        h23 = mul2(si23, u23);
      } else {
        const float r0 = relu_keep_nan(bf16_lo(G.x)), r1 = relu_keep_nan(bf16_hi(G.x));
        const float r2 = relu_keep_nan(bf16_lo(G.y)), r3 = relu_keep_nan(bf16_hi(G.y));
        const float2 two = make_float2(2.0f, 2.0f);
        dg01 = mul2(p01, mul2(two, make_float2(r0, r1)));
        dg23 = mul2(p23, mul2(two, make_float2(r2, r3)));
        du01 = du23 = make_float2(0.0f, 0.0f);
        h01 = mul2(make_float2(r0, r1), make_float2(r0, r1));
        h23 = mul2(make_float2(r2, r3), make_float2(r2, r3));
      }
      if (ACT != kClamped) {
        qg0 = pack_bf16x2(dg01.x, dg01.y);
        qg1 = pack_bf16x2(dg23.x, dg23.y);
        qu0 = pack_bf16x2(du01.x, du01.y);
        qu1 = pack_bf16x2(du23.x, du23.y);
      }
      const bool live = FULL || r < nrows;
      DG[r][0] = live ? qg0 : 0u;
      DG[r][1] = live ? qg1 : 0u;
      DU[r][0] = (live && ACT != kSReLU) ? qu0 : 0u;
      DU[r][1] = (live && ACT != kSReLU) ? qu1 : 0u;
      P[i] = live ? __fmaf_rn(d23.y, h23.y, __fmaf_rn(d23.x, h23.x,
                              __fmaf_rn(d01.y, h01.y, __fmul_rn(d01.x, h01.x))))
                  : 0.0f;
      if (p.dx != nullptr && (FULL || (colok && r < nrows))) {
        __stcs(dxb + r * Wq, make_uint2(DG[r][0], DG[r][1]));
        if (ACT != kSReLU) __stcs(dxb + r * Wq + Uq, make_uint2(DU[r][0], DU[r][1]));
      }
    }
    __syncwarp();
    if (lane == 0 && ring.k_issue < K) ring_issue<OPS, SLOTS, GROUPED>(p, m, ring, tm_x, tm_dy);
    if (p.dscale != nullptr) {
      // lane l ends with the warp sum of row 16h + (l >> 1)
      bfly_sum_f32<8>(P, lane, 16);
      bfly_sum_f32<4>(P, lane, 8);
      bfly_sum_f32<2>(P, lane, 4);
      bfly_sum_f32<1>(P, lane, 2);
      ph[h] = __fadd_rn(P[0], __shfl_xor_sync(kFull, P[0], 1));
    }
    if (DIRS & kRow) {
      // packed per-row block maxima over the lane's 4 columns: low half dgate,
      // high half dup
      uint32_t A[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * h + i;
        const uint32_t mg = __vmaxu2(DG[r][0] & 0x7FFF7FFFu, DG[r][1] & 0x7FFF7FFFu);
        const uint32_t mu = __vmaxu2(DU[r][0] & 0x7FFF7FFFu, DU[r][1] & 0x7FFF7FFFu);
        A[i] = __vmaxu2(__byte_perm(mg, mu, 0x5410), __byte_perm(mg, mu, 0x7632));
      }
      bfly_max_u16x2<8>(A, lane, 4);
      bfly_max_u16x2<4>(A, lane, 2);
      bfly_max_u16x2<2>(A, lane, 1);
      // lane l: rows 16h + 2(l & 7) + {0, 1} of block l >> 3
      const uint32_t bg0 = e8m0_from_amax(A[0] << 16), bu0 = e8m0_from_amax(A[0] & 0xFFFF0000u);
      const uint32_t bg1 = e8m0_from_amax(A[1] << 16), bu1 = e8m0_from_amax(A[1] & 0xFFFF0000u);
      bh[h] = bg0 | (bu0 << 8) | (bg1 << 16) | (bu1 << 24);
      const uint32_t mg0 = scale_multiplier(bg0), mg1 = scale_multiplier(bg1);
      const uint32_t mu0 = scale_multiplier(bu0), mu1 = scale_multiplier(bu1);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * h + i;
        const int src = (lane & 24) | (i >> 1);
        const uint32_t mg = __shfl_sync(kFull, (i & 1) ? mg1 : mg0, src);
        const uint32_t qg = e4m3x2_2(bf16x2_to_f2(DG[r][0]), mg, mg) |
                            (e4m3x2_2(bf16x2_to_f2(DG[r][1]), mg, mg) << 16);
        uint32_t qu = 0;
        if (ACT != kSReLU) {
          const uint32_t mu = __shfl_sync(kFull, (i & 1) ? mu1 : mu0, src);
          qu = e4m3x2_2(bf16x2_to_f2(DU[r][0]), mu, mu) |
               (e4m3x2_2(bf16x2_to_f2(DU[r][1]), mu, mu) << 16);
        }
        if (FULL || (colok && r < nrows)) {
          __stcs(rqb + r * Wq, qg);
          if (ACT != kSReLU) __stcs(rqb + r * Wq + Uq, qu);
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
    // lane l stores the block scales of row l (dgate blocks, then dup blocks)
    const uint32_t vg = gather_row_scales(bh[0], bh[1], lane, 0, 2);
    const uint32_t vu = gather_row_scales(bh[0], bh[1], lane, 1, 3);
    if (lane < nrows)
      store_bwd_row_scales<ACT, DIRS>(p, row0 + lane, tile, vg, vu,
                                      min(4, (N - tile * kTileCols) / 32));
  }
  if (DIRS & kCol) {
    uint32_t ag[2] = {0u, 0u}, au[2] = {0u, 0u};
#pragma unroll
    for (int r = 0; r < 32; r += 2)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        ag[c] = __vimax3_u16x2(ag[c], DG[r][c] & 0x7FFF7FFFu, DG[r + 1][c] & 0x7FFF7FFFu);
        au[c] = __vimax3_u16x2(au[c], DU[r][c] & 0x7FFF7FFFu, DU[r + 1][c] & 0x7FFF7FFFu);
      }
    uint32_t bg[4], bu[4], mg[4], mu[4];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      bg[2 * c] = e8m0_from_amax(ag[c] << 16);
      bg[2 * c + 1] = e8m0_from_amax(ag[c] & 0xFFFF0000u);
      bu[2 * c] = e8m0_from_amax(au[c] << 16);
      bu[2 * c + 1] = e8m0_from_amax(au[c] & 0xFFFF0000u);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      mg[c] = scale_multiplier(bg[c]);
      mu[c] = scale_multiplier(bu[c]);
    }
    if (colok) {
      if (DIRS & kGemm) {
        int64_t base;
        int j, kt;
        gemm_col_geom<GROUPED>(p, m, slab, base, j, kt);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          p.cs[gemm_col_scale_off(base, cs0 + c, j, kt)] = (uint8_t)bg[c];
          if (ACT != kSReLU)
            p.cs[gemm_col_scale_off(base, cs0 + p.up + c, j, kt)] = (uint8_t)bu[c];
        }
      } else {
        uint8_t* csr = p.cs + slab * (int64_t)W + cs0;
        __stcs(reinterpret_cast<unsigned int*>(csr),
               bg[0] | (bg[1] << 8) | (bg[2] << 16) | (bg[3] << 24));
        if (ACT != kSReLU)
          __stcs(reinterpret_cast<unsigned int*>(csr + p.up),
                 bu[0] | (bu[1] << 8) | (bu[2] << 16) | (bu[3] << 24));
      }
    }
    unsigned int* qb = reinterpret_cast<unsigned int*>(p.cq + row0 * (int64_t)W + cs0);
    const int Wqc = opaque(Wq);
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const uint32_t qg = e4m3x2_2(bf16x2_to_f2_p(DG[r][0]), mg[0], mg[1]) |
                          (e4m3x2_2(bf16x2_to_f2_p(DG[r][1]), mg[2], mg[3]) << 16);
      if (FULL || (colok && r < nrows)) {
        __stcs(qb + r * Wqc, qg);
        if (ACT != kSReLU) {
          const uint32_t qu = e4m3x2_2(bf16x2_to_f2_p(DU[r][0]), mu[0], mu[1]) |
                              (e4m3x2_2(bf16x2_to_f2_p(DU[r][1]), mu[2], mu[3]) << 16);
          __stcs(qb + r * Wqc + Uq, qu);
        }
      }
    }
  }
}

// The backward tile when dX is written (the usual case): the colwise pass
// re-reads each lane's own just-written dX columns (program order makes a
// thread's stores visible to its later loads; the 16 KiB per tile is still in
// L2), so only one 16-row half of gradients is held in registers.  Colwise
// maxima are accumulated on the fly.
// One 16-row half of a backward tile: waits for its ring slot, computes dX for
// the half (stored), the half's dscale partial (ph, rows 2(l&15) + {0,1}),
// its rowwise scales (bh, this lane's reduced E8M0 bytes) and codes, and folds
// the colwise maxima into acg / acu.  Returns false if the slot never landed.
template <int ACT, int DIRS, bool GROUPED, bool FULL, bool LB, int OPS, int SLOTS>
__device__ __forceinline__ bool bwd_half_rr(const Params& p, const Smem& m,
                                            Ring<OPS, SLOTS>& ring, int k0, int h, int K,
                                            int nrows, float sv, int lane, bool colok, int Wq,
                                            unsigned int* rqb, uint2* dxb, const void* tm_x,
                                            const void* tm_dy, float& ph, uint32_t& bh,
                                            uint32_t (&acg)[2], uint32_t (&acu)[2]) {
  // per-half copies the compiler cannot hoist out of the (rolled) half loop,
  // so that the 16 row offsets are not kept live across it
  const int Wqh = opaque(Wq), Nq = opaque(p.up >> 2);
  const int nrh = nrows - 16 * h;   // rows of this half that exist
  const int k = k0 + h;
  const int slot = k % SLOTS;
  if (!mbar_wait(ring.bars + slot, (uint32_t)(k / SLOTS) & 1u)) return false;
  const unsigned char* sm = ring.slots + slot * OPS * kOpHalfBytes + 8 * lane;
  uint32_t DG[16][2], DU[16][2];
  float P[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int r = 16 * h + i;
    const uint2 D = *reinterpret_cast<const uint2*>(sm + i * kRowBytes);
    const uint2 G = *reinterpret_cast<const uint2*>(sm + kOpHalfBytes + i * kRowBytes);
    uint2 U = make_uint2(0u, 0u);
    if (ACT != kSReLU) U = *reinterpret_cast<const uint2*>(sm + 2 * kOpHalfBytes + i * kRowBytes);
    const float sr = __shfl_sync(kFull, sv, r);
    float part;
    bwd_row<ACT, LB>(p, m.sig, D, G, U, sr, DG[i][0], DG[i][1], DU[i][0], DU[i][1], part);
    const bool live = FULL || i < nrh;
    // rows past the slab's end: past M they read as zero (and give zeros); in
    // a grouped call they are the next group's rows, which must not count
    if (GROUPED && !live) { DG[i][0] = DG[i][1] = DU[i][0] = DU[i][1] = 0u; part = 0.0f; }
    P[i] = part;
    if (FULL || (colok && live)) {
      dxb[r * Wqh] = make_uint2(DG[i][0], DG[i][1]);
      if (ACT != kSReLU) dxb[r * Wqh + Nq] = make_uint2(DU[i][0], DU[i][1]);
    }
    if (DIRS & kCol) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        acg[c] = __vmaxu2(acg[c], DG[i][c] & 0x7FFF7FFFu);
        if (ACT != kSReLU) acu[c] = __vmaxu2(acu[c], DU[i][c] & 0x7FFF7FFFu);
      }
    }
  }
  __syncwarp();
  if (lane == 0 && ring.k_issue < K) ring_issue<OPS, SLOTS, GROUPED>(p, m, ring, tm_x, tm_dy);
  if (p.dscale != nullptr) {
    bfly_sum_f32<8>(P, lane, 16);
    bfly_sum_f32<4>(P, lane, 8);
    bfly_sum_f32<2>(P, lane, 4);
    bfly_sum_f32<1>(P, lane, 2);
    ph = __fadd_rn(P[0], __shfl_xor_sync(kFull, P[0], 1));
  }
  if (DIRS & kRow) {
    uint32_t A[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t mg = __vmaxu2(DG[i][0] & 0x7FFF7FFFu, DG[i][1] & 0x7FFF7FFFu);
      const uint32_t mu = __vmaxu2(DU[i][0] & 0x7FFF7FFFu, DU[i][1] & 0x7FFF7FFFu);
      A[i] = __vmaxu2(__byte_perm(mg, mu, 0x5410), __byte_perm(mg, mu, 0x7632));
    }
    bfly_max_u16x2<8>(A, lane, 4);
    bfly_max_u16x2<4>(A, lane, 2);
    bfly_max_u16x2<2>(A, lane, 1);
    const uint32_t bg0 = e8m0_from_amax(A[0] << 16), bu0 = e8m0_from_amax(A[0] & 0xFFFF0000u);
    const uint32_t bg1 = e8m0_from_amax(A[1] << 16), bu1 = e8m0_from_amax(A[1] & 0xFFFF0000u);
    bh = bg0 | (bu0 << 8) | (bg1 << 16) | (bu1 << 24);
    const uint32_t mg0 = scale_multiplier(bg0), mg1 = scale_multiplier(bg1);
    const uint32_t mu0 = scale_multiplier(bu0), mu1 = scale_multiplier(bu1);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = 16 * h + i;
      const int src = (lane & 24) | (i >> 1);
      const uint32_t mg = __shfl_sync(kFull, (i & 1) ? mg1 : mg0, src);
      const uint32_t qg = e4m3x2_2(bf16x2_to_f2(DG[i][0]), mg, mg) |
                          (e4m3x2_2(bf16x2_to_f2(DG[i][1]), mg, mg) << 16);
      uint32_t qu = 0;
      if (ACT != kSReLU) {
        const uint32_t mu = __shfl_sync(kFull, (i & 1) ? mu1 : mu0, src);
        qu = e4m3x2_2(bf16x2_to_f2(DU[i][0]), mu, mu) |
             (e4m3x2_2(bf16x2_to_f2(DU[i][1]), mu, mu) << 16);
      }
      if (FULL || (colok && i < nrh)) {
        __stcs(rqb + r * Wqh, qg);
        if (ACT != kSReLU) __stcs(rqb + r * Wqh + Nq, qu);
      }
    }
  }
  return true;
}

// Colwise codes of a backward tile from dX re-read out of L2, in four chunks
// of 8 rows with double-buffered loads: the loads of the next chunk are in
// flight while the current one is quantized and stored, so one load latency
// per tile is exposed instead of one per chunk.
template <int ACT, bool FULL>
__device__ __forceinline__ void bwd_colwise_load8(int q, int U, int nrows, bool colok, int Wqc,
                                                  const uint2* dxb, uint2 (&RG)[8],
                                                  uint2 (&RU)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 8 * q + i;
    const bool ok = FULL || (colok && r < nrows);
    RG[i] = ok ? __ldcg(dxb + r * Wqc) : make_uint2(0u, 0u);
    if (ACT != kSReLU) RU[i] = ok ? __ldcg(dxb + r * Wqc + (U >> 2)) : make_uint2(0u, 0u);
  }
}

template <int ACT, bool FULL>
__device__ __forceinline__ void bwd_colwise_store8(int q, int U, int nrows, bool colok, int Wqc,
                                                   unsigned int* qb, const uint2 (&RG)[8],
                                                   const uint2 (&RU)[8], const uint32_t (&mg)[4],
                                                   const uint32_t (&mu)[4]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 8 * q + i;
    const uint32_t qg = e4m3x2_2(bf16x2_to_f2_p(RG[i].x), mg[0], mg[1]) |
                        (e4m3x2_2(bf16x2_to_f2_p(RG[i].y), mg[2], mg[3]) << 16);
    if (FULL || (colok && r < nrows)) {
      __stcs(qb + r * Wqc, qg);
      if (ACT != kSReLU) {
        const uint32_t qu = e4m3x2_2(bf16x2_to_f2_p(RU[i].x), mu[0], mu[1]) |
                            (e4m3x2_2(bf16x2_to_f2_p(RU[i].y), mu[2], mu[3]) << 16);
        __stcs(qb + r * Wqc + (U >> 2), qu);
      }
    }
  }
}

template <int ACT, bool FULL>
__device__ __forceinline__ void bwd_colwise_rr(int U, int nrows, bool colok, int Wqc,
                                               const uint2* dxb, unsigned int* qb,
                                               const uint32_t (&mg)[4], const uint32_t (&mu)[4]) {
  uint2 AG[8], AU[8], BG[8], BU[8];
  if (ACT == kClamped) {
    // ClampedSwiGLU's larger row body leaves fewer registers: 16 rows at a
    // time, loads first, nothing carried across the loop (the overlapped
    // form below spills there and measured slower)
#pragma unroll 1
    for (int q = 0; q < 4; q += 2) {
      bwd_colwise_load8<ACT, FULL>(q, U, nrows, colok, Wqc, dxb, AG, AU);
      bwd_colwise_load8<ACT, FULL>(q + 1, U, nrows, colok, Wqc, dxb, BG, BU);
      bwd_colwise_store8<ACT, FULL>(q, U, nrows, colok, Wqc, qb, AG, AU, mg, mu);
      bwd_colwise_store8<ACT, FULL>(q + 1, U, nrows, colok, Wqc, qb, BG, BU, mg, mu);
    }
    return;
  }
  bwd_colwise_load8<ACT, FULL>(0, U, nrows, colok, Wqc, dxb, AG, AU);
#pragma unroll 1
  for (int q = 0; q < 4; q += 2) {
    bwd_colwise_load8<ACT, FULL>(q + 1, U, nrows, colok, Wqc, dxb, BG, BU);
    bwd_colwise_store8<ACT, FULL>(q, U, nrows, colok, Wqc, qb, AG, AU, mg, mu);
    if (q + 2 < 4) bwd_colwise_load8<ACT, FULL>(q + 2, U, nrows, colok, Wqc, dxb, AG, AU);
    bwd_colwise_store8<ACT, FULL>(q + 1, U, nrows, colok, Wqc, qb, BG, BU, mg, mu);
  }
}

template <int ACT, int DIRS, bool GROUPED, bool FULL, bool LB, int OPS, int SLOTS>
__device__ __forceinline__ void bwd_tile_rr(const Params& p, const Smem& m,
                                            Ring<OPS, SLOTS>& ring, int k0, int K, int64_t slab,
                                            int tile, int64_t row0, int nrows, float sv, int lane,
                                            const void* tm_x, const void* tm_dy, bool& ok_flag) {
  const int N = p.N, W = p.W;
  const int Wq = W >> 2;   // row stride in 32-bit words (codes) / 8-byte words (dx)
  const int c0 = tile * kTileCols + 4 * lane;
  const bool colok = c0 < N;
  const int cs0 = glu_col(p, c0);   // stored column of the lane's first dgate column
  float ph[2] = {0.0f, 0.0f};
  uint32_t bh[2] = {0u, 0u};
  uint32_t acg[2] = {0u, 0u}, acu[2] = {0u, 0u};   // colwise maxima (packed bf16 magnitudes)
  unsigned int* rqb = reinterpret_cast<unsigned int*>(p.rq + row0 * (int64_t)W + cs0);
  uint2* dxb = reinterpret_cast<uint2*>(p.dx + row0 * (int64_t)W + cs0);
  // one copy of the half body (only scalars cross the halves): half the code
  // for the instruction cache to hold.  Measured faster than two unrolled
  // copies at every size, most of all when each warp sees only a few tiles
  // and the code is fetched cold.
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    float v;
    uint32_t b;
    if (!bwd_half_rr<ACT, DIRS, GROUPED, FULL, LB>(p, m, ring, k0, h, K, nrows, sv, lane, colok, Wq,
                                               rqb, dxb, tm_x, tm_dy, v, b, acg, acu)) {
      ok_flag = false;
      return;
    }
    if (h == 0) { ph[0] = v; bh[0] = b; } else { ph[1] = v; bh[1] = b; }
  }
  if (p.dscale != nullptr) {
    const int src = 2 * (lane & 15);
    const float v0 = __shfl_sync(kFull, ph[0], src), v1 = __shfl_sync(kFull, ph[1], src);
    if (lane < nrows) __stcg(p.part + (int64_t)tile * p.M + row0 + lane, lane < 16 ? v0 : v1);
  }
  if (DIRS & kRow) {
    const uint32_t vg = gather_row_scales(bh[0], bh[1], lane, 0, 2);
    const uint32_t vu = gather_row_scales(bh[0], bh[1], lane, 1, 3);
    if (lane < nrows)
      store_bwd_row_scales<ACT, DIRS>(p, row0 + lane, tile, vg, vu,
                                      min(4, (N - tile * kTileCols) / 32));
  }
  if (DIRS & kCol) {
    uint32_t bg[4], bu[4], mg[4], mu[4];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      bg[2 * c] = e8m0_from_amax(acg[c] << 16);
      bg[2 * c + 1] = e8m0_from_amax(acg[c] & 0xFFFF0000u);
      bu[2 * c] = e8m0_from_amax(acu[c] << 16);
      bu[2 * c + 1] = e8m0_from_amax(acu[c] & 0xFFFF0000u);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      mg[c] = scale_multiplier(bg[c]);
      mu[c] = scale_multiplier(bu[c]);
    }
    if (colok) {
      if (DIRS & kGemm) {
        int64_t base;
        int j, kt;
        gemm_col_geom<GROUPED>(p, m, slab, base, j, kt);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          p.cs[gemm_col_scale_off(base, cs0 + c, j, kt)] = (uint8_t)bg[c];
          if (ACT != kSReLU)
            p.cs[gemm_col_scale_off(base, cs0 + p.up + c, j, kt)] = (uint8_t)bu[c];
        }
      } else {
        uint8_t* csr = p.cs + slab * (int64_t)W + cs0;
        __stcs(reinterpret_cast<unsigned int*>(csr),
               bg[0] | (bg[1] << 8) | (bg[2] << 16) | (bg[3] << 24));
        if (ACT != kSReLU)
          __stcs(reinterpret_cast<unsigned int*>(csr + p.up),
                 bu[0] | (bu[1] << 8) | (bu[2] << 16) | (bu[3] << 24));
      }
    }
    unsigned int* qb = reinterpret_cast<unsigned int*>(p.cq + row0 * (int64_t)W + cs0);
    const int Wqc = opaque(Wq);
    bwd_colwise_rr<ACT, FULL>(p.up, nrows, colok, Wqc, dxb, qb, mg, mu);
  }
}

// REREAD: dX is written and the colwise pass re-reads it (from L2); without
// it the whole tile stays in registers for the colwise pass.
template <int ACT, int DIRS, bool GROUPED, bool REREAD>
__global__ void __launch_bounds__(Cfg<ACT, true>::kThreads, 1)
    act_bwd_kernel(const __grid_constant__ CUtensorMap tm_x,
                   const __grid_constant__ CUtensorMap tm_dy, const Params p) {
  using C = Cfg<ACT, true>;
  if (p.noop != nullptr && *p.noop != 0) return;   // a skipped replay: nothing issued yet
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const Smem m = carve<ACT, true>(smem_raw, GROUPED ? p.E : 0);
  uint64_t* sig_bar = m.bars + C::kWarps * C::kSlots;
  const int64_t n_slabs = stage_and_validate<C::kSig, GROUPED>(p, m, sig_bar);
  if (n_slabs < 0) {
    if (C::kSig && threadIdx.x == 0) mbar_wait(sig_bar, 0u);
    return;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t n_items = n_slabs * p.n_tiles;
  const int64_t first = first_item(n_items, C::kWarps, warp);
  const int64_t stride = (int64_t)gridDim.x * C::kWarps;
  const int count = first < n_items ? (int)((n_items - 1 - first) / stride + 1) : 0;
  const int K = 2 * count;
  Ring<C::kOps, C::kSlots> ring;
  ring.slots = m.ring + warp * C::kSlots * C::kOps * kOpHalfBytes;
  ring.bars = m.bars + warp * C::kSlots;
  ring.k_issue = 0;
  ring.row0 = 0;
  if (count > 0) ring.cur.init(first, stride, p.n_tiles);
  ring_prime<C::kOps, C::kSlots, GROUPED>(p, m, ring, &tm_x, &tm_dy, K, lane);
  if (C::kSig && !mbar_wait(sig_bar, 0u)) {
    if (lane == 0) {
      report_timeout(p, kErrTableWait);
      ring_drain(ring, 0);
    }
    return;
  }
  // the row scales of each item are loaded one item ahead
  Cursor cur;
  int64_t row0 = 0;
  int nrows = 0;
  float sv = 0.0f;
  if (count > 0) {
    cur.init(first, stride, p.n_tiles);
    slab_rows<GROUPED>(p, m, cur.slab, row0, nrows);
    sv = lane < nrows ? __ldg(p.s + row0 + lane) : 0.0f;
  }
  bool ok = true;
  for (int j = 0; j < count; ++j) {
    Cursor nx = cur;
    nx.next();
    int64_t row0n = 0;
    int nrowsn = 0;
    float svn = 0.0f;
    if (j + 1 < count) {
      slab_rows<GROUPED>(p, m, nx.slab, row0n, nrowsn);
      svn = lane < nrowsn ? __ldg(p.s + row0n + lane) : 0.0f;
    }
    const bool full = nrows == 32 && (cur.tile + 1) * kTileCols <= p.N;
    if (REREAD) {
      // (ClampedSwiGLU with a bf16 limit: the packed-clamp form of the tile)
      if (ACT == kClamped && p.clamp_bf16) {
        if (full)
          bwd_tile_rr<ACT, DIRS, GROUPED, true, ACT == kClamped>(
              p, m, ring, 2 * j, K, cur.slab, cur.tile, row0, nrows, sv, lane, &tm_x, &tm_dy, ok);
        else
          bwd_tile_rr<ACT, DIRS, GROUPED, false, ACT == kClamped>(
              p, m, ring, 2 * j, K, cur.slab, cur.tile, row0, nrows, sv, lane, &tm_x, &tm_dy, ok);
      } else if (full) {
        bwd_tile_rr<ACT, DIRS, GROUPED, true, false>(p, m, ring, 2 * j, K, cur.slab, cur.tile,
                                                     row0, nrows, sv, lane, &tm_x, &tm_dy, ok);
      } else {
        bwd_tile_rr<ACT, DIRS, GROUPED, false, false>(p, m, ring, 2 * j, K, cur.slab, cur.tile,
                                                      row0, nrows, sv, lane, &tm_x, &tm_dy, ok);
      }
    } else {
      bwd_tile<ACT, DIRS, GROUPED>(p, m, ring, 2 * j, K, cur.slab, cur.tile, row0, nrows, full,
                                   sv, lane, &tm_x, &tm_dy, ok);
    }
    cur = nx;
    row0 = row0n;
    nrows = nrowsn;
    sv = svn;
    if (!ok) {
      if (lane == 0) {
        report_timeout(p, kErrBwdWait);
        ring_drain(ring, 2 * j);
      }
      return;
    }
  }
}

}  // namespace moeact
