// Kernels of the host translation unit (capi.cu) only: the correctly rounded
// fp32 sigmoid tables, built once per device (and per slope alpha, for
// ClampedSwiGLU), the test hook that expands a table, splits_to_offsets and
// the dscale sum.  (The fused kernels, instantiated in their own translation
// units, stage a table from the device pointer they are given.)
#pragma once

#include "kernels.cuh"

namespace moeact {

// sigma(g) for SwiGLU lives in device global memory of this module, one copy
// per device, written by sigma_table_init before any activation kernel reads
// it, already in the shared-memory layout (positive gates at [0, 4097),
// negative at [8192, 12289)) so that a kernel stages it with one bulk copy.
__device__ __align__(16) float g_sigma_table[kSigBytes / 4];

// Builds a table of sigma(z), z = RN(alpha * g), for the bf16 gates g of the
// table's range (alpha = 1: sigma(g)).  For |z| < 2^-9, sigma(z) = 1/2 + z/4
// - z^3/48 + O(z^5): hi = 1/2 + z/4 is exact in binary64 (z has 24
// significant bits and |z| >= 2^-27 here) and the rest is far smaller than
// any distance from hi to an fp32 rounding boundary, except when hi sits
// exactly on one (a midpoint), where binary64 cannot see the remainder; there
// the remainder's sign (that of -z) decides.  Elsewhere the table comes from
// binary64 exp and division (error < 2^-51 relative), and entries whose
// binary64 value lies within 2^-48 (relative) of a rounding boundary are
// counted as uncertain (none are expected for alpha = 1: the closest true
// value stays 2^-37 away; the caller refuses a table with any).
//
// A ClampedSwiGLU table also takes the clamp of the gate at `limit`: every
// entry of a gate above it holds sig_limit = sigma(RN(alpha * limit))
// (certified by the caller).  The entries that stand for a range of gates
// stay right for every gate of their range: sigma is 1/2 on both sides of a
// limit below 2^-25 (the first entry, |g| <= 2^-25), and gates of 128 and
// above (the last entry) either all lie above the limit or, for a limit of
// 128 or more and alpha >= 13/16, have sigma 1 on both sides of it.
__global__ void sigma_table_init(float* tab, float alpha, float limit, float sig_limit,
                                 int* uncertain) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= kSigEntries) return;
  const uint32_t neg = i >= (int)kSigPerSign ? 1u : 0u;
  const uint32_t mag = (uint32_t)i - neg * kSigPerSign + kSigLo;
  const float g = __uint_as_float(((neg << 15) | mag) << 16);
  if (g > limit) {
    tab[sig_slot(i)] = sig_limit;
    return;
  }
  const float z = __fmul_rn(alpha, g);
  if (fabsf(z) < 0x1p-9f) {
    const double hi = 0.5 + 0.25 * (double)z;
    const float d = __double2float_rd(hi), u = __double2float_ru(hi);
    float f;
    if (d == u) {
      f = d;
    } else if (hi == 0.5 * ((double)d + (double)u)) {
      f = z > 0.0f ? d : u;
    } else {
      f = __double2float_rn(hi);
    }
    tab[sig_slot(i)] = f;
    return;
  }
  const double sd = 1.0 / (1.0 + exp(-(double)z));
  const float f = __double2float_rn(sd);
  const double up = 0.5 * ((double)f + (double)nextafterf(f, __int_as_float(0x7F800000)));
  const double dn = 0.5 * ((double)f + (double)nextafterf(f, __int_as_float(0xFF800000)));
  const double tol = fabs(sd) * 0x1p-48;
  if (!(fabs(sd - up) > tol && fabs(sd - dn) > tol)) atomicAdd(uncertain, 1);
  tab[sig_slot(i)] = f;
}

// Expands a table to all 65536 bf16 patterns (test hook), through the same
// shared-memory layout and pair lookup the fused kernels use: thread t looks
// up the packed pair (2t, 2t + 1).
__global__ void sigma_table_dump(const float* src, float* out) {
  extern __shared__ __align__(16) float tab[];
  for (int i = threadIdx.x; i < kSigBytes / 4; i += blockDim.x) tab[i] = src[i];
  __syncthreads();
  const uint32_t t = blockIdx.x * blockDim.x + threadIdx.x;
  // the table's address passes through a volatile move after the barrier, so
  // the lookups (plain ld.shared statements) cannot be scheduled before it
  uint32_t T;
  asm volatile("mov.u32 %0, %1;" : "=r"(T) : "r"(smem_addr(tab)));
  if (t < 32768 && T + kSigBytes <= 0x10000u) {
    float a, b;
    sigma_pair_s(sigma_key(T), (2 * t) | ((2 * t + 1) << 16), a, b);
    out[2 * t] = a;
    out[2 * t + 1] = b;
  }
}

// Shared-memory address at which dynamic shared memory begins (thread 0
// writes it to *out).  The fused kernels have no static shared memory, so
// theirs begins at the same address; the SwiGLU forward needs its sigmoid
// table, placed there, to end below 64 KiB.
__global__ void smem_base_probe(uint32_t* out) {
  extern __shared__ __align__(128) unsigned char raw[];
  if (threadIdx.x == 0) *out = smem_addr(raw);
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
  if (st) {
    // no offsets for bad splits: mark them invalid, so that a grouped call
    // given them reports MOEACT_DEV_BAD_OFFSETS and writes nothing (instead
    // of running on offsets left by an earlier call)
    if (t == 0) {
      ro[0] = -1;
      if (cb) cb[0] = -1;
    }
    return;
  }
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
                                                            float* __restrict__ dscale,
                                                            const int32_t* noop) {
  if (noop != nullptr && *noop != 0) return;
  const int64_t row = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= M) return;
  float acc = 0.0f;
#pragma unroll 8
  for (int t = 0; t < n_tiles; ++t) acc = __fadd_rn(acc, __ldcg(part + (int64_t)t * M + row));
  dscale[row] = acc;
}

// ---------------------------------------------------------------- wait check
// Exercises the bounded wait the fused kernels use on their copies: thread 0
// initialises an mbarrier that completes on one arrival, arrives on it only
// when `arrive` is set, and waits for it with mbar_wait_for(limit_ns).  A
// wait that gives up sets `code` in the device error word, as a fused kernel
// does.  out[0] = 1 if the wait saw the phase complete, 0 if it gave up;
// out[1] = the nanoseconds it waited.  Nothing else is touched.
__global__ void wait_probe_kernel(uint64_t limit_ns, int arrive, uint32_t* err, uint32_t code,
                                  uint64_t* out) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  mbar_init_fence();
  if (arrive)
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(&bar)) : "memory");
  const uint64_t t0 = global_ns();
  const bool done = mbar_wait_for(&bar, 0u, limit_ns);
  const uint64_t t1 = global_ns();
  if (!done) atomicOr(err, code);
  out[0] = done ? 1u : 0u;
  out[1] = t1 - t0;
}

}  // namespace moeact
