/*
 * moeact_oracle.c -- plain, slow, obviously-correct CPU oracle for the
 * per-row-scaled gated activation fused with MXFP8 quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or constant generator
 * with the CUDA library.
 *
 * What it follows (page titles, sections):
 *   - pytorch/ao PR #4743 "[mxfp8 training] Add a fused gated-activation
 *     (SwiGLU) + MXFP8 quantization kernel", sections "Summary" (gate/up read
 *     once, RCEIL MXFP8 cast, rowwise 1x32 / colwise 32x1 / both scales),
 *     "API" (gated input packs [gate | up]; backward returns [dGate | dUp])
 *     and the review reply on sigmoid / "dact = fma(silu, 1-s, s)".
 *   - TransformerEngine PR #3238 "Activation + GroupedLinear Fusion for MOE
 *     and other MOE optimizations", Greptile summary (per-row-scaled SReLU /
 *     SwiGLU, splits_to_offsets_multi) and its sequence diagram (grouped
 *     activation returns quantized grouped storage; grouped dactivation
 *     returns grouped_dy quantized, dense_dy and grad_scales).
 *   - TransformerEngine PR #2600 "[PyTorch] GroupedTensor integration",
 *     Key Changes (several tensors stored contiguously, addressed by offsets).
 *   - VeOmni PR #1340, "What does this PR do?" (SiLU rounded to the
 *     activation dtype before the multiply: staged rounding).
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes with its reason):
 *   sigma   : the correctly rounded fp32 value of 1/(1+exp(-g)) for the
 *             bf16 input g (computed in binary128 and certified).
 *   fp32    : every other step is one IEEE binary32 operation, in the order
 *             written, round-to-nearest-even, subnormals kept.
 *   y       : y = (silu(g) * u) * s_row  (scale applied after the product).
 *   staged  : a = bf16(silu), h = bf16(a * u), then y = h * s_row.
 *   E8M0    : b = 127 + e, e = smallest integer in [-127, 127] with
 *             amax <= 448 * 2^e (exact real comparison); +Inf -> e = 127;
 *             NaN amax -> b = 255.
 *   E4M3    : code = E4M3 nearest-even of y * 2^(127-b) (exact product),
 *             saturating to +-448, NaN -> 0x7F, sign of zero kept;
 *             a block with b = 255 has every code 0x7F.
 *   amax    : NaN-propagating max of |y| over the block.
 *   dscale  : sum over the row of dY * h (h unscaled, not staged), summed in
 *             binary64 and rounded once to fp32.
 *   backward MXFP8 quantizes the bf16-rounded gradient, width 2N.
 *   blocks  : rowwise blocks are 32 consecutive columns; colwise blocks are
 *             32 consecutive rows of one tensor (one expert); the last block
 *             of a tensor may be shorter (amax over its rows only).
 *
 * Parity pins for every function here are in tests/test_oracle_*.py.
 */
#define _GNU_SOURCE
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#include <quadmath.h>
#include <xmmintrin.h>
#include <pthread.h>

#define ORC_ROWWISE 1
#define ORC_COLWISE 2
#define ORC_SWIGLU 0
#define ORC_SRELU 1

/* ------------------------------------------------------------------ */
/* Floating-point environment: the oracle must keep subnormals.        */
/* ------------------------------------------------------------------ */
typedef struct { unsigned int csr; } orc_fpenv;
static orc_fpenv orc_enter(void) {
  orc_fpenv e; e.csr = _mm_getcsr();
  /* clear FTZ (bit 15) and DAZ (bit 6); round-to-nearest (bits 13-14 = 0) */
  _mm_setcsr(e.csr & ~((1u << 15) | (1u << 6) | (3u << 13)));
  return e;
}
static void orc_leave(orc_fpenv e) { _mm_setcsr(e.csr); }

/* ------------------------------------------------------------------ */
/* bf16                                                               */
/* ------------------------------------------------------------------ */
static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

float orc_bf16_to_f32(uint16_t b) { return f32_from_bits((uint32_t)b << 16); }

/* Value of a bf16 magnitude pattern (0..0x7F80) as a double, where the
 * pattern 0x7F80 is taken as 2^128: the next value above the largest finite
 * bf16 if the exponent range were unbounded (IEEE overflow rule). */
static double bf16_mag_value(uint32_t mag) {
  if (mag >= 0x7F80u) return ldexp(1.0, 128);
  return (double)f32_from_bits(mag << 16);
}

/* Round an fp32 value to the nearest bf16, ties to even (IEEE RNE).
 * NaN -> 0x7FC0 (quiet NaN); overflow -> +-Inf. */
uint16_t orc_f32_to_bf16(float f) {
  if (isnan(f)) return 0x7FC0;
  uint32_t u = bits_from_f32(f);
  uint32_t sign = u & 0x80000000u;
  uint32_t mag = u & 0x7FFFFFFFu;
  if (mag >= 0x7F800000u) return (uint16_t)((sign | 0x7F800000u) >> 16); /* Inf */
  uint32_t lo = mag >> 16;       /* truncation toward zero */
  uint32_t hi = lo + 1;          /* next bf16 magnitude away from zero */
  double a = (double)f32_from_bits(mag);
  double dlo = a - bf16_mag_value(lo);
  double dhi = bf16_mag_value(hi) - a;
  uint32_t pick;
  if (dlo < dhi) pick = lo;
  else if (dhi < dlo) pick = hi;
  else pick = (lo & 1u) ? hi : lo;  /* tie: even mantissa */
  return (uint16_t)((sign >> 16) | pick);
}

static float bf16_round(float f) { return orc_bf16_to_f32(orc_f32_to_bf16(f)); }

/* ------------------------------------------------------------------ */
/* E4M3 (OCP FP8: 1 sign, 4 exponent bits bias 7, 3 mantissa bits, no   */
/* infinities, S.1111.111 is NaN, largest finite 448).                  */
/* ------------------------------------------------------------------ */
double orc_e4m3_decode(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
  if (e == 0xF && m == 7) return NAN;
  double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

/* Nearest E4M3 value to x, ties to even, saturating to +-448 (also for
 * +-Inf), NaN -> 0x7F.  x is exact (a double). */
uint8_t orc_e4m3_encode(double x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs(x);
  if (a >= 448.0) return sign | 0x7E;
  double q; /* spacing of E4M3 values around a */
  if (a < ldexp(1.0, -6)) {
    q = ldexp(1.0, -9);            /* subnormals m * 2^-9 */
  } else {
    int ex; frexp(a, &ex);         /* a in [2^(ex-1), 2^ex) */
    q = ldexp(1.0, ex - 1 - 3);    /* 3 mantissa bits */
  }
  double k = nearbyint(a / q);     /* a/q exact (power-of-two scale); RNE */
  double v = k * q;                /* nearest representable, maybe 2^ex */
  if (v > 448.0) v = 448.0;        /* only reachable from a >= 464, handled */
  /* encode v exactly */
  if (v == 0.0) return sign;
  if (v < ldexp(1.0, -6)) return sign | (uint8_t)(v / ldexp(1.0, -9));
  int ex; double fr = frexp(v, &ex);  /* v = fr * 2^ex, fr in [0.5, 1) */
  int e = ex - 1 + 7;
  int m = (int)((fr * 2.0 - 1.0) * 8.0);
  return sign | (uint8_t)(e << 3) | (uint8_t)m;
}

/* ------------------------------------------------------------------ */
/* E8M0 shared scale, RCEIL                                           */
/* ------------------------------------------------------------------ */
/* thr[k] = 448 * 2^(k-127), k = 0..254: exact binary64 values. */
static double g_thr[255];
static pthread_once_t g_thr_once = PTHREAD_ONCE_INIT;
static void build_thr(void) { for (int k = 0; k < 255; ++k) g_thr[k] = ldexp(448.0, k - 127); }

int orc_e8m0_rceil(float amax) {
  pthread_once(&g_thr_once, build_thr);
  if (isnan(amax)) return 255;
  double a = fabs((double)amax);
  for (int k = 0; k < 255; ++k)   /* smallest e = k-127 with a <= 448*2^e */
    if (a <= g_thr[k]) return k;
  return 254; /* +Inf: e clamps at 127 */
}

/* Quantize n values (stride `stride` in `y`) as one MXFP8 block. */
static void quantize_block(const float* y, int64_t stride, int64_t n,
                           uint8_t* codes, int64_t cstride, uint8_t* scale) {
  float amax = 0.0f;
  for (int64_t k = 0; k < n; ++k) {
    float v = y[k * stride];
    if (isnan(v)) amax = v;
    else if (!isnan(amax) && fabsf(v) > amax) amax = fabsf(v);
  }
  int b = orc_e8m0_rceil(amax);
  *scale = (uint8_t)b;
  for (int64_t k = 0; k < n; ++k) {
    if (b == 255) { codes[k * cstride] = 0x7F; continue; }
    double v = (double)y[k * stride] * ldexp(1.0, 127 - b);
    codes[k * cstride] = orc_e4m3_encode(v);
  }
}

/* MXFP8 of a dense [M, W] fp32 matrix into the plain row-major layout:
 * row codes [M, W], row scales [M, W/32], col codes [M, W],
 * col scales [ceil(M/32), W]. */
static void mxfp8_quantize(const float* y, int64_t M, int64_t W, int dirs,
                           uint8_t* rq, uint8_t* rs, uint8_t* cq, uint8_t* cs) {
  if (dirs & ORC_ROWWISE)
    for (int64_t i = 0; i < M; ++i)
      for (int64_t jb = 0; jb < W / 32; ++jb)
        quantize_block(y + i * W + jb * 32, 1, 32,
                       rq + i * W + jb * 32, 1, rs + i * (W / 32) + jb);
  if (dirs & ORC_COLWISE)
    for (int64_t ib = 0; ib * 32 < M; ++ib) {
      int64_t n = (M - ib * 32 < 32) ? (M - ib * 32) : 32;
      for (int64_t j = 0; j < W; ++j)
        quantize_block(y + ib * 32 * W + j, W, n,
                       cq + ib * 32 * W + j, W, cs + ib * W + j);
    }
}

/* ------------------------------------------------------------------ */
/* sigma(g) for bf16 g, correctly rounded to fp32                      */
/* ------------------------------------------------------------------ */
static float g_sigma[65536];
static int g_sigma_bad = -1;   /* -1: not built; else number uncertified */
static pthread_once_t g_sigma_once = PTHREAD_ONCE_INIT;

/* 1/(1+exp(-g)) in binary128 (about 113 bits; expq is within a few ulps),
 * rounded once to fp32, and certified: the binary128 value must be farther
 * than 2^-100 (relative) from every fp32 rounding boundary. */
static float sigma_certified(float g, int* certified) {
  __float128 gq = (__float128)g;
  __float128 sq = 1.0Q / (1.0Q + expq(-gq));
  float f = (float)sq; /* one correct rounding from binary128 */
  float up = nextafterf(f, INFINITY), dn = nextafterf(f, -INFINITY);
  __float128 m_up = ((__float128)f + (__float128)up) / 2;
  __float128 m_dn = ((__float128)f + (__float128)dn) / 2;
  __float128 tol = fabsq(sq) * 0x1p-100Q;
  *certified = (fabsq(sq - m_up) > tol) && (fabsq(sq - m_dn) > tol);
  return f;
}

static void build_sigma(void) {
  orc_fpenv env = orc_enter();
  int bad = 0;
  for (uint32_t b = 0; b < 65536; ++b) {
    float g = orc_bf16_to_f32((uint16_t)b);
    if (isnan(g)) { g_sigma[b] = g; continue; }
    if (isinf(g)) { g_sigma[b] = g > 0 ? 1.0f : 0.0f; continue; }
    int ok;
    g_sigma[b] = sigma_certified(g, &ok);
    if (!ok) ++bad;
  }
  g_sigma_bad = bad;
  orc_leave(env);
}

/* Returns the number of bf16 inputs whose rounding could not be certified
 * (expected 0). */
int orc_sigma_init(void) { pthread_once(&g_sigma_once, build_sigma); return g_sigma_bad; }

float orc_sigmoid_bf16(uint16_t gbits) { orc_sigma_init(); return g_sigma[gbits]; }

/* ------------------------------------------------------------------ */
/* Activation values                                                   */
/* ------------------------------------------------------------------ */
/* SiLU pieces for one gate value (bf16 bits). */
static void silu_parts(uint16_t gb, float* g, float* sig, float* silu) {
  *g = orc_bf16_to_f32(gb);
  *sig = g_sigma[gb];
  *silu = *g * *sig;
}

static float relu_f(float v) { return (v > 0.0f || isnan(v)) ? v : 0.0f; }

/* y = act(x_row, j) * s, fp32, per the readings above. */
static float act_value(int act, const uint16_t* xrow, int64_t N, int64_t j, float s,
                       int staged) {
  if (act == ORC_SWIGLU) {
    float g, sig, silu;
    silu_parts(xrow[j], &g, &sig, &silu);
    float u = orc_bf16_to_f32(xrow[N + j]);
    float h;
    if (!staged) {
      h = silu * u;
    } else {
      float a = bf16_round(silu);
      h = bf16_round(a * u);
    }
    return h * s;
  } else {
    float r = relu_f(orc_bf16_to_f32(xrow[j]));
    float h = r * r;
    return h * s;
  }
}

/* ------------------------------------------------------------------ */
/* Forward                                                             */
/* ------------------------------------------------------------------ */
/* x: bf16 bits, [M, ldx] row-major; SwiGLU reads gate = x[:, 0:N],
 * up = x[:, N:2N]; SReLU reads x[:, 0:N].  s: fp32 [M].
 * Outputs (NULL for a disabled direction): row codes [M, N], row scales
 * [M, N/32], col codes [M, N], col scales [ceil(M/32), N]. */
int orc_act_fwd(int act, const uint16_t* x, int64_t ldx, const float* s,
                int64_t M, int64_t N, int dirs, int staged,
                uint8_t* rq, uint8_t* rs, uint8_t* cq, uint8_t* cs) {
  if (M < 0 || N <= 0 || N % 32 != 0) return 1;
  if (M == 0) return 0;
  orc_sigma_init();
  orc_fpenv env = orc_enter();
  float* y = (float*)malloc((size_t)(M * N) * sizeof(float));
  if (!y) { orc_leave(env); return 2; }
  for (int64_t i = 0; i < M; ++i)
    for (int64_t j = 0; j < N; ++j)
      y[i * N + j] = act_value(act, x + i * ldx, N, j, s[i], staged);
  mxfp8_quantize(y, M, N, dirs, rq, rs, cq, cs);
  free(y);
  orc_leave(env);
  return 0;
}

/* The fp32 activation itself, before quantization (for pins). */
int orc_act_values(int act, const uint16_t* x, int64_t ldx, const float* s,
                   int64_t M, int64_t N, int staged, float* y) {
  orc_sigma_init();
  orc_fpenv env = orc_enter();
  for (int64_t i = 0; i < M; ++i)
    for (int64_t j = 0; j < N; ++j)
      y[i * N + j] = act_value(act, x + i * ldx, N, j, s[i], staged);
  orc_leave(env);
  return 0;
}

/* Stand-alone MXFP8 quantizer of an fp32 [M, W] matrix (for pins). */
int orc_mxfp8_quantize(const float* y, int64_t M, int64_t W, int dirs,
                       uint8_t* rq, uint8_t* rs, uint8_t* cq, uint8_t* cs) {
  if (W <= 0 || W % 32 != 0 || M < 0) return 1;
  orc_fpenv env = orc_enter();
  mxfp8_quantize(y, M, W, dirs, rq, rs, cq, cs);
  orc_leave(env);
  return 0;
}

/* ------------------------------------------------------------------ */
/* Backward                                                            */
/* ------------------------------------------------------------------ */
/* dy: bf16 [M, lddy] (first N columns used); x as in the forward.
 * dx (nullable): bf16 [M, W] with W = 2N for SwiGLU ([dgate | dup]) and
 * W = N for SReLU.  dscale (nullable): fp32 [M].  MXFP8 of dx, width W. */
int orc_act_bwd(int act, const uint16_t* dy, int64_t lddy, const uint16_t* x,
                int64_t ldx, const float* s, int64_t M, int64_t N, int dirs,
                uint16_t* dx, float* dscale,
                uint8_t* rq, uint8_t* rs, uint8_t* cq, uint8_t* cs) {
  if (M < 0 || N <= 0 || N % 32 != 0) return 1;
  if (M == 0) return 0;
  orc_sigma_init();
  orc_fpenv env = orc_enter();
  int64_t W = (act == ORC_SWIGLU) ? 2 * N : N;
  float* d = (float*)malloc((size_t)(M * W) * sizeof(float));
  if (!d) { orc_leave(env); return 2; }
  for (int64_t i = 0; i < M; ++i) {
    const uint16_t* xr = x + i * ldx;
    double acc = 0.0;
    for (int64_t j = 0; j < N; ++j) {
      float gy = orc_bf16_to_f32(dy[i * lddy + j]);
      float p = gy * s[i];
      if (act == ORC_SWIGLU) {
        float g, sig, silu;
        silu_parts(xr[j], &g, &sig, &silu);
        float u = orc_bf16_to_f32(xr[N + j]);
        float one_m = 1.0f - sig;
        float dsilu = fmaf(silu, one_m, sig);     /* one rounding */
        float t = p * u;
        float dg = t * dsilu;
        float du = p * silu;
        d[i * W + j] = bf16_round(dg);
        d[i * W + N + j] = bf16_round(du);
        float h = silu * u;
        acc += (double)gy * (double)h;
      } else {
        float r = relu_f(orc_bf16_to_f32(xr[j]));
        float two_r = 2.0f * r;
        d[i * W + j] = bf16_round(p * two_r);
        float h = r * r;
        acc += (double)gy * (double)h;
      }
    }
    if (dscale) dscale[i] = (float)acc;
  }
  if (dx)
    for (int64_t k = 0; k < M * W; ++k) dx[k] = orc_f32_to_bf16(d[k]);
  mxfp8_quantize(d, M, W, dirs, rq, rs, cq, cs);
  free(d);
  orc_leave(env);
  return 0;
}

/* ------------------------------------------------------------------ */
/* Grouped: splits -> offsets, and per-expert tensors stored             */
/* contiguously.                                                       */
/* ------------------------------------------------------------------ */
/* row_offs[e] = sum of m_splits[0..e-1]; colblk_offs[e] = sum of
 * ceil(m_splits[k]/32) for k < e (the first col-scale row of expert e).
 * Returns the status: 0 ok, 1 a negative split, 2 splits that do not sum to
 * total_rows.  On a non-zero status nothing is written. */
int orc_splits_to_offsets(const int64_t* m_splits, int32_t E, int64_t total_rows,
                          int64_t* row_offs, int64_t* colblk_offs) {
  if (E < 0) return 1;
  for (int32_t e = 0; e < E; ++e) if (m_splits[e] < 0) return 1;
  int64_t sum = 0;
  for (int32_t e = 0; e < E; ++e) {
    if (m_splits[e] > total_rows - sum) return 2;
    sum += m_splits[e];
  }
  if (sum != total_rows) return 2;
  int64_t r = 0, c = 0;
  for (int32_t e = 0; e <= E; ++e) {
    if (row_offs) row_offs[e] = r;
    if (colblk_offs) colblk_offs[e] = c;
    if (e < E) { r += m_splits[e]; c += (m_splits[e] + 31) / 32; }
  }
  return 0;
}

/* Grouped forward: expert e is the tensor of rows [row_offs[e],
 * row_offs[e+1]); its codes start at row_offs[e]*N, its row scales at
 * row_offs[e]*N/32, its col scales at colblk_offs[e]*N. */
int orc_grouped_act_fwd(int act, const uint16_t* x, int64_t ldx, const float* s,
                        int64_t M, int64_t N, int dirs, int staged,
                        const int64_t* row_offs, const int64_t* colblk_offs, int32_t E,
                        uint8_t* rq, uint8_t* rs, uint8_t* cq, uint8_t* cs) {
  if (row_offs[E] != M) return 2;
  for (int32_t e = 0; e < E; ++e) {
    int64_t r0 = row_offs[e], me = row_offs[e + 1] - r0, c0 = colblk_offs[e];
    int rc = orc_act_fwd(act, x + r0 * ldx, ldx, s + r0, me, N, dirs, staged,
                         rq ? rq + r0 * N : NULL, rs ? rs + r0 * (N / 32) : NULL,
                         cq ? cq + r0 * N : NULL, cs ? cs + c0 * N : NULL);
    if (rc) return rc;
  }
  return 0;
}

int orc_grouped_act_bwd(int act, const uint16_t* dy, int64_t lddy, const uint16_t* x,
                        int64_t ldx, const float* s, int64_t M, int64_t N, int dirs,
                        const int64_t* row_offs, const int64_t* colblk_offs, int32_t E,
                        uint16_t* dx, float* dscale,
                        uint8_t* rq, uint8_t* rs, uint8_t* cq, uint8_t* cs) {
  if (row_offs[E] != M) return 2;
  int64_t W = (act == ORC_SWIGLU) ? 2 * N : N;
  for (int32_t e = 0; e < E; ++e) {
    int64_t r0 = row_offs[e], me = row_offs[e + 1] - r0, c0 = colblk_offs[e];
    int rc = orc_act_bwd(act, dy + r0 * lddy, lddy, x + r0 * ldx, ldx, s + r0, me, N, dirs,
                         dx ? dx + r0 * W : NULL, dscale ? dscale + r0 : NULL,
                         rq ? rq + r0 * W : NULL, rs ? rs + r0 * (W / 32) : NULL,
                         cq ? cq + r0 * W : NULL, cs ? cs + c0 * W : NULL);
    if (rc) return rc;
  }
  return 0;
}

/* ------------------------------------------------------------------ */
/* ClampedSwiGLU                                                       */
/* ------------------------------------------------------------------ */
/* The third per-row-scaled activation TransformerEngine PR #3238 names
 * (Greptile summary: SReLU / SwiGLU / ClampedSwiGLU); the pages give no
 * definition.  Reading taken (the clamped SwiGLU of the public gpt-oss
 * models, alpha and limit as parameters), in fp32 steps, x = [gate | up]:
 *   gc = min(g, L), uc = clamp(u, -L, L)   (NaN passes through)
 *   z = RN(alpha * gc);  sig = correctly rounded sigma(z)
 *   silu = RN(gc * sig);  v = RN(uc + 1);  h = RN(silu * v);  y = RN(h * s)
 * Backward (the SwiGLU form with the slope alpha; clamped inputs get a zero
 * gradient, as a clamp's gradient is):
 *   p = RN(dY * s)
 *   dsilu = g > L ? 0 : fma(RN(alpha * silu), RN(1 - sig), sig)
 *   dgate = g > L ? +0 : bf16(RN(RN(p * v) * dsilu))
 *   dup   = |u| > L ? +0 : bf16(RN(p * silu))
 *   dscale = sum_j dY * h (binary64, rounded once).
 * With alpha = 1 and L = +Inf it is SwiGLU with up + 1 in place of up. */
typedef struct { float g, u, gc, uc, z, sig, silu, v, h; } orc_clamped_parts;

static void clamped_parts(uint16_t gb, uint16_t ub, float alpha, float L,
                          orc_clamped_parts* c, int* certified) {
  c->g = orc_bf16_to_f32(gb);
  c->u = orc_bf16_to_f32(ub);
  c->gc = (c->g > L) ? L : c->g;
  c->uc = (c->u > L) ? L : ((c->u < -L) ? -L : c->u);
  c->z = alpha * c->gc;
  int ok = 1;
  if (isnan(c->z)) c->sig = c->z;
  else if (isinf(c->z)) c->sig = c->z > 0 ? 1.0f : 0.0f;
  else c->sig = sigma_certified(c->z, &ok);
  if (!ok) *certified = 0;
  c->silu = c->gc * c->sig;
  c->v = c->uc + 1.0f;
  c->h = c->silu * c->v;
}

/* sigma(RN(alpha * g)) for the bf16 gate g (no clamp), for the table pin;
 * *certified is cleared if the rounding could not be certified. */
float orc_clamped_sigmoid(float alpha, uint16_t gbits, int* certified) {
  orc_fpenv env = orc_enter();
  float z = alpha * orc_bf16_to_f32(gbits);
  float r;
  int ok = 1;
  if (isnan(z)) r = z;
  else if (isinf(z)) r = z > 0 ? 1.0f : 0.0f;
  else r = sigma_certified(z, &ok);
  if (!ok) *certified = 0;
  orc_leave(env);
  return r;
}

static int clamped_args_ok(float alpha, float L) {
  return alpha >= 0.8125f && alpha <= 2.0f && L > 0.0f;   /* L may be +Inf; NaN fails */
}

/* Forward: outputs as orc_act_fwd (width N).  Returns 1 on bad arguments,
 * 3 if a sigma rounding could not be certified. */
int orc_clamped_fwd(const uint16_t* x, int64_t ldx, const float* s, int64_t M, int64_t N,
                    int dirs, float alpha, float limit,
                    uint8_t* rq, uint8_t* rs, uint8_t* cq, uint8_t* cs) {
  if (M < 0 || N <= 0 || N % 32 != 0 || !clamped_args_ok(alpha, limit)) return 1;
  if (M == 0) return 0;
  orc_fpenv env = orc_enter();
  float* y = (float*)malloc((size_t)(M * N) * sizeof(float));
  if (!y) { orc_leave(env); return 2; }
  int cert = 1;
  for (int64_t i = 0; i < M; ++i)
    for (int64_t j = 0; j < N; ++j) {
      orc_clamped_parts c;
      clamped_parts(x[i * ldx + j], x[i * ldx + N + j], alpha, limit, &c, &cert);
      y[i * N + j] = c.h * s[i];
    }
  mxfp8_quantize(y, M, N, dirs, rq, rs, cq, cs);
  free(y);
  orc_leave(env);
  return cert ? 0 : 3;
}

/* The fp32 activation before quantization (for pins). */
int orc_clamped_values(const uint16_t* x, int64_t ldx, const float* s, int64_t M, int64_t N,
                       float alpha, float limit, float* y) {
  if (!clamped_args_ok(alpha, limit)) return 1;
  orc_fpenv env = orc_enter();
  int cert = 1;
  for (int64_t i = 0; i < M; ++i)
    for (int64_t j = 0; j < N; ++j) {
      orc_clamped_parts c;
      clamped_parts(x[i * ldx + j], x[i * ldx + N + j], alpha, limit, &c, &cert);
      y[i * N + j] = c.h * s[i];
    }
  orc_leave(env);
  return cert ? 0 : 3;
}

/* Backward: dx bf16 [M, 2N] = [dgate | dup], dscale fp32 [M], MXFP8 of dx. */
int orc_clamped_bwd(const uint16_t* dy, int64_t lddy, const uint16_t* x, int64_t ldx,
                    const float* s, int64_t M, int64_t N, int dirs, float alpha, float limit,
                    uint16_t* dx, float* dscale,
                    uint8_t* rq, uint8_t* rs, uint8_t* cq, uint8_t* cs) {
  if (M < 0 || N <= 0 || N % 32 != 0 || !clamped_args_ok(alpha, limit)) return 1;
  if (M == 0) return 0;
  orc_fpenv env = orc_enter();
  int64_t W = 2 * N;
  float* d = (float*)malloc((size_t)(M * W) * sizeof(float));
  if (!d) { orc_leave(env); return 2; }
  int cert = 1;
  for (int64_t i = 0; i < M; ++i) {
    double acc = 0.0;
    for (int64_t j = 0; j < N; ++j) {
      orc_clamped_parts c;
      clamped_parts(x[i * ldx + j], x[i * ldx + N + j], alpha, limit, &c, &cert);
      float gy = orc_bf16_to_f32(dy[i * lddy + j]);
      float p = gy * s[i];
      float dg = 0.0f, du = 0.0f;
      if (!(c.g > limit)) {
        float as = alpha * c.silu;
        float dsilu = fmaf(as, 1.0f - c.sig, c.sig);   /* one rounding */
        float t = p * c.v;
        dg = bf16_round(t * dsilu);
      }
      if (!(c.u > limit || c.u < -limit)) du = bf16_round(p * c.silu);
      d[i * W + j] = dg;
      d[i * W + N + j] = du;
      acc += (double)gy * (double)c.h;
    }
    if (dscale) dscale[i] = (float)acc;
  }
  if (dx)
    for (int64_t k = 0; k < M * W; ++k) dx[k] = orc_f32_to_bf16(d[k]);
  mxfp8_quantize(d, M, W, dirs, rq, rs, cq, cs);
  free(d);
  orc_leave(env);
  return cert ? 0 : 3;
}

int orc_grouped_clamped_fwd(const uint16_t* x, int64_t ldx, const float* s, int64_t M,
                            int64_t N, int dirs, float alpha, float limit,
                            const int64_t* row_offs, const int64_t* colblk_offs, int32_t E,
                            uint8_t* rq, uint8_t* rs, uint8_t* cq, uint8_t* cs) {
  if (row_offs[E] != M) return 2;
  for (int32_t e = 0; e < E; ++e) {
    int64_t r0 = row_offs[e], me = row_offs[e + 1] - r0, c0 = colblk_offs[e];
    int rc = orc_clamped_fwd(x + r0 * ldx, ldx, s + r0, me, N, dirs, alpha, limit,
                             rq ? rq + r0 * N : NULL, rs ? rs + r0 * (N / 32) : NULL,
                             cq ? cq + r0 * N : NULL, cs ? cs + c0 * N : NULL);
    if (rc) return rc;
  }
  return 0;
}

int orc_grouped_clamped_bwd(const uint16_t* dy, int64_t lddy, const uint16_t* x, int64_t ldx,
                            const float* s, int64_t M, int64_t N, int dirs, float alpha,
                            float limit, const int64_t* row_offs, const int64_t* colblk_offs,
                            int32_t E, uint16_t* dx, float* dscale,
                            uint8_t* rq, uint8_t* rs, uint8_t* cq, uint8_t* cs) {
  if (row_offs[E] != M) return 2;
  int64_t W = 2 * N;
  for (int32_t e = 0; e < E; ++e) {
    int64_t r0 = row_offs[e], me = row_offs[e + 1] - r0, c0 = colblk_offs[e];
    int rc = orc_clamped_bwd(dy + r0 * lddy, lddy, x + r0 * ldx, ldx, s + r0, me, N, dirs,
                             alpha, limit, dx ? dx + r0 * W : NULL,
                             dscale ? dscale + r0 : NULL, rq ? rq + r0 * W : NULL,
                             rs ? rs + r0 * (W / 32) : NULL, cq ? cq + r0 * W : NULL,
                             cs ? cs + c0 * W : NULL);
    if (rc) return rc;
  }
  return 0;
}

/* ------------------------------------------------------------------ */
/* GEMM-ready scale layout.                                            */
/* ------------------------------------------------------------------ */
/* The consumer of the quantized grouped tensors is a block-scaled grouped
 * GEMM (TransformerEngine PR #3238, sequence diagram: the activation feeds
 * quantized grouped storage to the next grouped linear).  The pages give no
 * layout for its scale factors; the reading taken is the one block-scaled
 * tensor-core GEMMs read: the E8M0 matrix S[R][C] (one byte per 32 elements
 * along the GEMM's K dimension) cut into tiles of 128 rows x 4 columns, 512
 * bytes each, tiles stored in row-major order of (row tile, column tile);
 * inside a tile, element (r, c) (r < 128, c < 4) is at byte
 * (r % 32) * 16 + (r / 32) * 4 + c.  Positions past R or C (when R or C is
 * not a whole number of tiles) are 0. */
void orc_scales_gemm_layout(const uint8_t* S, int64_t R, int64_t C, uint8_t* out) {
  int64_t rt = (R + 127) / 128, ct = (C + 3) / 4;
  memset(out, 0, (size_t)(rt * ct * 512));
  for (int64_t r = 0; r < R; ++r)
    for (int64_t c = 0; c < C; ++c) {
      int64_t tile = (r / 128) * ct + c / 4;
      int64_t rr = r % 128, cc = c % 4;
      out[tile * 512 + (rr % 32) * 16 + (rr / 32) * 4 + cc] = S[r * C + c];
    }
}

/* Colwise scales in the GEMM layout.  The colwise-quantized tensor of an
 * expert (m_e rows, W columns, 32x1 blocks) is read by the GEMM transposed:
 * W rows and K = m_e, so its scale matrix is the transpose of the expert's
 * [m_e/32][W] colwise scales, [W][m_e/32], laid out as above.  Experts
 * follow one another in expert order.  cs holds the row-major colwise
 * scales (expert e at rows colblk_offs[e] ..).  Returns 1 (nothing written)
 * unless every expert's row count and W are multiples of 128, the shapes
 * for which no tile needs padding. */
int orc_col_scales_gemm_layout(const uint8_t* cs, int64_t W, const int64_t* row_offs,
                               const int64_t* colblk_offs, int32_t E, uint8_t* out) {
  if (W % 128) return 1;
  for (int32_t e = 0; e < E; ++e)
    if ((row_offs[e + 1] - row_offs[e]) % 128) return 1;
  int64_t pos = 0;
  for (int32_t e = 0; e < E; ++e) {
    int64_t kb = (row_offs[e + 1] - row_offs[e]) / 32;   /* K blocks of expert e */
    uint8_t* t = (uint8_t*)malloc((size_t)(W * kb > 0 ? W * kb : 1));
    for (int64_t w = 0; w < W; ++w)
      for (int64_t j = 0; j < kb; ++j) t[w * kb + j] = cs[(colblk_offs[e] + j) * W + w];
    orc_scales_gemm_layout(t, W, kb, out + pos);
    pos += (W / 128) * (kb / 4) * 512;
    free(t);
  }
  return 0;
}
