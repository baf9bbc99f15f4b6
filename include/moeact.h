/*
 * moeact.h -- C ABI of libmoeact.so: per-row-scaled gated activation
 * (SwiGLU, SReLU) fused with MXFP8 quantization, forward and backward, dense
 * and grouped (MoE experts), for NVIDIA B200 (sm_100a).
 *
 * What the calls compute is defined by these pages (title, section):
 *   [AO]   pytorch/ao PR #4743 "[mxfp8 training] Add a fused gated-activation
 *          (SwiGLU) + MXFP8 quantization kernel" -- Summary (gate and up read
 *          once, the bf16 activation never materialised, RCEIL MXFP8 with
 *          rowwise 1x32, colwise 32x1 or both scales in one pass), API
 *          (gated input packs [gate | up]; backward returns [dGate | dUp];
 *          disabled directions produce nothing), review reply on the
 *          backward (dact = fma(silu, 1 - sigma, sigma)).
 *   [TE]   TransformerEngine PR #3238 "Activation + GroupedLinear Fusion for
 *          MOE and other MOE optimizations" -- Greptile summary (per-row-scaled
 *          SReLU / SwiGLU; splits_to_offsets_multi computes every offset array
 *          once, up front) and sequence diagram (grouped activation ->
 *          quantized grouped storage; grouped dactivation -> grouped_dy
 *          quantized, dense_dy, grad_scales).
 *   [GT]   TransformerEngine PR #2600 "[PyTorch] GroupedTensor integration" --
 *          Key Changes (several tensors stored contiguously, addressed by
 *          offsets).
 *   [VO]   VeOmni PR #1340 -- What does this PR do? (SiLU rounded to the
 *          activation dtype before the multiply; stride-aware; inputs are not
 *          mutated).
 *
 * Numerics (the same for every entry point; where the pages are silent the
 * reading is stated):
 *   sigma(g)  correctly rounded fp32 value of 1/(1+exp(-g)) for bf16 g.
 *   SwiGLU    y = RN(RN(RN(g*sigma) * u) * s_row)   (fp32, in this order);
 *             staged: y = RN(bf16(RN(bf16(RN(g*sigma)) * u)) * s_row)   [VO].
 *   SReLU     y = RN(RN(r*r) * s_row), r = relu(x) (NaN kept)            [TE].
 *   E8M0      per block, b = 127 + e, e the smallest integer in [-127, 127]
 *             with amax <= 448 * 2^e (RCEIL); amax = NaN-propagating max |y|;
 *             +Inf -> 254; NaN -> 255.
 *   E4M3      code = nearest-even E4M3 of y * 2^(127-b), saturating to
 *             +-448, sign of zero kept; a block with b = 255 has all codes
 *             0x7F.
 *   backward  p = RN(dY*s); dsilu = fma(g*sigma, RN(1-sigma), sigma);
 *             dgate = bf16(RN(RN(p*u)*dsilu)); dup = bf16(RN(p*silu));
 *             SReLU dx = bf16(RN(p*2r)); dscale_row = sum_j dY*h (h the
 *             unscaled activation, fp32 accumulation in a fixed order);
 *             the MXFP8 of the gradient quantizes the bf16 values.
 *
 * Layouts (all row-major, byte offsets from the given pointers):
 *   x        bf16 [M, ldx]; SwiGLU reads gate = x[:, 0:N], up = x[:, N:2N]
 *            (ldx >= 2N); SReLU reads x[:, 0:N] (ldx >= N).
 *   glu_interleave  (gated calls) G = 0: the [gate | up] halves above.
 *            G > 0: the 2N columns hold G gate columns, then the G up
 *            columns that pair with them, repeated N/G times: gate column j
 *            at (j / G) * 2G + j % G, its up column G further on [TE:
 *            Important Files Changed, swiglu.py row -- the GLU interleave
 *            reshaping now happens inside the scaled_swiglu / scaled_dswiglu
 *            kernels; the block order and granularity are a reading].  G
 *            must be 32, 64 or a multiple of 128 and divide N (G = N is the
 *            halves layout), else MOEACT_EINVAL.  The
 *            backward writes dx and the MXFP8 of [dgate | dup] in the same
 *            interleaved column order, with the 1x32 blocks taken along the
 *            stored columns (so each block is all dgate or all dup).
 *   dy       bf16 [M, lddy], first N columns (lddy >= N).
 *   s        fp32 [M] per-row scale (routing probability).
 *   W        width of the quantized tensor: N in the forward; 2N (SwiGLU,
 *            [dgate | dup]) or N (SReLU) in the backward.
 *   row codes  uint8 E4M3 [M, W];     row scales uint8 E8M0 [M, W/32].
 *   col codes  uint8 E4M3 [M, W] (same row-major layout as row codes);
 *   col scales uint8 E8M0 [S, W]; S = ceil(M/32) for dense calls; for grouped
 *            calls S = colblk_offs[E] = sum_e ceil(m_e/32) and the buffer must
 *            hold ceil(M/32) + E rows (rows >= S are not written).
 *   grouped  expert e owns rows [row_offs[e], row_offs[e+1]); its codes start
 *            at row row_offs[e], its row scales at row row_offs[e], its col
 *            scales at row colblk_offs[e]; colwise blocks never cross an
 *            expert boundary (the last block of an expert may be shorter;
 *            its amax covers the expert's rows only).
 *   dx       bf16 [M, W] (SwiGLU: [dgate | dup]).   dscale fp32 [M].
 *
 * Ownership and execution: the caller allocates every input, output and
 * workspace on the device; the library allocates nothing per call (it keeps
 * one 48 KiB sigmoid table per device, built at moeact_init or at the first
 * call on that device).  Calls are asynchronous on `stream` (a cudaStream_t
 * passed as void*, NULL = legacy default stream) and never synchronise the
 * host, except moeact_init.  Inputs are never written.  Outputs must not
 * overlap inputs or each other.
 *
 * Alignment: x, dy, dx, every code and scale array and the workspace must be
 * 16-byte aligned, ldx and lddy multiples of 8 elements; s and dscale
 * 4-byte aligned; offsets 8-byte aligned.  Violations return MOEACT_EALIGN
 * (there is no unaligned fallback).
 *
 * Errors: every call validates its arguments on the host and returns a status
 * without launching anything on failure; moeact_last_error() gives a
 * thread-local message.  Data errors only visible on the device (bad splits or
 * offsets) are written to the caller's int32 device status word, and the
 * kernels then do no work (their outputs are left untouched).
 */
#ifndef MOEACT_H
#define MOEACT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moeact_status {
  MOEACT_OK = 0,
  MOEACT_EINVAL = 1,        /* null required pointer, bad size, flag or stride */
  MOEACT_EALIGN = 2,        /* a pointer or stride breaks the alignment rules */
  MOEACT_EUNSUPPORTED = 3,  /* not an sm_100 device; first call inside capture */
  MOEACT_ERANGE = 4,        /* sizes beyond the supported index range */
  MOEACT_ECUDA = 5,         /* a CUDA runtime call or launch failed */
  MOEACT_EWORKSPACE = 6     /* dscale requested without a large enough workspace */
} moeact_status;

/* dirs bitmask: which MXFP8 outputs to produce. */
#define MOEACT_ROWWISE 1
#define MOEACT_COLWISE 2

/* Device status word values (grouped calls and splits_to_offsets). */
#define MOEACT_DEV_OK 0
#define MOEACT_DEV_NEGATIVE_SPLIT 1   /* a split < 0 */
#define MOEACT_DEV_SPLIT_SUM 2        /* splits do not sum to M */
#define MOEACT_DEV_BAD_OFFSETS 3      /* offsets not those of valid splits */
#define MOEACT_DEV_UNALIGNED_GROUPS 4 /* GEMM scale layout with a group whose rows
                                         are not a multiple of 128 */

/* Largest number of groups (experts) a grouped call accepts. */
#define MOEACT_MAX_GROUPS 2040
/* Largest M accepted (2^30 rows; TMA coordinates are 32-bit). */
#define MOEACT_MAX_ROWS (((int64_t)1) << 30)

/* Layouts of the E8M0 scale arrays (moeact_mx_out.scale_layout).
 * ROWMAJOR: row scales [M, W/32], col scales [S, W], row-major (see Layouts).
 * GEMM: the layout a block-scaled tensor-core GEMM reads its scale factors
 *   in (the pages name the consumer, a block-scaled grouped GEMM, but give no
 *   layout; this is the reading taken).  A scale matrix is cut into tiles of
 *   128 rows x 4 scale columns, 512 bytes each, stored in row-major order of
 *   (row tile, column tile); inside a tile, element (r, c) is at byte
 *   (r % 32) * 16 + (r / 32) * 4 + c.  Row scales: the [M, W/32] matrix
 *   (M * W / 32 bytes).  Col scales: each group's colwise data is read by
 *   the GEMM transposed (W rows, K = the group's rows), so its scales are the
 *   [W, m_e/32] matrix, tiled the same way, groups one after the other
 *   (group e from byte row_offs[e] / 32 * W; M * W / 32 bytes in all).
 *   Needs M, N and (grouped) every group's row count to be multiples of 128
 *   -- whole tiles, no padding -- else MOEACT_EINVAL on the host or
 *   MOEACT_DEV_UNALIGNED_GROUPS in the status word. */
#define MOEACT_SCALES_ROWMAJOR 0
#define MOEACT_SCALES_GEMM 1

/* MXFP8 outputs of one call; a disabled direction's two pointers must be NULL. */
typedef struct moeact_mx_out {
  uint8_t* row_codes;   /* [M, W]    E4M3, rowwise 1x32 blocks */
  uint8_t* row_scales;  /* [M, W/32] E8M0 (in `scale_layout`) */
  uint8_t* col_codes;   /* [M, W]    E4M3, colwise 32x1 blocks */
  uint8_t* col_scales;  /* [S, W]    E8M0 (in `scale_layout`) */
  int32_t scale_layout; /* MOEACT_SCALES_ROWMAJOR (0) or MOEACT_SCALES_GEMM */
  /* Optional device int32 (4-byte aligned), NULL for none: when it is
   * non-zero at the time the call's kernels run, the call writes nothing
   * (codes, scales, dX, dscale and the status word keep their contents), so
   * that a captured CUDA graph can skip the work on some replays without
   * changing any pointer [the device no-op flag of the pages' graph-safe
   * paths].  It is read on the device, in stream order. */
  const int32_t* noop_flag;
} moeact_mx_out;

/* Build the sigmoid table on the current device and set up its kernels.
 * Optional: the first call on a device does it, but that first call must not
 * be inside a stream capture.  Synchronises the current device once.
 * MOEACT_EUNSUPPORTED if the device is not sm_100, or if its dynamic shared
 * memory starts too high for the 16-bit table addressing of the SwiGLU
 * forward (not expected on sm_100). */
moeact_status moeact_init(void);

/* Static text of a status; thread-local detail of the last failure. */
const char* moeact_status_string(moeact_status status);
const char* moeact_last_error(void);

/* ---------------------------------------------------------------------
 * splits_to_offsets [TE: splits_to_offsets_multi, offsets computed once]
 *   m_splits     int64 [E] rows per group (device).
 *   row_offs     int64 [E+1] out: row_offs[e] = sum_{k<e} m_k (device).
 *   colblk_offs  int64 [E+1] out: sum_{k<e} ceil(m_k/32), the first
 *                col-scale row of group e (device).
 *   status       int32 out (device): MOEACT_DEV_OK, or NEGATIVE_SPLIT /
 *                SPLIT_SUM, in which case row_offs[0] (and colblk_offs[0])
 *                are set to -1 and nothing else is written: a grouped call
 *                given these offsets reports MOEACT_DEV_BAD_OFFSETS and
 *                writes nothing.
 * E = 0 is legal (offsets [0], M must be 0).  Element offsets of any array
 * are row_offs times its row length.
 * ------------------------------------------------------------------- */
moeact_status splits_to_offsets(const int64_t* m_splits, int32_t num_groups,
                                int64_t total_rows, int64_t* row_offs,
                                int64_t* colblk_offs, int32_t* status, void* stream);

/* ---------------------------------------------------------------------
 * Forward, dense [AO: gated_act_mxfp8_forward, plus TE's per-row scale].
 *   x [M, ldx] bf16, s [M] fp32, N % 32 == 0, dirs != 0; staged_rounding
 *   0/1 [VO]; glu_interleave as under Layouts (0: [gate | up]).  M == 0
 *   returns MOEACT_OK without launching.
 * ------------------------------------------------------------------- */
moeact_status scaled_swiglu_mxfp8_fwd(const void* x, int64_t ldx, const float* s,
                                      int64_t M, int64_t N, int dirs,
                                      int staged_rounding, int32_t glu_interleave,
                                      moeact_mx_out out, void* stream);
moeact_status scaled_srelu_mxfp8_fwd(const void* x, int64_t ldx, const float* s,
                                     int64_t M, int64_t N, int dirs,
                                     moeact_mx_out out, void* stream);

/* ---------------------------------------------------------------------
 * Forward, grouped [TE: _grouped_scaled_activation; GT layout].
 *   row_offs / colblk_offs int64 [E+1] (device), as splits_to_offsets
 *   writes them; status int32 (device) receives MOEACT_DEV_OK or
 *   MOEACT_DEV_BAD_OFFSETS (then nothing is written).  col_scales must hold
 *   ceil(M/32) + E rows.
 * ------------------------------------------------------------------- */
moeact_status grouped_scaled_swiglu_mxfp8_fwd(const void* x, int64_t ldx, const float* s,
                                              int64_t M, int64_t N, int dirs,
                                              int staged_rounding, int32_t glu_interleave,
                                              const int64_t* row_offs,
                                              const int64_t* colblk_offs,
                                              int32_t num_groups, int32_t* status,
                                              moeact_mx_out out, void* stream);
moeact_status grouped_scaled_srelu_mxfp8_fwd(const void* x, int64_t ldx, const float* s,
                                             int64_t M, int64_t N, int dirs,
                                             const int64_t* row_offs,
                                             const int64_t* colblk_offs,
                                             int32_t num_groups, int32_t* status,
                                             moeact_mx_out out, void* stream);

/* ---------------------------------------------------------------------
 * Backward [AO: gated_act_mxfp8_backward; TE: _grouped_scaled_dactivation
 * returning grouped_dy (MXFP8 of dX), dense_dy (bf16 dX) and grad_scales].
 *   dy [M, lddy] bf16; x, s as in the forward.
 *   dx     nullable, bf16 [M, W] (W = 2N SwiGLU, N SReLU).
 *   dscale nullable, fp32 [M].  Needs `workspace` of at least
 *          scaled_act_mxfp8_bwd_workspace_size(M, N, E) bytes (E = 1 for
 *          dense calls; the size does not depend on E): scratch for the
 *          per-tile partial sums (ceil(N/128) x M fp32), no initial content
 *          required.  dscale is then summed by a second kernel launched on
 *          the same stream.  Calls sharing one workspace must not overlap on
 *          the GPU.
 *   dirs   may be 0 (bf16 dx and/or dscale only); at least one output
 *          must be requested.
 * ------------------------------------------------------------------- */
size_t scaled_act_mxfp8_bwd_workspace_size(int64_t M, int64_t N, int32_t num_groups);

moeact_status scaled_swiglu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x,
                                      int64_t ldx, const float* s, int64_t M, int64_t N,
                                      int dirs, int32_t glu_interleave, void* dx, float* dscale,
                                      moeact_mx_out out, void* workspace,
                                      size_t workspace_bytes, void* stream);
moeact_status scaled_srelu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x,
                                     int64_t ldx, const float* s, int64_t M, int64_t N,
                                     int dirs, void* dx, float* dscale,
                                     moeact_mx_out out, void* workspace,
                                     size_t workspace_bytes, void* stream);
moeact_status grouped_scaled_swiglu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x,
                                              int64_t ldx, const float* s, int64_t M,
                                              int64_t N, int dirs, int32_t glu_interleave,
                                              const int64_t* row_offs,
                                              const int64_t* colblk_offs,
                                              int32_t num_groups, int32_t* status,
                                              void* dx, float* dscale, moeact_mx_out out,
                                              void* workspace, size_t workspace_bytes,
                                              void* stream);
moeact_status grouped_scaled_srelu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x,
                                             int64_t ldx, const float* s, int64_t M,
                                             int64_t N, int dirs,
                                             const int64_t* row_offs,
                                             const int64_t* colblk_offs,
                                             int32_t num_groups, int32_t* status,
                                             void* dx, float* dscale, moeact_mx_out out,
                                             void* workspace, size_t workspace_bytes,
                                             void* stream);

/* ---------------------------------------------------------------------
 * scaled_swiglu_mxfp8_bwd_noalloc -- the dense SwiGLU backward for callers
 * that cannot allocate device memory: for example code that runs where a
 * cudaMalloc (which may synchronise the device, at unbounded latency) is not
 * acceptable, or a framework that owns all device memory through its own
 * allocator and cannot pass this library a workspace.  The paper has no
 * counterpart; this is a convenience of this library.
 *   Arguments, outputs and results are those of scaled_swiglu_mxfp8_bwd
 *   with glu_interleave = 0 and without the workspace: the dscale partial sums go to a 16 MiB array built
 *   into the library (held by every GPU that loads it, until exit), so with
 *   dscale requested ceil(N/128) * M must not exceed 4194304 (else
 *   MOEACT_ERANGE, nothing launched; shapes are checked first, as for
 *   scaled_swiglu_mxfp8_bwd).  Allocates nothing.
 *   The array's device address is looked up (cudaGetSymbolAddress) with the
 *   rest of the per-device set-up, by moeact_init() or the first call of any
 *   entry point on the device; as for every entry point, that first call
 *   must not be inside a stream capture (MOEACT_EUNSUPPORTED).
 *   All calls share the array and it keeps the last call's contents; nothing
 *   in it needs to start at zero (every partial is written before it is
 *   read).  Calls that overlap on the GPU (other streams, other host threads)
 *   race on it and must be serialised by the caller.
 * ------------------------------------------------------------------- */
moeact_status scaled_swiglu_mxfp8_bwd_noalloc(const void* dy, int64_t lddy, const void* x,
                                              int64_t ldx, const float* s, int64_t M, int64_t N,
                                              int dirs, void* dx, float* dscale,
                                              moeact_mx_out out, void* stream);

/* ---------------------------------------------------------------------
 * ClampedSwiGLU [TE: the third per-row-scaled activation of the fused
 * grouped linear, Greptile summary; the pages name it without a definition,
 * so this is a reading: the clamped SwiGLU of the public gpt-oss models,
 * with the slope alpha and the limit L as arguments]:
 *   gc = min(g, L), uc = clamp(u, -L, L)   (NaN passes through)
 *   z = RN(alpha * gc); sig = correctly rounded fp32 sigma(z)
 *   y = RN(RN(RN(gc * sig) * RN(uc + 1)) * s_row)
 * Backward, the SwiGLU form with slope alpha; a clamped input gets a zero
 * gradient (+0):
 *   p = RN(dY * s); dsilu = fma(RN(alpha * RN(gc * sig)), RN(1 - sig), sig)
 *   dgate = g > L ? 0 : bf16(RN(RN(p * RN(uc + 1)) * dsilu))
 *   dup = |u| > L ? 0 : bf16(RN(p * RN(gc * sig)))
 *   dscale_row = sum_j dY * h (h = RN(RN(gc * sig) * RN(uc + 1))).
 * Layout, outputs, workspace and errors as for SwiGLU (x = [gate | up] or
 * interleaved by glu_interleave, W = 2N in the backward; no staged
 * rounding).  alpha must lie in
 * [0.8125, 2] and limit be > 0 (+Inf allowed), else MOEACT_EINVAL.  The
 * first call with a given (alpha, limit) on a device builds that pair's
 * sigmoid table, sigma(RN(alpha * min(g, limit))) for every bf16 gate g
 * (device memory, kept until exit; synchronises the device once; at most 32
 * distinct pairs per device, else MOEACT_ERANGE); it must not be inside a
 * stream capture (MOEACT_EUNSUPPORTED) -- call moeact_init_clamped(alpha,
 * limit) first.  With alpha = 1 and limit = +Inf it is SwiGLU with up + 1
 * for up.
 * ------------------------------------------------------------------- */
moeact_status moeact_init_clamped(float alpha, float limit);
moeact_status scaled_clamped_swiglu_mxfp8_fwd(const void* x, int64_t ldx, const float* s,
                                              int64_t M, int64_t N, int dirs, float alpha,
                                              float limit, int32_t glu_interleave,
                                              moeact_mx_out out, void* stream);
moeact_status grouped_scaled_clamped_swiglu_mxfp8_fwd(const void* x, int64_t ldx, const float* s,
                                                      int64_t M, int64_t N, int dirs,
                                                      float alpha, float limit,
                                                      int32_t glu_interleave,
                                                      const int64_t* row_offs,
                                                      const int64_t* colblk_offs,
                                                      int32_t num_groups, int32_t* status,
                                                      moeact_mx_out out, void* stream);
moeact_status scaled_clamped_swiglu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x,
                                              int64_t ldx, const float* s, int64_t M, int64_t N,
                                              int dirs, float alpha, float limit,
                                              int32_t glu_interleave, void* dx, float* dscale,
                                              moeact_mx_out out, void* workspace,
                                              size_t workspace_bytes, void* stream);
moeact_status grouped_scaled_clamped_swiglu_mxfp8_bwd(
    const void* dy, int64_t lddy, const void* x, int64_t ldx, const float* s, int64_t M,
    int64_t N, int dirs, float alpha, float limit, int32_t glu_interleave,
    const int64_t* row_offs, const int64_t* colblk_offs, int32_t num_groups, int32_t* status,
    void* dx, float* dscale, moeact_mx_out out, void* workspace, size_t workspace_bytes,
    void* stream);
/* Test hook: the table of sigma(RN(alpha * min(g, limit))) over all 65536
 * bf16 g, fp32 [65536] (as moeact_sigmoid_dump; limit = +Inf: the unclamped
 * sigma(RN(alpha * g))). */
moeact_status moeact_clamped_sigmoid_dump(float alpha, float limit, float* out, void* stream);

/* Reads and clears this device's error word: non-zero if a kernel gave up
 * waiting for its own input copies (bit 0 forward, bit 1 backward, bit 2 the
 * sigmoid table's copy) -- a defensive bound that ends the kernel instead of
 * letting it hang -- or found its shared-memory sigmoid table outside the
 * 16-bit address range its lookups use (bit 3); never expected in normal
 * operation.  Every wait gives up after one second of GPU time (the global
 * timer), and the kernel then waits (bounded again) for its copies in flight
 * and returns, its outputs incomplete.  Bit 4 is set only by
 * moeact_wait_selftest; bit 5 by the fused FC2 kernel
 * (grouped_scaled_swiglu_mxfp8_fc2).  Synchronous.  No counterpart on the pages. */
#define MOEACT_DEVERR_FWD_WAIT 0x1u
#define MOEACT_DEVERR_BWD_WAIT 0x2u
#define MOEACT_DEVERR_TABLE_WAIT 0x4u
#define MOEACT_DEVERR_TABLE_ADDR 0x8u
#define MOEACT_DEVERR_WAIT_SELFTEST 0x10u
#define MOEACT_DEVERR_FC2_WAIT 0x20u
moeact_status moeact_device_error(uint32_t* flags);

/* ---------------------------------------------------------------------
 * grouped_scaled_swiglu_mxfp8_fc2 -- the scaled SwiGLU + rowwise MXFP8 of
 * each expert's rows fused with that expert's FC2 GEMM on the tensor cores
 * [TE: the grouped scaled activation's quantized grouped tensor feeds the
 * grouped linear that follows it, ForwardScaledActivationGroupedLinear
 * (Greptile summary; sequence diagram)]:
 *   out[i, h] = sum_k A[i, k] * W_e[h, k]   for every row i of expert e,
 * where A is the rowwise MXFP8 (1 x 32 blocks along k) of y = SwiGLU(x) * s,
 * bit for bit what grouped_scaled_swiglu_mxfp8_fwd writes with dirs =
 * MOEACT_ROWWISE (staged rounding as there), and W_e is the expert's MXFP8
 * weight.  The products of the dequantized operands are summed in fp32 by
 * the tensor cores (tcgen05.mma, order not specified) and the sum is rounded
 * to bf16 (nearest even).  A itself is never written to memory.
 *   x, ldx, s, M, N, staged_rounding: as grouped_scaled_swiglu_mxfp8_fwd
 *     ([gate | up] halves only); N a multiple of 128 (else MOEACT_EINVAL),
 *     at most 768 (the quantized 128-row block stays in shared memory; else
 *     MOEACT_EUNSUPPORTED).
 *   row_offs [E + 1], num_groups = E, status: as the grouped forward
 *     (offsets from splits_to_offsets; every split size allowed: rows past
 *     an expert's end in its last 128-row block are neither read as its own
 *     nor written); offsets that are not those of valid splits set *status = 3
 *     and write nothing.
 *   w_codes: E4M3 codes of the weights, expert e's [H, N] matrix (row h =
 *     output column h, N k-values) in the tensor cores' K-major operand
 *     layout: tiles of 128 rows x 128 k (16 KiB), row blocks in order and,
 *     within a row block, k blocks in order; in a tile, row r's 128 bytes at
 *     offset 128 r, its 16-byte chunk c (k values 16c .. 16c + 15) at chunk
 *     position c ^ (r mod 8) (the 128-byte swizzle); experts one after
 *     another: E * H * N bytes, 16-byte aligned.  (A weight is tiled once;
 *     each tile then arrives in one contiguous bulk copy.)
 *   w_scales: E8M0 scales of the weight (1 x 32 blocks along k), per expert
 *     the [H, N/32] matrix in the GEMM-ready tiled layout of
 *     MOEACT_SCALES_GEMM (tiles of 128 rows x 4 scale columns, 512 bytes,
 *     in row-major tile order; element (r, c) of a tile at byte
 *     (r mod 32) * 16 + (r / 32) * 4 + c), experts one after another:
 *     E * H * N/32 bytes, 16-byte aligned.
 *   H: output width, a positive multiple of 128 (else MOEACT_EINVAL),
 *     E * H < 2^31 (else MOEACT_ERANGE).
 *   out: bf16 [M, ldo] (caller-owned, 16-byte aligned), ldo >= H (else
 *     MOEACT_EINVAL) and a multiple of 8 (else MOEACT_EALIGN); columns
 *     [0, H) of every row are written, the rest of each row is not touched.
 *   Null x, s, row_offs, status, w_codes, w_scales or out: MOEACT_EINVAL;
 *   row_offs not 8-byte, status or noop_flag not 4-byte, w_codes, w_scales or
 *   out not 16-byte aligned: MOEACT_EALIGN.  M == 0: MOEACT_OK, nothing
 *   launched.
 *   noop_flag: nullable device int32; non-zero at execution time makes the
 *     call write nothing (CUDA-graph replay, as moeact_mx_out.noop_flag).
 * Allocates nothing; asynchronous on `stream`.  Bounded waits report
 * MOEACT_DEVERR_FC2_WAIT through moeact_device_error.
 * ------------------------------------------------------------------- */
moeact_status grouped_scaled_swiglu_mxfp8_fc2(const void* x, int64_t ldx, const float* s,
                                              int64_t M, int64_t N, int staged_rounding,
                                              const int64_t* row_offs, int32_t num_groups,
                                              int32_t* status, const void* w_codes,
                                              const void* w_scales, int64_t H, void* out,
                                              int64_t ldo, const int32_t* noop_flag,
                                              void* stream);

/* ---------------------------------------------------------------------
 * moeact_wait_selftest -- checks the bounded wait of the fused kernels on the
 * GPU without any fault: one thread sets up an mbarrier that completes on
 * one arrival, arrives on it only when `arrive` is 1 (with 0 nothing ever
 * arrives), and waits for it through the same bounded-wait routine the fused
 * kernels use, with a limit of `limit_us` microseconds (1 .. 2000000, else
 * MOEACT_ERANGE) instead of their one second.  A wait that gives up sets
 * MOEACT_DEVERR_WAIT_SELFTEST in the device error word, as a fused kernel
 * sets its bit.  result: device memory, 2 x uint64, 8-byte aligned
 * (MOEACT_EALIGN): result[0] = 1 if the wait saw the barrier complete, 0 if
 * it gave up; result[1] = nanoseconds waited.  Asynchronous on `stream`.
 * No counterpart on the pages (failure detection of this library).
 * ------------------------------------------------------------------- */
moeact_status moeact_wait_selftest(int arrive, uint32_t limit_us, uint64_t* result,
                                   void* stream);

/* ---------------------------------------------------------------------
 * Test hook: sigma for every bf16 bit pattern (65536 fp32 values written to
 * `out`, device memory) exactly as the kernels compute it.  No counterpart on
 * the pages; it exposes the device table so it can be compared with an
 * independent CPU computation.
 * ------------------------------------------------------------------- */
moeact_status moeact_sigmoid_dump(float* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOEACT_H */
