// C ABI of libmoeact (declared in include/moeact.h): argument validation,
// per-device set-up and kernel dispatch.  Argument checks happen on the host
// before anything is launched; nothing here allocates device memory.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/moeact.h"
#include "kernels.cuh"

namespace moeact {
namespace {

thread_local char t_err[512] = "";

moeact_status fail(moeact_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_err, sizeof(t_err), fmt, ap);
  va_end(ap);
  return st;
}

moeact_status cuda_fail(cudaError_t e, const char* what) {
  return fail(MOEACT_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ------------------------------------------------------------ per device
constexpr int kMaxDevices = 64;
std::atomic<bool> g_ready[kMaxDevices];
int g_sms[kMaxDevices];
std::mutex g_mu;
__device__ int g_sigma_uncertain;

using KernelFn = void (*)(const Params);
struct Variant { KernelFn fn; int threads; };

template <int ACT, bool GROUPED>
void fwd_kernels(KernelFn* out, int& n) {
  out[n++] = act_fwd_kernel<ACT, kRow, false, GROUPED>;
  out[n++] = act_fwd_kernel<ACT, kCol, false, GROUPED>;
  out[n++] = act_fwd_kernel<ACT, kRow | kCol, false, GROUPED>;
  if (ACT == kSwiGLU) {
    out[n++] = act_fwd_kernel<ACT, kRow, true, GROUPED>;
    out[n++] = act_fwd_kernel<ACT, kCol, true, GROUPED>;
    out[n++] = act_fwd_kernel<ACT, kRow | kCol, true, GROUPED>;
  }
}

template <int ACT, bool GROUPED>
void bwd_kernels(KernelFn* out, int& n) {
  out[n++] = act_bwd_kernel<ACT, 0, GROUPED>;
  out[n++] = act_bwd_kernel<ACT, kRow, GROUPED>;
  out[n++] = act_bwd_kernel<ACT, kCol, GROUPED>;
  out[n++] = act_bwd_kernel<ACT, kRow | kCol, GROUPED>;
}

constexpr int kMaxSmem = kSigBytes + (MOEACT_MAX_GROUPS + 1 + 3) * 4;

moeact_status init_device(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_ready[dev].load()) return MOEACT_OK;
  cudaDeviceProp prop;
  cudaError_t e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
  if (prop.major != 10 || prop.minor != 0)
    return fail(MOEACT_EUNSUPPORTED, "device %d is sm_%d%d; libmoeact is built for sm_100a",
                dev, prop.major, prop.minor);
  g_sms[dev] = prop.multiProcessorCount;

  KernelFn ks[64];
  int n = 0;
  fwd_kernels<kSwiGLU, false>(ks, n);
  fwd_kernels<kSwiGLU, true>(ks, n);
  fwd_kernels<kSReLU, false>(ks, n);
  fwd_kernels<kSReLU, true>(ks, n);
  bwd_kernels<kSwiGLU, false>(ks, n);
  bwd_kernels<kSwiGLU, true>(ks, n);
  bwd_kernels<kSReLU, false>(ks, n);
  bwd_kernels<kSReLU, true>(ks, n);
  for (int i = 0; i < n; ++i) {
    e = cudaFuncSetAttribute(ks[i], cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  }

  cudaStream_t st;
  e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreate");
  const int zero = 0;
  int unc = -1;
  e = cudaMemcpyToSymbolAsync(g_sigma_uncertain, &zero, sizeof(int), 0,
                              cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) {
    int* d_unc = nullptr;
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d_unc), g_sigma_uncertain);
    if (e == cudaSuccess) {
      sigma_table_init<<<(kSigEntriesPadded + 255) / 256, 256, 0, st>>>(d_unc);
      e = cudaGetLastError();
    }
  }
  if (e == cudaSuccess)
    e = cudaMemcpyFromSymbolAsync(&unc, g_sigma_uncertain, sizeof(int), 0,
                                  cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  cudaStreamDestroy(st);
  if (e != cudaSuccess) return cuda_fail(e, "sigmoid table set-up");
  if (unc != 0)
    return fail(MOEACT_ECUDA, "sigmoid table: %d entries could not be certified", unc);
  g_ready[dev].store(true);
  return MOEACT_OK;
}

moeact_status ensure_ready(cudaStream_t st, int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MOEACT_EUNSUPPORTED, "device index %d", dev);
  *dev_out = dev;
  if (g_ready[dev].load()) return MOEACT_OK;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs != cudaStreamCaptureStatusNone)
    return fail(MOEACT_EUNSUPPORTED,
                "first call on device %d is inside a stream capture; call moeact_init() first",
                dev);
  return init_device(dev);
}

// ------------------------------------------------------------ validation
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

moeact_status check_mx(const moeact_mx_out& o, int dirs, bool allow_none) {
  if (dirs < 0 || dirs > 3 || (!allow_none && dirs == 0))
    return fail(MOEACT_EINVAL, "dirs must be a non-empty subset of ROWWISE|COLWISE (got %d)", dirs);
  const bool row = dirs & MOEACT_ROWWISE, col = dirs & MOEACT_COLWISE;
  if (row != (o.row_codes != nullptr) || row != (o.row_scales != nullptr))
    return fail(MOEACT_EINVAL, "row_codes/row_scales must be given exactly when ROWWISE is set");
  if (col != (o.col_codes != nullptr) || col != (o.col_scales != nullptr))
    return fail(MOEACT_EINVAL, "col_codes/col_scales must be given exactly when COLWISE is set");
  const void* ps[4] = {o.row_codes, o.row_scales, o.col_codes, o.col_scales};
  for (const void* p : ps)
    if (p && !aligned(p, 16)) return fail(MOEACT_EALIGN, "MXFP8 output pointers must be 16-byte aligned");
  return MOEACT_OK;
}

moeact_status check_shape(const void* x, int64_t ldx, const float* s, int64_t M, int64_t N,
                          int act) {
  if (!x || !s) return fail(MOEACT_EINVAL, "x and s are required");
  if (M < 0) return fail(MOEACT_EINVAL, "M must be >= 0 (got %lld)", (long long)M);
  if (N <= 0 || N % 32 != 0) return fail(MOEACT_EINVAL, "N must be a positive multiple of 32 (got %lld)", (long long)N);
  if (M > MOEACT_MAX_ROWS) return fail(MOEACT_ERANGE, "M above 2^36");
  if (N > (1 << 24)) return fail(MOEACT_ERANGE, "N above 2^24");
  const int64_t width = act == kSwiGLU ? 2 * N : N;
  if (ldx < width) return fail(MOEACT_EINVAL, "ldx (%lld) smaller than the input width %lld", (long long)ldx, (long long)width);
  if (ldx % 8 != 0) return fail(MOEACT_EALIGN, "ldx must be a multiple of 8 elements");
  if (ldx > (((int64_t)1) << 40) || M * ldx > (((int64_t)1) << 61)) return fail(MOEACT_ERANGE, "input extent too large");
  if (!aligned(x, 16)) return fail(MOEACT_EALIGN, "x must be 16-byte aligned");
  if (!aligned(s, 4)) return fail(MOEACT_EALIGN, "s must be 4-byte aligned");
  return MOEACT_OK;
}

moeact_status check_groups(const int64_t* ro, const int64_t* cb, int32_t E, int32_t* status) {
  if (!ro || !cb || !status) return fail(MOEACT_EINVAL, "row_offs, colblk_offs and status are required");
  if (E < 1 || E > MOEACT_MAX_GROUPS) return fail(MOEACT_EINVAL, "num_groups must be in [1, %d]", MOEACT_MAX_GROUPS);
  if (!aligned(ro, 8) || !aligned(cb, 8) || !aligned(status, 4)) return fail(MOEACT_EALIGN, "offsets must be 8-byte aligned, status 4-byte aligned");
  return MOEACT_OK;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct WsLayout { size_t tickets_off, part_off, total; };
WsLayout ws_layout(int64_t M, int64_t N, int32_t E) {
  const int64_t slabs = ceil_div(M, 32) + (E > 0 ? E : 1);
  const int64_t tiles = ceil_div(N, kTileCols);
  WsLayout w;
  w.tickets_off = 0;
  w.part_off = (size_t)ceil_div(slabs * 4, 256) * 256;
  w.total = w.part_off + (size_t)slabs * (size_t)tiles * 32 * 4;
  return w;
}

// ------------------------------------------------------------ launches
template <int ACT, int DIRS, bool STAGED, bool GROUPED>
Variant fwd_variant() { return {act_fwd_kernel<ACT, DIRS, STAGED, GROUPED>, fwd_threads(ACT, DIRS)}; }

template <int ACT, bool GROUPED>
Variant pick_fwd(int dirs, bool staged) {
  if (ACT == kSwiGLU && staged) {
    if (dirs == kRow) return fwd_variant<ACT, kRow, true, GROUPED>();
    if (dirs == kCol) return fwd_variant<ACT, kCol, true, GROUPED>();
    return fwd_variant<ACT, kRow | kCol, true, GROUPED>();
  }
  if (dirs == kRow) return fwd_variant<ACT, kRow, false, GROUPED>();
  if (dirs == kCol) return fwd_variant<ACT, kCol, false, GROUPED>();
  return fwd_variant<ACT, kRow | kCol, false, GROUPED>();
}

template <int ACT, int DIRS, bool GROUPED>
Variant bwd_variant() { return {act_bwd_kernel<ACT, DIRS, GROUPED>, bwd_threads(ACT, DIRS)}; }

template <int ACT, bool GROUPED>
Variant pick_bwd(int dirs) {
  if (dirs == 0) return bwd_variant<ACT, 0, GROUPED>();
  if (dirs == kRow) return bwd_variant<ACT, kRow, GROUPED>();
  if (dirs == kCol) return bwd_variant<ACT, kCol, GROUPED>();
  return bwd_variant<ACT, kRow | kCol, GROUPED>();
}

moeact_status launch(Variant v, const Params& p, int dev, int64_t slabs_upper, int act,
                     bool grouped, cudaStream_t st) {
  const int64_t items = slabs_upper * p.n_tiles;
  int64_t blocks = ceil_div(items, v.threads / 32);
  if (blocks > g_sms[dev]) blocks = g_sms[dev];
  if (blocks < 1) blocks = 1;
  size_t smem = (act == kSwiGLU ? kSigBytes : 0) + (grouped ? (size_t)(p.E + 1 + 3) / 4 * 16 : 0);
  v.fn<<<(unsigned)blocks, v.threads, smem, st>>>(p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return MOEACT_OK;
}

moeact_status fwd_common(int act, const void* x, int64_t ldx, const float* s, int64_t M,
                         int64_t N, int dirs, int staged, const int64_t* ro, const int64_t* cb,
                         int32_t E, int32_t* status, moeact_mx_out out, void* stream,
                         bool grouped) {
  t_err[0] = 0;
  moeact_status st = check_shape(x, ldx, s, M, N, act);
  if (st) return st;
  if ((st = check_mx(out, dirs, false))) return st;
  if (staged != 0 && staged != 1) return fail(MOEACT_EINVAL, "staged_rounding must be 0 or 1");
  if (grouped && (st = check_groups(ro, cb, E, status))) return st;
  if (M == 0) return MOEACT_OK;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int dev;
  if ((st = ensure_ready(cs, &dev))) return st;
  Params p{};
  p.x = static_cast<const uint16_t*>(x);
  p.ldx = ldx;
  p.s = s;
  p.M = M;
  p.N = (int)N;
  p.W = (int)N;
  p.rq = out.row_codes;
  p.rs = out.row_scales;
  p.cq = out.col_codes;
  p.cs = out.col_scales;
  p.row_offs = ro;
  p.cb_offs = cb;
  p.E = grouped ? E : 0;
  p.status = status;
  p.dense_slabs = ceil_div(M, 32);
  p.n_tiles = (int)ceil_div(N, kTileCols);
  const int64_t slabs_upper = grouped ? ceil_div(M, 32) + E : ceil_div(M, 32);
  Variant v;
  if (act == kSwiGLU) v = grouped ? pick_fwd<kSwiGLU, true>(dirs, staged) : pick_fwd<kSwiGLU, false>(dirs, staged);
  else v = grouped ? pick_fwd<kSReLU, true>(dirs, false) : pick_fwd<kSReLU, false>(dirs, false);
  return launch(v, p, dev, slabs_upper, act, grouped, cs);
}

moeact_status bwd_common(int act, const void* dy, int64_t lddy, const void* x, int64_t ldx,
                         const float* s, int64_t M, int64_t N, int dirs, const int64_t* ro,
                         const int64_t* cb, int32_t E, int32_t* status, void* dx,
                         float* dscale, moeact_mx_out out, void* ws, size_t ws_bytes,
                         void* stream, bool grouped) {
  t_err[0] = 0;
  moeact_status st = check_shape(x, ldx, s, M, N, act);
  if (st) return st;
  if ((st = check_mx(out, dirs, true))) return st;
  if (!dy) return fail(MOEACT_EINVAL, "dy is required");
  if (lddy < N) return fail(MOEACT_EINVAL, "lddy (%lld) smaller than N", (long long)lddy);
  if (lddy % 8 != 0) return fail(MOEACT_EALIGN, "lddy must be a multiple of 8 elements");
  if (lddy > (((int64_t)1) << 40) || M * lddy > (((int64_t)1) << 61)) return fail(MOEACT_ERANGE, "dy extent too large");
  if (!aligned(dy, 16)) return fail(MOEACT_EALIGN, "dy must be 16-byte aligned");
  if (dx && !aligned(dx, 16)) return fail(MOEACT_EALIGN, "dx must be 16-byte aligned");
  if (dscale && !aligned(dscale, 4)) return fail(MOEACT_EALIGN, "dscale must be 4-byte aligned");
  if (dirs == 0 && !dx && !dscale) return fail(MOEACT_EINVAL, "nothing requested: dirs == 0 and no dx / dscale");
  if (grouped && (st = check_groups(ro, cb, E, status))) return st;
  const WsLayout wl = ws_layout(M, N, grouped ? E : 1);
  if (dscale) {
    if (!ws) return fail(MOEACT_EWORKSPACE, "dscale needs a workspace");
    if (!aligned(ws, 16)) return fail(MOEACT_EALIGN, "workspace must be 16-byte aligned");
    if (ws_bytes < wl.total) return fail(MOEACT_EWORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, wl.total);
  }
  if (M == 0) return MOEACT_OK;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int dev;
  if ((st = ensure_ready(cs, &dev))) return st;
  Params p{};
  p.x = static_cast<const uint16_t*>(x);
  p.ldx = ldx;
  p.dy = static_cast<const uint16_t*>(dy);
  p.lddy = lddy;
  p.s = s;
  p.M = M;
  p.N = (int)N;
  p.W = (int)(act == kSwiGLU ? 2 * N : N);
  p.rq = out.row_codes;
  p.rs = out.row_scales;
  p.cq = out.col_codes;
  p.cs = out.col_scales;
  p.dx = static_cast<uint16_t*>(dx);
  p.dscale = dscale;
  if (dscale) {
    p.tickets = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + wl.tickets_off);
    p.part = reinterpret_cast<float*>(static_cast<char*>(ws) + wl.part_off);
  }
  p.row_offs = ro;
  p.cb_offs = cb;
  p.E = grouped ? E : 0;
  p.status = status;
  p.dense_slabs = ceil_div(M, 32);
  p.n_tiles = (int)ceil_div(N, kTileCols);
  const int64_t slabs_upper = grouped ? ceil_div(M, 32) + E : ceil_div(M, 32);
  Variant v;
  if (act == kSwiGLU) v = grouped ? pick_bwd<kSwiGLU, true>(dirs) : pick_bwd<kSwiGLU, false>(dirs);
  else v = grouped ? pick_bwd<kSReLU, true>(dirs) : pick_bwd<kSReLU, false>(dirs);
  return launch(v, p, dev, slabs_upper, act, grouped, cs);
}

}  // namespace
}  // namespace moeact

using namespace moeact;

extern "C" {

moeact_status moeact_init(void) {
  t_err[0] = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MOEACT_EUNSUPPORTED, "device index %d", dev);
  return init_device(dev);
}

const char* moeact_status_string(moeact_status s) {
  switch (s) {
    case MOEACT_OK: return "ok";
    case MOEACT_EINVAL: return "invalid argument";
    case MOEACT_EALIGN: return "misaligned pointer or stride";
    case MOEACT_EUNSUPPORTED: return "unsupported device or call context";
    case MOEACT_ERANGE: return "size out of range";
    case MOEACT_ECUDA: return "CUDA error";
    case MOEACT_EWORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

const char* moeact_last_error(void) { return t_err; }

moeact_status splits_to_offsets(const int64_t* m_splits, int32_t num_groups, int64_t total_rows,
                                int64_t* row_offs, int64_t* colblk_offs, int32_t* status,
                                void* stream) {
  t_err[0] = 0;
  if (!row_offs || !status || (num_groups > 0 && !m_splits))
    return fail(MOEACT_EINVAL, "m_splits, row_offs and status are required");
  if (num_groups < 0 || num_groups > MOEACT_MAX_GROUPS)
    return fail(MOEACT_EINVAL, "num_groups must be in [0, %d]", MOEACT_MAX_GROUPS);
  if (total_rows < 0) return fail(MOEACT_EINVAL, "total_rows must be >= 0");
  if (total_rows > MOEACT_MAX_ROWS) return fail(MOEACT_ERANGE, "total_rows above 2^36");
  if ((m_splits && !aligned(m_splits, 8)) || !aligned(row_offs, 8) ||
      (colblk_offs && !aligned(colblk_offs, 8)) || !aligned(status, 4))
    return fail(MOEACT_EALIGN, "offsets must be 8-byte aligned, status 4-byte aligned");
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int dev;
  moeact_status st = ensure_ready(cs, &dev);
  if (st) return st;
  splits_kernel<<<1, 1024, 0, cs>>>(m_splits, num_groups, total_rows, row_offs, colblk_offs, status);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "splits_to_offsets launch");
  return MOEACT_OK;
}

moeact_status scaled_swiglu_mxfp8_fwd(const void* x, int64_t ldx, const float* s, int64_t M,
                                      int64_t N, int dirs, int staged_rounding,
                                      moeact_mx_out out, void* stream) {
  return fwd_common(kSwiGLU, x, ldx, s, M, N, dirs, staged_rounding, nullptr, nullptr, 0,
                    nullptr, out, stream, false);
}

moeact_status scaled_srelu_mxfp8_fwd(const void* x, int64_t ldx, const float* s, int64_t M,
                                     int64_t N, int dirs, moeact_mx_out out, void* stream) {
  return fwd_common(kSReLU, x, ldx, s, M, N, dirs, 0, nullptr, nullptr, 0, nullptr, out, stream,
                    false);
}

moeact_status grouped_scaled_swiglu_mxfp8_fwd(const void* x, int64_t ldx, const float* s,
                                              int64_t M, int64_t N, int dirs,
                                              int staged_rounding, const int64_t* row_offs,
                                              const int64_t* colblk_offs, int32_t num_groups,
                                              int32_t* status, moeact_mx_out out,
                                              void* stream) {
  return fwd_common(kSwiGLU, x, ldx, s, M, N, dirs, staged_rounding, row_offs, colblk_offs,
                    num_groups, status, out, stream, true);
}

moeact_status grouped_scaled_srelu_mxfp8_fwd(const void* x, int64_t ldx, const float* s,
                                             int64_t M, int64_t N, int dirs,
                                             const int64_t* row_offs,
                                             const int64_t* colblk_offs, int32_t num_groups,
                                             int32_t* status, moeact_mx_out out, void* stream) {
  return fwd_common(kSReLU, x, ldx, s, M, N, dirs, 0, row_offs, colblk_offs, num_groups, status,
                    out, stream, true);
}

size_t scaled_act_mxfp8_bwd_workspace_size(int64_t M, int64_t N, int32_t num_groups) {
  if (M < 0 || N <= 0) return 0;
  return ws_layout(M, N, num_groups > 0 ? num_groups : 1).total;
}

moeact_status scaled_swiglu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x, int64_t ldx,
                                      const float* s, int64_t M, int64_t N, int dirs, void* dx,
                                      float* dscale, moeact_mx_out out, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  return bwd_common(kSwiGLU, dy, lddy, x, ldx, s, M, N, dirs, nullptr, nullptr, 0, nullptr, dx,
                    dscale, out, workspace, workspace_bytes, stream, false);
}

moeact_status scaled_srelu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x, int64_t ldx,
                                     const float* s, int64_t M, int64_t N, int dirs, void* dx,
                                     float* dscale, moeact_mx_out out, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  return bwd_common(kSReLU, dy, lddy, x, ldx, s, M, N, dirs, nullptr, nullptr, 0, nullptr, dx,
                    dscale, out, workspace, workspace_bytes, stream, false);
}

moeact_status grouped_scaled_swiglu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x,
                                              int64_t ldx, const float* s, int64_t M, int64_t N,
                                              int dirs, const int64_t* row_offs,
                                              const int64_t* colblk_offs, int32_t num_groups,
                                              int32_t* status, void* dx, float* dscale,
                                              moeact_mx_out out, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  return bwd_common(kSwiGLU, dy, lddy, x, ldx, s, M, N, dirs, row_offs, colblk_offs, num_groups,
                    status, dx, dscale, out, workspace, workspace_bytes, stream, true);
}

moeact_status grouped_scaled_srelu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x,
                                             int64_t ldx, const float* s, int64_t M, int64_t N,
                                             int dirs, const int64_t* row_offs,
                                             const int64_t* colblk_offs, int32_t num_groups,
                                             int32_t* status, void* dx, float* dscale,
                                             moeact_mx_out out, void* workspace,
                                             size_t workspace_bytes, void* stream) {
  return bwd_common(kSReLU, dy, lddy, x, ldx, s, M, N, dirs, row_offs, colblk_offs, num_groups,
                    status, dx, dscale, out, workspace, workspace_bytes, stream, true);
}

moeact_status moeact_sigmoid_dump(float* out, void* stream) {
  t_err[0] = 0;
  if (!out) return fail(MOEACT_EINVAL, "out is required");
  if (!aligned(out, 4)) return fail(MOEACT_EALIGN, "out must be 4-byte aligned");
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int dev;
  moeact_status st = ensure_ready(cs, &dev);
  if (st) return st;
  sigma_table_dump<<<256, 256, 0, cs>>>(out);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sigmoid dump launch");
  return MOEACT_OK;
}

}  // extern "C"
