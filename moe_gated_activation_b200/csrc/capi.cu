// C ABI of libmoeact (declared in include/moeact.h): argument validation,
// per-device set-up and kernel dispatch.  Argument checks happen on the host
// before anything is launched; nothing here allocates device memory.
#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "../../include/moeact.h"
#include "fc2.cuh"
#include "host_kernels.cuh"
#include "variants.cuh"

namespace moeact {
static_assert(kErrFwdWait == MOEACT_DEVERR_FWD_WAIT && kErrBwdWait == MOEACT_DEVERR_BWD_WAIT &&
                  kErrTableWait == MOEACT_DEVERR_TABLE_WAIT &&
                  kErrTableAddr == MOEACT_DEVERR_TABLE_ADDR,
              "device error bits differ from include/moeact.h");
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
__device__ uint32_t g_smem_base;

// The fused kernels of each activation (index kSwiGLU / kSReLU / kClamped),
// filled once.
FwdVariant g_fwd[3][kFwdSlots];
BwdVariant g_bwd[3][kBwdSlots];
bool g_tables_filled = false;

// Extra shared memory of a grouped call (its col-block offsets), at most.
constexpr int kGroupSmem = group_bytes(MOEACT_MAX_GROUPS);

__device__ uint32_t g_err_word;
uint32_t* g_err_ptr[kMaxDevices];
float* g_sig_ptr[kMaxDevices];   // g_sigma_table on each device
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Scratch of the allocation-free backward (scaled_swiglu_mxfp8_bwd_noalloc).
// Some callers cannot hand the library a workspace: code that runs where a
// device allocation is not acceptable at the point of the call (cudaMalloc
// may synchronise the device and its latency is unbounded), or a host
// framework that owns all device memory through its own allocator and offers
// the kernel layer no way to request scratch.  For them the dscale partial
// sums live in a fixed array compiled into this library (every GPU that loads
// the library holds it until the process exits).  In host code the array's
// name is only a host-side stand-in, so its device address is taken once per
// device, with that device current, by cudaGetSymbolAddress in init_device.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[kMaxDevices];

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
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
      return fail(MOEACT_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }

  if (!g_tables_filled) {
    fill_fwd_swiglu_dense(g_fwd[kSwiGLU]);
    fill_fwd_swiglu_grouped(g_fwd[kSwiGLU]);
    fill_fwd_swiglu_ilv_dense(g_fwd[kSwiGLU]);
    fill_fwd_swiglu_ilv_grouped(g_fwd[kSwiGLU]);
    fill_bwd_swiglu_dense(g_bwd[kSwiGLU]);
    fill_bwd_swiglu_grouped(g_bwd[kSwiGLU]);
    fill_fwd_srelu_dense(g_fwd[kSReLU]);
    fill_fwd_srelu_grouped(g_fwd[kSReLU]);
    fill_bwd_srelu_dense(g_bwd[kSReLU]);
    fill_bwd_srelu_grouped(g_bwd[kSReLU]);
    fill_fwd_clamped_dense(g_fwd[kClamped]);
    fill_fwd_clamped_grouped(g_fwd[kClamped]);
    fill_fwd_clamped_ilv_dense(g_fwd[kClamped]);
    fill_fwd_clamped_ilv_grouped(g_fwd[kClamped]);
    fill_bwd_clamped_dense(g_bwd[kClamped]);
    fill_bwd_clamped_grouped(g_bwd[kClamped]);
    g_tables_filled = true;
  }
  for (auto& tab : g_fwd)
    for (const FwdVariant& v : tab) {
      if (!v.fn) continue;
      e = cudaFuncSetAttribute(v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               v.smem_fixed + (v.sig ? 0 : kGroupSmem));
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    }
  for (auto& tab : g_bwd)
    for (const BwdVariant& v : tab) {
      if (!v.fn) continue;
      e = cudaFuncSetAttribute(v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               v.smem_fixed + (v.sig ? 0 : kGroupSmem));
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    }
  e = cudaFuncSetAttribute(sigma_table_dump, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSigBytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  e = fc2_prepare();
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (fused FC2)");
  e = cudaGetSymbolAddress(reinterpret_cast<void**>(&g_err_ptr[dev]), g_err_word);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
  e = cudaGetSymbolAddress(reinterpret_cast<void**>(&g_sig_ptr[dev]), g_sigma_table);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
  e = cudaGetSymbolAddress(&g_noalloc_ptr[dev], g_noalloc_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the built-in scratch");

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
      sigma_table_init<<<(kSigEntriesPadded + 255) / 256, 256, 0, st>>>(
          g_sig_ptr[dev], 1.0f, INFINITY, 1.0f, d_unc);
      e = cudaGetLastError();
    }
  }
  if (e == cudaSuccess)
    e = cudaMemcpyFromSymbolAsync(&unc, g_sigma_uncertain, sizeof(int), 0,
                                  cudaMemcpyDeviceToHost, st);
  uint32_t smem_base = 0xFFFFFFFFu;
  if (e == cudaSuccess) {
    uint32_t* d_base = nullptr;
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d_base), g_smem_base);
    if (e == cudaSuccess) {
      smem_base_probe<<<1, 32, 1024, st>>>(d_base);
      e = cudaGetLastError();
    }
    if (e == cudaSuccess)
      e = cudaMemcpyFromSymbolAsync(&smem_base, g_smem_base, sizeof(uint32_t), 0,
                                    cudaMemcpyDeviceToHost, st);
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  cudaStreamDestroy(st);
  if (e != cudaSuccess) return cuda_fail(e, "sigmoid table set-up");
  if (unc != 0)
    return fail(MOEACT_ECUDA, "sigmoid table: %d entries could not be certified", unc);
  // the forward's table sits at the (128-byte aligned) start of dynamic
  // shared memory and is looked up by 16-bit addresses
  if (smem_base + 127u + (uint32_t)kSigBytes > 0x10000u)
    return fail(MOEACT_EUNSUPPORTED, "dynamic shared memory starts at %u: above the 16-bit "
                "range the sigmoid lookups use", smem_base);
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
  if (o.noop_flag && !aligned(o.noop_flag, 4)) return fail(MOEACT_EALIGN, "noop_flag must be 4-byte aligned");
  return MOEACT_OK;
}

// The GEMM-ready scale layout is defined for whole 128 x 128 tiles only.
moeact_status check_layout(const moeact_mx_out& o, int64_t M, int64_t N) {
  if (o.scale_layout != MOEACT_SCALES_ROWMAJOR && o.scale_layout != MOEACT_SCALES_GEMM)
    return fail(MOEACT_EINVAL, "scale_layout must be MOEACT_SCALES_ROWMAJOR or MOEACT_SCALES_GEMM");
  if (o.scale_layout == MOEACT_SCALES_GEMM && (M % 128 != 0 || N % 128 != 0))
    return fail(MOEACT_EINVAL, "the GEMM scale layout needs M and N to be multiples of 128 "
                "(got M=%lld, N=%lld)", (long long)M, (long long)N);
  return MOEACT_OK;
}

moeact_status check_shape(const void* x, int64_t ldx, const float* s, int64_t M, int64_t N,
                          int act) {
  if (!x || !s) return fail(MOEACT_EINVAL, "x and s are required");
  if (M < 0) return fail(MOEACT_EINVAL, "M must be >= 0 (got %lld)", (long long)M);
  if (N <= 0 || N % 32 != 0) return fail(MOEACT_EINVAL, "N must be a positive multiple of 32 (got %lld)", (long long)N);
  if (M > MOEACT_MAX_ROWS) return fail(MOEACT_ERANGE, "M above 2^30");
  if (N > (1 << 24)) return fail(MOEACT_ERANGE, "N above 2^24");
  const int64_t width = act != kSReLU ? 2 * N : N;
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

// Backward workspace: the dscale partials, one fp32 per (128-column tile
// (kTileCols), row).
size_t ws_bytes_needed(int64_t M, int64_t N) {
  return (size_t)ceil_div(N, kTileCols) * (size_t)M * 4;
}

// ------------------------------------------------------------ launches
// Tensor map of a bf16 [rows, width] matrix with a row stride of `ld`
// elements, read in boxes of 128 columns x 16 rows; out-of-range elements read
// as zero.  Encoded on the host for every call (no allocation).
moeact_status make_map(CUtensorMap* map, const void* base, int64_t width, int64_t rows,
                       int64_t ld, int box_rows = kHalfRows) {
  const cuuint64_t dims[2] = {(cuuint64_t)width, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  const cuuint32_t box[2] = {(cuuint32_t)kTileCols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOEACT_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MOEACT_OK;
}

// Tensor map of a SwiGLU input [rows, 2N] (gate | up, row stride `ld`) as a
// [rows][2][N] view, read in boxes of 128 columns x 1 half x 16 rows: columns
// past N read as zero in the gate half as well as in the up half, so a ragged
// last column tile never sees the up values through its gate box (used by the
// backward, whose dscale sums across the lanes of a tile).
moeact_status make_map_gated(CUtensorMap* map, const void* base, int64_t N, int64_t rows,
                             int64_t ld) {
  const cuuint64_t dims[3] = {(cuuint64_t)N, 2, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)(N * 2), (cuuint64_t)(ld * 2)};
  const cuuint32_t box[3] = {(cuuint32_t)kTileCols, 1, (cuuint32_t)kHalfRows};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOEACT_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MOEACT_OK;
}

// Tensor map of a gated input whose gate and up columns alternate in blocks
// of G (G gate columns, then their G up columns, repeated) as a
// [rows][N/G][2][G] view.  Its box gathers 128 columns of one kind (gate or
// up) x 16 rows: {128, 1, 1, 16} when G is a multiple of 128, {G, 1, 128/G,
// 16} when G is 32 or 64, so the half-tile lands in shared memory as the
// same dense [16][128] block as with [gate | up] halves.
moeact_status make_map_ilv(CUtensorMap* map, const void* base, int64_t N, int64_t G,
                           int64_t rows, int64_t ld) {
  const cuuint64_t dims[4] = {(cuuint64_t)G, 2, (cuuint64_t)(N / G), (cuuint64_t)rows};
  const cuuint64_t strides[3] = {(cuuint64_t)(G * 2), (cuuint64_t)(G * 4), (cuuint64_t)(ld * 2)};
  const cuuint32_t box[4] = {(cuuint32_t)std::min<int64_t>(G, kTileCols), 1,
                             (cuuint32_t)std::max<int64_t>(1, kTileCols / G),
                             (cuuint32_t)kHalfRows};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOEACT_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MOEACT_OK;
}

// The backward's map of x: SReLU [rows][N]; gated [rows][2][N] or, with an
// interleave G, [rows][N/G][2][G].
moeact_status make_x_map(CUtensorMap* map, int act, const void* x, int64_t N, int ilv,
                         int64_t rows, int64_t ld) {
  if (act == kSReLU) return make_map(map, x, N, rows, ld);
  return ilv ? make_map_ilv(map, x, N, ilv, rows, ld) : make_map_gated(map, x, N, rows, ld);
}

int64_t grid_for(int64_t slabs_upper, int n_tiles, int threads, int dev) {
  const int64_t items = slabs_upper * n_tiles;
  int64_t blocks = ceil_div(items, threads / 32);
  if (blocks > g_sms[dev]) blocks = g_sms[dev];
  return blocks < 1 ? 1 : blocks;
}

int group_smem(bool sig, bool grouped, int E) { return (grouped && !sig) ? group_bytes(E) : 0; }

// ------------------------------------------------------------ ClampedSwiGLU
// The slope alpha of ClampedSwiGLU is folded into its sigmoid table (one table
// per alpha and device, built at the first call with that alpha, which
// synchronises the device once), so alpha must keep the table's bf16 range
// sufficient: for |g| < 2^-25, sigma(RN(alpha g)) rounds to 1/2 when alpha <=
// 2, and for |g| >= 128 it is 0 or 1 when alpha >= 13/16.
constexpr float kClampAlphaMin = 0.8125f, kClampAlphaMax = 2.0f;
constexpr int kMaxAlphaTables = 32;
struct AlphaTable {
  uint32_t alpha_bits;
  uint32_t limit_bits;
  float* tab;
};
AlphaTable g_alpha_tab[kMaxDevices][kMaxAlphaTables];
int g_n_alpha[kMaxDevices];

moeact_status check_clamp_args(float alpha, float limit) {
  if (!(alpha >= kClampAlphaMin && alpha <= kClampAlphaMax))
    return fail(MOEACT_EINVAL, "alpha must lie in [0.8125, 2] (got %g)", (double)alpha);
  if (!(limit > 0.0f)) return fail(MOEACT_EINVAL, "limit must be > 0 (got %g)", (double)limit);
  return MOEACT_OK;
}

bool sigmoid_f32_host(float z, float* out);

// The device table of a ClampedSwiGLU call, built on first use: sigma(RN(alpha
// * g)) for every bf16 gate g <= limit and sigma(RN(alpha * limit)) for every
// gate above it (limit = +Inf: the unclamped table), so that the kernels take
// a clamped gate's sigmoid from the table like any other.
moeact_status alpha_table(int dev, float alpha, float limit, cudaStream_t call_stream,
                          const float** out) {
  uint32_t bits, lbits;
  std::memcpy(&bits, &alpha, 4);
  std::memcpy(&lbits, &limit, 4);
  std::lock_guard<std::mutex> lk(g_mu);
  for (int i = 0; i < g_n_alpha[dev]; ++i)
    if (g_alpha_tab[dev][i].alpha_bits == bits && g_alpha_tab[dev][i].limit_bits == lbits) {
      *out = g_alpha_tab[dev][i].tab;
      return MOEACT_OK;
    }
  if (g_n_alpha[dev] == kMaxAlphaTables)
    return fail(MOEACT_ERANGE, "more than %d distinct (alpha, limit) pairs on one device",
                kMaxAlphaTables);
  float sig_limit = 1.0f;   // sigma(RN(alpha * limit)), fp32
  if (!sigmoid_f32_host(alpha * limit, &sig_limit))
    return fail(MOEACT_EUNSUPPORTED, "sigma(alpha * limit) could not be certified");
  cudaStreamCaptureStatus capt = cudaStreamCaptureStatusNone;
  if (call_stream && cudaStreamIsCapturing(call_stream, &capt) == cudaSuccess &&
      capt != cudaStreamCaptureStatusNone)
    return fail(MOEACT_EUNSUPPORTED,
                "first use of alpha %g, limit %g inside a stream capture; call "
                "moeact_init_clamped() first",
                (double)alpha, (double)limit);
  float* tab = nullptr;
  int* d_unc = nullptr;
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(&tab), kSigBytes);
  if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void**>(&d_unc), sizeof(int));
  cudaStream_t st = nullptr;
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
  int unc = -1;
  if (e == cudaSuccess) e = cudaMemsetAsync(tab, 0, kSigBytes, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(d_unc, 0, sizeof(int), st);
  if (e == cudaSuccess) {
    sigma_table_init<<<(kSigEntriesPadded + 255) / 256, 256, 0, st>>>(tab, alpha, limit,
                                                                        sig_limit, d_unc);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaMemcpyAsync(&unc, d_unc, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (st) cudaStreamDestroy(st);
  if (d_unc) cudaFree(d_unc);
  if (e != cudaSuccess || unc != 0) {
    if (tab) cudaFree(tab);
    if (e != cudaSuccess) return cuda_fail(e, "ClampedSwiGLU sigmoid table set-up");
    return fail(MOEACT_ECUDA, "sigmoid table for alpha %g: %d entries could not be certified",
                (double)alpha, unc);
  }
  g_alpha_tab[dev][g_n_alpha[dev]++] = {bits, lbits, tab};
  *out = tab;
  return MOEACT_OK;
}

// sigma(z) correctly rounded to fp32, for the sigmoid of a clamped gate: an
// x87 extended evaluation (64-bit significand, error a few units of 2^-64)
// rounded once, refused when it lies within 2^-56 (relative) of an fp32
// rounding boundary (not expected to happen).
bool sigmoid_f32_host(float z, float* out) {
  if (std::isinf(z)) {
    *out = z > 0 ? 1.0f : 0.0f;
    return true;
  }
  const long double sl = 1.0L / (1.0L + expl(-(long double)z));
  const float f = (float)sl;
  const long double up = 0.5L * ((long double)f + (long double)nextafterf(f, INFINITY));
  const long double dn = 0.5L * ((long double)f + (long double)nextafterf(f, -INFINITY));
  const long double tol = fabsl(sl) * 0x1p-56L;
  *out = f;
  return fabsl(sl - up) > tol && fabsl(sl - dn) > tol;
}

// What a fused call computes: the activation and its parameters.
struct ActArgs {
  int act;
  int staged;        // SwiGLU only
  float alpha;       // ClampedSwiGLU only
  float limit;       // ClampedSwiGLU only
  int32_t ilv;       // gated: interleave block of gate / up columns (0: halves)
};

ActArgs plain(int act, int staged = 0, int32_t ilv = 0) {
  return {act, staged, 1.0f, INFINITY, ilv};
}

// The interleave of a gated input: 0 ([gate | up] halves), or G columns of
// gate then G of up, with G = 32, 64 or a multiple of 128 dividing N (G = N
// is the halves layout).  On success *norm is 0 for halves, else G.
moeact_status check_ilv(int act, int64_t N, int32_t G, int32_t* norm) {
  *norm = 0;
  if (G == 0) return MOEACT_OK;
  if (act == kSReLU) return fail(MOEACT_EINVAL, "glu_interleave applies to gated activations only");
  if (G < 0 || G % 32 != 0 || N % G != 0)
    return fail(MOEACT_EINVAL, "glu_interleave (%d) must be a positive multiple of 32 dividing N",
                (int)G);
  if (G == N) return MOEACT_OK;
  if (G != 32 && G != 64 && G % kTileCols != 0)
    return fail(MOEACT_EINVAL, "glu_interleave (%d) must be 32, 64 or a multiple of 128",
                (int)G);
  *norm = G;
  return MOEACT_OK;
}

// Fills the activation-dependent parameters (the sigmoid table to stage and
// the clamp constants).
moeact_status act_params(const ActArgs& a, int dev, cudaStream_t cs, Params& p) {
  p.sig_src = g_sig_ptr[dev];
  p.clamp_L = a.limit;
  p.clamp_alpha = a.alpha;
  // the largest bf16 not above L (L > 0: its fp32 bits truncated), both halves
  uint32_t lb;
  std::memcpy(&lb, &a.limit, 4);
  lb >>= 16;
  p.clamp_Lb2 = lb | (lb << 16);
  {
    uint32_t lbits;
    std::memcpy(&lbits, &a.limit, 4);
    p.clamp_bf16 = (lbits & 0xFFFFu) == 0u;   // L is itself a bf16 value
  }
  if (a.act != kClamped) return MOEACT_OK;
  return alpha_table(dev, a.alpha, a.limit, cs, &p.sig_src);
}

moeact_status fwd_common(const ActArgs& a, const void* x, int64_t ldx, const float* s,
                         int64_t M, int64_t N, int dirs, const int64_t* ro, const int64_t* cb,
                         int32_t E, int32_t* status, moeact_mx_out out, void* stream,
                         bool grouped) {
  t_err[0] = 0;
  const int act = a.act, staged = a.staged;
  moeact_status st = check_shape(x, ldx, s, M, N, act);
  if (st) return st;
  if ((st = check_mx(out, dirs, false))) return st;
  if ((st = check_layout(out, M, N))) return st;
  if (staged != 0 && staged != 1) return fail(MOEACT_EINVAL, "staged_rounding must be 0 or 1");
  if (act == kClamped && (st = check_clamp_args(a.alpha, a.limit))) return st;
  int32_t ilv;
  if ((st = check_ilv(act, N, a.ilv, &ilv))) return st;
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
  p.ilv = ilv;
  p.up = ilv ? ilv : (int)N;
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
  p.gemm_scales = out.scale_layout == MOEACT_SCALES_GEMM;
  p.noop = out.noop_flag;
  p.err = g_err_ptr[dev];
  if ((st = act_params(a, dev, cs, p))) return st;
  const int64_t slabs_upper = grouped ? ceil_div(M, 32) + E : ceil_div(M, 32);
  const int kdirs = dirs | (p.gemm_scales ? kGemm : 0) | (ilv ? kIlv : 0);
  const FwdVariant& v = g_fwd[act][fwd_slot(grouped, act == kSwiGLU && staged, kdirs)];
  if (!v.fn) return fail(MOEACT_EUNSUPPORTED, "no forward kernel for this combination");
  CUtensorMap tx;
  if (ilv) st = make_map_ilv(&tx, x, N, ilv, M, ldx);
  else st = make_map(&tx, x, act != kSReLU ? 2 * N : N, M, ldx);
  if (st) return st;
  const int64_t blocks = grid_for(slabs_upper, p.n_tiles, v.threads, dev);
  v.fn<<<(unsigned)blocks, v.threads, v.smem_fixed + group_smem(v.sig, grouped, p.E), cs>>>(tx, p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return MOEACT_OK;
}

moeact_status bwd_common(const ActArgs& a, const void* dy, int64_t lddy, const void* x,
                         int64_t ldx, const float* s, int64_t M, int64_t N, int dirs,
                         const int64_t* ro, const int64_t* cb, int32_t E, int32_t* status,
                         void* dx, float* dscale, moeact_mx_out out, void* ws, size_t ws_bytes,
                         void* stream, bool grouped) {
  t_err[0] = 0;
  const int act = a.act;
  moeact_status st = check_shape(x, ldx, s, M, N, act);
  if (st) return st;
  if ((st = check_mx(out, dirs, true))) return st;
  if ((st = check_layout(out, M, N))) return st;
  if (!dy) return fail(MOEACT_EINVAL, "dy is required");
  if (lddy < N) return fail(MOEACT_EINVAL, "lddy (%lld) smaller than N", (long long)lddy);
  if (lddy % 8 != 0) return fail(MOEACT_EALIGN, "lddy must be a multiple of 8 elements");
  if (lddy > (((int64_t)1) << 40) || M * lddy > (((int64_t)1) << 61)) return fail(MOEACT_ERANGE, "dy extent too large");
  if (!aligned(dy, 16)) return fail(MOEACT_EALIGN, "dy must be 16-byte aligned");
  if (dx && !aligned(dx, 16)) return fail(MOEACT_EALIGN, "dx must be 16-byte aligned");
  if (dscale && !aligned(dscale, 4)) return fail(MOEACT_EALIGN, "dscale must be 4-byte aligned");
  if (dirs == 0 && !dx && !dscale) return fail(MOEACT_EINVAL, "nothing requested: dirs == 0 and no dx / dscale");
  if (act == kClamped && (st = check_clamp_args(a.alpha, a.limit))) return st;
  int32_t ilv;
  if ((st = check_ilv(act, N, a.ilv, &ilv))) return st;
  if (grouped && (st = check_groups(ro, cb, E, status))) return st;
  const size_t ws_need = ws_bytes_needed(M, N);
  if (dscale) {
    if (!ws) return fail(MOEACT_EWORKSPACE, "dscale needs a workspace");
    if (!aligned(ws, 16)) return fail(MOEACT_EALIGN, "workspace must be 16-byte aligned");
    if (ws_bytes < ws_need) return fail(MOEACT_EWORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, ws_need);
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
  p.W = (int)(act != kSReLU ? 2 * N : N);
  p.ilv = ilv;
  p.up = ilv ? ilv : (int)N;
  p.rq = out.row_codes;
  p.rs = out.row_scales;
  p.cq = out.col_codes;
  p.cs = out.col_scales;
  p.dx = static_cast<uint16_t*>(dx);
  p.dscale = dscale;
  if (dscale) p.part = static_cast<float*>(ws);
  p.row_offs = ro;
  p.cb_offs = cb;
  p.E = grouped ? E : 0;
  p.status = status;
  p.dense_slabs = ceil_div(M, 32);
  p.n_tiles = (int)ceil_div(N, kTileCols);
  p.gemm_scales = out.scale_layout == MOEACT_SCALES_GEMM;
  p.noop = out.noop_flag;
  p.err = g_err_ptr[dev];
  if ((st = act_params(a, dev, cs, p))) return st;
  const int64_t slabs_upper = grouped ? ceil_div(M, 32) + E : ceil_div(M, 32);
  // with dX written, the colwise pass re-reads it instead of keeping the
  // whole tile in registers
  const bool rr = dx != nullptr;
  const int kdirs = dirs | ((p.gemm_scales && dirs) ? kGemm : 0);
  const BwdVariant& v = g_bwd[act][bwd_slot(grouped, rr, kdirs)];
  if (!v.fn) return fail(MOEACT_EUNSUPPORTED, "no backward kernel for this combination");
  CUtensorMap tx, tdy;
  if ((st = make_x_map(&tx, act, x, N, ilv, M, ldx))) return st;
  if ((st = make_map(&tdy, dy, N, M, lddy))) return st;
  const int64_t blocks = grid_for(slabs_upper, p.n_tiles, v.threads, dev);
  v.fn<<<(unsigned)blocks, v.threads, v.smem_fixed + group_smem(v.sig, grouped, p.E), cs>>>(tx, tdy, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  if (dscale) {
    dscale_reduce_kernel<<<(unsigned)ceil_div(M, 256), 256, 0, cs>>>(p.part, p.n_tiles, M, dscale,
                                                                      p.noop);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "dscale reduction launch");
  }
  return MOEACT_OK;
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
  if (total_rows > MOEACT_MAX_ROWS) return fail(MOEACT_ERANGE, "total_rows above 2^30");
  if ((m_splits && !aligned(m_splits, 8)) || !aligned(row_offs, 8) ||
      (colblk_offs && !aligned(colblk_offs, 8)) || !aligned(status, 4))
    return fail(MOEACT_EALIGN, "offsets must be 8-byte aligned, status 4-byte aligned");
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int dev;
  moeact_status st = ensure_ready(cs, &dev);
  if (st) return st;
  // one thread per group up to 1024 (whole warps): a small E launches fewer
  // threads and synchronises fewer warps
  const int threads = (int)std::min<int64_t>(1024, std::max<int64_t>(32, ceil_div(num_groups, 32) * 32));
  splits_kernel<<<1, threads, 0, cs>>>(m_splits, num_groups, total_rows, row_offs, colblk_offs,
                                       status);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "splits_to_offsets launch");
  return MOEACT_OK;
}

moeact_status scaled_swiglu_mxfp8_fwd(const void* x, int64_t ldx, const float* s, int64_t M,
                                      int64_t N, int dirs, int staged_rounding,
                                      int32_t glu_interleave, moeact_mx_out out, void* stream) {
  return fwd_common(plain(kSwiGLU, staged_rounding, glu_interleave), x, ldx, s, M, N, dirs,
                    nullptr, nullptr, 0, nullptr, out, stream, false);
}

moeact_status scaled_srelu_mxfp8_fwd(const void* x, int64_t ldx, const float* s, int64_t M,
                                     int64_t N, int dirs, moeact_mx_out out, void* stream) {
  return fwd_common(plain(kSReLU), x, ldx, s, M, N, dirs, nullptr, nullptr, 0, nullptr, out,
                    stream, false);
}

moeact_status grouped_scaled_swiglu_mxfp8_fwd(const void* x, int64_t ldx, const float* s,
                                              int64_t M, int64_t N, int dirs,
                                              int staged_rounding, int32_t glu_interleave,
                                              const int64_t* row_offs,
                                              const int64_t* colblk_offs, int32_t num_groups,
                                              int32_t* status, moeact_mx_out out,
                                              void* stream) {
  return fwd_common(plain(kSwiGLU, staged_rounding, glu_interleave), x, ldx, s, M, N, dirs,
                    row_offs, colblk_offs, num_groups, status, out, stream, true);
}

moeact_status grouped_scaled_srelu_mxfp8_fwd(const void* x, int64_t ldx, const float* s,
                                             int64_t M, int64_t N, int dirs,
                                             const int64_t* row_offs,
                                             const int64_t* colblk_offs, int32_t num_groups,
                                             int32_t* status, moeact_mx_out out, void* stream) {
  return fwd_common(plain(kSReLU), x, ldx, s, M, N, dirs, row_offs, colblk_offs, num_groups,
                    status, out, stream, true);
}

size_t scaled_act_mxfp8_bwd_workspace_size(int64_t M, int64_t N, int32_t num_groups) {
  (void)num_groups;
  if (M < 0 || N <= 0) return 0;
  return ws_bytes_needed(M, N);
}

moeact_status scaled_swiglu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x, int64_t ldx,
                                      const float* s, int64_t M, int64_t N, int dirs,
                                      int32_t glu_interleave, void* dx, float* dscale,
                                      moeact_mx_out out, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  return bwd_common(plain(kSwiGLU, 0, glu_interleave), dy, lddy, x, ldx, s, M, N, dirs, nullptr,
                    nullptr, 0, nullptr, dx, dscale, out, workspace, workspace_bytes, stream,
                    false);
}

moeact_status scaled_srelu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x, int64_t ldx,
                                     const float* s, int64_t M, int64_t N, int dirs, void* dx,
                                     float* dscale, moeact_mx_out out, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  return bwd_common(plain(kSReLU), dy, lddy, x, ldx, s, M, N, dirs, nullptr, nullptr, 0, nullptr, dx,
                    dscale, out, workspace, workspace_bytes, stream, false);
}

moeact_status grouped_scaled_swiglu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x,
                                              int64_t ldx, const float* s, int64_t M, int64_t N,
                                              int dirs, int32_t glu_interleave,
                                              const int64_t* row_offs,
                                              const int64_t* colblk_offs, int32_t num_groups,
                                              int32_t* status, void* dx, float* dscale,
                                              moeact_mx_out out, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  return bwd_common(plain(kSwiGLU, 0, glu_interleave), dy, lddy, x, ldx, s, M, N, dirs, row_offs,
                    colblk_offs, num_groups, status, dx, dscale, out, workspace, workspace_bytes,
                    stream, true);
}

moeact_status grouped_scaled_srelu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x,
                                             int64_t ldx, const float* s, int64_t M, int64_t N,
                                             int dirs, const int64_t* row_offs,
                                             const int64_t* colblk_offs, int32_t num_groups,
                                             int32_t* status, void* dx, float* dscale,
                                             moeact_mx_out out, void* workspace,
                                             size_t workspace_bytes, void* stream) {
  return bwd_common(plain(kSReLU), dy, lddy, x, ldx, s, M, N, dirs, row_offs, colblk_offs, num_groups,
                    status, dx, dscale, out, workspace, workspace_bytes, stream, true);
}

// ---------------------------------------------------------------- ClampedSwiGLU
moeact_status moeact_init_clamped(float alpha, float limit) {
  t_err[0] = 0;
  moeact_status st = check_clamp_args(alpha, limit);
  if (st) return st;
  int dev;
  if ((st = ensure_ready(nullptr, &dev))) return st;
  const float* tab;
  return alpha_table(dev, alpha, limit, nullptr, &tab);
}

moeact_status scaled_clamped_swiglu_mxfp8_fwd(const void* x, int64_t ldx, const float* s,
                                              int64_t M, int64_t N, int dirs, float alpha,
                                              float limit, int32_t glu_interleave,
                                              moeact_mx_out out, void* stream) {
  return fwd_common({kClamped, 0, alpha, limit, glu_interleave}, x, ldx, s, M, N, dirs, nullptr,
                    nullptr, 0, nullptr, out, stream, false);
}

moeact_status grouped_scaled_clamped_swiglu_mxfp8_fwd(const void* x, int64_t ldx, const float* s,
                                                      int64_t M, int64_t N, int dirs,
                                                      float alpha, float limit,
                                                      int32_t glu_interleave,
                                                      const int64_t* row_offs,
                                                      const int64_t* colblk_offs,
                                                      int32_t num_groups, int32_t* status,
                                                      moeact_mx_out out, void* stream) {
  return fwd_common({kClamped, 0, alpha, limit, glu_interleave}, x, ldx, s, M, N, dirs, row_offs,
                    colblk_offs, num_groups, status, out, stream, true);
}

moeact_status scaled_clamped_swiglu_mxfp8_bwd(const void* dy, int64_t lddy, const void* x,
                                              int64_t ldx, const float* s, int64_t M, int64_t N,
                                              int dirs, float alpha, float limit,
                                              int32_t glu_interleave, void* dx, float* dscale,
                                              moeact_mx_out out, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  return bwd_common({kClamped, 0, alpha, limit, glu_interleave}, dy, lddy, x, ldx, s, M, N, dirs,
                    nullptr, nullptr, 0, nullptr, dx, dscale, out, workspace, workspace_bytes,
                    stream, false);
}

moeact_status grouped_scaled_clamped_swiglu_mxfp8_bwd(
    const void* dy, int64_t lddy, const void* x, int64_t ldx, const float* s, int64_t M,
    int64_t N, int dirs, float alpha, float limit, int32_t glu_interleave,
    const int64_t* row_offs, const int64_t* colblk_offs, int32_t num_groups, int32_t* status,
    void* dx, float* dscale, moeact_mx_out out, void* workspace, size_t workspace_bytes,
    void* stream) {
  return bwd_common({kClamped, 0, alpha, limit, glu_interleave}, dy, lddy, x, ldx, s, M, N, dirs,
                    row_offs, colblk_offs, num_groups, status, dx, dscale, out, workspace,
                    workspace_bytes, stream, true);
}

moeact_status moeact_clamped_sigmoid_dump(float alpha, float limit, float* out, void* stream) {
  t_err[0] = 0;
  if (!out) return fail(MOEACT_EINVAL, "out is required");
  if (!aligned(out, 4)) return fail(MOEACT_EALIGN, "out must be 4-byte aligned");
  moeact_status st = check_clamp_args(alpha, limit);
  if (st) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int dev;
  if ((st = ensure_ready(cs, &dev))) return st;
  const float* tab;
  if ((st = alpha_table(dev, alpha, limit, cs, &tab))) return st;
  sigma_table_dump<<<128, 256, kSigBytes, cs>>>(tab, out);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sigmoid dump launch");
  return MOEACT_OK;
}

moeact_status moeact_device_error(uint32_t* flags) {
  t_err[0] = 0;
  if (!flags) return fail(MOEACT_EINVAL, "flags is required");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  *flags = 0;
  if (dev < 0 || dev >= kMaxDevices || !g_ready[dev].load()) return MOEACT_OK;
  uint32_t v = 0;
  const uint32_t zero = 0;
  e = cudaMemcpyFromSymbol(&v, g_err_word, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_err_word, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  *flags = v;
  return MOEACT_OK;
}

moeact_status grouped_scaled_swiglu_mxfp8_fc2(const void* x, int64_t ldx, const float* s,
                                              int64_t M, int64_t N, int staged_rounding,
                                              const int64_t* row_offs, int32_t num_groups,
                                              int32_t* status, const void* w_codes,
                                              const void* w_scales, int64_t H, void* out,
                                              int64_t ldo, const int32_t* noop_flag,
                                              void* stream) {
  t_err[0] = 0;
  moeact_status st = check_shape(x, ldx, s, M, N, kSwiGLU);
  if (st) return st;
  if (N % 128 != 0) return fail(MOEACT_EINVAL, "N must be a multiple of 128 (got %lld)", (long long)N);
  if (N > kFc2MaxN)
    return fail(MOEACT_EUNSUPPORTED, "N above %d: the quantized 128-row block must fit in shared memory", kFc2MaxN);
  if (staged_rounding != 0 && staged_rounding != 1) return fail(MOEACT_EINVAL, "staged_rounding must be 0 or 1");
  if (!row_offs || !status) return fail(MOEACT_EINVAL, "row_offs and status are required");
  if (num_groups < 1 || num_groups > MOEACT_MAX_GROUPS) return fail(MOEACT_EINVAL, "num_groups must be in [1, %d]", MOEACT_MAX_GROUPS);
  if (!aligned(row_offs, 8) || !aligned(status, 4)) return fail(MOEACT_EALIGN, "row_offs must be 8-byte aligned, status 4-byte aligned");
  if (!w_codes || !w_scales || !out) return fail(MOEACT_EINVAL, "w_codes, w_scales and out are required");
  if (!aligned(w_codes, 16) || !aligned(w_scales, 16) || !aligned(out, 16))
    return fail(MOEACT_EALIGN, "w_codes, w_scales and out must be 16-byte aligned");
  if (H <= 0 || H % 128 != 0) return fail(MOEACT_EINVAL, "H must be a positive multiple of 128 (got %lld)", (long long)H);
  if (H * (int64_t)num_groups > INT32_MAX) return fail(MOEACT_ERANGE, "num_groups * H above 2^31 - 1");
  if (ldo < H) return fail(MOEACT_EINVAL, "ldo (%lld) smaller than H", (long long)ldo);
  if (ldo % 8 != 0) return fail(MOEACT_EALIGN, "ldo must be a multiple of 8 elements");
  if (ldo > (((int64_t)1) << 40) || M * ldo > (((int64_t)1) << 61)) return fail(MOEACT_ERANGE, "out extent too large");
  if (noop_flag && !aligned(noop_flag, 4)) return fail(MOEACT_EALIGN, "noop_flag must be 4-byte aligned");
  if (M == 0) return MOEACT_OK;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int dev;
  if ((st = ensure_ready(cs, &dev))) return st;
  CUtensorMap tx;
  if ((st = make_map(&tx, x, 2 * N, M, ldx, kFc2XBoxRows))) return st;
  Fc2Params p{};
  p.s = s;
  p.M = M;
  p.N = (int)N;
  p.H = (int)H;
  p.row_offs = row_offs;
  p.E = num_groups;
  p.status = status;
  p.w_codes = static_cast<const uint8_t*>(w_codes);
  p.w_scales = static_cast<const uint8_t*>(w_scales);
  p.out = static_cast<uint16_t*>(out);
  p.ldo = ldo;
  p.sig_src = g_sig_ptr[dev];
  p.noop = noop_flag;
  p.err = g_err_ptr[dev];
  p.n_sms = g_sms[dev];
  const int64_t grid = ceil_div(M, 128) + num_groups + g_sms[dev];
  const cudaError_t e = fc2_launch(p, tx, staged_rounding, (unsigned)grid, cs);
  if (e != cudaSuccess) return cuda_fail(e, "fused FC2 launch");
  return MOEACT_OK;
}

moeact_status moeact_wait_selftest(int arrive, uint32_t limit_us, uint64_t* result,
                                  void* stream) {
  t_err[0] = 0;
  if (!result) return fail(MOEACT_EINVAL, "result is required");
  if (!aligned(result, 8)) return fail(MOEACT_EALIGN, "result must be 8-byte aligned");
  if (arrive != 0 && arrive != 1) return fail(MOEACT_EINVAL, "arrive must be 0 or 1");
  if (limit_us < 1 || limit_us > 2000000u)
    return fail(MOEACT_ERANGE, "limit_us must be in [1, 2000000] (got %u)", limit_us);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int dev;
  moeact_status st = ensure_ready(cs, &dev);
  if (st) return st;
  wait_probe_kernel<<<1, 32, 0, cs>>>((uint64_t)limit_us * 1000u, arrive, g_err_ptr[dev],
                                      MOEACT_DEVERR_WAIT_SELFTEST, result);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "wait self-test launch");
  return MOEACT_OK;
}

moeact_status moeact_sigmoid_dump(float* out, void* stream) {
  t_err[0] = 0;
  if (!out) return fail(MOEACT_EINVAL, "out is required");
  if (!aligned(out, 4)) return fail(MOEACT_EALIGN, "out must be 4-byte aligned");
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int dev;
  moeact_status st = ensure_ready(cs, &dev);
  if (st) return st;
  sigma_table_dump<<<128, 256, kSigBytes, cs>>>(g_sig_ptr[dev], out);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sigmoid dump launch");
  return MOEACT_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward without any allocation (see g_noalloc_scratch above): the dense
// SwiGLU backward with the dscale partials in the built-in array.
extern "C" moeact_status scaled_swiglu_mxfp8_bwd_noalloc(
    const void* dy, int64_t lddy, const void* x, int64_t ldx, const float* s, int64_t M,
    int64_t N, int dirs, void* dx, float* dscale, moeact_mx_out out, void* stream) {
  t_err[0] = 0;
  // the shape checks first, so that a bad shape gets the error any entry
  // point gives it; then the scratch bound, in a form that cannot wrap
  moeact_status st = check_shape(x, ldx, s, M, N, kSwiGLU);
  if (st) return st;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  if (dscale != nullptr && M > 0) {
    const int64_t tiles = ceil_div(N, kTileCols);
    if (M > (int64_t)(kNoAllocScratchBytes / 4) / tiles)
      return fail(MOEACT_ERANGE,
                  "dscale for M=%lld, N=%lld needs %lld bytes of scratch; the built-in scratch "
                  "holds %zu (ceil(N/128) * M <= 4194304); use scaled_swiglu_mxfp8_bwd with a "
                  "workspace",
                  (long long)M, (long long)N, (long long)(tiles * M * 4), kNoAllocScratchBytes);
    int dev;
    if ((st = ensure_ready(static_cast<cudaStream_t>(stream), &dev))) return st;
    ws = g_noalloc_ptr[dev];
    ws_bytes = kNoAllocScratchBytes;
  }
  return scaled_swiglu_mxfp8_bwd(dy, lddy, x, ldx, s, M, N, dirs, 0, dx, dscale, out, ws,
                                 ws_bytes, stream);
}
