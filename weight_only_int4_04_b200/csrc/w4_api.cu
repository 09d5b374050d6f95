// C ABI entry points of libw4 (declared in include/w4.h): host-side argument checks, kernel
// selection and error reporting. No device memory is allocated here; the only device state
// is the static status words below (one per loaded library, shared by every call).
#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "w4_internal.cuh"
#include "w4_sync.cuh"

namespace {

// NVTX range around each entry point (a push/pop pair: near-free unless a profiler is
// attached, which then shows every call of the library on its timeline by name).
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

thread_local int g_last_cuda_error = 0;

// Device words: validation flags and the non-finite flag of a quantize call that was given
// no status pointer. Calls that use them synchronize their stream before returning, so one
// host thread never shares them in flight; calls from several threads or streams at once
// would (the header tells callers to pass their own status word then).
__device__ uint32_t g_validate_flags;
__device__ int32_t g_quant_status;
// Written by bounded device-side waits when they give up (read by w4_device_error).
__device__ int32_t g_device_error;

constexpr int64_t kMaxK = int64_t(1) << 24;
constexpr int64_t kMaxRows = 0x7fffffffLL;

w4_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return W4_ERR_CUDA;
}

bool sizes_ok(int64_t N, int64_t K) { return N >= 1 && K >= 1 && N <= kMaxRows && K <= kMaxK; }

template <typename T>
w4_status symbol_ptr(T **out, const T &sym) {
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, sym);
  if (e != cudaSuccess) return cuda_fail(e);
  *out = static_cast<T *>(p);
  return W4_OK;
}

// Decode launch policy (w4_set_weight_prefetch): stream codes and scales before the
// previous kernel of the stream has finished.
std::atomic<int> g_weight_prefetch{0};

// Kernel family the calling thread's last linear call launched (w4_last_linear_kernel).
thread_local const char *t_last_kernel = "none";

// Tensor-core GEMM is used above this M (and whenever the decode kernels do not apply).
constexpr int64_t kTcMinM = 17;

// The asymmetric tensor-core path gathers x into the workspace; everything else needs none.
bool asym_uses_tc(const w4i::LinearParams &p) {
  return p.asym && p.M >= kTcMinM && w4i::gemm_tc_supports(p);
}

w4_status run_linear(const w4i::LinearParams &p, void *workspace, size_t workspace_bytes,
                     cudaStream_t stream) {
  int32_t *err = nullptr;
  const w4_status st = symbol_ptr(&err, g_device_error);
  if (st != W4_OK) return st;
  // M dispatch: M <= 16 -> the TMA-fed tensor-core GEMV (symmetric codes, K a multiple of
  // 128, activations that fit in shared memory), else for M = 1 the register-streaming GEMV
  // and for M <= 16 the bulk-copy mma.sync kernel; larger M -> the tcgen05 GEMM; the other
  // kernels take the shapes the fast paths cannot (unaligned rows, odd widths, unsorted
  // act-order maps). The kernel chosen is recorded for w4_last_linear_kernel().
  cudaError_t e;
  // act-order beyond one short row: x is gathered into sorted column order once per call,
  // into the workspace, so that no CTA of the GEMV has to gather it (one row: every CTA
  // gathers it itself, which costs less than a launch)
  const bool asym_gather = p.asym && !w4i::gemv_tma_gathers_x(p);
  const bool ws_gather = workspace != nullptr && workspace_bytes >= w4i::gemm_tc_asym_workspace(p.M, p.K) &&
                         p.K % 8 == 0;
  if (w4i::gemv_tma_supports(p) && (!asym_gather || ws_gather)) {
    const __nv_bfloat16 *xs = nullptr;
    e = cudaSuccess;
    if (asym_gather) {
      xs = static_cast<const __nv_bfloat16 *>(workspace);
      e = w4i::launch_gather_x(p.x, p.perm, p.M, p.K, static_cast<__nv_bfloat16 *>(workspace), stream);
    }
    if (e == cudaSuccess)
      e = w4i::launch_gemv_tma(p, g_weight_prefetch.load(std::memory_order_relaxed) != 0, xs, err, stream);
    t_last_kernel = asym_gather ? "gather_x+gemv_tma" : "gemv_tma";
  } else if (w4i::gemv_rows_supports(p)) {
    e = w4i::launch_gemv_rows(p, stream);
    t_last_kernel = "gemv_rows";
  } else if (w4i::gemv_mma_supports(p)) {
    e = w4i::launch_gemv_mma(p, err, stream);
    t_last_kernel = "gemv_mma";
  } else if (w4i::gemv_supports(p)) {
    e = w4i::launch_gemv(p, stream);
    t_last_kernel = "gemv";
  } else if (p.M > 4 && w4i::gemm_tc_supports(p) &&
             (!p.asym || (workspace != nullptr && workspace_bytes >= w4i::gemm_tc_asym_workspace(p.M, p.K)))) {
    e = w4i::launch_gemm_tc(p, err, stream, workspace);
    t_last_kernel = p.asym ? "gather_x+gemm_tc" : "gemm_tc";
  } else {
    e = w4i::launch_linear_generic(p, stream);
    t_last_kernel = "linear_generic";
  }
  return e == cudaSuccess ? W4_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

int w4_version(void) { return 100; }

const char *w4_last_linear_kernel(void) { return t_last_kernel; }

int w4_last_cuda_error(void) { return g_last_cuda_error; }

const char *w4_status_string(w4_status s) {
  switch (s) {
    case W4_OK: return "ok";
    case W4_ERR_NULL: return "a required pointer is NULL";
    case W4_ERR_SHAPE: return "size out of range or sizes do not agree";
    case W4_ERR_DTYPE: return "unsupported dtype";
    case W4_ERR_NONFINITE: return "weight must be finite";
    case W4_ERR_SCALE: return "scales must be finite and positive";
    case W4_ERR_HIGH_NIBBLE: return "nonzero unused high nibble";
    case W4_ERR_RESERVED_CODE: return "reserved -8 code is outside the narrow signed range of format v1";
    case W4_ERR_VERSION: return "unsupported packed-weight version";
    case W4_ERR_GIDX: return "g_idx entry outside [0, n_groups)";
    case W4_ERR_ZERO: return "zero point outside [0, 15]";
    case W4_ERR_UNSUPPORTED: return "request not supported by this build";
    case W4_ERR_WORKSPACE: return "workspace too small or misaligned";
    case W4_ERR_TIMEOUT: return "a bounded device-side wait expired";
    case W4_ERR_CUDA: return "CUDA call failed";
  }
  return "unknown status";
}

w4_status w4_quantize_rtn(const float *W, int64_t N, int64_t K, uint8_t *codes, float *scales,
                          int32_t *d_status, w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_quantize_rtn");
  if (!W || !codes || !scales) return W4_ERR_NULL;
  if (!sizes_ok(N, K)) return W4_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t *status = d_status;
  if (!status) {
    const w4_status st = symbol_ptr(&status, g_quant_status);
    if (st != W4_OK) return st;
    const cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  cudaError_t e = w4i::launch_quantize_rtn(W, N, K, codes, scales, status, s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (!d_status) {
    int32_t host = 0;
    e = cudaMemcpyAsync(&host, status, sizeof(host), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (host != 0) return W4_ERR_NONFINITE;
  }
  return W4_OK;
}

w4_status w4_dequantize(const uint8_t *codes, const float *scales, int64_t N, int64_t K,
                        int format_version, w4_dtype out_dtype, void *out, w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_dequantize");
  if (!codes || !scales || !out) return W4_ERR_NULL;
  if (!sizes_ok(N, K)) return W4_ERR_SHAPE;
  if (format_version != 1 && format_version != 2) return W4_ERR_VERSION;
  if (out_dtype != W4_BF16 && out_dtype != W4_F16 && out_dtype != W4_F32 && out_dtype != W4_F64)
    return W4_ERR_DTYPE;
  const cudaError_t e = w4i::launch_dequantize(codes, scales, N, K, out_dtype, out,
                                               reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? W4_OK : cuda_fail(e);
}

size_t w4_linear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  (void)M;
  (void)N;
  (void)K;
  return 0;
}

w4_status w4_linear(const void *x, int64_t M, const uint8_t *codes, const float *scales, int64_t N,
                    int64_t K, const float *bias, void *y, w4_dtype y_dtype, void *workspace,
                    size_t workspace_bytes, w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_linear");
  if (!x || !codes || !scales || !y) return W4_ERR_NULL;
  if (!sizes_ok(N, K) || M < 1 || M > kMaxRows) return W4_ERR_SHAPE;
  if (y_dtype != W4_BF16 && y_dtype != W4_F32) return W4_ERR_DTYPE;
  const size_t need = w4_linear_workspace_bytes(M, N, K);
  if (need > 0 && (!workspace || workspace_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 256))
    return W4_ERR_WORKSPACE;
  w4i::LinearParams p{};
  p.x = static_cast<const __nv_bfloat16 *>(x);
  p.codes = codes;
  p.scales = scales;
  p.bias = bias;
  p.y = y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.y_dtype = y_dtype;
  p.asym = 0;
  return run_linear(p, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

size_t w4_linear_asym_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t n_groups) {
  // act-order kernels gather x through perm once per call: M * K bf16 (the tensor-core GEMM
  // above the decode sizes; the decode kernel when K is a multiple of 128)
  if (M < 1 || K < 1 || N < 1 || n_groups < 1 || K % 8 != 0) return 0;
  if (M < kTcMinM ? K % 128 != 0 : n_groups % 16 != 0) return 0;
  return w4i::gemm_tc_asym_workspace(M, K);
}

w4_status w4_asym_prepare(const uint8_t *codes_in, const int32_t *g_idx, int64_t N, int64_t K,
                          int64_t n_groups, uint8_t *codes_out, int32_t *perm, w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_asym_prepare");
  if (!codes_in || !g_idx || !codes_out || !perm) return W4_ERR_NULL;
  if (!sizes_ok(N, K) || n_groups < 1 || n_groups > K) return W4_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // One-time preparation: the stable sort of K column labels runs on the host.
  std::vector<int32_t> gi(static_cast<size_t>(K));
  cudaError_t e = cudaMemcpyAsync(gi.data(), g_idx, sizeof(int32_t) * K, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  for (int32_t g : gi)
    if (g < 0 || g >= n_groups) return W4_ERR_GIDX;
  std::vector<int32_t> order(static_cast<size_t>(K));
  for (int64_t k = 0; k < K; ++k) order[k] = static_cast<int32_t>(k);
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return gi[a] < gi[b]; });
  e = cudaMemcpyAsync(perm, order.data(), sizeof(int32_t) * K, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = w4i::launch_reorder_codes(codes_in, perm, N, K, codes_out, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);  // `order` is host memory in flight
  return e == cudaSuccess ? W4_OK : cuda_fail(e);
}

w4_status w4_linear_asym_gidx(const void *x, int64_t M, const uint8_t *codes, const float *scales,
                              const int8_t *zeros, const int32_t *g_idx, const int32_t *perm,
                              int64_t N, int64_t K, int64_t n_groups, const float *bias, void *y,
                              w4_dtype y_dtype, void *workspace, size_t workspace_bytes,
                              w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_linear_asym_gidx");
  if (!x || !codes || !scales || !zeros || !g_idx || !y) return W4_ERR_NULL;
  if (!sizes_ok(N, K) || M < 1 || M > kMaxRows || n_groups < 1 || n_groups > K) return W4_ERR_SHAPE;
  if (y_dtype != W4_BF16 && y_dtype != W4_F32) return W4_ERR_DTYPE;
  // With codes sorted by w4_asym_prepare (perm given) the tensor-core path needs the
  // workspace; without it a slower kernel serves the call (no error).
  if (workspace != nullptr && reinterpret_cast<uintptr_t>(workspace) % 256) return W4_ERR_WORKSPACE;
  w4i::LinearParams p{};
  p.x = static_cast<const __nv_bfloat16 *>(x);
  p.codes = codes;
  p.scales = scales;
  p.zeros = zeros;
  p.g_idx = g_idx;
  p.perm = perm;
  p.bias = bias;
  p.y = y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.n_groups = static_cast<int>(n_groups);
  p.y_dtype = y_dtype;
  p.asym = 1;
  return run_linear(p, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

static w4_status run_validate(const uint8_t *codes, const float *scales, const int8_t *zeros,
                              const int32_t *g_idx, int64_t N, int64_t K, int64_t n_groups,
                              int format_version, int asym, cudaStream_t s, uint32_t *flags_out) {
  uint32_t *flags = nullptr;
  w4_status st = symbol_ptr(&flags, g_validate_flags);
  if (st != W4_OK) return st;
  cudaError_t e = cudaMemsetAsync(flags, 0, sizeof(uint32_t), s);
  if (e == cudaSuccess)
    e = w4i::launch_validate(codes, scales, zeros, g_idx, N, K, n_groups, format_version, asym, flags, s);
  uint32_t host = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&host, flags, sizeof(host), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  *flags_out = host;
  return W4_OK;
}

w4_status w4_validate(const uint8_t *codes, const float *scales, int64_t N, int64_t K,
                      int format_version, w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_validate");
  if (!codes || !scales) return W4_ERR_NULL;
  if (!sizes_ok(N, K)) return W4_ERR_SHAPE;
  if (format_version != 1 && format_version != 2) return W4_ERR_VERSION;
  uint32_t f = 0;
  const w4_status st = run_validate(codes, scales, nullptr, nullptr, N, K, 0, format_version, 0,
                                    reinterpret_cast<cudaStream_t>(stream), &f);
  if (st != W4_OK) return st;
  if (f & w4i::FLAG_SCALE) return W4_ERR_SCALE;
  if (f & w4i::FLAG_HIGH_NIBBLE) return W4_ERR_HIGH_NIBBLE;
  if (f & w4i::FLAG_RESERVED) return W4_ERR_RESERVED_CODE;
  return W4_OK;
}

w4_status w4_validate_asym(const uint8_t *codes, const float *scales, const int8_t *zeros,
                           const int32_t *g_idx, int64_t N, int64_t K, int64_t n_groups,
                           w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_validate_asym");
  if (!codes || !scales || !zeros || !g_idx) return W4_ERR_NULL;
  if (!sizes_ok(N, K) || n_groups < 1 || n_groups > K) return W4_ERR_SHAPE;
  uint32_t f = 0;
  const w4_status st = run_validate(codes, scales, zeros, g_idx, N, K, n_groups, 2, 1,
                                    reinterpret_cast<cudaStream_t>(stream), &f);
  if (st != W4_OK) return st;
  if (f & w4i::FLAG_SCALE) return W4_ERR_SCALE;
  if (f & w4i::FLAG_HIGH_NIBBLE) return W4_ERR_HIGH_NIBBLE;
  if (f & w4i::FLAG_ZERO) return W4_ERR_ZERO;
  if (f & w4i::FLAG_GIDX) return W4_ERR_GIDX;
  return W4_OK;
}

w4_status w4_dequantize_q4_0(const uint8_t *blocks, int64_t N, int64_t K, w4_dtype out_dtype, void *out,
                             w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_dequantize_q4_0");
  if (!blocks || !out) return W4_ERR_NULL;
  if (!sizes_ok(N, K) || K % 32 != 0) return W4_ERR_SHAPE;
  if (out_dtype != W4_BF16 && out_dtype != W4_F16 && out_dtype != W4_F32 && out_dtype != W4_F64)
    return W4_ERR_DTYPE;
  const cudaError_t e =
      w4i::launch_q4_0_dequantize(blocks, N, K, out_dtype, out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? W4_OK : cuda_fail(e);
}

w4_status w4_q4_0_to_group32(const uint8_t *blocks, int64_t N, int64_t K, uint8_t *codes, float *scales,
                             w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_q4_0_to_group32");
  if (!blocks || !codes || !scales) return W4_ERR_NULL;
  if (!sizes_ok(N, K) || K % 32 != 0) return W4_ERR_SHAPE;
  const cudaError_t e =
      w4i::launch_q4_0_to_group32(blocks, N, K, codes, scales, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? W4_OK : cuda_fail(e);
}

w4_status w4_linear_q4_0(const void *x, int64_t M, const uint8_t *blocks, int64_t N, int64_t K,
                         const float *bias, void *y, w4_dtype y_dtype, w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_linear_q4_0");
  if (!x || !blocks || !y) return W4_ERR_NULL;
  if (!sizes_ok(N, K) || K % 32 != 0 || M < 1 || M > kMaxRows) return W4_ERR_SHAPE;
  if (y_dtype != W4_BF16 && y_dtype != W4_F32) return W4_ERR_DTYPE;
  int32_t *err = nullptr;
  const w4_status st = symbol_ptr(&err, g_device_error);
  if (st != W4_OK) return st;
  const cudaError_t e = w4i::launch_q4_0_linear(static_cast<const __nv_bfloat16 *>(x), M, blocks, N, K, bias, y,
                                                y_dtype, g_weight_prefetch.load(std::memory_order_relaxed) != 0,
                                                err, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? W4_OK : cuda_fail(e);
}

size_t w4_linear_backward_x_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return w4i::linear_backward_x_workspace(M, N, K);
}

w4_status w4_linear_backward_x(const void *dy, int64_t M, const uint8_t *codes, const float *scales, int64_t N,
                               int64_t K, void *dx, w4_dtype dx_dtype, void *workspace, size_t workspace_bytes,
                               w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_linear_backward_x");
  if (!dy || !codes || !scales || !dx) return W4_ERR_NULL;
  if (!sizes_ok(N, K) || M < 1 || M > kMaxRows) return W4_ERR_SHAPE;
  if (dx_dtype != W4_BF16 && dx_dtype != W4_F32) return W4_ERR_DTYPE;
  const size_t need = w4i::linear_backward_x_workspace(M, N, K);
  if (need > 0 && (!workspace || workspace_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 256))
    return W4_ERR_WORKSPACE;
  const cudaError_t e = w4i::launch_linear_backward_x(static_cast<const __nv_bfloat16 *>(dy), M, codes, scales, N,
                                                      K, dx, dx_dtype, workspace, workspace_bytes,
                                                      reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? W4_OK : cuda_fail(e);
}

w4_status w4_quantize_rtn_channel(const float *W, int64_t N, int64_t K, uint8_t *codes, float *scales,
                                  int32_t *d_status, w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_quantize_rtn_channel");
  if (!W || !codes || !scales) return W4_ERR_NULL;
  if (!sizes_ok(N, K)) return W4_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t *status = d_status;
  if (!status) {
    const w4_status st = symbol_ptr(&status, g_quant_status);
    if (st != W4_OK) return st;
    const cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  cudaError_t e = w4i::launch_quantize_rtn_channel(W, N, K, codes, scales, status, s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (!d_status) {
    int32_t host = 0;
    e = cudaMemcpyAsync(&host, status, sizeof(host), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (host != 0) return W4_ERR_NONFINITE;
  }
  return W4_OK;
}

size_t w4_linear_channel_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  // none for the per-row-scale decode kernel (M <= 16, K a multiple of 128, aligned x and
  // codes); otherwise the scales expanded to the group layout [N, ceil(K/32)] floats
  if (M >= 1 && M <= 16 && K % 128 == 0) return 0;
  if (N < 1 || K < 1) return 0;
  return static_cast<size_t>(((N * ((K + 31) / 32) * 4 + 255) / 256) * 256);
}

w4_status w4_linear_channel(const void *x, int64_t M, const uint8_t *codes, const float *scales, int64_t N,
                            int64_t K, const float *bias, void *y, w4_dtype y_dtype, void *workspace,
                            size_t workspace_bytes, w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_linear_channel");
  if (!x || !codes || !scales || !y) return W4_ERR_NULL;
  if (!sizes_ok(N, K) || M < 1 || M > kMaxRows) return W4_ERR_SHAPE;
  if (y_dtype != W4_BF16 && y_dtype != W4_F32) return W4_ERR_DTYPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  w4i::LinearParams p{};
  p.x = static_cast<const __nv_bfloat16 *>(x);
  p.codes = codes;
  p.scales = scales;
  p.bias = bias;
  p.y = y;
  p.M = M;
  p.N = N;
  p.K = K;
  p.y_dtype = y_dtype;
  p.channel = 1;
  if (w4i::gemv_tma_supports(p)) {
    int32_t *err = nullptr;
    const w4_status st = symbol_ptr(&err, g_device_error);
    if (st != W4_OK) return st;
    const cudaError_t e =
        w4i::launch_gemv_tma(p, g_weight_prefetch.load(std::memory_order_relaxed) != 0, nullptr, err, s);
    t_last_kernel = "gemv_tma_channel";
    return e == cudaSuccess ? W4_OK : cuda_fail(e);
  }
  // other shapes: the row scales expanded to the group layout in the workspace, then the
  // group-32 linear
  const size_t need = static_cast<size_t>(N * ((K + 31) / 32) * 4);
  if (!workspace || workspace_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 256) return W4_ERR_WORKSPACE;
  cudaError_t e = w4i::launch_expand_channel_scales(scales, N, K, static_cast<float *>(workspace), s);
  if (e != cudaSuccess) return cuda_fail(e);
  p.channel = 0;
  p.scales = static_cast<const float *>(workspace);
  return run_linear(p, nullptr, 0, s);
}

w4_status w4_expand_channel_scales(const float *scales, int64_t N, int64_t K, float *scales_out,
                                   w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_expand_channel_scales");
  if (!scales || !scales_out) return W4_ERR_NULL;
  if (!sizes_ok(N, K)) return W4_ERR_SHAPE;
  const cudaError_t e =
      w4i::launch_expand_channel_scales(scales, N, K, scales_out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? W4_OK : cuda_fail(e);
}

w4_status w4_lora_merge(const uint8_t *codes, const float *scales, int64_t N, int64_t K, const float *lora_b_t,
                        const float *lora_a_t, int64_t rank, float alpha_over_rank, uint8_t *codes_out,
                        float *scales_out, int32_t *d_status, w4_stream_t stream) {
  const NvtxRange nvtx_range("w4_lora_merge");
  if (!codes || !scales || !codes_out || !scales_out) return W4_ERR_NULL;
  if (rank > 0 && (!lora_b_t || !lora_a_t)) return W4_ERR_NULL;
  if (!sizes_ok(N, K) || rank < 0 || rank > 65536) return W4_ERR_SHAPE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t *status = d_status;
  if (!status) {
    const w4_status st = symbol_ptr(&status, g_quant_status);
    if (st != W4_OK) return st;
    const cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  cudaError_t e = w4i::launch_lora_merge(codes, scales, lora_b_t, lora_a_t, N, K, rank, alpha_over_rank, codes_out,
                                         scales_out, status, s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (!d_status) {
    int32_t host = 0;
    e = cudaMemcpyAsync(&host, status, sizeof(host), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (host != 0) return W4_ERR_NONFINITE;
  }
  return W4_OK;
}

int w4_set_weight_prefetch(int enable) {
  return g_weight_prefetch.exchange(enable != 0 ? 1 : 0);
}

w4_status w4_selftest_wait_timeout(uint64_t limit_ns, w4_stream_t stream) {
  if (limit_ns == 0 || limit_ns > w4i::kWaitLimitNs) return W4_ERR_SHAPE;
  int32_t *err = nullptr;
  const w4_status st = symbol_ptr(&err, g_device_error);
  if (st != W4_OK) return st;
  const cudaError_t e = w4i::launch_wait_selftest(limit_ns, err, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? W4_OK : cuda_fail(e);
}

w4_status w4_device_error(void) {
  cudaError_t e = cudaDeviceSynchronize();
  int32_t host = 0;
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&host, g_device_error, sizeof(host));
  if (e != cudaSuccess) return cuda_fail(e);
  if (host != 0) {
    const int32_t zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e);
    return static_cast<w4_status>(host);
  }
  return W4_OK;
}

}  // extern "C"
