// w4_linear_asym_gidx_noalloc: the act-order linear without any device allocation.
//
// Some callers cannot hand the library a workspace: a host program that runs inside a
// framework owning all device memory through its own pool, or a process that must not call
// cudaMalloc once it is serving (the call synchronizes the whole device, and it can fail
// when memory is fragmented). For them this entry point keeps its scratch memory -- the
// activations gathered into sorted column order for the tensor-core GEMM -- in one
// file-scope device array that exists on every GPU that loads the library, from load until
// process exit.
#include <nvtx3/nvToolsExt.h>

#include "w4_internal.cuh"

namespace {

// 16 MiB: M * K bf16 activations, e.g. M = 2048 rows at K = 4096 (exactly the limit).
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device. In host code the array's name
// is only a host-side stand-in, so the address is looked up with the device current. It is
// looked up on every call (a table lookup once the module is loaded): a cached address
// would dangle after a device reset reloads the module.
cudaError_t scratch_for_current_device(void **out) {
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  *out = p;
  return cudaSuccess;
}

w4_status noalloc_call(const void *x, int64_t M, const uint8_t *codes, const float *scales,
                       const int8_t *zeros, const int32_t *g_idx, const int32_t *perm, int64_t N, int64_t K,
                       int64_t n_groups, const float *bias, void *y, w4_dtype y_dtype, w4_stream_t stream) {
  // The limit is the gathered activations' size, M * K bf16, whichever kernel serves the
  // shape (the decode kernels need less, or none): larger shapes are rejected outright.
  // Exactly 16 MiB is accepted. Non-positive sizes fall through to the regular checks.
  if (M > 0 && K > 0 &&
      static_cast<uint64_t>(M) > kNoAllocScratchBytes / 2 / static_cast<uint64_t>(K))
    return W4_ERR_SHAPE;
  void *scratch = nullptr;
  const cudaError_t e = scratch_for_current_device(&scratch);
  if (e != cudaSuccess) return W4_ERR_CUDA;
  // Every element of the gathered activations is written before the GEMM reads it, so the
  // array needs no clearing between calls.
  return w4_linear_asym_gidx(x, M, codes, scales, zeros, g_idx, perm, N, K, n_groups, bias, y, y_dtype,
                             scratch, kNoAllocScratchBytes, stream);
}

}  // namespace

extern "C" w4_status w4_linear_asym_gidx_noalloc(const void *x, int64_t M, const uint8_t *codes,
                                                 const float *scales, const int8_t *zeros,
                                                 const int32_t *g_idx, const int32_t *perm, int64_t N,
                                                 int64_t K, int64_t n_groups, const float *bias, void *y,
                                                 w4_dtype y_dtype, w4_stream_t stream) {
  nvtxRangePushA("w4_linear_asym_gidx_noalloc");
  const w4_status st = noalloc_call(x, M, codes, scales, zeros, g_idx, perm, N, K, n_groups, bias, y, y_dtype, stream);
  nvtxRangePop();
  return st;
}
