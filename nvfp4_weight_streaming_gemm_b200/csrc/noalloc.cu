// nvfp4_gemm_skinny_noalloc: the tensor-core GEMM for callers that cannot
// allocate device memory and so cannot supply a workspace.
//
// Examples of such callers:
//   - a host whose device-memory plan is fixed at start-up and which forbids
//     allocation once it is serving;
//   - code that runs under another framework's pooling allocator, where a
//     stray cudaMalloc would bypass the pool's accounting;
//   - a plugin interface that hands over inputs and outputs but no scratch
//     buffer.
//
// For them the scratch the tensor-core kernel needs (its split-tile ticket
// counters and fp32 partial sums) lives in one file-scope device array of fixed
// size, kNoAllocScratchBytes. Every GPU that loads the library holds that array
// until the process exits. The caller still passes X, the packed weight and Y.
//
// On a device, the first call looks up the array's device address with
// cudaGetSymbolAddress and caches it. That first call should therefore come
// before any stream capture. In host code the array's name is only a host-side
// stand-in; it is never handed to a kernel.
//
// Every call reuses the same array and leaves its last contents there. Each
// call clears the ticket counters (cudaMemsetAsync on its stream, which
// allocates nothing). Two calls whose work overlaps on the GPU, for example on
// different streams, race on the array.
#include "common.cuh"
#include "mma.h"

#include <mutex>

namespace nvfp4ws {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static void* g_scratch_ptr[kNoAllocMaxDevices] = {};
static std::mutex g_scratch_mu;

// Device address of the scratch array on the current device, looked up once per device.
static int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
    return set_error(NVFP4WS_ERR_CUDA, "nvfp4_gemm_skinny_noalloc: cannot get the current device");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return set_error(NVFP4WS_ERR_CUDA, "nvfp4_gemm_skinny_noalloc: cudaGetSymbolAddress failed: %s",
                       cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return NVFP4WS_OK;
}

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

}  // namespace nvfp4ws

using namespace nvfp4ws;

extern "C" int nvfp4_gemm_skinny_noalloc(const void* X, const uint8_t* q, const uint8_t* sf,
                                         const float* tensor_scale, int64_t M, int64_t N, int64_t K, void* Y,
                                         int y_dtype, nvfp4ws_stream_t stream) {
  clear_error();
  if (!X || !q || !sf || !tensor_scale || !Y)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_gemm_skinny_noalloc: null pointer");
  if (M < 1 || N < 1 || K < 1)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_gemm_skinny_noalloc: M, N, K must be >= 1");
  if (!mma_supported(M, K))
    return set_error(NVFP4WS_ERR_UNSUPPORTED,
                     "nvfp4_gemm_skinny_noalloc: needs 1 <= M <= 128 and K a positive multiple of 256 "
                     "(M=%lld K=%lld)", (long long)M, (long long)K);
  if (((uintptr_t)X | (uintptr_t)q | (uintptr_t)sf | (uintptr_t)Y) & 15u)
    return set_error(NVFP4WS_ERR_MISALIGNED, "nvfp4_gemm_skinny_noalloc: X, q, sf and Y must be 16-byte aligned");
  if (y_dtype != NVFP4WS_Y_F32 && y_dtype != NVFP4WS_Y_BF16)
    return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_gemm_skinny_noalloc: bad y_dtype %d", y_dtype);
  if (N > (int64_t)0x7fffffff || K > ((int64_t)1 << 24))
    return set_error(NVFP4WS_ERR_UNSUPPORTED, "nvfp4_gemm_skinny_noalloc: N or K too large");
  const size_t need = mma_gemm_workspace_bytes(M, N, K);
  if (need > kNoAllocScratchBytes)
    return set_error(NVFP4WS_ERR_UNSUPPORTED,
                     "nvfp4_gemm_skinny_noalloc: this shape needs %zu bytes of scratch, more than the built-in "
                     "%zu; use nvfp4_gemm_skinny with a workspace", need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if (int e = scratch_address(&scratch)) return e;
  cudaStream_t s = (cudaStream_t)stream;
  // The leading ticket counters must start at zero.
  // (check_launch also counts the memset node, as nvfp4ws_kernel_launches documents.)
  const cudaError_t me = cudaMemsetAsync(scratch, 0, mma_gemm_counter_bytes(M, N, K), s);
  if (int e = check_launch("nvfp4_gemm_skinny_noalloc: counter clear")) return e;
  if (me != cudaSuccess)
    return set_error(NVFP4WS_ERR_CUDA, "nvfp4_gemm_skinny_noalloc: counter clear: %s", cudaGetErrorString(me));
  return launch_mma_gemm(static_cast<const uint16_t*>(X), q, sf, tensor_scale, M, N, K, Y, y_dtype, scratch,
                         kNoAllocScratchBytes, s);
}
