// tcgen05 tensor-core path (not built yet: reports unsupported).
#include "common.cuh"
#include "mma.h"

namespace nvfp4ws {

bool mma_supported(long long, long long) { return false; }
int mma_min_m() { return 1 << 30; }
size_t mma_gemm_workspace_bytes(long long, long long, long long) { return 0; }
size_t mma_verify_workspace_bytes(long long, long long, long long) { return 0; }
int launch_mma_gemm(const uint16_t*, const uint8_t*, const uint8_t*, const float*, long long, long long, long long,
                    void*, int, void*, size_t, cudaStream_t) {
  return set_error(NVFP4WS_ERR_UNSUPPORTED, "MMA path not available");
}
int launch_mma_verify(const uint16_t*, const uint8_t*, const uint8_t*, const float*, long long, long long, long long,
                      const int32_t*, int, int, int32_t*, int32_t*, float*, void*, cudaStream_t) {
  return set_error(NVFP4WS_ERR_UNSUPPORTED, "MMA path not available");
}

}  // namespace nvfp4ws
