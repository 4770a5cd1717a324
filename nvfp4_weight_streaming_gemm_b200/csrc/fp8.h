// Internal interface of the FP8 (E4M3, 128 x 128 block-scaled) weight path (not part of the C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"

namespace nvfp4ws {

// Rows and K elements covered by one fp32 block scale.
constexpr int kFp8Block = 128;

// The tensor-core kernel's shape limits: 1 <= M <= 128, K a positive multiple of 128.
bool fp8_supported(long long M, long long K);
size_t fp8_gemm_workspace_bytes_int(long long M, long long N, long long K);
size_t fp8_verify_workspace_bytes_int(long long M, long long N, long long K);
int launch_fp8_gemm(const uint16_t* X, const uint8_t* q, const float* scales, long long M, long long N, long long K,
                    void* Y, int y_dtype, void* workspace, cudaStream_t s);
int launch_fp8_verify(const uint16_t* X, const uint8_t* q, const float* scales, long long M, long long N,
                      long long K, const VerifyRule& v, void* workspace, cudaStream_t s);

// One GEMM of an FP8 weight pass, as the host sees it. verify: the pass's lm_head (last).
struct Fp8HostProblem {
  const uint16_t* X;
  const uint8_t* q;
  const float* scales;
  long long N, K;
  void* Y;
  int y_bf16, verify;
};
// Host state of an initialised FP8 pass lives in a caller-owned buffer of this many bytes.
constexpr size_t kFp8PassStateBytes = 256;
size_t fp8_pass_workspace_bytes_int(const Fp8HostProblem* hp, int n, long long M);
int fp8_pass_init_int(void* state, const Fp8HostProblem* hp, int n, long long M, const VerifyRule* vr,
                      void* workspace, size_t workspace_bytes);
int fp8_pass_run_int(const void* state, cudaStream_t s);

// The E4M3-term kernel (fp8q.cu): the codes straight into kind::f8f6f4, the activations as two
// residual E4M3 terms with a power-of-two row scale. Same limits as fp8_supported.
bool fp8q_supported(long long M, long long K);
size_t fp8q_workspace_bytes_int(long long M, long long N, long long K, bool verify);
int launch_fp8q_gemm(const uint16_t* X, const uint8_t* q, const float* scales, long long M, long long N, long long K,
                     void* Y, int y_dtype, void* workspace, cudaStream_t s);
int launch_fp8q_verify(const uint16_t* X, const uint8_t* q, const float* scales, long long M, long long N,
                       long long K, const VerifyRule& v, void* workspace, cudaStream_t s);
// FP8 weight passes on the E4M3-term kernel (state in the same caller-owned handle).
size_t fp8q_pass_workspace_bytes_int(const Fp8HostProblem* hp, int n, long long M);
int fp8q_pass_init_int(void* state, const Fp8HostProblem* hp, int n, long long M, const VerifyRule* vr,
                       void* workspace, size_t workspace_bytes);
int fp8q_pass_run_int(const void* state, cudaStream_t s);
bool fp8q_pass_owns(const void* state);

// fp32 W [N, K] -> E4M3 codes [N, K] and fp32 scales [ceil(N/128), ceil(K/128)].
int launch_fp8_pack(const float* W, long long N, long long K, uint8_t* q, float* scales, cudaStream_t s);

}  // namespace nvfp4ws
