// Internal interface of the tcgen05 tensor-core path (not part of the C ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"

namespace nvfp4ws {

bool mma_supported(long long M, long long K);
int mma_min_m();
size_t mma_gemm_workspace_bytes(long long M, long long N, long long K);
// Bytes of ticket counters at the start of the GEMM workspace (must be zero on entry).
size_t mma_gemm_counter_bytes(long long M, long long N, long long K);
size_t mma_verify_workspace_bytes(long long M, long long N, long long K);
int launch_mma_gemm(const uint16_t* X, const uint8_t* q, const uint8_t* sf, const float* ts, long long M, long long N,
                    long long K, void* Y, int y_dtype, void* workspace, size_t workspace_bytes, cudaStream_t s);
int launch_mma_verify(const uint16_t* X, const uint8_t* q, const uint8_t* sf, const float* ts, long long M,
                      long long N, long long K, const VerifyRule& v, void* workspace, cudaStream_t s);

// Block-scaled (kind::mxf4nvf4) path: activations as residual NVFP4 terms, kGemmTerms of them
// for a GEMM and kVerifyTerms for the verify; kGemmTermsFast for the GEMMs of a pass that asks
// for them (NVFP4WS_PASS_FOUR_TERMS); or (terms = 1) one NVFP4 quantisation per row: the W4A4
// product.
constexpr int kGemmTerms = 5;
constexpr int kVerifyTerms = 5;
constexpr int kGemmTermsFast = 4;
bool mxf4_supported(long long M, long long K, int terms = kGemmTerms);
size_t mxf4_workspace_bytes(long long M, long long N, long long K, int terms = kGemmTerms);
int launch_mxf4_gemm(const uint16_t* X, const uint8_t* q, const uint8_t* sf, const float* ts, long long M,
                     long long N, long long K, void* Y, int y_dtype, void* workspace, cudaStream_t s,
                     int terms = kGemmTerms);
int launch_mxf4_verify(const uint16_t* X, const uint8_t* q, const uint8_t* sf, const float* ts, long long M,
                       long long N, long long K, const VerifyRule& v, void* workspace, cudaStream_t s);

// A list of GEMMs sharing M, run by one persistent launch (a weight pass).
struct MxHostProblem {
  const uint16_t* X;
  const uint8_t* q;
  const uint8_t* sf;
  const float* ts;
  long long N, K;
  void* Y;
  int y_bf16, verify;
};
// Host state of an initialised pass lives in a caller-owned buffer of this many bytes.
constexpr size_t kMxPassStateBytes = 256;
// binv: a batch-invariant pass (one unit shape for every M). terms: activation terms of the
// GEMMs (kGemmTerms, kGemmTermsFast, or 1 for a W4A4 pass, which runs no verify); a verify
// problem, which must be the last, always takes kVerifyTerms.
size_t mxf4_pass_workspace_bytes(const MxHostProblem* hp, int n, long long M, bool binv, int terms);
int mxf4_pass_init(void* state, const MxHostProblem* hp, int n, long long M, const VerifyRule* vs, bool binv,
                   int terms, void* workspace, size_t workspace_bytes);
int mxf4_pass_run(const void* state, cudaStream_t s);

}  // namespace nvfp4ws
