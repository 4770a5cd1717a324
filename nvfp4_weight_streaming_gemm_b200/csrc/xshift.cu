// Per-row power-of-two shifts of bf16 activations for the kernels that multiply in f16
// (the f16 tensor-core GEMM and the FP8 GEMM). Their CTAs see X one K-slice at a time, so
// the row's amax comes from this small kernel first: one CTA per row, one reduction, and
// xe[m] = row_shift_of_amax(amax|x[m, :]|) (see common.cuh). The GEMM then converts
// x * 2^-xe[m] to f16, which is exact and never saturates, and multiplies its result
// by 2^xe[m].
#include "common.cuh"
#include "kernels.h"

namespace nvfp4ws {

constexpr int kShiftThreads = 256;

__global__ void __launch_bounds__(kShiftThreads) x_shift_kernel(const uint16_t* X, long long K, int* xe) {
  const int m = blockIdx.x, t = threadIdx.x;
  const uint32_t* row = reinterpret_cast<const uint32_t*>(X + (long long)m * K);   // bf16 pairs
  float v = 0.f;
  for (long long i = t; i < K / 2; i += kShiftThreads) v = fmaxf(v, bf16x2_absmax(__ldg(row + i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __shared__ float s_red[kShiftThreads / 32];
  if ((t & 31) == 0) s_red[t >> 5] = v;
  __syncthreads();
  if (t == 0) {
    float a = 0.f;
    for (int w = 0; w < kShiftThreads / 32; ++w) a = fmaxf(a, s_red[w]);
    xe[m] = row_shift_of_amax(a);
  }
}

int launch_row_shifts(const uint16_t* X, long long M, long long K, int* xe, cudaStream_t s) {
  x_shift_kernel<<<(unsigned)M, kShiftThreads, 0, s>>>(X, K, xe);
  return check_launch("x_shift_kernel");
}

}  // namespace nvfp4ws
