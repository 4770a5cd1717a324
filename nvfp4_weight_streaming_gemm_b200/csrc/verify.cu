// Stage 2 of the fused greedy verify.
//
// Rule ("TandemLLM", introduction, and its "How it works" flowchart): the target
// checks every drafted token. Drafts are kept up to the first one that differs
// from the target's greedy token, and the target's own token comes next. With
// M = B*(D+1) rows, row b*(D+1)+i holds the target's token for draft slot i of
// sequence b:
//   accept_len[b] = min{ i < D : drafts[b, i] != argmax[b*(D+1) + i] }, else D.
// One CTA per sequence b: it reduces the per-tile (max, lowest index) partials of its
// D+1 rows, 16 rows at a time, each thread reading every row of a partial together
// (they are contiguous), then computes that sequence's accept length. The (value,
// lowest index) order is total, so the result does not depend on reduction order.
#include "common.cuh"
#include "kernels.h"

#include <climits>
#include <cmath>

namespace nvfp4ws {

constexpr int kS2Threads = 512;
constexpr int kS2Rows = 16;

__global__ void __launch_bounds__(kS2Threads) verify_stage2_kernel(const float* __restrict__ pv,
                                                                   const int* __restrict__ pi, int nparts, int M,
                                                                   const int32_t* __restrict__ drafts, int B, int D,
                                                                   int32_t* __restrict__ argmax,
                                                                   int32_t* __restrict__ accept_len,
                                                                   float* __restrict__ max_logit) {
  // Launched as a programmatic dependent of the GEMM that wrote the partials.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float s_v[kS2Threads / 32][kS2Rows];
  __shared__ int s_i[kS2Threads / 32][kS2Rows];
  __shared__ int s_arg[NVFP4WS_MAX_M];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int b = blockIdx.x, R = D + 1, row0 = b * R;
  for (int r0 = 0; r0 < R; r0 += kS2Rows) {
    const int nr = (R - r0) < kS2Rows ? (R - r0) : kS2Rows;
    float bv[kS2Rows];
    int bi[kS2Rows];
#pragma unroll
    for (int j = 0; j < kS2Rows; ++j) { bv[j] = -INFINITY; bi[j] = INT_MAX; }
    for (int p = t; p < nparts; p += kS2Threads) {
      const float* v = pv + (long long)p * M + row0 + r0;
      const int* ix = pi + (long long)p * M + row0 + r0;
#pragma unroll
      for (int j = 0; j < kS2Rows; ++j) {
        if (j < nr) {
          const float vv = v[j];
          const int ii = ix[j];
          if (argmax_better(vv, ii, bv[j], bi[j])) { bv[j] = vv; bi[j] = ii; }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kS2Rows; ++j) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float v = __shfl_xor_sync(0xffffffffu, bv[j], o);
        const int i = __shfl_xor_sync(0xffffffffu, bi[j], o);
        if (argmax_better(v, i, bv[j], bi[j])) { bv[j] = v; bi[j] = i; }
      }
      if (lane == 0) { s_v[warp][j] = bv[j]; s_i[warp][j] = bi[j]; }
    }
    __syncthreads();
    if (t < nr) {
      float v = s_v[0][t];
      int i = s_i[0][t];
      for (int w = 1; w < kS2Threads / 32; ++w)
        if (argmax_better(s_v[w][t], s_i[w][t], v, i)) { v = s_v[w][t]; i = s_i[w][t]; }
      argmax[row0 + r0 + t] = i;
      s_arg[r0 + t] = i;
      if (max_logit) max_logit[row0 + r0 + t] = v;
    }
    __syncthreads();
  }
  if (t == 0) {
    int L = D;
    for (int i = 0; i < D; ++i) {
      if (drafts[(long long)b * D + i] != s_arg[i]) { L = i; break; }
    }
    accept_len[b] = L;
  }
}

int launch_verify_stage2(const float* part_val, const int* part_idx, int nparts, int M,
                         const int32_t* drafts, int B, int D, int32_t* argmax, int32_t* accept_len,
                         float* max_logit, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)B);
  cfg.blockDim = dim3(kS2Threads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, verify_stage2_kernel, part_val, part_idx, nparts, M, drafts, B, D, argmax,
                                     accept_len, max_logit);
  if (e != cudaSuccess) return set_error(NVFP4WS_ERR_CUDA, "verify_stage2_kernel launch: %s", cudaGetErrorString(e));
  return check_launch("verify_stage2_kernel");
}

}  // namespace nvfp4ws
