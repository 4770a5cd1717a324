// Stage 2 of the fused greedy verify.
//
// Rule ("TandemLLM", introduction, and its "How it works" flowchart): the target
// checks every drafted token. Drafts are kept up to the first one that differs
// from the target's greedy token, and the target's own token comes next. With
// M = B*(D+1) rows, row b*(D+1)+i holds the target's token for draft slot i of
// sequence b:
//   accept_len[b] = min{ i < D : drafts[b, i] != argmax[b*(D+1) + i] }, else D.
// One CTA: a fixed-order reduction of the per-CTA (max, lowest index) partials
// for every row, then one thread per sequence for the accept length.
#include "common.cuh"
#include "kernels.h"

#include <climits>
#include <cmath>

namespace nvfp4ws {

__global__ void __launch_bounds__(256) verify_stage2_kernel(const float* __restrict__ pv,
                                                            const int* __restrict__ pi, int nparts, int M,
                                                            const int32_t* __restrict__ drafts, int B, int D,
                                                            int32_t* __restrict__ argmax,
                                                            int32_t* __restrict__ accept_len,
                                                            float* __restrict__ max_logit) {
  __shared__ int s_arg[NVFP4WS_MAX_M];
  __shared__ float s_v[8];
  __shared__ int s_i[8];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  for (int m = 0; m < M; ++m) {
    float bv = -INFINITY;
    int bi = INT_MAX;
    for (int p = t; p < nparts; p += blockDim.x) {
      const float v = pv[(long long)p * M + m];
      const int i = pi[(long long)p * M + m];
      if (argmax_better(v, i, bv, bi)) { bv = v; bi = i; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float v = __shfl_xor_sync(0xffffffffu, bv, o);
      const int i = __shfl_xor_sync(0xffffffffu, bi, o);
      if (argmax_better(v, i, bv, bi)) { bv = v; bi = i; }
    }
    if (lane == 0) { s_v[warp] = bv; s_i[warp] = bi; }
    __syncthreads();
    if (t == 0) {
      for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
        if (argmax_better(s_v[w], s_i[w], bv, bi)) { bv = s_v[w]; bi = s_i[w]; }
      argmax[m] = bi;
      s_arg[m] = bi;
      if (max_logit) max_logit[m] = bv;
    }
    __syncthreads();
  }
  for (int b = t; b < B; b += blockDim.x) {
    int L = D;
    for (int i = 0; i < D; ++i) {
      if (drafts[(long long)b * D + i] != s_arg[b * (D + 1) + i]) { L = i; break; }
    }
    accept_len[b] = L;
  }
}

int launch_verify_stage2(const float* part_val, const int* part_idx, int nparts, int M,
                         const int32_t* drafts, int B, int D, int32_t* argmax, int32_t* accept_len,
                         float* max_logit, cudaStream_t s) {
  verify_stage2_kernel<<<1, 256, 0, s>>>(part_val, part_idx, nparts, M, drafts, B, D, argmax, accept_len,
                                         max_logit);
  return check_launch("verify_stage2_kernel");
}

}  // namespace nvfp4ws
