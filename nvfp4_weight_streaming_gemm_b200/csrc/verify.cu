// Stage 2 of the fused greedy verify.
//
// Rule ("TandemLLM", introduction, and its "How it works" flowchart): the target
// checks every drafted token. Drafts are kept up to the first one that differs
// from the target's greedy token, and the target's own token comes next. With
// M = B*(D+1) rows, row b*(D+1)+i holds the target's token for draft slot i of
// sequence b:
//   accept_len[b] = min{ i < D : drafts[b, i] != argmax[b*(D+1) + i] }, else D.
// A draft tree (parents non-null) generalises the chain: node k >= 1 holds
// drafts[b, k-1] under node parents[b, k-1] in [0, k-1]; it is accepted when its
// parent is and its draft equals the argmax at the parent's row; the kept path ends
// at the deepest accepted node (lowest index among equals).
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
                                                                   const VerifyRule v, unsigned int* err) {
  __shared__ float s_v[kS2Threads / 32][kS2Rows];
  __shared__ int s_i[kS2Threads / 32][kS2Rows];
  __shared__ int s_arg[NVFP4WS_MAX_M];
  __shared__ int s_draft[NVFP4WS_MAX_M], s_par[NVFP4WS_MAX_M];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int D = v.D, b = blockIdx.x, R = D + 1, row0 = b * R;
  // Launched as a programmatic dependent of the GEMM that wrote the partials (and the
  // drafts may come from a kernel before it in the stream): read nothing before this.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // Drafts and parents go to shared memory, so the accept walk below reads no global memory.
  for (int k = t; k < D; k += kS2Threads) {
    s_draft[k] = v.drafts[(long long)b * D + k];
    s_par[k] = v.parents ? v.parents[(long long)b * D + k] : k;   // a chain: node k+1 under node k
  }
  int32_t* argmax = v.argmax;
  float* max_logit = v.max_logit;
  for (int r0 = 0; r0 < R; r0 += kS2Rows) {
    const int nr = (R - r0) < kS2Rows ? (R - r0) : kS2Rows;
    float bv[kS2Rows];
    int bi[kS2Rows];
#pragma unroll
    for (int j = 0; j < kS2Rows; ++j) { bv[j] = -INFINITY; bi[j] = INT_MAX; }
    for (int p = t; p < nparts; p += kS2Threads) {
      const float* val = pv + (long long)p * M + row0 + r0;
      const int* ix = pi + (long long)p * M + row0 + r0;
#pragma unroll
      for (int j = 0; j < kS2Rows; ++j) {
        if (j < nr) {
          const float vv = val[j];
          const int ii = ix[j];
          if (argmax_better(vv, ii, bv[j], bi[j])) { bv[j] = vv; bi[j] = ii; }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kS2Rows; ++j) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv[j], o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi[j], o);
        if (argmax_better(ov, oi, bv[j], bi[j])) { bv[j] = ov; bi[j] = oi; }
      }
      if (lane == 0) { s_v[warp][j] = bv[j]; s_i[warp][j] = bi[j]; }
    }
    __syncthreads();
    if (t < nr) {
      float mv = s_v[0][t];
      int mi = s_i[0][t];
      for (int w = 1; w < kS2Threads / 32; ++w)
        if (argmax_better(s_v[w][t], s_i[w][t], mv, mi)) { mv = s_v[w][t]; mi = s_i[w][t]; }
      argmax[row0 + r0 + t] = mi;
      s_arg[r0 + t] = mi;
      if (max_logit) max_logit[row0 + r0 + t] = mv;
    }
    __syncthreads();
  }
  if (t == 0) {
    // Node k's acceptance and depth, in index order (a parent precedes its children).
    int best = 0, best_depth = 0;
    if (!v.parents) {                       // a chain: the first mismatch ends it
      best = D;
      for (int i = 0; i < D; ++i)
        if (s_draft[i] != s_arg[i]) { best = i; break; }
      best_depth = best;
    } else {
      __shared__ unsigned char s_ok[NVFP4WS_MAX_M];
      __shared__ short s_depth[NVFP4WS_MAX_M];
      s_ok[0] = 1;
      s_depth[0] = 0;
      bool bad = false;
      for (int k = 1; k <= D; ++k) {
        const int p = s_par[k - 1];
        if (p < 0 || p >= k) {
          bad = true;
          s_ok[k] = 0;
          s_depth[k] = 0;
          continue;
        }
        s_depth[k] = (short)(s_depth[p] + 1);
        s_ok[k] = (s_ok[p] && s_draft[k - 1] == s_arg[p]) ? 1 : 0;
        if (s_ok[k] && s_depth[k] > best_depth) { best = k; best_depth = s_depth[k]; }
      }
      if (bad) atomicOr(err, kDevErrBadTree);
    }
    v.accept_len[b] = best_depth;
    if (v.accept_node) v.accept_node[b] = best;
  }
}

int launch_verify_stage2(const float* part_val, const int* part_idx, int nparts, int M, const VerifyRule& v,
                         cudaStream_t s) {
  unsigned int* err = device_error_word();
  if (!err) return set_error(NVFP4WS_ERR_CUDA, "cannot resolve the device error word");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)v.B);
  cfg.blockDim = dim3(kS2Threads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, verify_stage2_kernel, part_val, part_idx, nparts, M, v, err);
  if (e != cudaSuccess) return set_error(NVFP4WS_ERR_CUDA, "verify_stage2_kernel launch: %s", cudaGetErrorString(e));
  return check_launch("verify_stage2_kernel");
}

}  // namespace nvfp4ws
