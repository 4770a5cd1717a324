// Internal launch interfaces of libnvfp4ws (not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4ws {

struct GemvArgs {
  const uint16_t* X;        // bf16 [M, K]
  const uint8_t* q;         // [N, K/2]
  const uint8_t* sf;        // [N, K/16]
  const float* ts;          // [1]
  long long M, N, K;
  int m0;                   // first token of this launch
  void* Y;                  // [M, N] (GEMM mode)
  int y_bf16;
  float* part_val;          // [grid, M] (verify mode)
  int* part_idx;            // [grid, M]
  int verify;               // staged kernel: write argmax partials instead of Y
  unsigned int* err;        // device error word (bounded waits)
};

struct GemvPlan {
  int mt, cpt, rows, threads, grid;
  int staged;               // 1: bulk-copy-staged kernel (threads includes the producer warp)
  int stages;
  unsigned int stage_bytes;
  size_t smem;
};

GemvPlan gemv_plan(long long M, long long N, long long K, bool regs_only);
bool gemv_supported(long long K);
int launch_gemv(const GemvArgs& a, bool verify, bool regs_only, cudaStream_t s);

// xe[m] = the power-of-two shift of activation row m (bf16 [M, K], K even) that the f16
// kernels apply before converting it (row_shift_of_amax in common.cuh).
int launch_row_shifts(const uint16_t* X, long long M, long long K, int* xe, cudaStream_t s);

int launch_pack(const float* W, long long N, long long K, uint8_t* q, uint8_t* sf, float* ts,
                const float* ts_in, cudaStream_t s);

// The verify's inputs and outputs: drafts [B, D]; parents [B, D] (node k >= 1 hangs
// under parents[b, k-1]) or null for a chain; argmax [M], accept_len [B], and the
// kept path's end node accept_node [B] and the winning logits max_logit [M] (both
// optional, null to skip).
struct VerifyRule {
  const int32_t* drafts;
  const int32_t* parents;
  int B, D;
  int32_t* argmax;
  int32_t* accept_len;
  int32_t* accept_node;
  float* max_logit;
};

// Stage 2 of the verify: reduce per-CTA (max, index) partials to argmax[M], then
// the accept length (and end node) of every sequence.
int launch_verify_stage2(const float* part_val, const int* part_idx, int nparts, int M, const VerifyRule& v,
                         cudaStream_t s);

}  // namespace nvfp4ws
