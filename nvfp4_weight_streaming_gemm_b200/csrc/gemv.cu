// CUDA-core streaming GEMV for small M:
//   y[m, n] = ts * sum_b S[n, b] * sum_{k in block b} x[m, k] * e2m1(code[n, k])
//
// Why this shape. At M = 1 a weight pass streams ~0.56 bytes per element and does
// 2 flops per element: it is HBM-bound by a factor of ~500 ("veloGB10",
// "Unique aspects: Engineered to the roofline": "~94% GEMM and
// weight-bandwidth-bound"). The only arithmetic that matters is keeping the
// dequantisation ahead of HBM. On B200 the cheapest exact form measured was a
// hardware E2M1x2 -> f16x2 conversion followed by mixed f16 x f16 -> f32 FMAs.
//
// Mapping. The threads of a CTA span K. Thread t owns the 32-element chunks
// c = t + j*T (j < CPT, T = blockDim.x). Its slice of X stays in registers as
// f16x2 for the whole kernel. A CTA walks row groups of R rows, grid-stride. For
// each row it loads one 16-byte nibble word per chunk
// (ld.global.nc.L1::no_allocate) and one 2-byte scale pair. The next group is
// prefetched into registers while the current one is computed. Per-row partial
// sums are reduced with warp shuffles, then across warps through shared memory,
// in a fixed order. The result is deterministic and uses no atomics.
//
// In verify mode the reducing thread of each token keeps a running (max, lowest
// index) over the rows the CTA visits, and writes one partial per CTA. Logits
// never reach HBM.
#include "common.cuh"
#include "kernels.h"
#include "sync.cuh"

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>

namespace nvfp4ws {

// x[m][k] as raw bf16 pairs: thread t owns the 32-element chunks t + j*T of rows m0..m0+MT-1.
template <int MT, int CPT>
__device__ __forceinline__ void load_x_rows(const GemvArgs& a, int t, int T, int C, uint32_t (&xr)[MT][CPT][16]) {
#pragma unroll
  for (int m = 0; m < MT; ++m) {
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      const int c = t + j * T;
      const int mm = a.m0 + m;
      if (c < C && mm < a.M) {
        const uint4* src = reinterpret_cast<const uint4*>(a.X + (long long)mm * a.K + (long long)c * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 b = src[v];
          xr[m][j][4 * v + 0] = b.x;
          xr[m][j][4 * v + 1] = b.y;
          xr[m][j][4 * v + 2] = b.z;
          xr[m][j][4 * v + 3] = b.w;
        }
      } else {
#pragma unroll
        for (int v = 0; v < 16; ++v) xr[m][j][v] = 0u;
      }
    }
  }
}

// Each row's power-of-two shift (row_shift_of_amax) from the amax over the threads that hold
// it: warp shuffles, then one value per warp in `red` between two barriers (`sync`).
template <int MT, int CPT, typename Sync>
__device__ __forceinline__ void row_shifts(const uint32_t (&xr)[MT][CPT][16], float* red, int lane, int warp,
                                           int nwarps, int (&xe)[MT], Sync sync) {
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float v = 0.f;
#pragma unroll
    for (int j = 0; j < CPT; ++j)
#pragma unroll
      for (int e = 0; e < 16; ++e) v = fmaxf(v, bf16x2_absmax(xr[m][j][e]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[warp * MT + m] = v;
  }
  sync();
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float v = 0.f;
    for (int w = 0; w < nwarps; ++w) v = fmaxf(v, red[w * MT + m]);
    xe[m] = row_shift_of_amax(v);
  }
  sync();                                        // `red` is reused by the caller
}

template <int MT, int CPT>
__device__ __forceinline__ void convert_x_rows(uint32_t (&xr)[MT][CPT][16], const int (&xe)[MT]) {
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int j = 0; j < CPT; ++j)
#pragma unroll
      for (int v = 0; v < 16; ++v) xr[m][j][v] = bf16x2_to_f16x2_shifted(xr[m][j][v], xe[m]);
}

// xe[m] for a run-time m < MT without dynamic register indexing.
template <int MT>
__device__ __forceinline__ int pick(const int (&xe)[MT], int m) {
  int r = xe[0];
#pragma unroll
  for (int k = 1; k < MT; ++k) r = (m == k) ? xe[k] : r;
  return r;
}

template <int MT, int CPT, int R, bool VERIFY>
__global__ void __launch_bounds__(512) gemv_kernel(GemvArgs a) {
  const int T = blockDim.x;
  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5, nwarps = T >> 5;
  const int C = a.K >> 5;                       // 32-element chunks per row
  const long long rowq = a.K >> 1;              // bytes of q per row
  const long long rows = a.K >> 4;              // bytes of sf per row

  // X slice -> registers, zero outside [0, C) and beyond M; then each row's shift from its
  // amax (every CTA holds whole rows) and the conversion to f16x2
  extern __shared__ float red[];                // [2][nwarps][R][MT]
  uint32_t xr[MT][CPT][16];
  int xe[MT];
  load_x_rows<MT, CPT>(a, t, T, C, xr);
  row_shifts<MT>(xr, red, lane, warp, nwarps, xe, [] { __syncthreads(); });
  convert_x_rows<MT, CPT>(xr, xe);
  const float ts = *a.ts;
  const int ngroups = (int)((a.N + R - 1) / R);

  float bestv = -INFINITY;
  int besti = INT_MAX;

  uint4 cur[R][CPT];
  uint32_t curs[R][CPT];

  auto load_group = [&](int g, uint4 (&qv)[R][CPT], uint32_t (&sv)[R][CPT]) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const long long n = (long long)g * R + r;
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const int c = t + j * T;
        if (n < a.N && c < C) {
          qv[r][j] = ld_stream_v4(a.q + n * rowq + (long long)c * 16);
          sv[r][j] = ld_stream_u16(a.sf + n * rows + (long long)c * 2);
        } else {
          qv[r][j] = make_uint4(0, 0, 0, 0);
          sv[r][j] = 0u;
        }
      }
    }
  };

  int g = blockIdx.x;
  if (g < ngroups) load_group(g, cur, curs);
  int buf = 0;
  for (; g < ngroups; g += gridDim.x) {
    uint4 nxt[R][CPT];
    uint32_t nxts[R][CPT];
    const int gn = g + gridDim.x;
    if (gn < ngroups) load_group(gn, nxt, nxts);

    float acc[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;

#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const uint32_t s2 = e4m3x2_to_f16x2(curs[r][j]);
        const float S0 = f16lo_to_f32(s2), S1 = f16hi_to_f32(s2);
        const uint32_t w[4] = {cur[r][j].x, cur[r][j].y, cur[r][j].z, cur[r][j].w};
        uint32_t h[16];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int b = 0; b < 4; ++b) h[4 * i + b] = e2m1x2_to_f16x2(w[i] >> (8 * b));
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) dot2_f16_f32(p0, p1, h[e], xr[m][j][e]);
#pragma unroll
          for (int e = 8; e < 16; ++e) dot2_f16_f32(p2, p3, h[e], xr[m][j][e]);
          acc[r][m] = fmaf(S0, p0 + p1, acc[r][m]);
          acc[r][m] = fmaf(S1, p2 + p3, acc[r][m]);
        }
      }
    }

    // reduce over the CTA: shuffles within each warp, then warps in order
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float v = acc[r][m];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[((buf * nwarps + warp) * R + r) * MT + m] = v;
      }
    __syncthreads();
    if constexpr (!VERIFY) {
      if (t < R * MT) {
        const int r = t / MT, m = t - r * MT;
        const long long n = (long long)g * R + r;
        const int mm = a.m0 + m;
        if (n < a.N && mm < a.M) {
          float s = 0.f;
          for (int w = 0; w < nwarps; ++w) s += red[((buf * nwarps + w) * R + r) * MT + m];
          const float y = mul_pow2(s * ts, pick<MT>(xe, m));
          if (a.y_bf16)
            reinterpret_cast<uint16_t*>(a.Y)[(long long)mm * a.N + n] = f32_to_bf16_rn(y);
          else
            reinterpret_cast<float*>(a.Y)[(long long)mm * a.N + n] = y;
        }
      }
    } else {
      if (t < MT) {
        const int et = pick<MT>(xe, t);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const long long n = (long long)g * R + r;
          if (n < a.N) {
            float s = 0.f;
            for (int w = 0; w < nwarps; ++w) s += red[((buf * nwarps + w) * R + r) * MT + t];
            const float y = mul_pow2(s * ts, et);
            if (argmax_better(y, (int)n, bestv, besti)) { bestv = y; besti = (int)n; }
          }
        }
      }
    }
    buf ^= 1;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int j = 0; j < CPT; ++j) { cur[r][j] = nxt[r][j]; curs[r][j] = nxts[r][j]; }
  }
  if constexpr (VERIFY) {
    if (t < MT && a.m0 + t < a.M) {
      a.part_val[(long long)blockIdx.x * a.M + a.m0 + t] = bestv;
      a.part_idx[(long long)blockIdx.x * a.M + a.m0 + t] = besti;
    }
  }
}

// ---------------------------------------------------------------------------
// Bulk-copy-staged variant (K % 256 == 0). One CTA per SM: T compute threads
// that span K as above, plus one producer warp. The producer copies RG whole
// rows per stage (RG*K/2 bytes of nibbles and RG*K/16 bytes of scales, each one
// contiguous range) with cp.async.bulk into an mbarrier ring of up to 8 stages.
// That keeps 100-190 KB of weights in flight per SM without spending registers
// on prefetch.
// ---------------------------------------------------------------------------

template <int MT, int CPT, int RG>
__global__ void __launch_bounds__(544, 1) gemv_staged_kernel(GemvArgs a, int stages, uint32_t stage_bytes) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int T = (int)blockDim.x - 32;           // compute threads (multiple of 32)
  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5, nwarps = T >> 5;
  const int C = (int)(a.K >> 5);
  const long long rowq = a.K >> 1, rows = a.K >> 4;
  const int ngroups = (int)((a.N + RG - 1) / RG);
  const int S = stages;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)S * stage_bytes);
  volatile int* s_abort = reinterpret_cast<volatile int*>(bars + 2 * S);
  float* red = reinterpret_cast<float*>(bars + 2 * S + 2);     // [2][nwarps][RG][MT]
  auto bar_full = [&](int s) { return smem_u32(bars + s); };
  auto bar_empty = [&](int s) { return smem_u32(bars + S + s); };

  if (t == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(bar_full(s), 1); mbar_init(bar_empty(s), nwarps); }
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == nwarps) {
    // ---------------- producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int i = 0;
      for (int g = blockIdx.x; g < ngroups; g += gridDim.x, ++i) {
        const int s = i % S;
        if (!mbar_wait(bar_empty(s), ((uint32_t)(i / S) & 1u) ^ 1u, s_abort, a.err)) break;
        const long long n0 = (long long)g * RG;
        const long long nr = (a.N - n0 < RG) ? (a.N - n0) : RG;
        uint8_t* st = smem + (size_t)s * stage_bytes;
        mbar_arrive_expect_tx(bar_full(s), (uint32_t)(nr * rowq + nr * rows));
        bulk_load(smem_u32(st), a.q + n0 * rowq, (uint32_t)(nr * rowq), bar_full(s), pol);
        bulk_load(smem_u32(st + RG * rowq), a.sf + n0 * rows, (uint32_t)(nr * rows), bar_full(s), pol);
      }
      if (*s_abort) {                            // drain the copies still in flight (bounded)
        for (int k = (i > S ? i - S : 0); k < i; ++k) {
          const unsigned long long t0 = globaltimer();
          while (!mbar_try_wait(bar_full(k % S), (uint32_t)(k / S) & 1u) && globaltimer() - t0 < kWaitLimitNs) {}
        }
      }
    }
    return;    // the producer warp takes no part in the compute threads' named barriers
  }

  // ---------------- compute threads
  uint32_t xr[MT][CPT][16];
  int xe[MT];
  load_x_rows<MT, CPT>(a, t, T, C, xr);
  row_shifts<MT>(xr, red, lane, warp, nwarps, xe, [T] { named_bar(1, T); });
  convert_x_rows<MT, CPT>(xr, xe);
  const float ts = *a.ts;
  float bestv = -INFINITY;
  int besti = INT_MAX;
  int buf = 0, i = 0;
  for (int g = blockIdx.x; g < ngroups; g += gridDim.x, ++i) {
    const int s = i % S;
    if (!mbar_wait(bar_full(s), (uint32_t)(i / S) & 1u, s_abort, a.err)) break;
    const uint8_t* st = smem + (size_t)s * stage_bytes;
    float acc[RG][MT];
#pragma unroll
    for (int r = 0; r < RG; ++r) {
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        const int c = t + j * T;
        if (c < C && (long long)g * RG + r < a.N) {
          const uint4 w4 = *reinterpret_cast<const uint4*>(st + r * rowq + (long long)c * 16);
          const uint32_t sc = *reinterpret_cast<const uint16_t*>(st + RG * rowq + r * rows + (long long)c * 2);
          const uint32_t s2 = e4m3x2_to_f16x2(sc);
          const float S0 = f16lo_to_f32(s2), S1 = f16hi_to_f32(s2);
          const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
          uint32_t h[16];
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int b = 0; b < 4; ++b) h[4 * q + b] = e2m1x2_to_f16x2(w[q] >> (8 * b));
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) dot2_f16_f32(p0, p1, h[e], xr[m][j][e]);
#pragma unroll
            for (int e = 8; e < 16; ++e) dot2_f16_f32(p2, p3, h[e], xr[m][j][e]);
            acc[r][m] = fmaf(S0, p0 + p1, acc[r][m]);
            acc[r][m] = fmaf(S1, p2 + p3, acc[r][m]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty(s));      // this warp is done reading the stage
#pragma unroll
    for (int r = 0; r < RG; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float v = acc[r][m];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[((buf * nwarps + warp) * RG + r) * MT + m] = v;
      }
    named_bar(1, T);
    if (!a.verify) {
      if (t < RG * MT) {
        const int r = t / MT, m = t - r * MT;
        const long long n = (long long)g * RG + r;
        const int mm = a.m0 + m;
        if (n < a.N && mm < a.M) {
          float sum = 0.f;
          for (int w = 0; w < nwarps; ++w) sum += red[((buf * nwarps + w) * RG + r) * MT + m];
          const float y = mul_pow2(sum * ts, pick<MT>(xe, m));
          if (a.y_bf16)
            reinterpret_cast<uint16_t*>(a.Y)[(long long)mm * a.N + n] = f32_to_bf16_rn(y);
          else
            reinterpret_cast<float*>(a.Y)[(long long)mm * a.N + n] = y;
        }
      }
    } else if (t < MT) {
      const int et = pick<MT>(xe, t);
#pragma unroll
      for (int r = 0; r < RG; ++r) {
        const long long n = (long long)g * RG + r;
        if (n < a.N) {
          float sum = 0.f;
          for (int w = 0; w < nwarps; ++w) sum += red[((buf * nwarps + w) * RG + r) * MT + t];
          const float y = mul_pow2(sum * ts, et);
          if (argmax_better(y, (int)n, bestv, besti)) { bestv = y; besti = (int)n; }
        }
      }
    }
    buf ^= 1;
  }
  if (a.verify && t < MT && a.m0 + t < a.M) {
    a.part_val[(long long)blockIdx.x * a.M + a.m0 + t] = bestv;
    a.part_idx[(long long)blockIdx.x * a.M + a.m0 + t] = besti;
  }
}

// ---------------------------------------------------------------------------
// Host side: pick (MT, CPT, R, T) and the grid
// ---------------------------------------------------------------------------

template <int MT, int CPT, int R, bool VERIFY>
static int launch_one(const GemvArgs& a, int T, int grid, cudaStream_t s) {
  const int nwarps = T / 32;
  const size_t smem = sizeof(float) * 2 * nwarps * R * MT;
  gemv_kernel<MT, CPT, R, VERIFY><<<grid, T, smem, s>>>(a);
  return check_launch("gemv_kernel");
}

template <int MT, int CPT, int R, bool VERIFY>
static int occupancy_of(int T) {
  const int nwarps = T / 32;
  const size_t smem = sizeof(float) * 2 * nwarps * R * MT;
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, gemv_kernel<MT, CPT, R, VERIFY>, T, smem) != cudaSuccess)
    return 1;
  return std::max(nb, 1);
}

template <int MT, int CPT, int RG>
static int launch_staged(const GemvArgs& a, const GemvPlan& p, cudaStream_t s) {
  static std::atomic<bool> attr[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(gemv_staged_kernel<MT, CPT, RG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024) != cudaSuccess)
      return check_launch("cudaFuncSetAttribute(gemv_staged_kernel)");
    attr[dev].store(true, std::memory_order_release);
  }
  gemv_staged_kernel<MT, CPT, RG><<<p.grid, p.threads, p.smem, s>>>(a, p.stages, p.stage_bytes);
  return check_launch("gemv_staged_kernel");
}

GemvPlan gemv_plan(long long M, long long N, long long K, bool regs_only) {
  GemvPlan p{};
  const int C = (int)(K / 32);
  p.cpt = C <= 512 ? 1 : (C <= 1024 ? 2 : 4);
  int per = (C + p.cpt - 1) / p.cpt;
  const int T = std::max(32, ((per + 31) / 32) * 32);
  const int sms = std::max(1, device_sm_count());
  p.staged = (K % 256 == 0) && !regs_only;
  if (p.staged) {
    p.mt = (M >= 2 && p.cpt <= 2) ? 2 : 1;
    p.rows = K <= 8192 ? 8 : (K <= 16384 ? 4 : 2);
    p.threads = T + 32;
    p.stage_bytes = (unsigned int)(p.rows * (K / 2) + p.rows * (K / 16));
    p.stage_bytes = (p.stage_bytes + 127) / 128 * 128;
    p.stages = (int)std::min<long long>(8, (200 * 1024) / p.stage_bytes);
    if (p.stages < 2) { p.staged = 0; }
    const size_t tail = 16 * 8 + 16 + 2 * (size_t)(T / 32) * p.rows * p.mt * 4;
    p.smem = (size_t)p.stages * p.stage_bytes + tail + 128;
    const long long ngroups = (N + p.rows - 1) / p.rows;
    p.grid = (int)std::max<long long>(1, std::min<long long>(ngroups, sms));
    if (p.staged) return p;
  }
  p.threads = T;
  p.mt = (M >= 4 && p.cpt == 1) ? 4 : (M >= 2 && p.cpt <= 2 ? 2 : 1);
  p.rows = p.cpt == 1 ? 4 : (p.cpt == 2 ? 2 : 1);
  int occ = 1;
#define OCC(MT_, CPT_, R_) if (p.mt == MT_ && p.cpt == CPT_) occ = occupancy_of<MT_, CPT_, R_, true>(p.threads);
  OCC(1, 1, 4) OCC(1, 2, 2) OCC(1, 4, 1) OCC(2, 1, 4) OCC(2, 2, 2) OCC(4, 1, 4)
#undef OCC
  const long long ngroups = (N + p.rows - 1) / p.rows;
  p.grid = (int)std::max<long long>(1, std::min<long long>(ngroups, (long long)sms * occ));
  return p;
}

bool gemv_supported(long long K) { return K % 32 == 0 && K / 32 <= 2048; }

int launch_gemv(const GemvArgs& base, bool verify, bool regs_only, cudaStream_t s) {
  const GemvPlan p = gemv_plan(base.M, base.N, base.K, regs_only);
  for (long long m0 = 0; m0 < base.M;) {
    GemvArgs a = base;
    a.m0 = (int)m0;
    a.verify = verify ? 1 : 0;
    a.err = device_error_word();
    const long long left = base.M - m0;
    int mt = p.mt;
    while (mt > 1 && mt > left) mt >>= 1;
    int e = 0;
    if (p.staged) {
#define LS(MT_, CPT_, RG_)                                                              \
  if (mt == MT_ && p.cpt == CPT_ && p.rows == RG_) { e = launch_staged<MT_, CPT_, RG_>(a, p, s); } else
      LS(1, 1, 8) LS(2, 1, 8) LS(1, 1, 4) LS(2, 1, 4) LS(1, 2, 4) LS(2, 2, 4) LS(1, 2, 2) LS(2, 2, 2)
      LS(1, 4, 2) LS(1, 4, 4) LS(1, 1, 2) LS(2, 1, 2) {
        return set_error(NVFP4WS_ERR_UNSUPPORTED, "no staged GEMV variant for mt=%d cpt=%d rg=%d", mt, p.cpt,
                         p.rows);
      }
#undef LS
    } else {
#define L(MT_, CPT_, R_)                                                              \
  if (mt == MT_ && p.cpt == CPT_) {                                                   \
    e = verify ? launch_one<MT_, CPT_, R_, true>(a, p.threads, p.grid, s)             \
               : launch_one<MT_, CPT_, R_, false>(a, p.threads, p.grid, s);           \
  } else
      L(1, 1, 4) L(1, 2, 2) L(1, 4, 1) L(2, 1, 4) L(2, 2, 2) L(4, 1, 4) {
        return set_error(NVFP4WS_ERR_UNSUPPORTED, "no GEMV variant for mt=%d cpt=%d", mt, p.cpt);
      }
#undef L
    }
    if (e) return e;
    m0 += mt;
  }
  return NVFP4WS_OK;
}

}  // namespace nvfp4ws
