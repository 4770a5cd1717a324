// FP8 (E4M3, 128 x 128 block-scaled) weight GEMM on tcgen05 kind::f8f6f4: the codes are the
// MMA's A operand straight from shared memory, and the bf16 activations are written as residual
// E4M3 terms, the MMA's B operand.
//
//   Y[m, n] = sum_kb s[n / 128, kb] * g[m] * sum_t 16^-t * sum_{k in kb} c_t[m, k] * e4m3(code[n, k])
//
// Why. One kind::f16 MMA (M=128, K=16) costs about as much as its weights take to stream at
// full clock, so the dequantising kernel (fp8.cu) is bound by MMA issue. kind::f8f6f4 takes
// K = 32 per instruction from the packed codes, with no per-element work on the CUDA cores.
//
// Activation terms. Per row, g = 2^(e - 8) with amax|x| = f * 2^e (f in [0.5, 1)), so |x|/g is
// below 256 and x/g keeps bf16's 8 significant bits. Term t takes c_t = E4M3_rn(r_t * 16^t),
// r_0 = x/g, r_{t+1} = r_t - 16^-t * c_t: each term takes the next 4 of those bits, so two
// terms hold x exactly unless E4M3's subnormal step (2^-9 in term 0's units) cuts the second,
// and the rest is below 2^-14 g. The terms are extra B rows (token m, term t -> row m*T + t);
// the epilogue folds them with exact power-of-two weights before the block scale, and applies
// g at the end.
//
// One GEMM, or a whole list of them (an FP8 weight pass) in one persistent launch, as fp8.cu.
//
// Roles per CTA (one persistent CTA per SM, 8 warps):
//   warp 0        TMA producer: the unit's 16 KB code tiles (2-D, 128-byte swizzle) and the
//                 matching term images (one contiguous bulk copy each; the prep kernel wrote
//                 them in the shared-memory operand layout). No multicast.
//   warp 1        TMEM allocator and MMA issuer: 4 x kind::f8f6f4 (K = 32) per block, each
//                 block into its own P of one of np rotating P sets.
//   warps 4-11    promotion and epilogue, as in fp8.cu: two warpgroups, each lane quarter's rows
//                 served by two warps that take alternate groups of 16 tokens (the promotion's
//                 TMEM round trips grow with M).
// Scheduling, split tiles and bounded waits are those of fp8.cu.
#include "common.cuh"
#include "fp8.h"
#include "kernels.h"
#include "sync.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstring>
#include <vector>

namespace nvfp4ws {
namespace fp8q {

constexpr int kThreads = 384;
constexpr int kEpiThreads = 256;                     // warps 4-11
constexpr int kTileRows = 128;
constexpr int kKB = kFp8Block;                       // K elements of one scale block
constexpr uint32_t kWBytes = kTileRows * kKB;        // 16 KB of codes per block
constexpr int kT = 2;                                // activation terms
constexpr int kMaxM = 128;
constexpr int kMaxP = 4;
constexpr int kMaxStages = 8;
constexpr size_t kTailBytes = 8192;
constexpr int kPrepThreads = 256;

// One GEMM of a launch. A pass keeps an array of these in device memory; TMA reads the tensor
// map from there.
struct alignas(64) Problem {
  CUtensorMap tm_w;        // codes [N, K] u8, box 128 B x 128 rows, 128-byte swizzle
  const uint16_t* X;       // [M, K] bf16 (read by the prep kernel)
  const float* scales;     // [tiles][K / 128]
  uint8_t* img;            // [K / 128][npadB][128] term images (shared-memory operand layout)
  float* gx;               // [M] per-row power-of-two scales
  void* Y;                 // [M, N] fp32 or bf16 (unused by the verify problem)
  float* part_val;         // verify problem: per-tile row maxima [tiles][M]
  int* part_idx;           //                 and their indices
  long long N, K;
  long long unit0;         // first unit of this problem in the launch's numbering
  int tile0;               // first ticket counter of this problem
  int kus;                 // units per tile: K / (128 * BPU)
  int tiles, y_bf16, verify;
};

struct Params {
  const Problem* probs;    // device array of a pass, or nullptr: the single problem passed by value
  int nprob;
  uint32_t img_bytes;      // one block's image: npadB * 128
  int M, npad, npadB, np;
  long long units;
  int grid;
  int stages;
  uint32_t stage_bytes;
  unsigned int* counters;  // [tiles of all problems], zero between calls
  float* partials;         // [2 * grid][M][128]
  unsigned int* err;
};

// Position of a unit: its problem, the tile within that problem and the unit within the tile.
// The problem's unit and tile counts are kept in registers and read again only when the walk
// enters the next problem.
struct Cursor {
  int pi;
  long long tile;
  int ku, kus, tiles;
  __device__ __forceinline__ void init(const Problem* probs, int nprob, long long u) {
    pi = 0;
    while (pi + 1 < nprob && probs[pi + 1].unit0 <= u) ++pi;
    const Problem& pr = probs[pi];
    kus = pr.kus;
    tiles = pr.tiles;
    const long long r = u - pr.unit0;
    tile = r / kus;
    ku = (int)(r - tile * kus);
  }
  // Steps to the next unit. Past the launch's last unit pi equals nprob and nothing is read.
  __device__ __forceinline__ void next(const Problem* probs, int nprob) {
    if (++ku < kus) return;
    ku = 0;
    if (++tile < tiles) return;
    tile = 0;
    if (++pi < nprob) { kus = probs[pi].kus; tiles = probs[pi].tiles; }
  }
};

// What the epilogue needs of the problem it is in, in registers (read once per problem).
struct ProbView {
  long long N, unit0;
  int tile0, y_bf16, verify;
  const float* gx;
  void* Y;
  float* part_val;
  int* part_idx;
  __device__ __forceinline__ void load(const Problem& pr) {
    N = pr.N; unit0 = pr.unit0; tile0 = pr.tile0; y_bf16 = pr.y_bf16; verify = pr.verify;
    gx = pr.gx; Y = pr.Y; part_val = pr.part_val; part_idx = pr.part_idx;
  }
};

// ---------------------------------------------------------------- activation terms

// Two fp32 values -> two E4M3 codes (first value in bits 0..7), nearest even, saturating.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float first, float second) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(second), "f"(first));
  return r;
}

// One CTA per (problem, row m): g[m], then the kT terms of every element into the block images.
// Image of block kb: npadB rows of 128 B, row m*kT + t, 16-byte chunk j of a row stored at chunk
// j ^ (row % 8) (the 128-byte swizzle the MMA's descriptor names).
__global__ void __launch_bounds__(kPrepThreads) fp8q_prep_kernel(const __grid_constant__ Problem single,
                                                                   const Problem* probs, int M, uint32_t img_bytes) {
  const Problem& pr = probs ? probs[blockIdx.x / M] : single;
  const uint16_t* X = pr.X;
  const long long K = pr.K;
  uint8_t* img = pr.img;
  float* gx = pr.gx;
  const int m = blockIdx.x % M, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const uint16_t* xr = X + (long long)m * K;
  const long long nchunk = K / 16;
  __shared__ float s_red[kPrepThreads / 32];
  float amax = 0.f;
  for (long long j = t; j < nchunk; j += kPrepThreads) {
    const uint4 a = *reinterpret_cast<const uint4*>(xr + j * 16);
    const uint4 b = *reinterpret_cast<const uint4*>(xr + j * 16 + 8);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[i] << 16)), fabsf(__uint_as_float(w[i] & 0xFFFF0000u))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) s_red[warp] = amax;
  __syncthreads();
  amax = 0.f;
#pragma unroll
  for (int w = 0; w < kPrepThreads / 32; ++w) amax = fmaxf(amax, s_red[w]);
  int e = 0;
  if (amax > 0.f) frexpf(amax, &e);                  // amax = f * 2^e, f in [0.5, 1)
  const float g = amax > 0.f ? ldexpf(1.0f, e - 8) : 1.0f;     // >= 2^-141: an fp32 subnormal at worst
  // 1/g = 2^(8-e) can exceed fp32's range for tiny rows, so it is applied as two exact factors
  const int sh = amax > 0.f ? 8 - e : 0;
  const float inv_a = ldexpf(1.0f, sh / 2), inv_b = ldexpf(1.0f, sh - sh / 2);
  if (t == 0) gx[m] = g;
  for (long long j = t; j < nchunk; j += kPrepThreads) {
    const uint4 a = *reinterpret_cast<const uint4*>(xr + j * 16);
    const uint4 b = *reinterpret_cast<const uint4*>(xr + j * 16 + 8);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float r[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      r[2 * i] = __uint_as_float(w[i] << 16) * inv_a * inv_b;   // exact: power-of-two scalings
      r[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u) * inv_a * inv_b;
    }
    const long long kb = j / 8;                                 // 8 chunks of 16 per 128-wide block
    const int cj = (int)(j % 8);
#pragma unroll
    for (int term = 0; term < kT; ++term) {
      uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t c2 = f32x2_to_e4m3x2(r[2 * i], r[2 * i + 1]);
        packed[i >> 1] |= c2 << ((i & 1) * 16);
        // residual for the next term, scaled by 16 (exact: the code's value has 4 significant bits)
        const uint32_t h2 = e4m3x2_to_f16x2(c2);
        r[2 * i] = (r[2 * i] - f16lo_to_f32(h2)) * 16.0f;
        r[2 * i + 1] = (r[2 * i + 1] - f16hi_to_f32(h2)) * 16.0f;
      }
      const int row = m * kT + term;
      uint8_t* dst = img + kb * img_bytes + (size_t)(row >> 3) * 1024 + (row & 7) * 128 + ((cj ^ (row & 7)) << 4);
      *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
  }
}

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// D[128 x N] (+)= A[128 x 32] * B[32 x N], A and B E4M3 in shared memory, fp32 accumulation.
__device__ __forceinline__ void tc_mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_st_x16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tc_ld_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFF) >> 4);          // start address
  d |= (uint64_t)1 << 16;                           // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;                 // stride byte offset
  d |= (uint64_t)1 << 46;                           // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                           // SWIZZLE_128B
  return d;
}

// ---------------------------------------------------------------- schedule helpers

__device__ __forceinline__ long long unit_begin(long long c, long long U, int G) { return c * U / G; }

__device__ __forceinline__ int cta_of_unit(long long u, long long U, int G) {
  int c = (int)(u * G / U);
  while (c + 1 < G && unit_begin(c + 1, U, G) <= u) ++c;
  while (c > 0 && unit_begin(c, U, G) > u) --c;
  return c;
}

// ---------------------------------------------------------------- epilogue pieces

__device__ __forceinline__ void write_y(const Params& p, const ProbView& pr, long long n, int m0,
                                        const float (&y)[16]) {
  if (n >= pr.N) return;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int m = m0 + j;
    if (m < p.M) {
      if (pr.y_bf16)
        reinterpret_cast<uint16_t*>(pr.Y)[(long long)m * pr.N + n] = f32_to_bf16_rn(y[j]);
      else
        reinterpret_cast<float*>(pr.Y)[(long long)m * pr.N + n] = y[j];
    }
  }
}

__device__ __forceinline__ void warp_argmax(const ProbView& pr, long long n, int m0, const float (&y)[16],
                                            float* s_val, int* s_idx, int q, int lane) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float v = (n < pr.N) ? y[j] : -INFINITY;
    int i = (n < pr.N) ? (int)n : INT_MAX;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, v, o);
      const int oi = __shfl_xor_sync(0xffffffffu, i, o);
      if (argmax_better(ov, oi, v, i)) { v = ov; i = oi; }
    }
    if (lane == 0) { s_val[q * kMaxM + m0 + j] = v; s_idx[q * kMaxM + m0 + j] = i; }
  }
}

__device__ __forceinline__ void tile_argmax_out(const Params& p, const ProbView& pr, long long tile, int et,
                                                const float* s_val, const int* s_idx) {
  if (et >= p.M) return;
  float bv = s_val[et];
  int bi = s_idx[et];
  for (int w = 1; w < 4; ++w)
    if (argmax_better(s_val[w * kMaxM + et], s_idx[w * kMaxM + et], bv, bi)) {
      bv = s_val[w * kMaxM + et];
      bi = s_idx[w * kMaxM + et];
    }
  pr.part_val[tile * p.M + et] = bv;
  pr.part_idx[tile * p.M + et] = bi;
}

// ---------------------------------------------------------------- the GEMM kernel

template <int BPU>
__global__ void __launch_bounds__(kThreads, 1)
    fp8q_kernel(const __grid_constant__ Problem single, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages, NP = p.np;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)S * p.stage_bytes);
  // [0,S) full, [S,2S) empty, 2S+b p_full, 2S+kMaxP+b p_empty, 2S+2kMaxP drain
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * S + 1 + 2 * kMaxP);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_last = reinterpret_cast<int*>(s_tmem + 2);
  float* s_val = reinterpret_cast<float*>(s_tmem + 4);                  // [4][kMaxM]
  int* s_idx = reinterpret_cast<int*>(s_val + 4 * kMaxM);               // [4][kMaxM]

  auto bar_full = [&](int s) { return smem_u32(bars + s); };
  auto bar_empty = [&](int s) { return smem_u32(bars + S + s); };
  auto bar_pfull = [&](int b) { return smem_u32(bars + 2 * S + b); };
  auto bar_pempty = [&](int b) { return smem_u32(bars + 2 * S + kMaxP + b); };
  const uint32_t bar_drain = smem_u32(bars + 2 * S + 2 * kMaxP);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const long long U = p.units;
  const long long u_begin = unit_begin(c, U, p.grid), u_end = unit_begin(c + 1, U, p.grid);
  const int nunits = (int)(u_end - u_begin);
  const int npadB = p.npadB;
  const Problem* probs = p.probs ? p.probs : &single;
  const uint32_t img_bytes = p.img_bytes;
  const uint32_t kR = 0;                           // running sums: columns [0, npad)
  const uint32_t pcol0 = (uint32_t)p.npad;         // P set b, block h at pcol0 + (b*BPU + h)*npadB

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(bar_full(s), 1); mbar_init(bar_empty(s), 1); }
    for (int b = 0; b < kMaxP; ++b) { mbar_init(bar_pfull(b), 1); mbar_init(bar_pempty(b), kEpiThreads); }
    mbar_init(bar_drain, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {   // whole warp allocates all 512 TMEM columns (one CTA per SM)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
      const uint32_t tx = (uint32_t)BPU * (kWBytes + img_bytes);
      int issued = 0;
      Cursor cur;
      cur.init(probs, p.nprob, u_begin);
      int s = 0;
      uint32_t ph = 0;
      for (int i = 0; i < nunits; ++i) {
        if (!mbar_wait(bar_empty(s), ph ^ 1u, s_abort, p.err)) break;
        uint8_t* st = smem + (size_t)s * p.stage_bytes;
        mbar_arrive_expect_tx(bar_full(s), tx);
        const Problem& pr = probs[cur.pi];
#pragma unroll
        for (int h = 0; h < BPU; ++h) {
          const int kb = cur.ku * BPU + h;
          tma_load_2d(smem_u32(st + h * kWBytes), &pr.tm_w, kb * kKB, (int)(cur.tile * kTileRows), bar_full(s),
                      pol_w);
          bulk_load(smem_u32(st + BPU * kWBytes + h * img_bytes), pr.img + (size_t)kb * img_bytes, img_bytes,
                    bar_full(s), pol_x);
        }
        issued = i + 1;
        cur.next(probs, p.nprob);
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (*s_abort) {       // drain: wait (bounded) for every copy this thread issued
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i) {
          const unsigned long long t0 = globaltimer();
          while (!mbar_try_wait(bar_full(i % S), (uint32_t)(i / S) & 1u) && globaltimer() - t0 < kWaitLimitNs) {}
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // kind::f8f6f4: f32 accumulator, A and B E4M3 (format 0), both K-major, N = npadB, M = 128
      const uint32_t idesc = (1u << 4) | ((uint32_t)(npadB >> 3) << 17) | ((uint32_t)(kTileRows >> 4) << 24);
      int s = 0;
      uint32_t ph = 0;
      for (int i = 0; i < nunits; ++i) {
        const int b = i % NP, k = i / NP;
        const bool ok = mbar_wait(bar_pempty(b), ((uint32_t)k & 1u) ^ 1u, s_abort, p.err) &&
                        mbar_wait(bar_full(s), ph, s_abort, p.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t st = smem_u32(smem + (size_t)s * p.stage_bytes);
#pragma unroll
        for (int h = 0; h < BPU; ++h) {
          const uint32_t d_tmem = tmem + pcol0 + (uint32_t)((b * BPU + h) * npadB);
          const uint32_t wa = st + h * kWBytes, xb = st + BPU * kWBytes + h * img_bytes;
#pragma unroll
          for (int kk = 0; kk < kKB / 32; ++kk)    // 32 one-byte elements = 32 B of each swizzled row
            tc_mma_f8(d_tmem, sw128_desc(wa + kk * 32), sw128_desc(xb + kk * 32), idesc, kk == 0 ? 0u : 1u);
        }
        tc_commit(bar_empty(s));       // stage reusable once these MMAs retire
        tc_commit(bar_pfull(b));       // the blocks' sums are ready for promotion
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      tc_commit(bar_drain);            // completes when every MMA issued above has retired
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(bar_drain, 0) && globaltimer() - t0 < kWaitLimitNs) {}
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ promotion and epilogue warpgroup
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;                // token groups m0 / 16 of this parity
    const int rowl = q * 32 + lane;
    const int et = threadIdx.x - 4 * 32;             // 0..255
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    // Block scales, four units ahead: block h of unit (tile, ku) has scale [tile][ku * BPU + h]
    // of its problem; the L2 round trip is then off every unit's path.
    Cursor ahead;
    ahead.init(probs, p.nprob, u_begin);
    int ahead_pi = ahead.pi;
    const float* ahead_scales = probs[ahead_pi].scales;
    int ia = 0;                                      // unit of this CTA's range that `ahead` is at
    auto load_ahead = [&](float (&dst)[BPU]) {
      if (ia < nunits) {
        if (ahead.pi != ahead_pi) { ahead_pi = ahead.pi; ahead_scales = probs[ahead_pi].scales; }
        const float* sp = ahead_scales + (ahead.tile * ahead.kus + ahead.ku) * BPU;
#pragma unroll
        for (int h = 0; h < BPU; ++h) dst[h] = __ldg(sp + h);
        ahead.next(probs, p.nprob);
      } else {
#pragma unroll
        for (int h = 0; h < BPU; ++h) dst[h] = 0.0f;
      }
      ++ia;
    };
    float scn[4][BPU];
#pragma unroll
    for (int a = 0; a < 4; ++a) load_ahead(scn[a]);
    Cursor cur;
    cur.init(probs, p.nprob, u_begin);
    ProbView pr;
    int view_pi = cur.pi;
    pr.load(probs[view_pi]);
    for (int i = 0; i < nunits; ++i) {
      const long long u = u_begin + i;
      if (cur.pi != view_pi) { view_pi = cur.pi; pr.load(probs[view_pi]); }
      const long long tile = cur.tile;
      const int ku = cur.ku, kus = cur.kus;
      if (i + 1 < nunits) cur.next(probs, p.nprob);
      const bool seg_first = (i == 0) || (ku == 0);
      const bool seg_last = (i == nunits - 1) || (ku == kus - 1);
      const int b = i % NP, k = i / NP;
      float sc[BPU];
#pragma unroll
      for (int h = 0; h < BPU; ++h) {
        sc[h] = scn[0][h];
        scn[0][h] = scn[1][h];
        scn[1][h] = scn[2][h];
        scn[2][h] = scn[3][h];
      }
      load_ahead(scn[3]);
      // Every thread reaches the barrier and leaves with the same decision, so a give-up seen by
      // any of them ends the loop for all.
      const bool got = mbar_wait(bar_pfull(b), (uint32_t)k & 1u, s_abort, p.err);
      if (named_bar_any(1, kEpiThreads, !got || ld_shared_volatile(s_abort) != 0)) break;
      tc_fence_after();
      const long long n = tile * kTileRows + rowl;
      const long long tile_u0 = pr.unit0 + tile * kus, tile_u1 = tile_u0 + kus;
      const long long seg_u0 = u_begin > tile_u0 ? u_begin : tile_u0;
      const bool complete = (seg_u0 == tile_u0) && (u + 1 == tile_u1);
      const int slot = (seg_u0 == u_begin) ? 2 * c : 2 * c + 1;
      const uint32_t pcol = pcol0 + (uint32_t)(b * BPU * npadB);
      for (int m0 = 16 * half; m0 < p.M; m0 += 32) {
        // tokens m0 .. m0+15: their 2 x 16 term columns of each block, and the running sums
        float y[16];
        uint32_t rv[16];
        if (!seg_first) tc_ld_x16(lane_base + kR + m0, rv);
#pragma unroll
        for (int h = 0; h < BPU; ++h) {
          uint32_t lo[16], hi[16];
          tc_ld_x16(lane_base + pcol + (uint32_t)(h * npadB + kT * m0), lo);
          tc_ld_x16(lane_base + pcol + (uint32_t)(h * npadB + kT * m0 + 16), hi);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t* src = j < 8 ? lo : hi;
            const int jj = (j & 7) * 2;
            const float blk = __uint_as_float(src[jj]) + 0.0625f * __uint_as_float(src[jj + 1]);   // term fold
            if (h == 0)
              y[j] = seg_first ? sc[0] * blk : fmaf(sc[0], blk, __uint_as_float(rv[j]));
            else
              y[j] = fmaf(sc[h], blk, y[j]);
          }
        }
        if (!seg_last) {
          uint32_t o[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(y[j]);
          tc_st_x16(lane_base + kR + m0, o);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) y[j] *= (m0 + j < p.M) ? __ldg(pr.gx + m0 + j) : 0.0f;   // exact: 2^e
          if (complete) {
            if (pr.verify) warp_argmax(pr, n, m0, y, s_val, s_idx, q, lane);
            else write_y(p, pr, n, m0, y);
          } else {
            float* dst = p.partials + ((long long)slot * p.M) * kTileRows;
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (m0 + j < p.M) dst[(long long)(m0 + j) * kTileRows + rowl] = y[j];
          }
        }
      }
      if (!seg_last) tc_wait_st();
      tc_fence_before();
      mbar_arrive(bar_pempty(b));
      if (!seg_last) continue;
      if (complete) {
        if (pr.verify) {
          named_bar(1, kEpiThreads);
          tile_argmax_out(p, pr, tile, et, s_val, s_idx);
          named_bar(1, kEpiThreads);
        }
        continue;
      }
      // split tile: publish the partial, take a ticket; the last arrival finishes the tile
      __threadfence();
      named_bar(1, kEpiThreads);
      if (et == 0) {
        const int c0 = cta_of_unit(tile_u0, U, p.grid), c1 = cta_of_unit(tile_u1 - 1, U, p.grid);
        int expected = 0;
        for (int cc = c0; cc <= c1; ++cc)
          if (unit_begin(cc + 1, U, p.grid) > unit_begin(cc, U, p.grid)) ++expected;
        const unsigned int prev = atomicAdd(p.counters + pr.tile0 + tile, 1u);
        *s_last = (prev + 1 == (unsigned int)expected) ? 1 : 0;
      }
      named_bar(1, kEpiThreads);
      if (*s_last) {
        __threadfence();
        const int c0 = cta_of_unit(tile_u0, U, p.grid), c1 = cta_of_unit(tile_u1 - 1, U, p.grid);
        for (int m0 = 16 * half; m0 < p.M; m0 += 32) {
          float y[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) y[j] = 0.0f;
          for (int cc = c0; cc <= c1; ++cc) {
            const long long b0 = unit_begin(cc, U, p.grid), b1 = unit_begin(cc + 1, U, p.grid);
            if (b1 <= b0) continue;
            const int sl = (b0 >= tile_u0) ? 2 * cc : 2 * cc + 1;
            const float* src = p.partials + ((long long)sl * p.M) * kTileRows;
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              v[j] = (m0 + j < p.M) ? __ldcg(src + (long long)(m0 + j) * kTileRows + rowl) : 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) y[j] += v[j];
          }
          if (pr.verify) warp_argmax(pr, n, m0, y, s_val, s_idx, q, lane);
          else write_y(p, pr, n, m0, y);
        }
        if (pr.verify) {
          named_bar(1, kEpiThreads);
          tile_argmax_out(p, pr, tile, et, s_val, s_idx);
        }
        if (et == 0) p.counters[pr.tile0 + tile] = 0u;   // ready for the next call
      }
      named_bar(1, kEpiThreads);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

}  // namespace fp8q

// ============================================================================ host side

using namespace fp8q;

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn_fp8q() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    return nullptr;
  }();
  return fn;
}

bool fp8q_supported(long long M, long long K) {
  return M >= 1 && M <= kMaxM && K >= kKB && K % kKB == 0 && K / kKB <= (1ll << 24);
}

static size_t al256_q(size_t v) { return (v + 255) / 256 * 256; }

// The launch shape and the workspace layout of a list of FP8 GEMMs sharing M.
struct QPlan {
  int npad, npadB, bpu, np, grid, stages;
  int tiles, vtiles;       // tiles of all problems; of the verify problem (0 without one)
  long long units;
  uint32_t img_bytes, stage_bytes;
  size_t smem;
  size_t off_partials, off_verify, off_img, off_gx, off_desc, bytes;
  std::vector<size_t> img_off;   // per problem, from off_img
};

static QPlan q_plan(long long M, const Fp8HostProblem* hp, int n, bool with_desc) {
  QPlan pl{};
  pl.npad = (int)std::max<long long>(16, (M + 15) / 16 * 16);
  pl.npadB = kT * pl.npad;                          // the epilogue reads 16 tokens' terms at a time
  pl.img_bytes = (uint32_t)pl.npadB * 128u;
  bool even = true;
  for (int i = 0; i < n; ++i) even = even && ((hp[i].K / kKB) % 2 == 0);
  // TMEM: R (npad), then np P sets of bpu * npadB columns.
  const int room = 512 - pl.npad;
  pl.bpu = (even && room / (2 * pl.npadB) >= 2) ? 2 : 1;
  pl.np = std::max(1, std::min(kMaxP, room / (pl.bpu * pl.npadB)));
  size_t img = 0;
  for (int i = 0; i < n; ++i) {
    const int tiles = (int)((hp[i].N + kTileRows - 1) / kTileRows);
    pl.units += (long long)tiles * (hp[i].K / kKB / pl.bpu);
    pl.tiles += tiles;
    if (hp[i].verify) pl.vtiles = tiles;
    pl.img_off.push_back(img);
    img += (size_t)(hp[i].K / kKB) * pl.img_bytes;   // multiples of 1024: npadB is a multiple of 16
  }
  const int sms = std::max(1, device_sm_count());
  pl.grid = (int)std::min<long long>(sms, pl.units);
  pl.stage_bytes = (uint32_t)pl.bpu * (kWBytes + pl.img_bytes);
  const size_t budget = 227 * 1024 - 1024 - kTailBytes;
  pl.stages = (int)std::min<size_t>(kMaxStages, budget / pl.stage_bytes);
  pl.smem = 1024 + (size_t)pl.stages * pl.stage_bytes + kTailBytes;
  pl.off_partials = al256_q((size_t)pl.tiles * 4);
  pl.off_verify = pl.off_partials + al256_q((size_t)2 * pl.grid * M * kTileRows * 4);
  pl.off_img = pl.off_verify + (pl.vtiles ? 2 * al256_q((size_t)pl.vtiles * M * 4) : 0);
  pl.off_img = (pl.off_img + 1023) / 1024 * 1024;
  pl.off_gx = pl.off_img + img;
  pl.off_desc = pl.off_gx + al256_q((size_t)n * M * 4);
  pl.bytes = pl.off_desc + (with_desc ? al256_q((size_t)n * sizeof(Problem)) : 0);
  return pl;
}

static int fill_problem(Problem* P, const Fp8HostProblem& h, long long M, const QPlan& pl, long long unit0, int tile0,
                        char* ws, int index) {
  memset(static_cast<void*>(P), 0, sizeof(*P));
  auto fn = encode_fn_fp8q();
  if (!fn) return set_error(NVFP4WS_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)h.K, (cuuint64_t)h.N};
  cuuint64_t strides[1] = {(cuuint64_t)h.K};
  cuuint32_t box[2] = {kKB, kTileRows};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&P->tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(h.q), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return set_error(NVFP4WS_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  P->X = h.X;
  P->scales = h.scales;
  P->img = reinterpret_cast<uint8_t*>(ws + pl.off_img + pl.img_off[index]);
  P->gx = reinterpret_cast<float*>(ws + pl.off_gx) + (size_t)index * M;
  P->Y = h.Y;
  P->N = h.N;
  P->K = h.K;
  P->unit0 = unit0;
  P->tile0 = tile0;
  P->kus = (int)(h.K / kKB / pl.bpu);
  P->tiles = (int)((h.N + kTileRows - 1) / kTileRows);
  P->y_bf16 = h.y_bf16;
  P->verify = h.verify;
  if (h.verify) {
    P->part_val = reinterpret_cast<float*>(ws + pl.off_verify);
    P->part_idx = reinterpret_cast<int*>(ws + pl.off_verify + al256_q((size_t)pl.vtiles * M * 4));
  }
  return NVFP4WS_OK;
}

// Enqueue the term prep (one CTA per problem and row) and the GEMM. `single` is used when
// `probs_dev` is null (one problem).
static int launch_kernels(const Problem& single, const Problem* probs_dev, int nprob, long long M, const QPlan& pl,
                          char* ws, cudaStream_t s) {
  if (pl.stages < 2) return set_error(NVFP4WS_ERR_UNSUPPORTED, "fp8 term path: stage does not fit shared memory");
  fp8q_prep_kernel<<<(unsigned)(M * nprob), kPrepThreads, 0, s>>>(single, probs_dev, (int)M, pl.img_bytes);
  if (int e = check_launch("fp8q_prep_kernel")) return e;
  Params p{};
  p.probs = probs_dev;
  p.nprob = nprob;
  p.img_bytes = pl.img_bytes;
  p.M = (int)M;
  p.npad = pl.npad;
  p.npadB = pl.npadB;
  p.np = pl.np;
  p.units = pl.units;
  p.grid = pl.grid;
  p.stages = pl.stages;
  p.stage_bytes = pl.stage_bytes;
  p.counters = reinterpret_cast<unsigned int*>(ws);
  p.partials = reinterpret_cast<float*>(ws + pl.off_partials);
  p.err = device_error_word();
  if (!p.err) return set_error(NVFP4WS_ERR_CUDA, "cannot resolve the device error word");
  static std::atomic<bool> attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(fp8q_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess ||
        cudaFuncSetAttribute(fp8q_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
      return check_launch("cudaFuncSetAttribute(fp8q_kernel)");
    attr_set[dev].store(true, std::memory_order_release);
  }
  if (pl.bpu == 2) fp8q_kernel<2><<<pl.grid, kThreads, pl.smem, s>>>(single, p);
  else fp8q_kernel<1><<<pl.grid, kThreads, pl.smem, s>>>(single, p);
  return check_launch("fp8q_kernel");
}

// ---------------------------------------------------------------------------- one GEMM

static Fp8HostProblem one_q(const uint16_t* X, const uint8_t* q, const float* scales, long long N, long long K,
                            void* Y, int y_dtype, bool verify) {
  return Fp8HostProblem{X, q, scales, N, K, Y, y_dtype == NVFP4WS_Y_BF16 ? 1 : 0, verify ? 1 : 0};
}

size_t fp8q_workspace_bytes_int(long long M, long long N, long long K, bool verify) {
  if (!fp8q_supported(M, K) || N < 1) return 0;
  const Fp8HostProblem h = one_q(nullptr, nullptr, nullptr, N, K, nullptr, 0, verify);
  return q_plan(M, &h, 1, false).bytes;
}

static int launch_one_q(const Fp8HostProblem& h, long long M, void* workspace, cudaStream_t s, QPlan* out) {
  const QPlan pl = q_plan(M, &h, 1, false);
  char* ws = static_cast<char*>(workspace);
  alignas(64) Problem P;
  if (int e = fill_problem(&P, h, M, pl, 0, 0, ws, 0)) return e;
  *out = pl;
  return launch_kernels(P, nullptr, 1, M, pl, ws, s);
}

int launch_fp8q_gemm(const uint16_t* X, const uint8_t* q, const float* scales, long long M, long long N, long long K,
                     void* Y, int y_dtype, void* workspace, cudaStream_t s) {
  QPlan pl;
  return launch_one_q(one_q(X, q, scales, N, K, Y, y_dtype, false), M, workspace, s, &pl);
}

int launch_fp8q_verify(const uint16_t* X, const uint8_t* q, const float* scales, long long M, long long N,
                       long long K, const VerifyRule& v, void* workspace, cudaStream_t s) {
  QPlan pl;
  if (int e = launch_one_q(one_q(X, q, scales, N, K, nullptr, 0, true), M, workspace, s, &pl)) return e;
  char* ws = static_cast<char*>(workspace);
  return launch_verify_stage2(reinterpret_cast<const float*>(ws + pl.off_verify),
                              reinterpret_cast<const int*>(ws + pl.off_verify + al256_q((size_t)pl.vtiles * M * 4)),
                              pl.vtiles, (int)M, v, s);
}

// ---------------------------------------------------------------------------- FP8 weight passes

// Host state of an initialised pass on this kernel: plain data in the caller's nvfp4_pass.
struct QPassState {
  uint32_t magic;
  int nprob, has_verify, vtiles;
  long long M;
  const Problem* probs;    // device copy, in the workspace
  char* ws;
  int npad, npadB, bpu, np, grid, stages;
  long long units;
  uint32_t img_bytes, stage_bytes;
  size_t smem, off_partials, off_verify;
  VerifyRule vr;
};
static_assert(sizeof(QPassState) <= kFp8PassStateBytes, "pass state does not fit the caller's handle");
constexpr uint32_t kQPassMagic = 0x46503851u;

bool fp8q_pass_owns(const void* state) {
  uint32_t m;
  memcpy(&m, state, sizeof(m));
  return m == kQPassMagic;
}

size_t fp8q_pass_workspace_bytes_int(const Fp8HostProblem* hp, int n, long long M) {
  return q_plan(M, hp, n, true).bytes;
}

int fp8q_pass_init_int(void* state, const Fp8HostProblem* hp, int n, long long M, const VerifyRule* vr,
                       void* workspace, size_t workspace_bytes) {
  const QPlan pl = q_plan(M, hp, n, true);
  if (workspace_bytes < pl.bytes)
    return set_error(NVFP4WS_ERR_WORKSPACE, "fp8_pass_init: workspace needs %zu bytes", pl.bytes);
  if (pl.stages < 2) return set_error(NVFP4WS_ERR_UNSUPPORTED, "fp8 term path: stage does not fit shared memory");
  char* ws = static_cast<char*>(workspace);
  std::vector<Problem> P(n);
  long long unit0 = 0;
  int tile0 = 0;
  for (int i = 0; i < n; ++i) {
    if (int e = fill_problem(&P[i], hp[i], M, pl, unit0, tile0, ws, i)) return e;
    unit0 += (long long)P[i].tiles * P[i].kus;
    tile0 += P[i].tiles;
  }
  Problem* dev = reinterpret_cast<Problem*>(ws + pl.off_desc);
  if (cudaMemcpy(dev, P.data(), (size_t)n * sizeof(Problem), cudaMemcpyHostToDevice) != cudaSuccess)
    return check_launch("fp8_pass_init: descriptor copy");
  QPassState st{};
  st.magic = kQPassMagic;
  st.nprob = n;
  st.has_verify = vr != nullptr;
  st.vtiles = pl.vtiles;
  st.M = M;
  st.probs = dev;
  st.ws = ws;
  st.npad = pl.npad; st.npadB = pl.npadB; st.bpu = pl.bpu; st.np = pl.np; st.grid = pl.grid; st.stages = pl.stages;
  st.units = pl.units;
  st.img_bytes = pl.img_bytes; st.stage_bytes = pl.stage_bytes;
  st.smem = pl.smem; st.off_partials = pl.off_partials; st.off_verify = pl.off_verify;
  if (vr) st.vr = *vr;
  memcpy(state, &st, sizeof(st));
  return NVFP4WS_OK;
}

int fp8q_pass_run_int(const void* state, cudaStream_t s) {
  QPassState st;
  memcpy(&st, state, sizeof(st));
  if (st.magic != kQPassMagic) return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_pass_run: pass is not initialised");
  QPlan pl{};
  pl.npad = st.npad; pl.npadB = st.npadB; pl.bpu = st.bpu; pl.np = st.np; pl.grid = st.grid; pl.stages = st.stages;
  pl.units = st.units;
  pl.img_bytes = st.img_bytes; pl.stage_bytes = st.stage_bytes;
  pl.smem = st.smem; pl.off_partials = st.off_partials; pl.off_verify = st.off_verify;
  alignas(64) Problem unused;
  memset(static_cast<void*>(&unused), 0, sizeof(unused));
  if (int e = launch_kernels(unused, st.probs, st.nprob, st.M, pl, st.ws, s)) return e;
  if (!st.has_verify) return NVFP4WS_OK;
  return launch_verify_stage2(reinterpret_cast<const float*>(st.ws + st.off_verify),
                              reinterpret_cast<const int*>(st.ws + st.off_verify +
                                                           al256_q((size_t)st.vtiles * st.M * 4)),
                              st.vtiles, (int)st.M, st.vr, s);
}

}  // namespace nvfp4ws
