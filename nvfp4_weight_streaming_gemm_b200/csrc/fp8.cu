// FP8 (E4M3) block-scaled weight GEMMs and fused verify on the tcgen05 tensor cores (sm_100a):
// one GEMM, or a whole list of them (an FP8 weight pass) in one persistent launch.
//
//   Y[m, n] = sum_kb s[n / 128, kb] * sum_{k in block kb} x16[m, k] * e4m3(code[n, k])
//
// The weight format is one E4M3 code per element and one fp32 scale per 128 x 128 block
// (rows x K), s = fp32(amax_block / 448) ("TandemLLM", "The parts": the lm_head in FP8 E4M3;
// "Qwen3.8 on DGX Spark (GB10)", the model list: FP8 block-scaled projections). The pages
// name no block shape; 128 x 128 is the reading taken here.
//
// Exactness. An E4M3 value has at most 4 significant bits and lies in [2^-9, 448], so it is
// exact in f16. Each activation row is multiplied by a power of two 2^-e (e from the row's
// amax, computed by fp8_x_shift_kernel first) so that its amax lies in [2^14, 2^15): the
// bf16 -> f16 conversion is then exact for every value above 2^-25 of the amax and never
// saturates, and the output is multiplied by 2^e. Every product is exact in the fp32
// accumulator. The block scale is an
// arbitrary fp32 and would round if folded into either f16 operand, so the tensor core sums
// each 128 x 128 block's 128 products per (row, token) into a fresh TMEM buffer P, and the
// epilogue promotes it into a running sum R = s * P, then R += s * P, in fp32 (R also lives
// in TMEM). A unit of work is BPU = 1 or 2 such blocks of one 128-row tile: two while TMEM
// leaves room for two rotating P sets (npad <= 48) and every problem's K is a multiple of 256,
// which halves the per-unit hand-offs per weight byte.
//
// Roles per CTA (one persistent CTA per SM, 16 warps):
//   warp 0        TMA producer: the unit's 16 KB code tiles (128 rows x 128 B, 128-byte
//                 swizzle) and its bf16 X slice (2*BPU 64-wide swizzled atoms) into a ring.
//                 No multicast.
//   warp 1        TMEM allocator and the single MMA-issuing thread: 8 x kind::f16 (K = 16)
//                 per block, A from TMEM, B from shared memory, each block into its own P of
//                 one of np rotating P sets.
//   warps 4-7,    two dequantisation warpgroups taking alternate units. Each thread owns one
//   warps 8-11    weight row (its TMEM lane): E4M3 pairs -> f16 pairs (cvt.rn.f16x2.e4m3x2)
//                 written into TMEM as the A operand. The same threads convert the unit's X
//                 rows from bf16 to f16 in place.
//   warps 12-15   promotion and epilogue: at the end of a tile's K range, Y (or the tile's
//                 per-token argmax for the verify problem, or a split-K partial).
//
// TMEM columns (512, one CTA per SM): two A buffers of 64*BPU columns (64 f16 pairs per row
// and block), then R (npad columns), then np P sets of BPU*npad columns.
//
// Scheduling is stream-K over the concatenated (problem, tile, K-range) units of all the
// launch's problems: they are cut into equal contiguous ranges, one per CTA, so every SM
// streams the same number of bytes however the list's shapes fall. A tile whose K range spans
// several CTAs is finished by the last to arrive: each publishes its fp32 partial, takes a
// ticket, and the holder of the last ticket sums the partials in K order, so results are
// deterministic and no CTA waits for another. Every mbarrier wait is bounded; on expiry the
// thread records kDevErrWaitTimeout and the CTA winds down (drains its copies and MMAs, frees
// its TMEM).
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
namespace fp8k {

constexpr int kThreads = 512;
constexpr int kTileRows = 128;
constexpr int kKB = kFp8Block;                       // K elements of one scale block
constexpr uint32_t kWBytes = kTileRows * kKB;        // 16 KB of codes per block
constexpr int kMaxNpad = 128;
constexpr int kACols = kKB / 2;                      // f16 pairs per row and block = TMEM columns
constexpr int kMaxP = 4;
constexpr int kMaxStages = 8;
constexpr size_t kTailBytes = 8192;

// One GEMM of a launch. A pass keeps an array of these in device memory; TMA reads the tensor
// maps from there.
struct alignas(64) Problem {
  CUtensorMap tm_w;        // codes [N, K] u8, box 128 B x 128 rows, 128-byte swizzle
  CUtensorMap tm_x;        // X [M, K] bf16, box 64 x npad, 128-byte swizzle
  const float* scales;     // [tiles][K / 128]
  void* Y;                 // [M, N] fp32 or bf16 (unused by the verify problem)
  float* part_val;         // verify problem: per-tile row maxima [tiles][M]
  int* part_idx;           //                 and their indices
  long long N;
  long long unit0;         // first unit of this problem in the launch's numbering
  int tile0;               // first ticket counter of this problem
  int kus;                 // units per tile: K / (128 * BPU)
  int tiles, y_bf16, verify;
  const uint16_t* X;       // [M, K] bf16 (read by the row-shift kernel)
  long long K;
  int* xe;                 // [M] power-of-two shift of each X row (fp8_x_shift_kernel)
};

struct Params {
  const Problem* probs;    // device array of a pass, or nullptr: the single problem passed by value
  int nprob;
  int M, npad, np;
  long long units;
  int grid;
  int stages;
  uint32_t stage_bytes;
  unsigned int* counters;  // [tiles of all problems], zero between calls
  float* partials;         // [2 * grid][M][128]
  unsigned int* err;
};

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// D[128 x N] (+)= A[128 x 16] (TMEM, f16) * B[16 x N] (shared memory, f16), fp32 accumulation.
__device__ __forceinline__ void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_st_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
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

// Position of a unit: its problem, the tile within that problem and the unit within the tile.
struct Cursor {
  int pi;
  long long tile;
  int ku;
  __device__ __forceinline__ void init(const Problem* probs, int nprob, long long u) {
    pi = 0;
    while (pi + 1 < nprob && probs[pi + 1].unit0 <= u) ++pi;
    const Problem& pr = probs[pi];
    const long long r = u - pr.unit0;
    tile = r / pr.kus;
    ku = (int)(r - tile * pr.kus);
  }
  // Steps to the next unit. Past the launch's last unit pi equals nprob; do not read it then.
  __device__ __forceinline__ void next(const Problem* probs) {
    const Problem& pr = probs[pi];
    if (++ku == pr.kus) {
      ku = 0;
      if (++tile == pr.tiles) { tile = 0; ++pi; }
    }
  }
};

// ---------------------------------------------------------------- epilogue pieces

// Writes y for tokens [m0, m0+16) of weight row n of problem pr.
__device__ __forceinline__ void write_y(const Params& p, const Problem& pr, long long n, int m0,
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

// Per-token argmax over the 32 rows of this warp; lane 0 stages the warp's winner.
__device__ __forceinline__ void warp_argmax(const Problem& pr, long long n, int m0, const float (&y)[16],
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
    if (lane == 0) { s_val[q * kMaxNpad + m0 + j] = v; s_idx[q * kMaxNpad + m0 + j] = i; }
  }
}

// Combines the 4 warps' staged winners into the tile's partial (one thread per token).
__device__ __forceinline__ void tile_argmax_out(const Params& p, const Problem& pr, long long tile, int et,
                                                const float* s_val, const int* s_idx) {
  if (et >= p.M) return;
  float bv = s_val[et];
  int bi = s_idx[et];
  for (int w = 1; w < 4; ++w)
    if (argmax_better(s_val[w * kMaxNpad + et], s_idx[w * kMaxNpad + et], bv, bi)) {
      bv = s_val[w * kMaxNpad + et];
      bi = s_idx[w * kMaxNpad + et];
    }
  pr.part_val[tile * p.M + et] = bv;
  pr.part_idx[tile * p.M + et] = bi;
}

// ---------------------------------------------------------------- the kernel

// BPU scale blocks (128 K each) per unit. Two blocks per unit halve the per-unit fixed costs
// (barrier hand-offs, the epilogue's TMEM round trips) per weight byte; the sums are the same
// fma sequence either way, so the result does not depend on BPU.
template <int BPU>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_kernel(const __grid_constant__ Problem single, const Params p) {
  constexpr uint32_t kUW = BPU * kWBytes;           // code bytes per unit
  constexpr int kUACols = BPU * kACols;             // TMEM columns of one A buffer
  constexpr uint32_t kR = 2 * kUACols;              // running sums after the two A buffers
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages, NP = p.np;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)S * p.stage_bytes);
  // [0,S) full, [S,2S) empty, 2S+{0,1} a_full, 2S+{2,3} a_empty, 2S+4+b p_full, 2S+4+kMaxP+b p_empty,
  // 2S+4+2kMaxP drain
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * S + 5 + 2 * kMaxP);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_last = reinterpret_cast<int*>(s_tmem + 2);
  float* s_val = reinterpret_cast<float*>(s_tmem + 4);                  // [4][kMaxNpad]
  int* s_idx = reinterpret_cast<int*>(s_val + 4 * kMaxNpad);            // [4][kMaxNpad]
  // row shifts of the problem each stage holds, written by the producer before its arrive
  const int** s_stage_xe = reinterpret_cast<const int**>(s_idx + 4 * kMaxNpad);   // [kMaxStages]

  auto bar_full = [&](int s) { return smem_u32(bars + s); };
  auto bar_empty = [&](int s) { return smem_u32(bars + S + s); };
  auto bar_afull = [&](int g) { return smem_u32(bars + 2 * S + g); };
  auto bar_aempty = [&](int g) { return smem_u32(bars + 2 * S + 2 + g); };
  auto bar_pfull = [&](int b) { return smem_u32(bars + 2 * S + 4 + b); };
  auto bar_pempty = [&](int b) { return smem_u32(bars + 2 * S + 4 + kMaxP + b); };
  const uint32_t bar_drain = smem_u32(bars + 2 * S + 4 + 2 * kMaxP);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const long long U = p.units;
  const long long u_begin = unit_begin(c, U, p.grid), u_end = unit_begin(c + 1, U, p.grid);
  const int nunits = (int)(u_end - u_begin);
  const int npad = p.npad;
  const Problem* probs = p.probs ? p.probs : &single;
  const uint32_t pcol0 = kR + (uint32_t)npad;      // first P buffer; buffer b, block h at + (b*BPU + h)*npad

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(bar_full(s), 1); mbar_init(bar_empty(s), 1); }
    for (int g = 0; g < 2; ++g) { mbar_init(bar_afull(g), 128); mbar_init(bar_aempty(g), 1); }
    for (int b = 0; b < kMaxP; ++b) { mbar_init(bar_pfull(b), 1); mbar_init(bar_pempty(b), 128); }
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
      const uint32_t tx = kUW + (uint32_t)(BPU * npad) * 256u;
      int issued = 0;
      Cursor cur;
      cur.init(probs, p.nprob, u_begin);
      int s = 0;
      uint32_t ph = 0;
      for (int i = 0; i < nunits; ++i) {
        if (!mbar_wait(bar_empty(s), ph ^ 1u, s_abort, p.err)) break;
        uint8_t* st = smem + (size_t)s * p.stage_bytes;
        const Problem& pr = probs[cur.pi];
        const int k0 = cur.ku * BPU * kKB;             // first K element of the unit
        s_stage_xe[s] = pr.xe;                         // published by the arrive below
        mbar_arrive_expect_tx(bar_full(s), tx);
#pragma unroll
        for (int h = 0; h < BPU; ++h)
          tma_load_2d(smem_u32(st + h * kWBytes), &pr.tm_w, k0 + h * kKB, (int)(cur.tile * kTileRows), bar_full(s),
                      pol_w);
#pragma unroll
        for (int a = 0; a < 2 * BPU; ++a)
          tma_load_2d(smem_u32(st + kUW + a * npad * 128), &pr.tm_x, k0 + a * 64, 0, bar_full(s), pol_x);
        issued = i + 1;
        cur.next(probs);
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
      // kind::f16: f32 accumulator, A and B f16, both K-major, N = npad, M = 128
      const uint32_t idesc = (1u << 4) | ((uint32_t)(npad >> 3) << 17) | ((uint32_t)(kTileRows >> 4) << 24);
      int s = 0;
      uint32_t ph = 0;
      for (int i = 0; i < nunits; ++i) {
        const int g = i & 1, b = i % NP, k = i / NP;
        const bool ok = mbar_wait(bar_pempty(b), ((uint32_t)k & 1u) ^ 1u, s_abort, p.err) &&
                        mbar_wait(bar_full(s), ph, s_abort, p.err) &&
                        mbar_wait(bar_afull(g), (uint32_t)(i >> 1) & 1u, s_abort, p.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t xbase = smem_u32(smem + (size_t)s * p.stage_bytes + kUW);
#pragma unroll
        for (int h = 0; h < BPU; ++h) {            // each block into its own P: its scale comes later
          const uint32_t d_tmem = tmem + pcol0 + (uint32_t)((b * BPU + h) * npad);
          const uint32_t a_tmem = tmem + (uint32_t)(g * kUACols + h * kACols);
#pragma unroll
          for (int kk = 0; kk < kKB / 16; ++kk) {
            const uint64_t bdesc = sw128_desc(xbase + (2 * h + (kk >> 2)) * npad * 128 + (kk & 3) * 32);
            tc_mma_f16_ts(d_tmem, a_tmem + kk * 8, bdesc, idesc, kk == 0 ? 0u : 1u);
          }
        }
        tc_commit(bar_empty(s));       // stage reusable once these MMAs retire
        tc_commit(bar_aempty(g));      // A buffer reusable
        tc_commit(bar_pfull(b));       // the blocks' sums are ready for promotion
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      tc_commit(bar_drain);            // completes when every MMA issued above has retired
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(bar_drain, 0) && globaltimer() - t0 < kWaitLimitNs) {}
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ dequantisation warpgroups
    const int g = (warp - 4) >> 2;                   // warpgroup 0 or 1
    const int q = warp & 3;                          // TMEM lane quarter
    const int r = q * 32 + lane;                     // row within the tile
    const int tg = threadIdx.x - (4 + 4 * g) * 32;   // 0..127 within the warpgroup
    int s = g % S;
    uint32_t ph = (uint32_t)(g / S) & 1u;
    for (int i = g; i < nunits; i += 2) {
      if (i != g) {                                   // advance the ring position by two units
        s += 2;
        if (s >= S) { s -= S; ph ^= 1u; }
      }
      if (!mbar_wait(bar_full(s), ph, s_abort, p.err)) break;
      if (!mbar_wait(bar_aempty(g), ((uint32_t)(i >> 1) & 1u) ^ 1u, s_abort, p.err)) break;
      tc_fence_after();
      uint8_t* st = smem + (size_t)s * p.stage_bytes;
      // X slice: bf16 -> f16 in place, each row shifted by its power of two (rows < M; TMA
      // zero-filled the rest)
      {
        uint8_t* xs = st + kUW;
        const int* xe = s_stage_xe[s];
        const int words = 2 * BPU * p.M * 8;         // 16-byte words: 2*BPU atoms x M rows x 8
        for (int w = tg; w < words; w += 128) {
          const int a = w / (p.M * 8), rem = w - a * (p.M * 8);
          uint4* ptr = reinterpret_cast<uint4*>(xs + a * npad * 128 + (rem >> 3) * 128 + (rem & 7) * 16);
          uint4 v = *ptr;
          const int e = __ldg(xe + (rem >> 3));
          v.x = bf16x2_to_f16x2_shifted(v.x, e); v.y = bf16x2_to_f16x2_shifted(v.y, e);
          v.z = bf16x2_to_f16x2_shifted(v.z, e); v.w = bf16x2_to_f16x2_shifted(v.w, e);
          *ptr = v;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      // weight row r of each block: 128 codes in eight swizzled 16-byte chunks -> 64 f16 pairs
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(g * kUACols);
#pragma unroll
      for (int h = 0; h < BPU; ++h) {
        const uint8_t* row = st + h * kWBytes + r * 128;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t out[32];
#pragma unroll
          for (int j2 = 0; j2 < 4; ++j2) {
            const int j = half * 4 + j2;              // logical chunk: elements 16j .. 16j+15
            const uint4 w = *reinterpret_cast<const uint4*>(row + ((j ^ (r & 7)) << 4));
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) out[j2 * 8 + e] = e4m3x2_to_f16x2(ww[e >> 1] >> ((e & 1) * 16));
          }
          tc_st_x32(taddr + (uint32_t)(h * kACols + half * 32), out);
        }
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(bar_afull(g));
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ promotion and epilogue warpgroup
    const int q = warp & 3;
    const int rowl = q * 32 + lane;
    const int et = threadIdx.x - 12 * 32;            // 0..127
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    // Block scales, four units ahead: the L2 round trip would otherwise sit on every unit's
    // path. Block h of unit (tile, ku) has scale [tile][ku * BPU + h].
    Cursor ahead;
    ahead.init(probs, p.nprob, u_begin);
    int ia = 0;                                      // unit of this CTA's range that `ahead` is at
    auto load_ahead = [&](float (&dst)[BPU]) {
      if (ia < nunits) {
        const Problem& pa = probs[ahead.pi];
        const float* sp = pa.scales + (ahead.tile * pa.kus + ahead.ku) * BPU;
#pragma unroll
        for (int h = 0; h < BPU; ++h) dst[h] = __ldg(sp + h);
        ahead.next(probs);
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
    for (int i = 0; i < nunits; ++i) {
      const long long u = u_begin + i;
      const Problem& pr = probs[cur.pi];
      const long long tile = cur.tile;
      const int ku = cur.ku, kus = pr.kus;
      cur.next(probs);
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
      if (named_bar_any(1, 128, !got || ld_shared_volatile(s_abort) != 0)) break;
      tc_fence_after();
      const long long n = tile * kTileRows + rowl;
      const long long tile_u0 = pr.unit0 + tile * kus, tile_u1 = tile_u0 + kus;
      const long long seg_u0 = u_begin > tile_u0 ? u_begin : tile_u0;
      const bool complete = (seg_u0 == tile_u0) && (u + 1 == tile_u1);
      const int slot = (seg_u0 == u_begin) ? 2 * c : 2 * c + 1;
      const uint32_t pcol = pcol0 + (uint32_t)(b * BPU * npad);
      for (int m0 = 0; m0 < p.M; m0 += 16) {
        uint32_t pv[BPU][16], rv[16];
#pragma unroll
        for (int h = 0; h < BPU; ++h) tc_ld_x16(lane_base + pcol + (uint32_t)(h * npad + m0), pv[h]);
        if (!seg_first) tc_ld_x16(lane_base + kR + m0, rv);
        tc_wait_ld();
        float y[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float acc = seg_first ? sc[0] * __uint_as_float(pv[0][j]) : fmaf(sc[0], __uint_as_float(pv[0][j]), __uint_as_float(rv[j]));
#pragma unroll
          for (int h = 1; h < BPU; ++h) acc = fmaf(sc[h], __uint_as_float(pv[h][j]), acc);
          y[j] = acc;
        }
        if (!seg_last) {
          uint32_t o[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(y[j]);
          tc_st_x16(lane_base + kR + m0, o);
        } else if (complete) {
#pragma unroll
          for (int j = 0; j < 16; ++j) y[j] = mul_pow2(y[j], m0 + j < p.M ? __ldg(pr.xe + m0 + j) : 0);
          if (pr.verify) warp_argmax(pr, n, m0, y, s_val, s_idx, q, lane);
          else write_y(p, pr, n, m0, y);
        } else {
          float* dst = p.partials + ((long long)slot * p.M) * kTileRows;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (m0 + j < p.M) dst[(long long)(m0 + j) * kTileRows + rowl] = y[j];
        }
      }
      if (!seg_last) tc_wait_st();
      tc_fence_before();
      mbar_arrive(bar_pempty(b));
      if (!seg_last) continue;
      if (complete) {
        if (pr.verify) {
          named_bar(1, 128);
          tile_argmax_out(p, pr, tile, et, s_val, s_idx);
          named_bar(1, 128);
        }
        continue;
      }
      // split tile: publish the partial, take a ticket; the last arrival finishes the tile
      __threadfence();
      named_bar(1, 128);
      if (et == 0) {
        const int c0 = cta_of_unit(tile_u0, U, p.grid), c1 = cta_of_unit(tile_u1 - 1, U, p.grid);
        int expected = 0;
        for (int cc = c0; cc <= c1; ++cc)
          if (unit_begin(cc + 1, U, p.grid) > unit_begin(cc, U, p.grid)) ++expected;
        const unsigned int prev = atomicAdd(p.counters + pr.tile0 + tile, 1u);
        *s_last = (prev + 1 == (unsigned int)expected) ? 1 : 0;
      }
      named_bar(1, 128);
      if (*s_last) {
        __threadfence();
        const int c0 = cta_of_unit(tile_u0, U, p.grid), c1 = cta_of_unit(tile_u1 - 1, U, p.grid);
        for (int m0 = 0; m0 < p.M; m0 += 16) {
          float y[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) y[j] = 0.0f;
          for (int cc = c0; cc <= c1; ++cc) {
            const long long b0 = unit_begin(cc, U, p.grid), b1 = unit_begin(cc + 1, U, p.grid);
            if (b1 <= b0) continue;
            const int sl = (b0 >= tile_u0) ? 2 * cc : 2 * cc + 1;
            const float* src = p.partials + ((long long)sl * p.M) * kTileRows;
            float v[16];   // all loads of the chunk first: one L2 round trip per contributor
#pragma unroll
            for (int j = 0; j < 16; ++j)
              v[j] = (m0 + j < p.M) ? __ldcg(src + (long long)(m0 + j) * kTileRows + rowl) : 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) y[j] += v[j];
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) y[j] = mul_pow2(y[j], m0 + j < p.M ? __ldg(pr.xe + m0 + j) : 0);
          if (pr.verify) warp_argmax(pr, n, m0, y, s_val, s_idx, q, lane);
          else write_y(p, pr, n, m0, y);
        }
        if (pr.verify) {
          named_bar(1, 128);
          tile_argmax_out(p, pr, tile, et, s_val, s_idx);
        }
        if (et == 0) p.counters[pr.tile0 + tile] = 0u;   // ready for the next call
      }
      named_bar(1, 128);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}


// Row shifts of every problem's X (one CTA per (problem, row)): xe[m] from the row's amax,
// as row_shift_of_amax defines it. The GEMM converts x * 2^-xe[m] to f16 and multiplies its
// output by 2^xe[m].
constexpr int kShiftThreads = 256;

__global__ void __launch_bounds__(kShiftThreads)
    fp8_x_shift_kernel(const __grid_constant__ Problem single, const Problem* probs, int M) {
  const Problem& pr = probs ? probs[blockIdx.x / M] : single;
  const int m = blockIdx.x % M, t = threadIdx.x;
  const uint32_t* row = reinterpret_cast<const uint32_t*>(pr.X + (long long)m * pr.K);   // bf16 pairs
  float v = 0.f;
  for (long long i = t; i < pr.K / 2; i += kShiftThreads) v = fmaxf(v, bf16x2_absmax(__ldg(row + i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __shared__ float s_red[kShiftThreads / 32];
  if ((t & 31) == 0) s_red[t >> 5] = v;
  __syncthreads();
  if (t == 0) {
    float a = 0.f;
    for (int w = 0; w < kShiftThreads / 32; ++w) a = fmaxf(a, s_red[w]);
    pr.xe[m] = row_shift_of_amax(a);
  }
}

}  // namespace fp8k

// ============================================================================ host side

using namespace fp8k;

// Looked up once per process; a function-local static is initialised exactly once even
// when several host threads make their first call together.
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn_fp8() {
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

static bool make_map_fp8(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                         uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto fn = encode_fn_fp8();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool fp8_supported(long long M, long long K) {
  return M >= 1 && M <= kMaxNpad && K >= kKB && K % kKB == 0 && K / kKB <= (1ll << 24);
}

static size_t al256_fp8(size_t v) { return (v + 255) / 256 * 256; }

// The launch shape and the workspace layout of a list of GEMMs sharing M.
struct Fp8Plan {
  int npad, bpu, np, grid, stages;
  int tiles, vtiles;       // tiles of all problems; of the verify problem (0 without one)
  long long units;
  uint32_t stage_bytes;
  size_t smem;
  size_t off_partials, off_verify, off_xe, off_desc, bytes;
};

static Fp8Plan fp8_plan(long long M, const Fp8HostProblem* hp, int n, bool with_desc) {
  Fp8Plan pl{};
  pl.npad = (int)std::max<long long>(16, (M + 15) / 16 * 16);
  // TMEM: two A buffers (64 columns per block each), R (npad), np rotating P sets (bpu * npad
  // each). Two blocks per unit while that leaves at least two P sets and every K allows it.
  bool even = true;
  for (int i = 0; i < n; ++i) even = even && ((hp[i].K / kKB) % 2 == 0);
  pl.bpu = (even && (512 - 2 * 2 * kACols - pl.npad) / (2 * pl.npad) >= 2) ? 2 : 1;
  pl.np = std::min(kMaxP, (512 - 2 * pl.bpu * kACols - pl.npad) / (pl.bpu * pl.npad));
  for (int i = 0; i < n; ++i) {
    const int tiles = (int)((hp[i].N + kTileRows - 1) / kTileRows);
    pl.units += (long long)tiles * (hp[i].K / kKB / pl.bpu);
    pl.tiles += tiles;
    if (hp[i].verify) pl.vtiles = tiles;
  }
  const int sms = std::max(1, device_sm_count());
  pl.grid = (int)std::min<long long>(sms, pl.units);
  pl.stage_bytes = (uint32_t)pl.bpu * (kWBytes + (uint32_t)pl.npad * 256u);
  const size_t budget = 227 * 1024 - 1024 - kTailBytes;
  pl.stages = (int)std::min<size_t>(kMaxStages, budget / pl.stage_bytes);
  pl.smem = 1024 + (size_t)pl.stages * pl.stage_bytes + kTailBytes;
  pl.off_partials = al256_fp8((size_t)pl.tiles * 4);
  pl.off_verify = pl.off_partials + al256_fp8((size_t)2 * pl.grid * M * kTileRows * 4);
  pl.off_xe = pl.off_verify + (pl.vtiles ? 2 * al256_fp8((size_t)pl.vtiles * M * 4) : 0);
  pl.off_desc = pl.off_xe + al256_fp8((size_t)n * M * 4);                 // row shifts [n][M]
  pl.bytes = pl.off_desc + (with_desc ? al256_fp8((size_t)n * sizeof(Problem)) : 0);
  return pl;
}

static int fill_problem(Problem* P, const Fp8HostProblem& h, long long M, const Fp8Plan& pl, long long unit0,
                        int tile0, char* ws, int index) {
  memset(P, 0, sizeof(*P));
  if (!make_map_fp8(&P->tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, h.q, h.K, h.N, h.K, kKB, kTileRows) ||
      !make_map_fp8(&P->tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h.X, h.K, M, h.K * 2, 64, pl.npad))
    return set_error(NVFP4WS_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  P->scales = h.scales;
  P->Y = h.Y;
  P->N = h.N;
  P->unit0 = unit0;
  P->tile0 = tile0;
  P->kus = (int)(h.K / kKB / pl.bpu);
  P->tiles = (int)((h.N + kTileRows - 1) / kTileRows);
  P->y_bf16 = h.y_bf16;
  P->verify = h.verify;
  P->X = h.X;
  P->K = h.K;
  P->xe = reinterpret_cast<int*>(ws + pl.off_xe) + (size_t)index * M;
  if (h.verify) {
    P->part_val = reinterpret_cast<float*>(ws + pl.off_verify);
    P->part_idx = reinterpret_cast<int*>(ws + pl.off_verify + al256_fp8((size_t)pl.vtiles * M * 4));
  }
  return NVFP4WS_OK;
}

static int launch_kernel(const Problem& single, const Problem* probs_dev, int nprob, long long M, const Fp8Plan& pl,
                         char* ws, cudaStream_t s) {
  Params p{};
  p.probs = probs_dev;
  p.nprob = nprob;
  p.M = (int)M;
  p.npad = pl.npad;
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
    if (cudaFuncSetAttribute(fp8_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess ||
        cudaFuncSetAttribute(fp8_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
      return check_launch("cudaFuncSetAttribute(fp8_kernel)");
    attr_set[dev].store(true, std::memory_order_release);
  }
  fp8_x_shift_kernel<<<(unsigned)(M * nprob), kShiftThreads, 0, s>>>(single, probs_dev, (int)M);
  if (int e = check_launch("fp8_x_shift_kernel")) return e;
  if (pl.bpu == 2) fp8_kernel<2><<<pl.grid, kThreads, pl.smem, s>>>(single, p);
  else fp8_kernel<1><<<pl.grid, kThreads, pl.smem, s>>>(single, p);
  return check_launch("fp8_kernel");
}

// ---------------------------------------------------------------------------- one GEMM

static Fp8HostProblem one(const uint16_t* X, const uint8_t* q, const float* scales, long long N, long long K, void* Y,
                          int y_dtype, bool verify) {
  return Fp8HostProblem{X, q, scales, N, K, Y, y_dtype == NVFP4WS_Y_BF16 ? 1 : 0, verify ? 1 : 0};
}

size_t fp8_gemm_workspace_bytes_int(long long M, long long N, long long K) {
  if (!fp8_supported(M, K) || N < 1) return 0;
  const Fp8HostProblem h = one(nullptr, nullptr, nullptr, N, K, nullptr, 0, false);
  return fp8_plan(M, &h, 1, false).bytes;
}

size_t fp8_verify_workspace_bytes_int(long long M, long long N, long long K) {
  if (!fp8_supported(M, K) || N < 1) return 0;
  const Fp8HostProblem h = one(nullptr, nullptr, nullptr, N, K, nullptr, 0, true);
  return fp8_plan(M, &h, 1, false).bytes;
}

static int launch_one(const Fp8HostProblem& h, long long M, void* workspace, cudaStream_t s, Fp8Plan* out) {
  const Fp8Plan pl = fp8_plan(M, &h, 1, false);
  char* ws = static_cast<char*>(workspace);
  alignas(64) Problem P;
  if (int e = fill_problem(&P, h, M, pl, 0, 0, ws, 0)) return e;
  *out = pl;
  return launch_kernel(P, nullptr, 1, M, pl, ws, s);
}

int launch_fp8_gemm(const uint16_t* X, const uint8_t* q, const float* scales, long long M, long long N, long long K,
                    void* Y, int y_dtype, void* workspace, cudaStream_t s) {
  Fp8Plan pl;
  return launch_one(one(X, q, scales, N, K, Y, y_dtype, false), M, workspace, s, &pl);
}

int launch_fp8_verify(const uint16_t* X, const uint8_t* q, const float* scales, long long M, long long N,
                      long long K, const VerifyRule& v, void* workspace, cudaStream_t s) {
  Fp8Plan pl;
  if (int e = launch_one(one(X, q, scales, N, K, nullptr, 0, true), M, workspace, s, &pl)) return e;
  char* ws = static_cast<char*>(workspace);
  return launch_verify_stage2(reinterpret_cast<const float*>(ws + pl.off_verify),
                              reinterpret_cast<const int*>(ws + pl.off_verify + al256_fp8((size_t)pl.vtiles * M * 4)),
                              pl.vtiles, (int)M, v, s);
}

// ---------------------------------------------------------------------------- FP8 weight passes

struct Fp8PassState {
  uint32_t magic;
  int nprob, has_verify;
  long long M;
  const Problem* probs;    // device copy, in the workspace
  char* ws;
  Fp8Plan pl;
  VerifyRule vr;
};
static_assert(sizeof(Fp8PassState) <= kFp8PassStateBytes, "pass state does not fit the caller's handle");
constexpr uint32_t kFp8PassMagic = 0x46503850u;

size_t fp8_pass_workspace_bytes_int(const Fp8HostProblem* hp, int n, long long M) {
  return fp8_plan(M, hp, n, true).bytes;
}

int fp8_pass_init_int(void* state, const Fp8HostProblem* hp, int n, long long M, const VerifyRule* vr,
                      void* workspace, size_t workspace_bytes) {
  const Fp8Plan pl = fp8_plan(M, hp, n, true);
  if (workspace_bytes < pl.bytes)
    return set_error(NVFP4WS_ERR_WORKSPACE, "fp8_pass_init: workspace needs %zu bytes", pl.bytes);
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
  Fp8PassState st{};
  st.magic = kFp8PassMagic;
  st.nprob = n;
  st.has_verify = vr != nullptr;
  st.M = M;
  st.probs = dev;
  st.ws = ws;
  st.pl = pl;
  if (vr) st.vr = *vr;
  memcpy(state, &st, sizeof(st));
  return NVFP4WS_OK;
}

int fp8_pass_run_int(const void* state, cudaStream_t s) {
  Fp8PassState st;
  memcpy(&st, state, sizeof(st));
  if (st.magic != kFp8PassMagic) return set_error(NVFP4WS_ERR_INVALID_ARG, "fp8_pass_run: pass is not initialised");
  alignas(64) Problem unused;
  memset(&unused, 0, sizeof(unused));
  if (int e = launch_kernel(unused, st.probs, st.nprob, st.M, st.pl, st.ws, s)) return e;
  if (!st.has_verify) return NVFP4WS_OK;
  return launch_verify_stage2(reinterpret_cast<const float*>(st.ws + st.pl.off_verify),
                              reinterpret_cast<const int*>(st.ws + st.pl.off_verify +
                                                           al256_fp8((size_t)st.pl.vtiles * st.M * 4)),
                              st.pl.vtiles, (int)st.M, st.vr, s);
}

}  // namespace nvfp4ws
