// tcgen05 tensor-core path of the skinny NVFP4 GEMM and the fused verify (sm_100a).
//
//   Y[m, n] = ts * sum_k x16[m, k] * (e2m1(code[n, k]) * S[n, k/16])
//
// At M = 17 or 68 the pass does 68-272 flops per weight byte, too much for CUDA
// cores at HBM speed, so the contraction runs on the 5th-generation tensor cores.
// The MMA is swap-AB: weight rows are the MMA's M dimension (128 per tile), and
// the tokens are its N dimension (M padded to a multiple of 16).
//
// Data flow per CTA (one persistent CTA per SM, 16 warps):
//   warp 0        TMA producer. It streams the weight tile for each 256-wide
//                 K-chunk (128 rows x 128 B of nibbles, 128 x 16 B of E4M3
//                 scales) and the matching bf16 X chunk into a shared-memory
//                 ring of stages, on mbarriers. No multicast.
//   warp 1        TMEM allocator and MMA issuer (one thread): 16 x tcgen05.mma
//                 kind::f16 per chunk, A from TMEM, B from shared memory, fp32
//                 accumulators in TMEM.
//   warps 4-7,    Two dequantisation warpgroups taking alternate chunks. Each
//   warps 8-11    thread owns one weight row (its TMEM lane). It converts its
//                 E2M1 pairs with cvt.rn.f16x2.e2m1x2 and multiplies by the
//                 E4M3 block scale in f16 (exact). It writes the f16 A operand
//                 straight into TMEM with tcgen05.st, so A never takes a round
//                 trip through shared memory. The same threads convert the
//                 chunk's X rows from bf16 to f16 in place, each row shifted by
//                 its power of two xe[m] (x_shift_kernel, launched first), so the
//                 conversion is exact and never saturates.
//   warps 12-15   Epilogue warpgroup: tcgen05.ld of the accumulators, times ts
//                 and 2^xe[m], then Y (or, in verify mode, the per-tile argmax).
//
// Scheduling. The units are (128-row tile, 256-wide K-chunk) pairs. They are
// split into equal contiguous ranges, one per CTA (stream-K), so every SM streams
// the same number of bytes even when N/128 is smaller than the SM count (the down
// projection has 40 tiles). A tile whose K range spans several CTAs is finished
// by the last of them to arrive: each writes its fp32 partial to the workspace,
// takes a ticket, and the holder of the last ticket sums the partials in K
// order. The sum order is fixed, so results are deterministic. No CTA ever waits
// for another.
//
// Every mbarrier wait is bounded by a timer. On expiry the thread records
// kDevErrWaitTimeout in the device error word and the CTA winds down: it drains
// its own TMA copies and MMAs, then frees its TMEM.
#include "common.cuh"
#include "kernels.h"
#include "mma.h"
#include "sync.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>

namespace nvfp4ws {
namespace mmak {

constexpr int kThreads = 512;
constexpr int kTileRows = 128;
constexpr int kKC = 256;                          // K elements per stage
constexpr int kNibBytes = kTileRows * kKC / 2;    // 16 KB
constexpr int kSfBytes = kTileRows * kKC / 16;    // 2 KB
constexpr int kMaxNpad = 128;
constexpr int kAColsPerBuf = kKC / 2;             // f16 pairs per row per chunk = TMEM columns
// barriers, TMEM address, flags and the [4][kMaxNpad] argmax staging after the stages
constexpr size_t kTailBytes = 8192;

struct Params {
  const uint16_t* X;
  float* Y;                // fp32 or bf16 (y_bf16)
  int y_bf16;
  const float* ts;
  int M, npad;
  long long N, K;
  int tiles, kch;
  long long units;
  int grid;
  int stages;
  uint32_t stage_bytes;
  // workspace
  unsigned int* counters;  // [tiles], zero between calls
  float* partials;         // [2 * grid][M][128]
  const int* xe;           // [M] power-of-two shift of each X row (x_shift_kernel)
  // verify mode
  int verify;
  float* part_val;         // [tiles][M]
  int* part_idx;
  unsigned int* err;
};

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

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

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

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

struct EpiRow {
  int rowl;        // row within the tile (= TMEM lane)
  long long n;     // global weight row
};

// Writes y (already scaled) for tokens [m0, m0+16) of this thread's row.
__device__ __forceinline__ void write_y(const Params& p, const EpiRow& r, int m0, const float (&y)[16]) {
  if (r.n >= p.N) return;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int m = m0 + j;
    if (m < p.M) {
      if (p.y_bf16)
        reinterpret_cast<uint16_t*>(p.Y)[(long long)m * p.N + r.n] = f32_to_bf16_rn(y[j]);
      else
        p.Y[(long long)m * p.N + r.n] = y[j];
    }
  }
}

// Per-token argmax across the 128 rows of the tile (verify mode). Each warp
// reduces its 32 rows; the 4 warp results are combined in shared memory.
__device__ __forceinline__ void tile_argmax(const Params& p, const EpiRow& r, int m0, const float (&y)[16],
                                            float* s_val, int* s_idx, int q, int lane) {
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float v = (r.n < p.N) ? y[j] : -INFINITY;
    int i = (r.n < p.N) ? (int)r.n : INT_MAX;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, v, o);
      const int oi = __shfl_xor_sync(0xffffffffu, i, o);
      if (argmax_better(ov, oi, v, i)) { v = ov; i = oi; }
    }
    if (lane == 0) { s_val[q * kMaxNpad + m0 + j] = v; s_idx[q * kMaxNpad + m0 + j] = i; }
  }
}

// ---------------------------------------------------------------- the kernel

__global__ void __launch_bounds__(kThreads, 1)
    mma_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_sf,
               const __grid_constant__ CUtensorMap tm_x, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  // barriers and small state after the stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)S * p.stage_bytes);
  // [0,S) full, [S,2S) empty, 2S+{0,1} a_full, 2S+{2,3} a_empty, 2S+{4,5} acc_full, 2S+{6,7} acc_empty, 2S+8 drain
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * S + 9);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_last = reinterpret_cast<int*>(s_tmem + 2);
  float* s_val = reinterpret_cast<float*>(s_tmem + 4);                  // [4][kMaxNpad]
  int* s_idx = reinterpret_cast<int*>(s_val + 4 * kMaxNpad);            // [4][kMaxNpad]
  int* s_xe = s_idx + 4 * kMaxNpad;                                     // [kMaxNpad] row shifts

  auto bar_full = [&](int s) { return smem_u32(bars + s); };
  auto bar_empty = [&](int s) { return smem_u32(bars + S + s); };
  auto bar_afull = [&](int g) { return smem_u32(bars + 2 * S + g); };
  auto bar_aempty = [&](int g) { return smem_u32(bars + 2 * S + 2 + g); };
  auto bar_accfull = [&](int b) { return smem_u32(bars + 2 * S + 4 + b); };
  auto bar_accempty = [&](int b) { return smem_u32(bars + 2 * S + 6 + b); };
  const uint32_t bar_drain = smem_u32(bars + 2 * S + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const long long U = p.units;
  const long long u_begin = unit_begin(c, U, p.grid), u_end = unit_begin(c + 1, U, p.grid);
  const int nunits = (int)(u_end - u_begin);
  const int npad = p.npad;
  const uint32_t acc_col0 = 2 * kAColsPerBuf;      // accumulators after the two A buffers

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(bar_full(s), 1); mbar_init(bar_empty(s), 1); }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar_afull(g), 128); mbar_init(bar_aempty(g), 1);
      mbar_init(bar_accfull(g), 1); mbar_init(bar_accempty(g), 128);
    }
    mbar_init(bar_drain, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int m = threadIdx.x; m < kMaxNpad; m += kThreads) s_xe[m] = m < p.M ? p.xe[m] : 0;
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
      const uint32_t tx = kNibBytes + kSfBytes + (uint32_t)npad * 512u;
      int issued = 0;
      int s = 0, tile = (int)(u_begin / p.kch), kc = (int)(u_begin % p.kch);   // advanced incrementally below
      uint32_t ph = 0;
      for (int i = 0; i < nunits; ++i) {
        if (!mbar_wait(bar_empty(s), ph ^ 1u, s_abort, p.err)) break;
        uint8_t* st = smem + (size_t)s * p.stage_bytes;
        mbar_arrive_expect_tx(bar_full(s), tx);
        tma_load_2d(smem_u32(st), &tm_q, kc * (kKC / 2), tile * kTileRows, bar_full(s), pol_w);
        tma_load_2d(smem_u32(st + kNibBytes + npad * 512), &tm_sf, kc * (kKC / 16), tile * kTileRows, bar_full(s),
                    pol_w);
#pragma unroll
        for (int a = 0; a < 4; ++a)
          tma_load_2d(smem_u32(st + kNibBytes + a * npad * 128), &tm_x, kc * kKC + a * 64, 0, bar_full(s), pol_x);
        issued = i + 1;
        if (++kc == p.kch) { kc = 0; ++tile; }
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
      const uint32_t idesc = (1u << 4) | ((uint32_t)(npad >> 3) << 17) | ((uint32_t)(kTileRows >> 4) << 24);
      int seg = 0;
      bool ok = true;
      int s = 0, kc = (int)(u_begin % p.kch);
      uint32_t ph = 0;
      for (int i = 0; i < nunits && ok; ++i) {
        const int g = i & 1;
        const bool seg_first = (i == 0) || (kc == 0);
        const bool seg_last = (i == nunits - 1) || (kc == p.kch - 1);
        const int ab = seg & 1;
        if (seg_first) {
          ok = mbar_wait(bar_accempty(ab), ((uint32_t)(seg >> 1) & 1u) ^ 1u, s_abort, p.err);
          if (!ok) break;
        }
        ok = mbar_wait(bar_full(s), ph, s_abort, p.err) &&
             mbar_wait(bar_afull(g), (uint32_t)(i >> 1) & 1u, s_abort, p.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t xbase = smem_u32(smem + (size_t)s * p.stage_bytes + kNibBytes);
        const uint32_t d_tmem = tmem + acc_col0 + ab * npad;
        const uint32_t a_tmem = tmem + g * kAColsPerBuf;
#pragma unroll
        for (int kk = 0; kk < kKC / 16; ++kk) {
          const uint64_t bdesc = sw128_desc(xbase + (kk >> 2) * npad * 128 + (kk & 3) * 32);
          tc_mma_f16_ts(d_tmem, a_tmem + kk * 8, bdesc, idesc, (seg_first && kk == 0) ? 0u : 1u);
        }
        tc_commit(bar_empty(s));       // stage reusable once these MMAs retire
        tc_commit(bar_aempty(g));      // A buffer reusable
        if (seg_last) { tc_commit(bar_accfull(ab)); ++seg; }
        if (++kc == p.kch) kc = 0;
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
      // X chunk: bf16 -> f16 in place (rows < M; TMA zero-filled the rest)
      {
        uint8_t* xs = st + kNibBytes;
        const int words = 4 * p.M * 8;               // 16-byte words: 4 atoms x M rows x 8
        for (int w = tg; w < words; w += 128) {
          const int a = w / (p.M * 8), rem = w - a * (p.M * 8);
          uint4* ptr = reinterpret_cast<uint4*>(xs + a * npad * 128 + (rem >> 3) * 128 + (rem & 7) * 16);
          uint4 v = *ptr;
          const int e = s_xe[rem >> 3];
          v.x = bf16x2_to_f16x2_shifted(v.x, e); v.y = bf16x2_to_f16x2_shifted(v.y, e);
          v.z = bf16x2_to_f16x2_shifted(v.z, e); v.w = bf16x2_to_f16x2_shifted(v.w, e);
          *ptr = v;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      // weight row r: 128 bytes of nibbles (swizzled 16-byte chunks) and 16 scale bytes
      const uint8_t* nib = st + r * 128;
      const uint4 sc = *reinterpret_cast<const uint4*>(st + kNibBytes + npad * 512 + r * 16);
      const uint32_t scw[4] = {sc.x, sc.y, sc.z, sc.w};
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + g * kAColsPerBuf;
#pragma unroll
      for (int part = 0; part < 4; ++part) {
        uint32_t out[32];
#pragma unroll
        for (int j2 = 0; j2 < 2; ++j2) {
          const int j = part * 2 + j2;                // 16-byte chunk = 32 elements = 2 blocks
          const uint4 w = *reinterpret_cast<const uint4*>(nib + ((j ^ (r & 7)) << 4));
          const uint32_t s2 = e4m3x2_to_f16x2(scw[j >> 1] >> ((j & 1) * 16));
          const uint32_t hs0 = (s2 & 0xFFFFu) * 0x10001u, hs1 = (s2 >> 16) * 0x10001u;
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint32_t h = e2m1x2_to_f16x2(ww[e >> 2] >> (8 * (e & 3)));
            out[j2 * 16 + e] = hmul2(h, e < 8 ? hs0 : hs1);
          }
        }
        tc_st_x32(taddr + part * 32, out);
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(bar_afull(g));
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue warpgroup
    const int q = warp & 3;
    EpiRow row;
    row.rowl = q * 32 + lane;
    const int et = threadIdx.x - 12 * 32;            // 0..127
    const float ts = *p.ts;
    int seg = 0;
    int tile_it = (int)(u_begin / p.kch), kc_it = (int)(u_begin % p.kch);
    for (int i = 0; i < nunits; ++i) {
      const long long u = u_begin + i;
      const int tile = tile_it;
      const bool seg_last = (i == nunits - 1) || (kc_it == p.kch - 1);
      if (++kc_it == p.kch) { kc_it = 0; ++tile_it; }
      if (!seg_last) continue;
      // this segment covers units [seg_u0, u] of `tile`
      const long long tile_u0 = (long long)tile * p.kch, tile_u1 = tile_u0 + p.kch;
      const long long seg_u0 = u_begin > tile_u0 ? u_begin : tile_u0;
      const bool complete = (seg_u0 == tile_u0) && (u + 1 == tile_u1);
      const int ab = seg & 1;
      if (!mbar_wait(bar_accfull(ab), (uint32_t)(seg >> 1) & 1u, s_abort, p.err)) break;
      tc_fence_after();
      row.n = (long long)tile * kTileRows + row.rowl;
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + acc_col0 + ab * npad;
      const int slot = (seg_u0 == u_begin) ? 2 * c : 2 * c + 1;
      for (int m0 = 0; m0 < npad; m0 += 16) {
        uint32_t v[16];
        tc_ld_x16(taddr + m0, v);
        tc_wait_ld();
        if (m0 >= p.M) continue;
        if (complete) {
          float y[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) y[j] = mul_pow2(__uint_as_float(v[j]) * ts, s_xe[m0 + j]);
          if (p.verify) tile_argmax(p, row, m0, y, s_val, s_idx, q, lane);
          else write_y(p, row, m0, y);
        } else {
          float* dst = p.partials + ((long long)slot * p.M) * kTileRows;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (m0 + j < p.M) dst[(long long)(m0 + j) * kTileRows + row.rowl] = __uint_as_float(v[j]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_accempty(ab));
      ++seg;
      if (complete) {
        if (p.verify) {
          named_bar(1, 128);
          if (et < p.M) {
            float bv = s_val[et];
            int bi = s_idx[et];
            for (int w = 1; w < 4; ++w)
              if (argmax_better(s_val[w * kMaxNpad + et], s_idx[w * kMaxNpad + et], bv, bi)) {
                bv = s_val[w * kMaxNpad + et]; bi = s_idx[w * kMaxNpad + et];
              }
            p.part_val[(long long)tile * p.M + et] = bv;
            p.part_idx[(long long)tile * p.M + et] = bi;
          }
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
        const unsigned int prev = atomicAdd(p.counters + tile, 1u);
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
              v[j] = (m0 + j < p.M) ? __ldcg(src + (long long)(m0 + j) * kTileRows + row.rowl) : 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) y[j] += v[j];
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) y[j] = mul_pow2(y[j] * ts, s_xe[m0 + j]);
          if (p.verify) tile_argmax(p, row, m0, y, s_val, s_idx, q, lane);
          else write_y(p, row, m0, y);
        }
        if (p.verify) {
          named_bar(1, 128);
          if (et < p.M) {
            float bv = s_val[et];
            int bi = s_idx[et];
            for (int w = 1; w < 4; ++w)
              if (argmax_better(s_val[w * kMaxNpad + et], s_idx[w * kMaxNpad + et], bv, bi)) {
                bv = s_val[w * kMaxNpad + et]; bi = s_idx[w * kMaxNpad + et];
              }
            p.part_val[(long long)tile * p.M + et] = bv;
            p.part_idx[(long long)tile * p.M + et] = bi;
          }
        }
        if (et == 0) p.counters[tile] = 0u;          // ready for the next call
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

}  // namespace mmak

// ============================================================================ host side

using namespace mmak;

// Looked up once per process; a function-local static is initialised exactly once even
// when several host threads make their first call together.
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

static bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static int npad_of(long long M) { return (int)std::max<long long>(16, (M + 15) / 16 * 16); }

bool mma_supported(long long M, long long K) { return M >= 1 && M <= kMaxNpad && K % kKC == 0 && K >= kKC; }

int mma_min_m() { return 2; }

struct MmaPlan {
  int npad, tiles, kch, grid, stages;
  long long units;
  uint32_t stage_bytes;
  size_t smem;
};

static MmaPlan plan_of(long long M, long long N, long long K) {
  MmaPlan pl{};
  pl.npad = npad_of(M);
  pl.tiles = (int)((N + kTileRows - 1) / kTileRows);
  pl.kch = (int)(K / kKC);
  pl.units = (long long)pl.tiles * pl.kch;
  const int sms = std::max(1, device_sm_count());
  pl.grid = (int)std::min<long long>(sms, pl.units);
  pl.stage_bytes = kNibBytes + kSfBytes + (uint32_t)pl.npad * 512u;
  const size_t budget = 227 * 1024 - 1024 - kTailBytes;
  pl.stages = (int)std::min<size_t>(8, budget / pl.stage_bytes);
  pl.smem = 1024 + (size_t)pl.stages * pl.stage_bytes + kTailBytes;
  return pl;
}

static size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// GEMM workspace: ticket counters [tiles] | partials [2 * grid][M][128] | row shifts [M].
static size_t xe_offset(const MmaPlan& pl, long long M) {
  return align256((size_t)pl.tiles * 4) + align256((size_t)2 * pl.grid * M * kTileRows * 4);
}

size_t mma_gemm_workspace_bytes(long long M, long long N, long long K) {
  if (!mma_supported(M, K)) return 0;
  MmaPlan pl = plan_of(M, N, K);
  return xe_offset(pl, M) + align256((size_t)M * 4);
}

size_t mma_gemm_counter_bytes(long long M, long long N, long long K) {
  if (!mma_supported(M, K)) return 0;
  return align256((size_t)plan_of(M, N, K).tiles * 4);
}

size_t mma_verify_workspace_bytes(long long M, long long N, long long K) {
  if (!mma_supported(M, K)) return 0;
  MmaPlan pl = plan_of(M, N, K);
  return mma_gemm_workspace_bytes(M, N, K) + 2 * align256((size_t)pl.tiles * M * 4);
}

static int launch_mma(const uint16_t* X, const uint8_t* q, const uint8_t* sf, const float* ts, long long M,
                      long long N, long long K, void* Y, int y_dtype, void* workspace, bool verify, float** pv_out,
                      int** pi_out, int* nparts_out, cudaStream_t s) {
  MmaPlan pl = plan_of(M, N, K);
  alignas(64) CUtensorMap tq, tsf, tx;
  if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K / 2, N, K / 2, kKC / 2, kTileRows,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tsf, CU_TENSOR_MAP_DATA_TYPE_UINT8, sf, K / 16, N, K / 16, kKC / 16, kTileRows,
                CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, K, M, K * 2, 64, pl.npad, CU_TENSOR_MAP_SWIZZLE_128B))
    return set_error(NVFP4WS_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  Params p{};
  p.X = X;
  p.Y = static_cast<float*>(Y);
  p.y_bf16 = (y_dtype == NVFP4WS_Y_BF16);
  p.ts = ts;
  p.M = (int)M;
  p.npad = pl.npad;
  p.N = N;
  p.K = K;
  p.tiles = pl.tiles;
  p.kch = pl.kch;
  p.units = pl.units;
  p.grid = pl.grid;
  p.stages = pl.stages;
  p.stage_bytes = pl.stage_bytes;
  char* ws = static_cast<char*>(workspace);
  p.counters = reinterpret_cast<unsigned int*>(ws);
  p.partials = reinterpret_cast<float*>(ws + align256((size_t)pl.tiles * 4));
  int* xe = reinterpret_cast<int*>(ws + xe_offset(pl, M));
  p.xe = xe;
  p.verify = verify ? 1 : 0;
  if (verify) {
    char* v = ws + mma_gemm_workspace_bytes(M, N, K);
    p.part_val = reinterpret_cast<float*>(v);
    p.part_idx = reinterpret_cast<int*>(v + align256((size_t)pl.tiles * M * 4));
    *pv_out = p.part_val;
    *pi_out = p.part_idx;
    *nparts_out = pl.tiles;
  }
  p.err = device_error_word();
  if (!p.err) return set_error(NVFP4WS_ERR_CUDA, "cannot resolve the device error word");
  static std::atomic<bool> attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
      return check_launch("cudaFuncSetAttribute(mma_kernel)");
    attr_set[dev].store(true, std::memory_order_release);
  }
  if (int e = launch_row_shifts(X, M, K, xe, s)) return e;
  mma_kernel<<<pl.grid, kThreads, pl.smem, s>>>(tq, tsf, tx, p);
  return check_launch("mma_kernel");
}

int launch_mma_gemm(const uint16_t* X, const uint8_t* q, const uint8_t* sf, const float* ts, long long M, long long N,
                    long long K, void* Y, int y_dtype, void* workspace, size_t, cudaStream_t s) {
  return launch_mma(X, q, sf, ts, M, N, K, Y, y_dtype, workspace, false, nullptr, nullptr, nullptr, s);
}

int launch_mma_verify(const uint16_t* X, const uint8_t* q, const uint8_t* sf, const float* ts, long long M,
                      long long N, long long K, const VerifyRule& v, void* workspace, cudaStream_t s) {
  float* pv = nullptr;
  int* pi = nullptr;
  int nparts = 0;
  if (int e = launch_mma(X, q, sf, ts, M, N, K, nullptr, 0, workspace, true, &pv, &pi, &nparts, s)) return e;
  return launch_verify_stage2(pv, pi, nparts, (int)M, v, s);
}

}  // namespace nvfp4ws
