// Block-scaled tensor-core path: tcgen05.mma kind::mxf4nvf4 on packed NVFP4 weights.
//
// Why. On B200 a tcgen05.mma kind::f16 instruction (M=128, K=16) costs ~70-96 SM
// cycles for every N up to 128 (measured). So a path that dequantises W to f16
// is capped near 29 weights/clk/SM (~4.6 TB/s), before the cost of
// dequantisation itself. kind::mxf4nvf4 instead consumes the packed E2M1 weights
// straight from shared memory with their E4M3 block scales: K=64 per
// instruction, with no per-element work on the CUDA cores at all.
//
// The catch is that both operands must be NVFP4. The activations are bf16, so
// they are represented as T residual NVFP4 terms:
//   r_0 = x;  for t < T:  g_t = amax|r_t| / 2688,  S_t = E4M3(amax_block(r_t) / (6 g_t)),
//                          c_t = E2M1(r_t / (S_t g_t)),  r_{t+1} = r_t - c_t S_t g_t
// so x = sum_t g_t S_t c_t + r_T. Every term is an ordinary two-level NVFP4
// quantisation of the residual left by the previous ones. Each term cuts the
// error about 10x. With T = 5 the GEMM matches the exact float64 result to ~1e-5
// relative, and logits to ~4e-5 absolute. The terms are extra B columns (token m,
// term t -> column m*T + t). The epilogue folds them: y[m] = ts * sum_t g_t acc[m*T+t].
//
// Kernels.
//   x_prep_kernel   one CTA per activation row: the T-term decomposition into the
//                   workspace (codes [M*T, K/2], scales [M*T, K/16], g [M, T]). It
//                   triggers dependent launch at once, so the GEMM's prologue and
//                   first weight loads overlap it.
//   mxf4_kernel     one persistent CTA per SM, 12 warps:
//     warp 0        TMA producer: the W tile (128 rows x 128 B nibbles, SW128; 128 x 16 B
//                   scales) and the X-term tile (codes SW128, scales) per 256-wide
//                   K-chunk. The first stages' weight loads are issued before waiting
//                   on x_prep.
//     warp 1        TMEM allocator and MMA issuer: 4 K-steps x B-tiles of
//                   tcgen05.mma kind::mxf4nvf4.block_scale.block16 per chunk.
//     warps 4-7     scale-factor warpgroup: copies the chunk's W and X block scales
//                   from shared memory into TMEM in the layout the MMA reads (the 4
//                   scales of row m0 + 32*j in column j of lane m0, replicated over the
//                   four lane quarters).
//     warps 8-11    epilogue: tcgen05.ld of the accumulators, fold of the terms,
//                   x ts, then Y or the per-tile argmax. Split tiles are finished as on
//                   the f16 path.
// Scheduling (stream-K over (tile, chunk) units, last-arriver fixed-order split-tile
// reduction) and bounded waits are the same as on the f16 path.
#include "common.cuh"
#include "kernels.h"
#include "mma.h"
#include "sync.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>

namespace nvfp4ws {
namespace mxk {

// Optional per-unit timeline of CTA 0 (clock64 at each hand-off), for pipeline
// analysis. Compiled out unless NVFP4WS_TRACE is defined; it changes no work.
#ifdef NVFP4WS_TRACE
__device__ unsigned long long g_trace[16 * 64];
#define MX_TRACE(f, i) do { if (blockIdx.x == 0 && (i) < 64) g_trace[(f) * 64 + (i)] = clock64(); } while (0)
// per-CTA events on the global timer (ns): [cta][event]
__device__ unsigned long long g_cta_trace[256 * 16];
#define MX_CTA(e) do { if (blockIdx.x < 256) g_cta_trace[blockIdx.x * 16 + (e)] = globaltimer(); } while (0)
#else
#define MX_TRACE(f, i) do { } while (0)
#define MX_CTA(e) do { } while (0)
#endif

constexpr int kThreads = 384;
constexpr int kTileRows = 128;
constexpr int kKC = 256;
constexpr int kNibBytes = kTileRows * kKC / 2;     // 16 KB
constexpr int kSfBytes = kTileRows * kKC / 16;     // 2 KB
constexpr int kMaxB = 352;                         // B rows (tokens x terms) the TMEM budget allows
constexpr size_t kTailBytes = 8192;

// ------------------------------------------------------------------ activation decomposition

struct XPrepArgs {
  const uint16_t* X;
  int M, T;
  long long K;
  uint8_t* xq;     // [M*T, K/2]
  uint8_t* xs;     // [M*T, K/16]
  float* xg;       // [M, T]
};

constexpr int kPrepThreads = 512;                 // K <= 512 * 4 * 16 = 32768 with 4 blocks per thread

__device__ __forceinline__ float block_amax16(const float (&v)[16]) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[i]));
  return a;
}

template <int BPT>
__global__ void __launch_bounds__(kPrepThreads) x_prep_kernel(XPrepArgs a) {
  asm volatile("griddepcontrol.launch_dependents;");
#ifdef NVFP4WS_TRACE
  if (threadIdx.x == 0 && blockIdx.x < 56) g_cta_trace[(200 + blockIdx.x) * 16 + 0] = globaltimer();
#endif
  const int m = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int nblk = (int)(a.K / 16);
  __shared__ float s_red[kPrepThreads / 32];
  float r[BPT][16];
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    const int b = t + j * kPrepThreads;
    if (b < nblk) {
      const uint4* src = reinterpret_cast<const uint4*>(a.X + (long long)m * a.K + (long long)b * 16);
      const uint4 u0 = src[0], u1 = src[1];
      const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        r[j][2 * i] = __uint_as_float(w[i] << 16);
        r[j][2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) r[j][i] = 0.f;
    }
  }
  for (int term = 0; term < a.T; ++term) {
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < BPT; ++j) amax = fmaxf(amax, block_amax16(r[j]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) s_red[warp] = amax;
    __syncthreads();
    float row_amax = 0.f;
#pragma unroll
    for (int w = 0; w < kPrepThreads / 32; ++w) row_amax = fmaxf(row_amax, s_red[w]);
    __syncthreads();
    const float g = row_amax / 2688.0f;
    if (t == 0) a.xg[m * a.T + term] = g;
    const long long brow = (long long)m * a.T + term;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      const int b = t + j * kPrepThreads;
      if (b >= nblk) continue;
      uint32_t sbits = 0, lo = 0, hi = 0;
      if (g > 0.f) {
        const float want = block_amax16(r[j]) / (6.0f * g);
        uint16_t s2;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(s2) : "f"(0.0f), "f"(want));
        sbits = s2 & 0xFFu;
        const uint32_t sh = e4m3x2_to_f16x2(sbits);
        const float S = f16lo_to_f32(sh);
        const float den = S * g;
        if (den > 0.f) {
          const float inv = 1.0f / den;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            uint16_t c2;
            asm("{ .reg .b8 b; cvt.rn.satfinite.e2m1x2.f32 b, %1, %2; cvt.u16.u8 %0, b; }"
                : "=h"(c2) : "f"(r[j][2 * i + 1] * inv), "f"(r[j][2 * i] * inv));
            const uint32_t h = e2m1x2_to_f16x2(c2);
            r[j][2 * i] = fmaf(-f16lo_to_f32(h), den, r[j][2 * i]);
            r[j][2 * i + 1] = fmaf(-f16hi_to_f32(h), den, r[j][2 * i + 1]);
            if (i < 4) lo |= (uint32_t)(c2 & 0xFF) << (8 * i);
            else hi |= (uint32_t)(c2 & 0xFF) << (8 * (i - 4));
          }
        }
      }
      *reinterpret_cast<uint2*>(a.xq + brow * (a.K / 2) + (long long)b * 8) = make_uint2(lo, hi);
      a.xs[brow * (a.K / 16) + b] = (uint8_t)sbits;
    }
  }
#ifdef NVFP4WS_TRACE
  __syncthreads();
  if (threadIdx.x == 0 && blockIdx.x < 56) g_cta_trace[(200 + blockIdx.x) * 16 + 1] = globaltimer();
#endif
}

// ------------------------------------------------------------------ GEMM

struct Params {
  float* Y;
  int y_bf16;
  const float* ts;
  const float* xg;          // [M, T]
  int M, T, nb;             // nb = M*T B rows
  int nbt, nb_tile;         // B tiles per MMA K-step and rows per B tile (multiple of 8)
  int nsfb;                 // TMEM columns of B scales per (K-step, B tile): 4 (<=128 rows) or 8
  long long N, K;
  int tiles, kch;
  long long units;
  int grid, stages;
  uint32_t stage_bytes, xq_off, sfw_off, xs_off;
  int acc_bufs;             // 1 or 2 accumulator buffers
  int sf_bufs;              // scale-factor TMEM buffers (2..stages); unit i uses buffer i % sf_bufs
  uint32_t sf_cols;         // TMEM columns per scale-factor buffer
  uint32_t acc_col0, acc_stride;
  unsigned int* counters;
  float* partials;
  int verify;
  float* part_val;
  int* part_idx;
  unsigned int* err;
};

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_mma_mxf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                            uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p; }" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
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
__device__ __forceinline__ void tc_st_x8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
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

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// K-major, 128-byte-swizzle shared-memory descriptor (8-row groups 1024 B apart).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__device__ __forceinline__ long long unit_begin(long long c, long long U, int G) { return c * U / G; }
__device__ __forceinline__ int cta_of_unit(long long u, long long U, int G) {
  int c = (int)(u * G / U);
  while (c + 1 < G && unit_begin(c + 1, U, G) <= u) ++c;
  while (c > 0 && unit_begin(c, U, G) > u) --c;
  return c;
}

template <int NBT>
__global__ void __launch_bounds__(kThreads, 1)
    mxf4_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_sf,
                const __grid_constant__ CUtensorMap tm_xq, const __grid_constant__ CUtensorMap tm_xs,
                const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int S = p.stages;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)S * p.stage_bytes);
  // [0,S) full  [S,2S) mma_done (one commit per unit: frees the stage and the unit's scale buffer)
  // 2S+{0,1} acc_full  2S+{2,3} acc_empty  2S+4 drain  2S+5+{0..7} sf_full
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * S + 13);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_last = reinterpret_cast<int*>(s_tmem + 2);
  float* s_val = reinterpret_cast<float*>(s_tmem + 4);                 // [4][72]
  int* s_idx = reinterpret_cast<int*>(s_val + 4 * 72);                 // [4][72]
  float* s_g = reinterpret_cast<float*>(s_idx + 4 * 72);               // [kMaxB]

  auto bar_full = [&](int s) { return smem_u32(bars + s); };
  auto bar_empty = [&](int s) { return smem_u32(bars + S + s); };
  auto bar_accfull = [&](int b) { return smem_u32(bars + 2 * S + b); };
  auto bar_accempty = [&](int b) { return smem_u32(bars + 2 * S + 2 + b); };
  const uint32_t bar_drain = smem_u32(bars + 2 * S + 4);
  auto bar_sffull = [&](int b) { return smem_u32(bars + 2 * S + 5 + b); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const long long U = p.units;
  const long long u_begin = unit_begin(c, U, p.grid), u_end = unit_begin(c + 1, U, p.grid);
  const int nunits = (int)(u_end - u_begin);

  if (threadIdx.x == 0) MX_CTA(0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(bar_full(s), 1); mbar_init(bar_empty(s), 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(bar_accfull(b), 1); mbar_init(bar_accempty(b), 128); }
    for (int b = 0; b < p.sf_bufs; ++b) mbar_init(bar_sffull(b), 128);
    mbar_init(bar_drain, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) MX_CTA(1);
  const uint32_t tmem = *s_tmem;
  const uint32_t bytes_x = (uint32_t)(p.nbt * p.nb_tile) * (128u + 16u);
  const uint32_t tx = kNibBytes + kSfBytes + bytes_x;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
      int issued = 0;
      // (tile, kc) of unit u_begin + i advance incrementally: no 64-bit divisions in the loop
      const int tile0 = (int)(u_begin / p.kch), kc0 = (int)(u_begin % p.kch);
      auto load_w = [&](int s, int tile, int kc) {
        const uint32_t st = sbase + (uint32_t)s * p.stage_bytes;
        mbar_arrive_expect_tx(bar_full(s), tx);
        tma_load_2d(st, &tm_q, kc * (kKC / 2), tile * kTileRows, bar_full(s), pol_w);
        tma_load_2d(st + p.sfw_off, &tm_sf, kc * (kKC / 16), tile * kTileRows, bar_full(s), pol_w);
      };
      auto load_x = [&](int s, int kc) {
        const uint32_t st = sbase + (uint32_t)s * p.stage_bytes;
        for (int bt = 0; bt < p.nbt; ++bt) {
          tma_load_2d(st + p.xq_off + bt * p.nb_tile * 128, &tm_xq, kc * (kKC / 2), bt * p.nb_tile, bar_full(s), pol_x);
          tma_load_2d(st + p.xs_off + bt * p.nb_tile * 16, &tm_xs, kc * (kKC / 16), bt * p.nb_tile, bar_full(s), pol_x);
        }
      };
      // weights of the first stages do not depend on the activation prep: load them first
      const int pre = nunits < S ? nunits : S;
      {
        int tile = tile0, kc = kc0;
        for (int i = 0; i < pre; ++i) {
          load_w(i, tile, kc);
          issued = i + 1;
          if (++kc == p.kch) { kc = 0; ++tile; }
        }
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
      {
        int kc = kc0;
        for (int i = 0; i < pre; ++i) {
          load_x(i, kc);
          if (++kc == p.kch) kc = 0;
        }
      }
      {
        int tile = tile0 + (kc0 + pre) / p.kch, kc = (kc0 + pre) % p.kch;
        int s = pre % S;
        uint32_t ph = (uint32_t)(pre / S) & 1u;
        for (int i = pre; i < nunits; ++i) {
          if (!mbar_wait(bar_empty(s), ph ^ 1u, s_abort, p.err)) break;
          MX_TRACE(0, i);
          load_w(s, tile, kc);
          load_x(s, kc);
          issued = i + 1;
          if (++kc == p.kch) { kc = 0; ++tile; }
          if (++s == S) { s = 0; ph ^= 1u; }
        }
      }
      if (*s_abort) {
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i) {
          const unsigned long long t0 = globaltimer();
          while (!mbar_try_wait(bar_full(i % S), (uint32_t)(i / S) & 1u) && globaltimer() - t0 < kWaitLimitNs) {}
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int seg = 0;
      bool ok = true;
      int s = 0, kc = (int)(u_begin % p.kch);
      uint32_t ph = 0;
      const uint32_t idesc = (1u << 7) | (1u << 10) | ((uint32_t)(p.nb_tile >> 3) << 17) |
                             ((uint32_t)(kTileRows >> 4) << 24);
      // Everything an MMA needs is precomputed: the single issuing thread is
      // latency-bound on scalar work between MMAs, so the loop does adds only.
      const uint64_t adesc_base = sw128_desc(sbase);
      const uint64_t bdesc_base = sw128_desc(sbase + p.xq_off);
      const uint64_t stage_step = (uint64_t)(p.stage_bytes >> 4);
      uint64_t adesc = adesc_base, bdesc = bdesc_base;
      uint32_t boff[NBT], doff[NBT], sfboff[4][NBT];
#pragma unroll
      for (int bt = 0; bt < NBT; ++bt) {
        boff[bt] = (uint32_t)(bt * p.nb_tile * 8);
        doff[bt] = (uint32_t)(bt * p.nb_tile);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) sfboff[kk][bt] = 16u + (uint32_t)((kk * NBT + bt) * p.nsfb);
      }
      int fb = 0;                                     // scale-factor buffer of unit i
      uint32_t fph = 0;
      const uint32_t acc0 = tmem + p.acc_col0, acc1 = tmem + p.acc_col0 + p.acc_stride;
      for (int i = 0; i < nunits && ok; ++i) {
        const bool seg_first = (i == 0) || (kc == 0);
        const bool seg_last = (i == nunits - 1) || (kc == p.kch - 1);
        const int ab = (p.acc_bufs == 2) ? (seg & 1) : 0;
        if (seg_first) {
          const uint32_t acc_use = (p.acc_bufs == 2) ? (uint32_t)(seg >> 1) : (uint32_t)seg;
          ok = mbar_wait(bar_accempty(ab), (acc_use & 1u) ^ 1u, s_abort, p.err);
          if (!ok) break;
        }
        MX_TRACE(11, i);
        ok = mbar_wait(bar_full(s), ph, s_abort, p.err);
        MX_TRACE(1, i);
        ok = ok && mbar_wait(bar_sffull(fb), fph, s_abort, p.err);
        if (!ok) break;
        MX_TRACE(2, i);
        if (i == 0) MX_CTA(2);
        tc_fence_after();
        const uint32_t sf = tmem + (uint32_t)fb * p.sf_cols;
        const uint32_t d0 = ab ? acc1 : acc0;
        const uint32_t first = seg_first ? 0u : 1u;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
          for (int bt = 0; bt < NBT; ++bt)
            tc_mma_mxf4(d0 + doff[bt], adesc + (uint64_t)(kk * 2), bdesc + (uint64_t)(boff[bt] + kk * 2), idesc,
                        sf + (uint32_t)(kk * 4), sf + sfboff[kk][bt], kk == 0 ? first : 1u);
        }
        MX_TRACE(3, i);
        tc_commit(bar_empty(s));                      // stage s and scale buffer fb are free once these retire
        if (seg_last) { tc_commit(bar_accfull(ab)); ++seg; }
        MX_TRACE(4, i);
        if (++kc == p.kch) kc = 0;
        if (++fb == p.sf_bufs) { fb = 0; fph ^= 1u; }
        if (++s == S) { s = 0; ph ^= 1u; adesc = adesc_base; bdesc = bdesc_base; }
        else { adesc += stage_step; bdesc += stage_step; }
      }
      MX_CTA(3);
      tc_commit(bar_drain);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(bar_drain, 0) && globaltimer() - t0 < kWaitLimitNs) {}
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ scale factors -> TMEM
    const int q = warp & 3;                 // lane quarter; every quarter holds the same values
    const int m0 = lane;
    int s = 0;
    uint32_t ph = 0;
    const int NF = p.sf_bufs;
    int s2 = S - NF;                // ring position of unit i - NF (valid once i >= NF)
    uint32_t ph2 = 1u;
    int fb = 0;
    uint32_t fph = 0;
    for (int i = 0; i < nunits; ++i) {
      if (!mbar_wait(bar_full(s), ph, s_abort, p.err)) break;
      if (lane == 0 && warp == 4) MX_TRACE(5, i);
      // scale buffer fb was last read by the MMAs of unit i - NF
      if (i >= NF && !mbar_wait(bar_empty(s2), ph2, s_abort, p.err)) break;
      if (lane == 0 && warp == 4) MX_TRACE(6, i);
      tc_fence_after();
      const uint32_t st = sbase + (uint32_t)s * p.stage_bytes;
      const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)fb * p.sf_cols;
      {   // W scales: column 4*kk + j of lane m0 = the 4 block scales (K-step kk) of tile row m0 + 32*j
        uint4 R[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) R[j] = lds128(st + p.sfw_off + (uint32_t)((m0 + 32 * j) * 16));
        uint32_t out[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          out[0 + j] = R[j].x; out[4 + j] = R[j].y; out[8 + j] = R[j].z; out[12 + j] = R[j].w;
        }
        tc_st_x16(lane_base, out);
      }
      for (int bt = 0; bt < p.nbt; ++bt) {   // X-term scales, per B tile: nsfb columns per K-step
        uint4 R[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int row = m0 + 32 * j;
          R[j] = (j < p.nsfb && row < p.nb_tile) ? lds128(st + p.xs_off + (uint32_t)((bt * p.nb_tile + row) * 16))
                                                 : make_uint4(0, 0, 0, 0);
        }
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t out[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) out[j] = kk == 0 ? R[j].x : kk == 1 ? R[j].y : kk == 2 ? R[j].z : R[j].w;
          const uint32_t col = 16u + (uint32_t)((kk * p.nbt + bt) * p.nsfb);
          if (p.nsfb == 8) {
            tc_st_x8(lane_base + col, out);
          } else {
            uint32_t o4[8] = {out[0], out[1], out[2], out[3], 0, 0, 0, 0};
            asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(lane_base + col),
                         "r"(o4[0]), "r"(o4[1]), "r"(o4[2]), "r"(o4[3])
                         : "memory");
          }
        }
      }
      tc_wait_st();
      tc_fence_before();
      if (lane == 0 && warp == 4) MX_TRACE(7, i);
      if (lane == 0 && warp == 7) MX_TRACE(8, i);
      mbar_arrive(bar_sffull(fb));
      (void)fph;
      if (++fb == NF) { fb = 0; fph ^= 1u; }
      if (++s == S) { s = 0; ph ^= 1u; }
      if (++s2 == S) { s2 = 0; ph2 ^= 1u; }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ epilogue
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int q = warp & 3;
    const int rowl = q * 32 + lane;
    const int et = threadIdx.x - 8 * 32;
    for (int j = et; j < p.nb; j += 128) s_g[j] = p.xg[j];
    named_bar(1, 128);
    const float ts = *p.ts;
    int seg = 0;
    int tile = (int)(u_begin / p.kch), kc = (int)(u_begin % p.kch);
    for (int i = 0; i < nunits; ++i) {
      const long long u = u_begin + i;
      const bool seg_last = (i == nunits - 1) || (kc == p.kch - 1);
      const int cur_tile = tile;
      if (++kc == p.kch) { kc = 0; ++tile; }
      if (!seg_last) continue;
      const long long tile_u0 = (long long)cur_tile * p.kch, tile_u1 = tile_u0 + p.kch;
      const long long seg_u0 = u_begin > tile_u0 ? u_begin : tile_u0;
      const bool complete = (seg_u0 == tile_u0) && (u + 1 == tile_u1);
      const int ab = (p.acc_bufs == 2) ? (seg & 1) : 0;
      const uint32_t acc_use = (p.acc_bufs == 2) ? (uint32_t)(seg >> 1) : (uint32_t)seg;
      if (!mbar_wait(bar_accfull(ab), acc_use & 1u, s_abort, p.err)) break;
      if (et == 0) MX_TRACE(9, seg);
      if (et == 0 && seg < 2) MX_CTA(8 + 4 * seg);
      tc_fence_after();
      const long long n = (long long)cur_tile * kTileRows + rowl;
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + p.acc_col0 + (uint32_t)ab * p.acc_stride;
      const int slot = (seg_u0 == u_begin) ? 2 * c : 2 * c + 1;
      float* dst = p.partials + ((long long)slot * p.M) * kTileRows;
      // Fold the T terms of each token: y[m] = sum_t g[m,t] * acc[m*T + t]. Accumulator
      // column c holds B row c, so token m's terms are columns m*T .. m*T+T-1. Tokens are
      // taken 16 at a time: up to 5 TMEM loads of 16 columns are issued back to back and
      // waited for once, and the fold uses the compile-time term count.
      static_assert(kMxf4Terms == 5, "the fold below is written for 5 terms");
      const int nb16 = (p.nb + 15) & ~15;                 // columns that exist in the accumulator
      for (int mc = 0; mc < p.M; mc += 16) {
        const int col0 = mc * kMxf4Terms;                 // multiple of 80
        const int nld = (nb16 - col0) / 16 < 5 ? (nb16 - col0) / 16 : 5;
        uint32_t v[80];
        tc_ld_x16(taddr + (uint32_t)col0, *reinterpret_cast<uint32_t(*)[16]>(v));
        if (nld > 1) tc_ld_x16(taddr + (uint32_t)(col0 + 16), *reinterpret_cast<uint32_t(*)[16]>(v + 16));
        if (nld > 2) tc_ld_x16(taddr + (uint32_t)(col0 + 32), *reinterpret_cast<uint32_t(*)[16]>(v + 32));
        if (nld > 3) tc_ld_x16(taddr + (uint32_t)(col0 + 48), *reinterpret_cast<uint32_t(*)[16]>(v + 48));
        if (nld > 4) tc_ld_x16(taddr + (uint32_t)(col0 + 64), *reinterpret_cast<uint32_t(*)[16]>(v + 64));
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = mc + j;
          if (m >= p.M) break;
          float ym = 0.f;
#pragma unroll
          for (int t = 0; t < kMxf4Terms; ++t)
            ym = fmaf(s_g[m * kMxf4Terms + t], __uint_as_float(v[j * kMxf4Terms + t]), ym);
          if (complete) {
            const float y = ym * ts;
            if (p.verify) {
              float bv = (n < p.N) ? y : -INFINITY;
              int bi = (n < p.N) ? (int)n : INT_MAX;
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (argmax_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
              }
              if (lane == 0) { s_val[q * 72 + m] = bv; s_idx[q * 72 + m] = bi; }
            } else if (n < p.N) {
              if (p.y_bf16) reinterpret_cast<uint16_t*>(p.Y)[(long long)m * p.N + n] = f32_to_bf16_rn(y);
              else p.Y[(long long)m * p.N + n] = y;
            }
          } else {
            dst[(long long)m * kTileRows + rowl] = ym;
          }
        }
      }
      tc_fence_before();
      if (et == 0) MX_TRACE(10, seg);
      if (et == 0 && seg < 2) MX_CTA(9 + 4 * seg);
      mbar_arrive(bar_accempty(ab));
      ++seg;
      if (complete) {
        if (p.verify) {
          named_bar(1, 128);
          if (et < p.M) {
            float bv = s_val[et];
            int bi = s_idx[et];
            for (int w = 1; w < 4; ++w)
              if (argmax_better(s_val[w * 72 + et], s_idx[w * 72 + et], bv, bi)) { bv = s_val[w * 72 + et]; bi = s_idx[w * 72 + et]; }
            p.part_val[(long long)cur_tile * p.M + et] = bv;
            p.part_idx[(long long)cur_tile * p.M + et] = bi;
          }
          named_bar(1, 128);
        }
        continue;
      }
      __threadfence();
      if (et == 0 && seg <= 2) MX_CTA(10 + 4 * (seg - 1));
      named_bar(1, 128);
      if (et == 0) {
        const int c0 = cta_of_unit(tile_u0, U, p.grid), c1 = cta_of_unit(tile_u1 - 1, U, p.grid);
        int expected = 0;
        for (int cc = c0; cc <= c1; ++cc)
          if (unit_begin(cc + 1, U, p.grid) > unit_begin(cc, U, p.grid)) ++expected;
        const unsigned int prev = atomicAdd(p.counters + cur_tile, 1u);
        *s_last = (prev + 1 == (unsigned int)expected) ? 1 : 0;
      }
      named_bar(1, 128);
      if (*s_last) {
        __threadfence();
        const int c0 = cta_of_unit(tile_u0, U, p.grid), c1 = cta_of_unit(tile_u1 - 1, U, p.grid);
        // 16 tokens at a time: issue all partial loads of a chunk before summing them, so
        // the fix-up costs one L2 round trip per (chunk, contributor), not one per token.
        for (int mc = 0; mc < p.M; mc += 16) {
          float acc[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[j] = 0.f;
          for (int cc = c0; cc <= c1; ++cc) {
            const long long b0 = unit_begin(cc, U, p.grid), b1 = unit_begin(cc + 1, U, p.grid);
            if (b1 <= b0) continue;
            const int sl = (b0 >= tile_u0) ? 2 * cc : 2 * cc + 1;
            const float* src = p.partials + ((long long)sl * p.M) * kTileRows + rowl;
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = (mc + j < p.M) ? __ldcg(src + (long long)(mc + j) * kTileRows) : 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] += v[j];
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = mc + j;
            if (m >= p.M) break;
            const float y = acc[j] * ts;
            if (p.verify) {
              float bv = (n < p.N) ? y : -INFINITY;
              int bi = (n < p.N) ? (int)n : INT_MAX;
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (argmax_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
              }
              if (lane == 0) { s_val[q * 72 + m] = bv; s_idx[q * 72 + m] = bi; }
            } else if (n < p.N) {
              if (p.y_bf16) reinterpret_cast<uint16_t*>(p.Y)[(long long)m * p.N + n] = f32_to_bf16_rn(y);
              else p.Y[(long long)m * p.N + n] = y;
            }
          }
        }
        if (p.verify) {
          named_bar(1, 128);
          if (et < p.M) {
            float bv = s_val[et];
            int bi = s_idx[et];
            for (int w = 1; w < 4; ++w)
              if (argmax_better(s_val[w * 72 + et], s_idx[w * 72 + et], bv, bi)) { bv = s_val[w * 72 + et]; bi = s_idx[w * 72 + et]; }
            p.part_val[(long long)cur_tile * p.M + et] = bv;
            p.part_idx[(long long)cur_tile * p.M + et] = bi;
          }
        }
        if (et == 0) p.counters[cur_tile] = 0u;
      }
      named_bar(1, 128);
      if (et == 0 && seg <= 2) MX_CTA(11 + 4 * (seg - 1));
    }
  }

  if (threadIdx.x == 8 * 32) MX_CTA(4);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
  if (threadIdx.x == 0) MX_CTA(5);
}

}  // namespace mxk

// ============================================================================ host side

using namespace mxk;

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn_mx() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

static bool map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                   uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto fn = encode_fn_mx();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct MxPlan {
  int T, nb, nbt, nb_tile, nsfb, tiles, kch, grid, stages, acc_bufs, sf_bufs;
  long long units;
  uint32_t stage_bytes, xq_off, sfw_off, xs_off, sf_cols, acc_col0, acc_stride;
  size_t smem;
};

static size_t al256(size_t v) { return (v + 255) / 256 * 256; }

static MxPlan mx_plan(long long M, long long N, long long K) {
  MxPlan pl{};
  pl.T = kMxf4Terms;
  pl.nb = (int)M * pl.T;
  pl.nbt = (pl.nb + 255) / 256;
  pl.nb_tile = ((pl.nb + pl.nbt - 1) / pl.nbt + 15) / 16 * 16;   // MMA N; a multiple of 16 keeps x16 loads inside the tile
  pl.nsfb = pl.nb_tile <= 128 ? 4 : 8;
  pl.sf_cols = 16u + 4u * (uint32_t)(pl.nbt * pl.nsfb);
  pl.acc_stride = (uint32_t)(pl.nbt * pl.nb_tile);
  pl.acc_bufs = (2 * pl.sf_cols + 2 * pl.acc_stride <= 512) ? 2 : 1;
  pl.tiles = (int)((N + kTileRows - 1) / kTileRows);
  pl.kch = (int)(K / kKC);
  pl.units = (long long)pl.tiles * pl.kch;
  const int sms = std::max(1, device_sm_count());
  pl.grid = (int)std::min<long long>(sms, pl.units);
  const uint32_t xq = (uint32_t)(pl.nbt * pl.nb_tile) * 128u;
  const uint32_t xs = (uint32_t)(pl.nbt * pl.nb_tile) * 16u;
  pl.xq_off = kNibBytes;
  pl.sfw_off = (pl.xq_off + xq + 1023) / 1024 * 1024;
  pl.xs_off = pl.sfw_off + kSfBytes;
  pl.stage_bytes = (pl.xs_off + xs + 1023) / 1024 * 1024;
  const size_t budget = 227 * 1024 - 1024 - kTailBytes;
  pl.stages = (int)std::min<size_t>(8, budget / pl.stage_bytes);
  pl.smem = 1024 + (size_t)pl.stages * pl.stage_bytes + kTailBytes;
  // scale-factor buffers: one per ring stage when TMEM allows (the scale copy then runs ahead like TMA)
  const uint32_t acc_cols = (uint32_t)pl.acc_bufs * pl.acc_stride;
  pl.sf_bufs = (int)std::min<uint32_t>((uint32_t)pl.stages, (512u - acc_cols) / pl.sf_cols);
  if (pl.sf_bufs < 2) pl.sf_bufs = 2;
  pl.acc_col0 = (uint32_t)pl.sf_bufs * pl.sf_cols;
  return pl;
}

bool mxf4_supported(long long M, long long K) {
  return M >= 1 && M * kMxf4Terms <= kMaxB && K % kKC == 0 && K >= kKC && K <= 32768;
}

// workspace: counters | partials [2*grid][M][128] | xq [nb][K/2] | xs [nb][K/16] | xg [M][T] | (verify) part val/idx
static void mx_ws_layout(long long M, long long N, long long K, size_t* off_part, size_t* off_xq, size_t* off_xs,
                         size_t* off_xg, size_t* off_pv, size_t* off_pi, size_t* total) {
  MxPlan pl = mx_plan(M, N, K);
  size_t o = al256((size_t)pl.tiles * 4);
  *off_part = o; o += al256((size_t)2 * pl.grid * M * kTileRows * 4);
  *off_xq = o; o += al256((size_t)pl.nb * (K / 2));
  *off_xs = o; o += al256((size_t)pl.nb * (K / 16));
  *off_xg = o; o += al256((size_t)pl.nb * 4);
  *off_pv = o; o += al256((size_t)pl.tiles * M * 4);
  *off_pi = o; o += al256((size_t)pl.tiles * M * 4);
  *total = o;
}

size_t mxf4_workspace_bytes(long long M, long long N, long long K) {
  if (!mxf4_supported(M, K)) return 0;
  size_t a, b, c, d, e, f, t;
  mx_ws_layout(M, N, K, &a, &b, &c, &d, &e, &f, &t);
  return t;
}

size_t mxf4_counter_bytes(long long M, long long N, long long K) {
  return mxf4_supported(M, K) ? al256((size_t)mx_plan(M, N, K).tiles * 4) : 0;
}

static int launch_mxf4(const uint16_t* X, const uint8_t* q, const uint8_t* sf, const float* ts, long long M,
                       long long N, long long K, void* Y, int y_dtype, void* workspace, bool verify, float** pv_out,
                       int** pi_out, int* nparts_out, cudaStream_t s) {
  MxPlan pl = mx_plan(M, N, K);
  size_t off_part, off_xq, off_xs, off_xg, off_pv, off_pi, total;
  mx_ws_layout(M, N, K, &off_part, &off_xq, &off_xs, &off_xg, &off_pv, &off_pi, &total);
  char* ws = static_cast<char*>(workspace);

  // 1) activation decomposition
  XPrepArgs xa{};
  xa.X = X; xa.M = (int)M; xa.T = pl.T; xa.K = K;
  xa.xq = reinterpret_cast<uint8_t*>(ws + off_xq);
  xa.xs = reinterpret_cast<uint8_t*>(ws + off_xs);
  xa.xg = reinterpret_cast<float*>(ws + off_xg);
  const int bpt = (int)((K / 16 + kPrepThreads - 1) / kPrepThreads);
  if (bpt <= 1) x_prep_kernel<1><<<(int)M, kPrepThreads, 0, s>>>(xa);
  else if (bpt == 2) x_prep_kernel<2><<<(int)M, kPrepThreads, 0, s>>>(xa);
  else if (bpt == 3) x_prep_kernel<3><<<(int)M, kPrepThreads, 0, s>>>(xa);
  else x_prep_kernel<4><<<(int)M, kPrepThreads, 0, s>>>(xa);
  if (int e = check_launch("x_prep_kernel")) return e;

  // 2) the GEMM, launched as a programmatic dependent of the prep kernel
  alignas(64) CUtensorMap tq, tsf, txq, txs;
  if (!map_u8(&tq, q, K / 2, N, kKC / 2, kTileRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map_u8(&tsf, sf, K / 16, N, kKC / 16, kTileRows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !map_u8(&txq, ws + off_xq, K / 2, pl.nb, kKC / 2, pl.nb_tile, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map_u8(&txs, ws + off_xs, K / 16, pl.nb, kKC / 16, pl.nb_tile, CU_TENSOR_MAP_SWIZZLE_NONE))
    return set_error(NVFP4WS_ERR_CUDA, "cuTensorMapEncodeTiled failed (mxf4 path)");
  Params p{};
  p.Y = static_cast<float*>(Y);
  p.y_bf16 = (y_dtype == NVFP4WS_Y_BF16);
  p.ts = ts;
  p.xg = reinterpret_cast<const float*>(ws + off_xg);
  p.M = (int)M; p.T = pl.T; p.nb = pl.nb; p.nbt = pl.nbt; p.nb_tile = pl.nb_tile; p.nsfb = pl.nsfb;
  p.N = N; p.K = K; p.tiles = pl.tiles; p.kch = pl.kch; p.units = pl.units; p.grid = pl.grid; p.stages = pl.stages;
  p.stage_bytes = pl.stage_bytes; p.xq_off = pl.xq_off; p.sfw_off = pl.sfw_off; p.xs_off = pl.xs_off;
  p.acc_bufs = pl.acc_bufs; p.sf_bufs = pl.sf_bufs; p.sf_cols = pl.sf_cols; p.acc_col0 = pl.acc_col0; p.acc_stride = pl.acc_stride;
  p.counters = reinterpret_cast<unsigned int*>(ws);
  p.partials = reinterpret_cast<float*>(ws + off_part);
  p.verify = verify ? 1 : 0;
  p.part_val = reinterpret_cast<float*>(ws + off_pv);
  p.part_idx = reinterpret_cast<int*>(ws + off_pi);
  if (verify) { *pv_out = p.part_val; *pi_out = p.part_idx; *nparts_out = pl.tiles; }
  p.err = device_error_word();
  if (!p.err) return set_error(NVFP4WS_ERR_CUDA, "cannot resolve the device error word");
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(mxf4_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess ||
        cudaFuncSetAttribute(mxf4_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
      return check_launch("cudaFuncSetAttribute(mxf4_kernel)");
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = (pl.nbt == 1) ? cudaLaunchKernelEx(&cfg, mxf4_kernel<1>, tq, tsf, txq, txs, p)
                                 : cudaLaunchKernelEx(&cfg, mxf4_kernel<2>, tq, tsf, txq, txs, p);
  if (e != cudaSuccess) return set_error(NVFP4WS_ERR_CUDA, "mxf4_kernel launch: %s", cudaGetErrorString(e));
  return check_launch("mxf4_kernel");
}

int launch_mxf4_gemm(const uint16_t* X, const uint8_t* q, const uint8_t* sf, const float* ts, long long M,
                     long long N, long long K, void* Y, int y_dtype, void* workspace, cudaStream_t s) {
  return launch_mxf4(X, q, sf, ts, M, N, K, Y, y_dtype, workspace, false, nullptr, nullptr, nullptr, s);
}

int launch_mxf4_verify(const uint16_t* X, const uint8_t* q, const uint8_t* sf, const float* ts, long long M,
                       long long N, long long K, const int32_t* drafts, int B, int D, int32_t* argmax,
                       int32_t* accept_len, float* max_logit, void* workspace, cudaStream_t s) {
  float* pv = nullptr;
  int* pi = nullptr;
  int nparts = 0;
  if (int e = launch_mxf4(X, q, sf, ts, M, N, K, nullptr, 0, workspace, true, &pv, &pi, &nparts, s)) return e;
  return launch_verify_stage2(pv, pi, nparts, (int)M, drafts, B, D, argmax, accept_len, max_logit, s);
}

}  // namespace nvfp4ws

#ifdef NVFP4WS_TRACE
// Copies the timeline of the last traced launch (16 fields x 64 units of CTA 0) to the host.
extern "C" int nvfp4ws_trace_read(unsigned long long* host, int n) {
  if (n > 16 * 64) n = 16 * 64;
  return cudaMemcpyFromSymbol(host, nvfp4ws::mxk::g_trace, sizeof(unsigned long long) * n) == cudaSuccess ? 0 : 5;
}
// Per-CTA global-timer events: [256][8] (GEMM CTAs 0..147; prep kernel rows at 200+m).
extern "C" int nvfp4ws_trace_cta_read(unsigned long long* host) {
  return cudaMemcpyFromSymbol(host, nvfp4ws::mxk::g_cta_trace, sizeof(unsigned long long) * 256 * 16) == cudaSuccess ? 0 : 5;
}
#endif
