// Block-scaled tensor-core path: tcgen05.mma kind::mxf4nvf4 on packed NVFP4 weights,
// for one GEMM or for a whole list of them (a weight pass) in one persistent launch.
//
// Why. On B200 a tcgen05.mma kind::f16 instruction (M=128, K=16) costs ~70-96 SM
// cycles for every N up to 128 (measured). So a path that dequantises W to f16
// is capped near 29 weights/clk/SM (~4.6 TB/s), before the cost of
// dequantisation itself. kind::mxf4nvf4 instead consumes the packed E2M1 weights
// straight from shared memory with their E4M3 block scales: K=64 per
// instruction, with no per-element work on the CUDA cores at all.
//
// The catch is that both operands must be NVFP4. The activations are bf16, so
// they are represented as T residual NVFP4 terms with one row amax:
//   g_0 = amax|x| / 2688,  g_t = g_0 / 4^t,  r_0 = x,  for t < T:
//       S_t = E4M3(amax_block(r_t) / (6 g_t)),  c_t = E2M1(r_t / (S_t g_t)),  r_{t+1} = r_t - c_t S_t g_t
// so x = sum_t g_t S_t c_t + r_T. One E2M1 code with its E4M3 block scale leaves
// at most ~0.18 of the block magnitude behind, so r_t stays below 6 * 448 * g_t
// and every S_t fits E4M3. Each term cuts the error about 10x; with T = 5 the
// GEMM matches the exact float64 result to ~1e-5 relative and logits to ~5e-5
// absolute. The terms are extra B rows (token m, term t -> row m*T + t). The
// epilogue folds them: y[m] = ts * sum_t g_t acc[m*T+t]. With T = 1 (the W4A4
// product) the single term is the NVFP4 quantisation of the row, its code taken
// and scale taken from the exact quotients, rounded once (the weights' rule).
//
// Kernels.
//   x_prep_kernel   one CTA per (activation row, problem; a single GEMM splits each row over
//                   several CTAs along K): the T-term decomposition,
//                   written as per-K-chunk images that are byte-for-byte the shared
//                   memory operand (128-byte-swizzled code rows, then 16 scale bytes
//                   per row). The GEMM fetches each with ONE contiguous bulk copy:
//                   measured on B200, a 2D tensor box gathering R rows of 128 B from
//                   L2 cuts the concurrent HBM weight stream by 11% (R=16) to 50%
//                   (R=352); a contiguous bulk copy of the same bytes costs ~3%.
//   pass_kernel     one persistent CTA per SM, 12 warps, over the concatenated units
//                   of all problems: a group of 1-2 128-row tiles x 1-2 256-wide
//                   K-chunks. Consecutive problems whose images fit L2 together form a
//                   wave, and each wave's units are split evenly across the CTAs
//                   (stream-K), so a tile is split between CTAs only at the G-1 range
//                   boundaries of a wave.
//     warp 0        TMA producer: the W tiles (128 rows x 128 B nibbles, SW128) and
//                   their 128 x 16 B scales (2D tensor loads), then the activation
//                   images (1D bulk). Codes stream evict-first; scale lines and images,
//                   which are read again, evict-last. The first stages' weight loads
//                   are issued before waiting on the prep kernel.
//     warp 1        TMEM allocator and MMA issuer: 4 K-steps x B-tiles x tiles of
//                   tcgen05.mma kind::mxf4nvf4.block_scale.block16 per K-chunk.
//     warps 4-7     scale-factor warpgroup: copies the unit's W and X block scales
//                   from shared memory into TMEM in the layout the MMA reads (the 4
//                   scales of row m0 + 32*j in column j of lane m0, replicated over the
//                   four lane quarters), all of a chunk's shared loads first.
//     warps 8-11    epilogue: tcgen05.ld of the accumulators; several terms (5, or 4 in
//                   a pass that asks for them) are folded into registers and the
//                   accumulator is released before any store, one term is streamed 16
//                   tokens at a time; then x ts and Y, the per-tile argmax of a verify
//                   problem, or a split tile's partials, which the last CTA to finish the
//                   tile sums in CTA order (with tile-pair units, the CTA's final such sum
//                   is done by all 12 warps once the role loops end).
// Every wait is bounded (see sync.cuh); a timeout sets the device error word.
#include "common.cuh"
#include "kernels.h"
#include "mma.h"
#include "sync.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <vector>

namespace nvfp4ws {
namespace mxk {

// Optional timelines for pipeline analysis, compiled out unless NVFP4WS_TRACE is
// defined; they change no work. g_trace: clock64 per unit of CTA 0 at each hand-off.
// g_cta_trace: per-CTA global-timer events (ns): [cta][event].
#ifdef NVFP4WS_TRACE
__device__ unsigned long long g_trace[16 * 64];
#define MX_TRACE(f, i) do { if (blockIdx.x == 0 && (i) < 64) g_trace[(f) * 64 + (i)] = clock64(); } while (0)
__device__ unsigned long long g_cta_trace[256 * 16];
#define MX_CTA(e) do { if (blockIdx.x < 256) g_cta_trace[blockIdx.x * 16 + (e)] = globaltimer(); } while (0)
#else
#define MX_TRACE(f, i) do { } while (0)
#define MX_CTA(e) do { } while (0)
#endif

constexpr int kThreads = 384;
constexpr int kTileRows = 128;
constexpr int kKC = 256;                           // one K-chunk; a unit is 1 or 2 chunks (Geom::ku)
constexpr int kNibBytes = kTileRows * kKC / 2;     // 16 KB of W codes per chunk (one SW128 block)
constexpr int kSfBytes = kTileRows * kKC / 16;     // 2 KB of W scales per chunk
constexpr uint32_t kWChunk = kNibBytes + kSfBytes; // weight bytes per chunk (1024-aligned)
constexpr int kMaxStages = 12;
constexpr int kMaxB = 352;                         // B rows (tokens x terms) the TMEM budget allows
constexpr size_t kTailBytes = 8192;
constexpr int kMaxSfBufs = 8;
constexpr int kFixupBatch = 12;                    // contributors whose partials a deferred sum loads at once

// One GEMM of a launch. Lives in device memory (a pass) or in the kernel's parameter
// space (a single GEMM); the tensor maps are read by TMA from wherever it lives.
struct alignas(64) Problem {
  CUtensorMap tm_q;        // W codes [N, K/2] u8, box 128 B x 128 rows, 128-byte swizzle
  CUtensorMap tm_sf;       // W scales [N, K/16] u8, box 16 B x 128 rows
  const uint16_t* X;       // [M, K] bf16
  uint8_t* ximg;           // [K/256][img_stride] activation-term images, one per 256-wide chunk
  float* xg;               // [M*T] per-term global scales
  const float* ts;         // W tensor scale (device)
  void* Y;                 // [M, N] f32 or bf16 (unused by a verify problem)
  float* part_val;         // verify problem: per-tile row maxima [tiles][M]
  int* part_idx;           //                 and their indices
  long long N;
  unsigned int unit0;      // first unit of this problem in the launch's unit numbering
  int K, kch, tiles, y_bf16, verify;
  int groups;              // groups of tpu tiles: units are (group, K-chunk)
};

// What depends on M alone, shared by every problem of a launch.
struct Geom {
  int M, T, nb, nbt, nb_tile, nsfb;
  int ku;                  // 256-wide K-chunks per unit (1 or 2)
  int tpu;                 // 128-row weight tiles per unit (1 or 2); they share the unit's activation images
  uint32_t img_bytes;      // one chunk's image: nbt*nb_tile rows x (128 B codes + 16 B scales)
  uint32_t img_stride;     // images are 1024-byte aligned (the MMA operand's swizzle atom)
  uint32_t img_xs_off;     // offset of the scale rows in an image
  uint32_t wbytes;         // weight bytes of a unit: tpu x ku x (codes + scales)
};

struct PassParams {
  Geom g;
  const Problem* probs;    // device array, or nullptr: the single problem passed by value
  int nprob;
  // Waves: consecutive problems whose activation images fit L2 together. Units of wave w
  // are [wave_u0[w], wave_u0[w+1]); each is split evenly across the CTAs (stream-K), so
  // at any time every CTA works on the same few problems. nullptr: one wave of `units`.
  const uint32_t* wave_u0; // [nwave + 1]
  const int* cta_prob;     // [nwave][grid] problem holding each CTA's first unit of a wave
  const int* cta_units;    // [grid] units of each CTA over all waves
  int nwave;
  unsigned int units;
  int grid, stages;
  uint32_t stage_bytes;    // one stage: W codes (tpu x ku blocks), W scales (tpu tiles), then ku activation images
  int acc_bufs, sf_bufs;
  uint32_t sf_cols, acc_col0, acc_stride;
  unsigned int* counters;  // [nwave][grid] split-tile tickets, zero on entry and on exit
  float* partials;         // [nwave][2*grid][tpu][128 rows][Mp] split-tile partial sums, Mp = M rounded up to 4
  unsigned int* err;
};

// ------------------------------------------------------------------ activation decomposition

__device__ __forceinline__ float block_amax16(const float (&v)[16]) {
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[i]));
  return a;
}

// One CTA per (activation row, problem). A first sweep over the row finds amax|x|
// (one CTA reduction; each thread has four blocks' loads in flight before it uses any),
// a second re-reads it (from L2) and writes the T terms of each 16-element block. On the
// path of a single GEMM the prep's latency is paid in full, so its registers are not
// squeezed for occupancy (measured: 40 registers with spills and one round trip per block
// made the prep 4-8 us after the previous kernel ended; 64 registers and the unrolled
// sweep, 3-5 us). Per-thread state is small, so several CTAs fit an SM and the many
// short rows of a pass are prepared at once. Repeated
// multiplication by 0.25 is exact unless g underflows; the decomposition and the stored
// g follow the same sequence. The code and scale choices only need to be consistent
// with the residual they leave (which is exact), so they use reciprocal multiplies.
constexpr int kPrepThreads = 256;

__device__ __forceinline__ void load_block16(const uint16_t* X, int b, float (&r)[16]) {
  const uint4* src = reinterpret_cast<const uint4*>(X + (long long)b * 16);
  const uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
  const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    r[2 * i] = __uint_as_float(w[i] << 16);
    r[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// v narrowed to fp32 by rounding to odd: the result rounded to nearest (ties to even) in any
// format with at most 22 significant bits equals the single rounding of v itself, when v is
// the correctly rounded double of a quotient of an 8-bit by a <= 28-bit number (such a
// quotient is either exact in fp32 or at least 2^-52 away from every fp32 value, so the
// double rounding loses no sticky bit).
__device__ __forceinline__ float to_f32_odd(double v) {
  float r = __double2float_rz(v);
  if ((double)r != v) r = __uint_as_float(__float_as_uint(r) | 1u);
  return r;
}

// |q| within a relative 2^-20 of a point where E2M1 rounding changes (0.25, 0.75, 1.25,
// 1.75, 2.5, 3.5, 5): an fp32 quotient with a few ulps of error may decide such a q wrongly.
__device__ __forceinline__ bool near_e2m1_midpoint(float q) {
  const float a = fabsf(q), t = a * 0x1p-20f;
  return (fabsf(a - 0.25f) <= t) | (fabsf(a - 0.75f) <= t) | (fabsf(a - 1.25f) <= t) | (fabsf(a - 1.75f) <= t) |
         (fabsf(a - 2.5f) <= t) | (fabsf(a - 3.5f) <= t) | (fabsf(a - 5.0f) <= t);
}

// One NVFP4 term of block b (the W4A4 activations): the weights' two-level rule with the
// row scale g in place of the tensor scale, both quotients exact and rounded once:
//   S = E4M3_rne_satfinite(amax_block / (6 g)),  c = E2M1_rne_satfinite(x / (S g)).
// 6 g and S g are exact in double. The scale takes a correctly rounded double quotient; the
// codes take an fp32 quotient and, within 2^-20 of a rounding point, the exact one.
__device__ __forceinline__ void quantise_block_single(const float (&r)[16], int b, int m, float g0, const Geom& g,
                                                      uint8_t* img) {
  const int kc = b >> 4, bi = b & 15;
  uint8_t* base = img + (size_t)kc * g.img_stride;
  uint32_t sbits = 0, lo = 0, hi = 0;
  if (g0 > 0.f) {
    const double g64 = (double)g0;
    uint16_t s2;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
        : "=h"(s2) : "f"(0.0f), "f"(to_f32_odd(__ddiv_rn((double)block_amax16(r), 6.0 * g64))));
    sbits = s2 & 0xFFu;
    const double den = (double)f16lo_to_f32(e4m3x2_to_f16x2(sbits)) * g64;
    if (den > 0.0) {
      const bool fast = den >= 0x1p-100;
      const float inv = fast ? __frcp_rn((float)den) : 0.f;
      float q[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        q[i] = r[i] * inv;
        if (!fast || near_e2m1_midpoint(q[i])) q[i] = to_f32_odd(__ddiv_rn((double)r[i], den));
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint16_t c2;
        asm("{ .reg .b8 b; cvt.rn.satfinite.e2m1x2.f32 b, %1, %2; cvt.u16.u8 %0, b; }"
            : "=h"(c2) : "f"(q[2 * i + 1]), "f"(q[2 * i]));
        if (i < 4) lo |= (uint32_t)(c2 & 0xFF) << (8 * i);
        else hi |= (uint32_t)(c2 & 0xFF) << (8 * (i - 4));
      }
    }
  }
  const uint32_t off = (uint32_t)m * 128u + ((uint32_t)((bi >> 1) ^ (m & 7)) << 4) + ((uint32_t)(bi & 1) << 3);
  *reinterpret_cast<uint2*>(base + off) = make_uint2(lo, hi);
  base[g.img_xs_off + (uint32_t)m * 16u + (uint32_t)bi] = (uint8_t)sbits;
}

// The T terms of block b (16 values in r) into the chunk images; gt0 = g_0, inv6 = 1/(6 g_t).
template <int T>
__device__ __forceinline__ void quantise_block(float (&r)[16], int b, int m, float gt0, const float (&inv6)[T],
                                               const Geom& g, uint8_t* img) {
  if constexpr (T == 1) {
    quantise_block_single(r, b, m, gt0, g, img);
    return;
  }
  const int kc = b >> 4, bi = b & 15;           // K-chunk and block within it
  uint8_t* base = img + (size_t)kc * g.img_stride;
  float gt = gt0;
#pragma unroll
  for (int term = 0; term < T; ++term, gt *= 0.25f) {
    uint32_t sbits = 0, lo = 0, hi = 0;
    if (gt > 0.f) {
      uint16_t s2;
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(s2) : "f"(0.0f), "f"(block_amax16(r) * inv6[term]));
      sbits = s2 & 0xFFu;
      const float den = f16lo_to_f32(e4m3x2_to_f16x2(sbits)) * gt;
      if (den > 0.f) {
        const float inv = rcp_approx(den);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint16_t c2;
          // Approximate codes are fine here: each residual is exact and the next term corrects it.
          const float q1 = r[2 * i + 1] * inv;
          const float q0 = r[2 * i] * inv;
          asm("{ .reg .b8 b; cvt.rn.satfinite.e2m1x2.f32 b, %1, %2; cvt.u16.u8 %0, b; }"
              : "=h"(c2) : "f"(q1), "f"(q0));
          const uint32_t h = e2m1x2_to_f16x2(c2);
          r[2 * i] = fmaf(-f16lo_to_f32(h), den, r[2 * i]);
          r[2 * i + 1] = fmaf(-f16hi_to_f32(h), den, r[2 * i + 1]);
          if (i < 4) lo |= (uint32_t)(c2 & 0xFF) << (8 * i);
          else hi |= (uint32_t)(c2 & 0xFF) << (8 * (i - 4));
        }
      }
    }
    // B row of (token m, term): its 128 code bytes for this chunk, with the 16-byte
    // pieces permuted by the 128-byte swizzle (piece p of row r at p ^ (r & 7)).
    const int row = m * T + term;
    const uint32_t off = (uint32_t)row * 128u + ((uint32_t)((bi >> 1) ^ (row & 7)) << 4) + ((uint32_t)(bi & 1) << 3);
    *reinterpret_cast<uint2*>(base + off) = make_uint2(lo, hi);
    base[g.img_xs_off + (uint32_t)row * 16u + (uint32_t)bi] = (uint8_t)sbits;
  }
}

// slices: CTAs per activation row. Each takes the row's amax over all of K, then writes the
// terms of its share of the row's blocks. One slice serves a pass (thousands of rows run at
// once); a single GEMM splits each row so that the prep's latency, which the GEMM waits for,
// does not grow with K.
template <int T>
__global__ void __launch_bounds__(kPrepThreads, 4) x_prep_kernel(const __grid_constant__ Problem single,
                                                                  const Problem* probs, const Geom g, int slices) {
  asm volatile("griddepcontrol.launch_dependents;");
  // X may come from the previous kernel of the stream, and the previous GEMM may still
  // read this workspace: nothing is read or written before that kernel has finished.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int row_cta = blockIdx.x / slices, sl = blockIdx.x - row_cta * slices;
  const int m = row_cta % g.M;
  const Problem* pr = probs ? probs + row_cta / g.M : &single;
  const int nblk = pr->K / 16;
  const uint16_t* X = pr->X + (long long)m * pr->K;
  uint8_t* img = pr->ximg;
  __shared__ float s_red[kPrepThreads / 32];
  // amax over the row, four blocks' loads in flight per thread before any is used (a loop
  // that uses each load before issuing the next costs one memory round trip per block)
  float amax = 0.f;
  for (int b = t; b < nblk; b += 4 * kPrepThreads) {
    uint4 u[4][2];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int bb = b + k * kPrepThreads;
      const uint4* src = reinterpret_cast<const uint4*>(X + (long long)bb * 16);
      u[k][0] = bb < nblk ? __ldg(src) : make_uint4(0u, 0u, 0u, 0u);
      u[k][1] = bb < nblk ? __ldg(src + 1) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t w[8] = {u[k][0].x, u[k][0].y, u[k][0].z, u[k][0].w, u[k][1].x, u[k][1].y, u[k][1].z, u[k][1].w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
        amax = fmaxf(amax, fmaxf(__uint_as_float((w[i] << 16) & 0x7FFFFFFFu), __uint_as_float(w[i] & 0x7FFF0000u)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) s_red[warp] = amax;
  __syncthreads();
  amax = 0.f;
#pragma unroll
  for (int w = 0; w < kPrepThreads / 32; ++w) amax = fmaxf(amax, s_red[w]);
  const float g0 = amax / 2688.0f;
  float inv6[T];
  {
    float gt = g0;
#pragma unroll
    for (int term = 0; term < T; ++term, gt *= 0.25f) {
      inv6[term] = gt > 0.f ? 1.0f / (6.0f * gt) : 0.f;
      if (t == 0 && sl == 0) pr->xg[m * T + term] = gt;
    }
  }
  const int b1 = (int)((long long)(sl + 1) * nblk / slices);
  for (int b = (int)((long long)sl * nblk / slices) + t; b < b1; b += kPrepThreads) {
    float r[16];
    load_block16(X, b, r);
    quantise_block<T>(r, b, m, g0, inv6, g, img);
  }
}

// ------------------------------------------------------------------ GEMM

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
__device__ __forceinline__ void tc_st_x4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ void tc_ld_x16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tc_ld_x8(uint32_t taddr, uint32_t* v) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
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

// Stream-K partition: CTA c owns units [floor(c*U/G), floor((c+1)*U/G)). The host keeps
// G <= U (every CTA owns at least one unit) and U * G < 2^32, so 32-bit arithmetic is exact.
__device__ __forceinline__ uint32_t unit_begin(uint32_t c, uint32_t U, uint32_t G) { return c * U / G; }
// The CTA owning unit u: the largest c with floor(c*U/G) <= u.
__device__ __forceinline__ uint32_t cta_of_unit(uint32_t u, uint32_t U, uint32_t G) { return ((u + 1) * G - 1) / U; }

// Position of a unit: problem, tile group, K-chunk. Advances without divisions; a
// problem's sizes are read once when the walk enters it.
struct Cursor {
  int pi, tile, kc, kch, tiles;   // tile: the tile group; tiles: groups in the problem
  __device__ __forceinline__ void init(const Problem* probs, int p0, uint32_t u) {
    pi = p0;
    kch = probs[pi].kch;
    tiles = probs[pi].groups;
    const uint32_t rel = u - probs[pi].unit0;
    tile = (int)(rel / (uint32_t)kch);
    kc = (int)(rel - (uint32_t)tile * (uint32_t)kch);
  }
  __device__ __forceinline__ void advance(const Problem* probs, int nprob) {
    if (++kc < kch) return;
    kc = 0;
    if (++tile < tiles) return;
    tile = 0;
    if (++pi < nprob) { kch = probs[pi].kch; tiles = probs[pi].groups; }
  }
};

// The units one CTA processes, wave by wave: in wave w of Uw units starting at w0,
// CTA c owns [w0 + floor(c*Uw/G), w0 + floor((c+1)*Uw/G)) (at least one unit: the host
// makes every wave at least G units long).
struct Walk {
  int w;                   // current wave
  uint32_t w0, Uw;         // its first unit and size
  uint32_t r0, r1;         // this CTA's range in it
  uint32_t u;              // current unit
  Cursor cu;
  __device__ __forceinline__ void start(const PassParams& p, const Problem* probs, int c, int w_) {
    w = w_;
    w0 = p.wave_u0 ? p.wave_u0[w] : 0u;
    Uw = (p.wave_u0 ? p.wave_u0[w + 1] : p.units) - w0;
    r0 = w0 + unit_begin((uint32_t)c, Uw, (uint32_t)p.grid);
    r1 = w0 + unit_begin((uint32_t)c + 1u, Uw, (uint32_t)p.grid);
    u = r0;
    cu.init(probs, p.cta_prob ? p.cta_prob[w * p.grid + c] : 0, u);
  }
  // Advance one unit; at the end of a wave's range jump to the next wave (callers stop
  // after the CTA's unit count, so no wave past the last is started).
  __device__ __forceinline__ void next(const PassParams& p, const Problem* probs, int c) {
    if (++u < r1) { cu.advance(probs, p.nprob); return; }
    if (w + 1 < p.nwave) start(p, probs, c, w + 1);
  }
  __device__ __forceinline__ bool first() const { return u == r0; }
  __device__ __forceinline__ bool last() const { return u + 1 == r1; }
  // Units left in the current segment: to the end of the tile or of this wave's range.
  __device__ __forceinline__ int seg_units() const {
    const uint32_t to_tile = (uint32_t)(cu.kch - cu.kc), to_range = r1 - u;
    return (int)(to_tile < to_range ? to_tile : to_range);
  }
  // Skip the n units that finish the current segment (n == seg_units()).
  __device__ __forceinline__ void skip_segment(const PassParams& p, const Problem* probs, int c, int n) {
    u += (uint32_t)n;
    if (u == r1) {
      if (w + 1 < p.nwave) start(p, probs, c, w + 1);
      return;
    }
    cu.kc = 0;
    if (++cu.tile < cu.tiles) return;
    cu.tile = 0;
    if (++cu.pi < p.nprob) { cu.kch = probs[cu.pi].kch; cu.tiles = probs[cu.pi].groups; }
  }
};

// Most tokens a kernel instance serves, rounded up to 8 (the fold takes 8 tokens at a
// time). Several terms: the row is folded in registers; two B tiles hold M*T <= 352 rows
// (T = 5: M <= 70), one B tile M*T <= 256, and a tile pair needs a double-buffered
// accumulator, which leaves N <= 104 per tile (T = 5: M <= 20). One term (W4A4): the row
// is streamed from TMEM, so only the B rows bound M (352).
__host__ __device__ constexpr int pass_max_tokens(int nbt, int tpu, int terms) {
  return terms == 1 ? kMaxB : ((tpu == 2 ? 104 : nbt == 2 ? kMaxB : 256) / terms + 7) / 8 * 8;
}


// T: activation terms (kGemmTerms or kVerifyTerms residual terms, or 1 for NVFP4 activations).
template <int NBT, int KU, int TPU, int T>
__global__ void __launch_bounds__(kThreads, 1)
    pass_kernel(const __grid_constant__ Problem single, const PassParams p) {
  // The next kernel of the stream may launch as soon as SMs free up: the library's prep
  // kernel waits for this grid to finish before touching the workspace or its input.
  asm volatile("griddepcontrol.launch_dependents;");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int S = p.stages;
  const Geom& g = p.g;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)S * p.stage_bytes);
  // [0,S) full  [S,2S) empty (one MMA commit per unit frees the stage and the unit's scale
  // buffer)  2S+{0,1} acc_full  2S+{2,3} acc_empty  2S+4 drain  2S+5+{0..7} sf_full
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * S + 5 + kMaxSfBufs);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_last = reinterpret_cast<int*>(s_tmem + 2);
  float* s_val = reinterpret_cast<float*>(s_tmem + 4);                 // [4][72]
  int* s_idx = reinterpret_cast<int*>(s_val + 4 * 72);                 // [4][72]
  // g_0 of each token of the current problem, 16-byte aligned for float4 reads [kMaxB]
  float* s_g0 = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(s_idx + 4 * 72) + 15) & ~uintptr_t(15));
  // the split tile group whose partials the whole CTA sums after the role loops (on = 0: none)
  struct DeferredFixup {
    int on, pi, group, c0, c1, wave;
    uint32_t tile_u0, w0, Uw;
  };
  DeferredFixup* s_def = reinterpret_cast<DeferredFixup*>(s_g0 + kMaxB);

  auto bar_full = [&](int s) { return smem_u32(bars + s); };
  auto bar_empty = [&](int s) { return smem_u32(bars + S + s); };
  auto bar_accfull = [&](int b) { return smem_u32(bars + 2 * S + b); };
  auto bar_accempty = [&](int b) { return smem_u32(bars + 2 * S + 2 + b); };
  const uint32_t bar_drain = smem_u32(bars + 2 * S + 4);
  auto bar_sffull = [&](int b) { return smem_u32(bars + 2 * S + 5 + b); };

  constexpr int MT = pass_max_tokens(NBT, TPU, T);
  const Problem* probs = p.probs ? p.probs : &single;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const uint32_t G = (uint32_t)p.grid;
  const int nunits = p.cta_units ? p.cta_units[c]
                                 : (int)(unit_begin((uint32_t)c + 1u, p.units, G) - unit_begin((uint32_t)c, p.units, G));

  if (threadIdx.x == 0) MX_CTA(0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(bar_full(s), 1); mbar_init(bar_empty(s), 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(bar_accfull(b), 1); mbar_init(bar_accempty(b), 128); }
    for (int b = 0; b < p.sf_bufs; ++b) mbar_init(bar_sffull(b), 128);
    mbar_init(bar_drain, 1);
    *s_abort = 0;
    s_def->on = 0;
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // Weight codes stream through L2 once (evict-first). A row's 128-byte scale line
      // serves eight consecutive K-chunks, and every CTA of a problem reads the same
      // activation images, so both stay (evict-last).
      const uint64_t pol_w = policy_evict_first(), pol_sf = policy_evict_last(), pol_x = policy_evict_last();
      const uint32_t xbytes = (uint32_t)g.ku * g.img_stride;
      const uint32_t tx = g.wbytes + xbytes;
      int issued = 0;
      auto load_w = [&](int s, const Cursor& cu) {
        const uint32_t st = sbase + (uint32_t)s * p.stage_bytes;
        const Problem* pr = probs + cu.pi;
        mbar_arrive_expect_tx(bar_full(s), tx);
        for (int j = 0; j < g.tpu; ++j) {
          const int row = (cu.tile * g.tpu + j) * kTileRows;   // rows past N read as zeros
          for (int h = 0; h < g.ku; ++h)
            tma_load_2d(st + (uint32_t)(j * g.ku + h) * kNibBytes, &pr->tm_q, (cu.kc * g.ku + h) * (kKC / 2), row,
                        bar_full(s), pol_w);
          tma_load_2d(st + (uint32_t)(g.tpu * g.ku) * kNibBytes + (uint32_t)j * (kTileRows * 16u * g.ku), &pr->tm_sf,
                      cu.kc * g.ku * (kKC / 16), row, bar_full(s), pol_sf);
        }
      };
      auto load_x = [&](int s, const Cursor& cu) {
        bulk_load(sbase + (uint32_t)s * p.stage_bytes + g.wbytes, probs[cu.pi].ximg + (size_t)cu.kc * xbytes, xbytes,
                  bar_full(s), pol_x);
      };
      // weights of the first stages do not depend on the activation prep: load them first
      const int pre = nunits < S ? nunits : S;
      Walk wk;
      wk.start(p, probs, c, 0);
      for (int i = 0; i < pre; ++i) { load_w(i, wk.cu); issued = i + 1; wk.next(p, probs, c); }
      asm volatile("griddepcontrol.wait;" ::: "memory");
      {
        Walk wx;
        wx.start(p, probs, c, 0);
        for (int i = 0; i < pre; ++i) { load_x(i, wx.cu); wx.next(p, probs, c); }
      }
      int s = pre % S;
      uint32_t ph = (uint32_t)(pre / S) & 1u;
      for (int i = pre; i < nunits; ++i) {
        if (!mbar_wait(bar_empty(s), ph ^ 1u, s_abort, p.err)) break;
        MX_TRACE(0, i);
        load_w(s, wk.cu);
        load_x(s, wk.cu);
        issued = i + 1;
        wk.next(p, probs, c);
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (*s_abort) {   // let the copies in flight land before the CTA exits
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i) {
          const unsigned long long t0 = globaltimer();
          while (!mbar_try_wait(bar_full(i % S), (uint32_t)(i / S) & 1u) && globaltimer() - t0 < kWaitLimitNs) {}
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The single issuing thread is latency-bound, so its loop is kept minimal: it waits
    // only for the unit's scale buffer. The scale warps arrive on it after observing the
    // stage's TMA completion, and that arrive/wait pair (release/acquire) orders the
    // landed operands before the MMAs. Descriptors are precomputed and advanced by adds.
    if (lane == 0) {
      int seg = 0;
      bool ok = true;
      int s = 0;
      Walk wk;
      wk.start(p, probs, c, 0);
      const uint32_t idesc = (1u << 7) | (1u << 10) | ((uint32_t)(g.nb_tile >> 3) << 17) |
                             ((uint32_t)(kTileRows >> 4) << 24);
      const uint64_t adesc_base = sw128_desc(sbase), bdesc_base = sw128_desc(sbase + g.wbytes);
      const uint64_t step = (uint64_t)(p.stage_bytes >> 4);
      uint64_t adesc = adesc_base, bdesc = bdesc_base;
      // K-step kk of chunk h: A (tile j) at block j*KU + h, B in image h, scales in columns
      // laid out as the scale warps store them (W: 4 per K-step and tile, tile-major; then X:
      // nsfb per K-step and B tile). Tile j accumulates at column j*NBT*nb_tile.
      uint32_t boff[KU][NBT], doff[TPU][NBT], sfboff[KU][4][NBT];
#pragma unroll
      for (int bt = 0; bt < NBT; ++bt) {
#pragma unroll
        for (int j = 0; j < TPU; ++j) doff[j][bt] = (uint32_t)((j * NBT + bt) * g.nb_tile);
#pragma unroll
        for (int h = 0; h < KU; ++h) {
          boff[h][bt] = (h * g.img_stride >> 4) + (uint32_t)(bt * g.nb_tile * 8);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            sfboff[h][kk][bt] = 16u * KU * TPU + (uint32_t)(((h * 4 + kk) * NBT + bt) * g.nsfb);
        }
      }
      int fb = 0;                                     // scale-factor buffer of unit i
      uint32_t fph = 0;
      const uint32_t acc0 = tmem + p.acc_col0, acc1 = tmem + p.acc_col0 + p.acc_stride;
      // Segment bookkeeping is a countdown: the walk is consulted once per segment.
      int seg_len = 0, seg_left = 0;
      const bool two_acc = p.acc_bufs == 2;
      for (int i = 0; i < nunits && ok; ++i) {
        const bool seg_first = seg_left == 0;
        const int ab = two_acc ? (seg & 1) : 0;
        if (seg_first) {
          seg_len = seg_left = wk.seg_units();
          const uint32_t acc_use = two_acc ? (uint32_t)(seg >> 1) : (uint32_t)seg;
          ok = mbar_wait(bar_accempty(ab), (acc_use & 1u) ^ 1u, s_abort, p.err);
          if (!ok) break;
        }
        ok = mbar_wait(bar_sffull(fb), fph, s_abort, p.err);
        if (!ok) break;
        MX_TRACE(2, i);
        if (i == 0) MX_CTA(2);
        tc_fence_after();
        const uint32_t sf = tmem + (uint32_t)fb * p.sf_cols;
        const uint32_t d0 = ab ? acc1 : acc0;
        const uint32_t first = seg_first ? 0u : 1u;
#pragma unroll
        for (int h = 0; h < KU; ++h) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int j = 0; j < TPU; ++j) {
#pragma unroll
              for (int bt = 0; bt < NBT; ++bt)
                tc_mma_mxf4(d0 + doff[j][bt], adesc + (uint64_t)((j * KU + h) * (kNibBytes >> 4) + kk * 2),
                            bdesc + (uint64_t)(boff[h][bt] + kk * 2), idesc,
                            sf + (uint32_t)((j * 4 * KU + h * 4 + kk) * 4), sf + sfboff[h][kk][bt],
                            (h == 0 && kk == 0) ? first : 1u);
            }
          }
        }
        MX_TRACE(3, i);
        tc_commit(bar_empty(s));                      // stage s and scale buffer fb are free once these retire
        if (--seg_left == 0) {
          tc_commit(bar_accfull(ab));
          ++seg;
          wk.skip_segment(p, probs, c, seg_len);
        }
        if (++fb == p.sf_bufs) { fb = 0; fph ^= 1u; }
        if (++s == S) { s = 0; adesc = adesc_base; bdesc = bdesc_base; }
        else { adesc += step; bdesc += step; }
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
    const int NF = p.sf_bufs;               // <= S
    int s2 = S - NF;                        // ring position of unit i - NF (valid once i >= NF)
    uint32_t ph2 = 1u;
    int fb = 0;
    const uint32_t wsf_row = 16u * (uint32_t)g.ku;                          // W scales: row m has 16*ku bytes
    const uint32_t wsf_off = (uint32_t)(g.tpu * g.ku) * kNibBytes;          // tile j's scales at + j*128*wsf_row
    const uint32_t xsf_col = 16u * (uint32_t)(g.ku * g.tpu);                // X scale columns follow the W ones
    for (int i = 0; i < nunits; ++i) {
      if (!mbar_wait(bar_full(s), ph, s_abort, p.err)) break;
      if (lane == 0 && warp == 4) MX_TRACE(5, i);
      // scale buffer fb was last read by the MMAs of unit i - NF
      if (i >= NF && !mbar_wait(bar_empty(s2), ph2, s_abort, p.err)) break;
      tc_fence_after();
      const uint32_t st = sbase + (uint32_t)s * p.stage_bytes;
      const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)fb * p.sf_cols;
      // All of a chunk's shared loads are issued before its first TMEM store: under a
      // saturated ring one round trip to shared memory costs ~250 cycles, and three
      // dependent rounds (W, then each B tile) made this copy the slowest hand-off at M=68.
#pragma unroll
      for (int h = 0; h < KU; ++h) {
        uint4 RW[TPU][4], RX[NBT][8];
        const uint32_t xs = st + g.wbytes + (uint32_t)h * g.img_stride + g.img_xs_off;
#pragma unroll
        for (int t = 0; t < TPU; ++t) {
          const uint32_t wsf = st + wsf_off + (uint32_t)t * (kTileRows * wsf_row);
#pragma unroll
          for (int j = 0; j < 4; ++j) RW[t][j] = lds128(wsf + (uint32_t)(m0 + 32 * j) * wsf_row + (uint32_t)h * 16u);
        }
#pragma unroll
        for (int bt = 0; bt < NBT; ++bt) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int row = m0 + 32 * j;
            RX[bt][j] = (j < g.nsfb && row < g.nb_tile) ? lds128(xs + (uint32_t)((bt * g.nb_tile + row) * 16))
                                                        : make_uint4(0, 0, 0, 0);
          }
        }
        // W scales of tile t: column 16*(t*ku + h) + 4*kk + j of lane m0 = the 4 block scales
        // (K-step kk of chunk h) of row m0 + 32*j
#pragma unroll
        for (int t = 0; t < TPU; ++t) {
          uint32_t out[16];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            out[0 + j] = RW[t][j].x; out[4 + j] = RW[t][j].y; out[8 + j] = RW[t][j].z; out[12 + j] = RW[t][j].w;
          }
          tc_st_x16(lane_base + (uint32_t)(t * KU + h) * 16u, out);
        }
        if (NBT == 1 && g.nsfb == 4) {
          // one B tile of <= 128 rows: the chunk's 4 K-steps x 4 columns are contiguous, so
          // column 4*kk + j of lane m0 (B row m0 + 32*j, K-step kk) goes in one x16 store
          uint32_t out[16];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            out[0 + j] = RX[0][j].x; out[4 + j] = RX[0][j].y; out[8 + j] = RX[0][j].z; out[12 + j] = RX[0][j].w;
          }
          tc_st_x16(lane_base + xsf_col + (uint32_t)h * 16u, out);
          continue;
        }
#pragma unroll
        for (int bt = 0; bt < NBT; ++bt) {   // X-term scales, per B tile: nsfb columns per K-step
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            uint32_t out[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              out[j] = kk == 0 ? RX[bt][j].x : kk == 1 ? RX[bt][j].y : kk == 2 ? RX[bt][j].z : RX[bt][j].w;
            const uint32_t col = xsf_col + (uint32_t)(((h * 4 + kk) * NBT + bt) * g.nsfb);
            if (g.nsfb == 8) tc_st_x8(lane_base + col, out);
            else tc_st_x4(lane_base + col, out[0], out[1], out[2], out[3]);
          }
        }
      }
      tc_wait_st();
      tc_fence_before();
      if (lane == 0 && warp == 4) MX_TRACE(7, i);
      mbar_arrive(bar_sffull(fb));
      if (++fb == NF) fb = 0;
      if (++s == S) { s = 0; ph ^= 1u; }
      if (++s2 == S) { s2 = 0; ph2 ^= 1u; }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ epilogue
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int q = warp & 3;
    const int rowl = q * 32 + lane;
    const int et = threadIdx.x - 8 * 32;
    const int M = g.M;
    int gprob = -1;                         // problem whose term scales are in s_g
    int seg = 0;
    Walk wk;
    wk.start(p, probs, c, 0);
    for (int done = 0; done < nunits;) {   // one iteration per segment
      const int n_seg = wk.seg_units();
      const uint32_t u = wk.u + (uint32_t)(n_seg - 1), r0 = wk.r0, w0 = wk.w0, Uw = wk.Uw;   // u: the segment's last unit
      const int wave = wk.w;
      const int pi = wk.cu.pi, group = wk.cu.tile, kch = wk.cu.kch;
      wk.skip_segment(p, probs, c, n_seg);
      done += n_seg;
      const Problem* pr = probs + pi;
      const uint32_t tile_u0 = pr->unit0 + (uint32_t)group * (uint32_t)kch, tile_u1 = tile_u0 + (uint32_t)kch;
      const uint32_t seg_u0 = r0 > tile_u0 ? r0 : tile_u0;
      const bool complete = (seg_u0 == tile_u0) && (u + 1 == tile_u1);
      if (pi != gprob) {
        named_bar(1, 128);
        for (int j = et; j < M; j += 128) s_g0[j] = pr->xg[j * T];
        named_bar(1, 128);
        gprob = pi;
      }
      const float ts = *pr->ts;
      const long long N = pr->N;
      const int verify = pr->verify, y_bf16 = pr->y_bf16, tiles = pr->tiles;
      float* Yf = static_cast<float*>(pr->Y);
      const int ab = (p.acc_bufs == 2) ? (seg & 1) : 0;
      const uint32_t acc_use = (p.acc_bufs == 2) ? (uint32_t)(seg >> 1) : (uint32_t)seg;
      if (!mbar_wait(bar_accfull(ab), acc_use & 1u, s_abort, p.err)) break;
      if (et == 0 && seg < 2) MX_CTA(8 + 4 * seg);
      tc_fence_after();
      const uint32_t taddr0 = tmem + ((uint32_t)(q * 32) << 16) + p.acc_col0 + (uint32_t)ab * p.acc_stride;
      const int Mp = (M + 3) & ~3;
      float* wave_part = p.partials + (long long)wave * 2 * G * g.tpu * kTileRows * Mp;
      const int slot = (seg_u0 == r0) ? 2 * c : 2 * c + 1;
      // Finished outputs of row n for tokens mc .. mc+15 (y[j], already x ts).
      // Verify problem: each token's argmax candidate of the 4 warps' rows. Otherwise Y,
      // one token per warp-wide 128-byte store (measured: a 4x4 shuffle transpose into
      // 16-byte stores was slower here, Y rows being N floats apart).
      auto emit16 = [&](long long n, int mc, const float (&y)[16]) {
        if (verify) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = mc + j;
            if (m >= M) break;
            float bv = (n < N) ? y[j] : -INFINITY;
            int bi = (n < N) ? (int)n : INT_MAX;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
              const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
              if (argmax_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
            }
            if (lane == 0) { s_val[q * 72 + m] = bv; s_idx[q * 72 + m] = bi; }
          }
          return;
        }
        if (n < N) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = mc + j;
            if (m >= M) break;
            if (y_bf16) reinterpret_cast<uint16_t*>(Yf)[(long long)m * N + n] = f32_to_bf16_rn(y[j]);
            else Yf[(long long)m * N + n] = y[j];
          }
        }
      };
      auto tile_argmax = [&](int tile) {  // combine the 4 warps' candidates of each row
        named_bar(1, 128);
        if (et < M) {
          float bv = s_val[et];
          int bi = s_idx[et];
          for (int w = 1; w < 4; ++w)
            if (argmax_better(s_val[w * 72 + et], s_idx[w * 72 + et], bv, bi)) { bv = s_val[w * 72 + et]; bi = s_idx[w * 72 + et]; }
          pr->part_val[(long long)tile * M + et] = bv;
          pr->part_idx[(long long)tile * M + et] = bi;
        }
        named_bar(1, 128);
      };
      // Fold the T terms of each token: y[m] = sum_t g_t acc[m*T + t] with g_t = g_0 / 4^t,
      // i.e. g_0 * (acc_0 + (acc_1 + (... + acc_{T-1}/4)/4)/4) (the multiplications by 1/4
      // are exact; the prep kernel's g_t are the same sequence unless it underflows).
      // Accumulator column j holds B row j, so token m's terms are columns m*T .. m*T+T-1.
      // Tokens are taken 8 at a time: T TMEM loads of 8 columns are issued back to back and
      // waited for once. The folded row (at most MT tokens) stays in registers, so the
      // accumulator is handed back to the MMA thread before any global store: with one
      // accumulator buffer (M=68) the stores of a tile then overlap the next tile's MMAs
      // (measured: holding the buffer through the stores stalled the MMA thread ~15 us per
      // tile under full HBM load).
      if constexpr (T > 1) {
        const int nb16 = (g.nb + 15) & ~15;                 // columns that exist in the accumulator
        float yr[TPU][MT];
#pragma unroll
        for (int tj = 0; tj < TPU; ++tj) {
          const uint32_t taddr = taddr0 + (uint32_t)(tj * NBT * g.nb_tile);
#pragma unroll
          for (int mc = 0; mc < MT; mc += 8) {
            if (mc < M) {
              const int col0 = mc * T;                        // multiple of 8T
              const int n8 = (nb16 - col0) >> 3;              // >= 1: loads stay inside the accumulator
              uint32_t v[8 * T];
#pragma unroll
              for (int k = 0; k < T; ++k)
                if (k < n8) tc_ld_x8(taddr + (uint32_t)(col0 + 8 * k), v + 8 * k);
              const float4 ga = reinterpret_cast<const float4*>(s_g0 + mc)[0];
              const float4 gb = reinterpret_cast<const float4*>(s_g0 + mc)[1];
              const float g0[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
              tc_wait_ld();
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                float a = __uint_as_float(v[j * T + T - 1]);
#pragma unroll
                for (int t = T - 2; t >= 0; --t) a = fmaf(a, 0.25f, __uint_as_float(v[j * T + t]));
                yr[tj][mc + j] = (mc + j < M) ? a * g0[j] : 0.f;   // columns past the tokens are never loaded
              }
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j) yr[tj][mc + j] = 0.f;
            }
          }
        }
        tc_fence_before();
        if (et == 0 && seg < 2) MX_CTA(9 + 4 * seg);
        mbar_arrive(bar_accempty(ab));
#pragma unroll
        for (int tj = 0; tj < TPU; ++tj) {
          const int tile = group * TPU + tj;
          const long long n = (long long)tile * kTileRows + rowl;
          if (complete) {
#pragma unroll
            for (int mc = 0; mc < MT; mc += 16) {
              if (mc < M) {
                float y16[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  const int m = mc + j < MT ? mc + j : MT - 1;    // static index; tokens >= M are zeros
                  y16[j] = (mc + j < MT) ? yr[tj][m] * ts : 0.f;
                }
                emit16(n, mc, y16);
              }
            }
            if (verify && tile < tiles) tile_argmax(tile);
          } else {
            float* dst = wave_part + ((long long)(slot * TPU + tj) * kTileRows + rowl) * Mp;   // this row's partials
#pragma unroll
            for (int b = 0; b < MT / 4; ++b)
              if (4 * b < Mp)
                *reinterpret_cast<float4*>(dst + 4 * b) =
                    make_float4(yr[tj][4 * b], yr[tj][4 * b + 1], yr[tj][4 * b + 2], yr[tj][4 * b + 3]);
          }
        }
      } else {
        // One term (W4A4): accumulator column j is token j, so there is nothing to fold.
        // Up to 352 tokens do not fit in registers: the row is scaled and stored 16 tokens
        // at a time while the accumulator is held, and handed back after the last load.
        // (The host runs no verify problem here: its candidates are kept for <= 72 rows.)
        static_assert(T == 1, "one term or several");
        for (int tj = 0; tj < TPU; ++tj) {
          const uint32_t taddr = taddr0 + (uint32_t)(tj * NBT * g.nb_tile);
          const int tile = group * TPU + tj;
          const long long n = (long long)tile * kTileRows + rowl;
          float* dst = wave_part + ((long long)(slot * TPU + tj) * kTileRows + rowl) * Mp;   // this row's partials
          for (int mc = 0; mc < M; mc += 16) {
            uint32_t v[16];
            tc_ld_x16(taddr + (uint32_t)mc, v);            // mc + 16 <= (M + 15) & ~15 <= NBT * nb_tile
            float g0[16];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float4 t4 = reinterpret_cast<const float4*>(s_g0 + mc)[k];
              g0[4 * k] = t4.x; g0[4 * k + 1] = t4.y; g0[4 * k + 2] = t4.z; g0[4 * k + 3] = t4.w;
            }
            tc_wait_ld();
            if (tj + 1 == TPU && mc + 16 >= M) {             // last load of the buffer: release it
              tc_fence_before();
              mbar_arrive(bar_accempty(ab));
            }
            float y16[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) y16[j] = (mc + j < M) ? __uint_as_float(v[j]) * g0[j] : 0.f;
            if (complete) {
#pragma unroll
              for (int j = 0; j < 16; ++j) y16[j] *= ts;
              emit16(n, mc, y16);
            } else {
#pragma unroll
              for (int b = 0; b < 4; ++b)
                if (mc + 4 * b < Mp)
                  *reinterpret_cast<float4*>(dst + mc + 4 * b) =
                      make_float4(y16[4 * b], y16[4 * b + 1], y16[4 * b + 2], y16[4 * b + 3]);
            }
          }
        }
      }
      ++seg;
      if (complete) continue;
      // Split tile group: count this CTA's arrival. The barrier orders every epilogue
      // thread's partial stores before thread 0's release; the acquire side of the same
      // atomic orders the last arriver's loads of the other contributors' partials after
      // it. The ticket of a split group is indexed by its first contributing CTA, which
      // has at most one split group starting in its range.
      const int c0 = (int)cta_of_unit(tile_u0 - w0, Uw, G), c1 = (int)cta_of_unit(tile_u1 - 1u - w0, Uw, G);
      unsigned int* ticket = p.counters + (long long)wave * G + c0;
      named_bar(1, 128);
      if (et == 0) {
        unsigned int prev;
        asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(prev) : "l"(ticket) : "memory");
        *s_last = (prev + 1 == (unsigned int)(c1 - c0 + 1)) ? 1 : 0;   // every CTA owns >= 1 unit
      }
      named_bar(1, 128);
      if (et == 0 && seg <= 2) MX_CTA(10 + 4 * (seg - 1));
      // The CTA's final segment of a GEMM with tile-pair units: every warp is free once the
      // role loops end, so the whole CTA sums the partials then (below), with a row's
      // contributors 12 at a time in flight. (Measured on single GEMMs: M=17, tile pairs, a
      // chained 27B pass 7.1 -> 6.7 ms; one tile per unit (M=1, M=68) slightly slower, so
      // those keep the epilogue's own sum.)
      const bool defer = TPU == 2 && *s_last && !verify && done >= nunits;
      if (defer && et == 0) {
        s_def->pi = pi; s_def->group = group; s_def->c0 = c0; s_def->c1 = c1; s_def->wave = wave;
        s_def->tile_u0 = tile_u0; s_def->w0 = w0; s_def->Uw = Uw;
        s_def->on = 1;
        *ticket = 0u;                      // ready for the next launch
      }
      if (*s_last && !defer) {
        // Sum the contributors' partials in CTA order (deterministic), 16 tokens per pass. The
        // loads of four contributors are issued together: a tile split across many CTAs (the
        // down projection's 40 tiles over 148 CTAs) then costs a quarter of the dependent L2
        // round trips, which set the tail of a single GEMM.
        for (int tj = 0; tj < g.tpu; ++tj) {
          const int tile = group * g.tpu + tj;
          const long long n = (long long)tile * kTileRows + rowl;
          for (int mc = 0; mc < M; mc += 16) {
            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = 0.f;
            for (int cc = c0; cc <= c1; cc += 4) {
              float4 v[4][4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int cx = cc + k;
                const bool on = cx <= c1;
                const int sl = on ? ((w0 + unit_begin((uint32_t)cx, Uw, G) >= tile_u0) ? 2 * cx : 2 * cx + 1) : 0;
                const float4* src =
                    reinterpret_cast<const float4*>(wave_part + ((long long)(sl * g.tpu + tj) * kTileRows + rowl) * Mp + mc);
#pragma unroll
                for (int b = 0; b < 4; ++b)
                  v[k][b] = (on && mc + 4 * b < Mp) ? __ldcg(src + b) : make_float4(0.f, 0.f, 0.f, 0.f);
              }
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                if (cc + k <= c1) {
#pragma unroll
                  for (int b = 0; b < 4; ++b) {
                    acc[4 * b] += v[k][b].x; acc[4 * b + 1] += v[k][b].y;
                    acc[4 * b + 2] += v[k][b].z; acc[4 * b + 3] += v[k][b].w;
                  }
                }
              }
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = (mc + j < M) ? acc[j] * ts : 0.f;
            emit16(n, mc, acc);
          }
          if (verify && tile < tiles) tile_argmax(tile);
        }
        if (et == 0) *ticket = 0u;           // ready for the next launch
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
  if (TPU == 2 && s_def->on) {
    // The deferred sum of a split tile group, by all warps: one work item per (tile, row,
    // 8 tokens), its contributors' partials loaded 12 CTAs at a time and added in CTA order,
    // as the epilogue's own sum does (the same bits). The epilogue thread that took the last
    // ticket acquired the other CTAs' partials before the barrier above.
    const DeferredFixup d = *s_def;
    const Problem* pr = probs + d.pi;
    const int M = g.M, Mp = (M + 3) & ~3, ng8 = (M + 7) >> 3;
    const float* wave_part = p.partials + (long long)d.wave * 2 * G * g.tpu * kTileRows * Mp;
    const float ts = *pr->ts;
    const long long N = pr->N;
    const int items = g.tpu * kTileRows * ng8;
    for (int it = threadIdx.x; it < items; it += kThreads) {
      const int row = it % kTileRows, rest = it / kTileRows, mg = rest % ng8, tj = rest / ng8;
      const int mc = mg * 8;
      float acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = 0.f;
      for (int cc = d.c0; cc <= d.c1; cc += kFixupBatch) {
        float4 v[kFixupBatch][2];
#pragma unroll
        for (int k = 0; k < kFixupBatch; ++k) {
          const int cx = cc + k;
          const bool on = cx <= d.c1;
          const int sl =
              on ? ((d.w0 + unit_begin((uint32_t)cx, d.Uw, G) >= d.tile_u0) ? 2 * cx : 2 * cx + 1) : 0;
          const float4* src =
              reinterpret_cast<const float4*>(wave_part + ((long long)(sl * g.tpu + tj) * kTileRows + row) * Mp + mc);
#pragma unroll
          for (int b = 0; b < 2; ++b)
            v[k][b] = (on && mc + 4 * b < Mp) ? __ldcg(src + b) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < kFixupBatch; ++k) {
          if (cc + k <= d.c1) {
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              acc[4 * b] += v[k][b].x; acc[4 * b + 1] += v[k][b].y;
              acc[4 * b + 2] += v[k][b].z; acc[4 * b + 3] += v[k][b].w;
            }
          }
        }
      }
      const long long n = (long long)(d.group * g.tpu + tj) * kTileRows + row;
      if (n < N) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int m = mc + j;
          if (m < M) {
            if (pr->y_bf16) reinterpret_cast<uint16_t*>(pr->Y)[(long long)m * N + n] = f32_to_bf16_rn(acc[j] * ts);
            else static_cast<float*>(pr->Y)[(long long)m * N + n] = acc[j] * ts;
          }
        }
      }
    }
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

static size_t al256(size_t v) { return (v + 255) / 256 * 256; }

// Launch geometry: depends on M, and on whether every K of the launch is a multiple of
// 512 (then a unit may span two 256-wide chunks).
struct MxPlan {
  Geom g;
  int stages, acc_bufs, sf_bufs;
  uint32_t stage_bytes, sf_cols, acc_col0, acc_stride;
  size_t smem;
};

static MxPlan mx_plan_ku(long long M, int ku, int tpu, int terms) {
  MxPlan pl{};
  Geom& g = pl.g;
  g.M = (int)M;
  g.T = terms;
  g.nb = (int)M * g.T;
  g.nbt = (g.nb + 255) / 256;
  g.nb_tile = ((g.nb + g.nbt - 1) / g.nbt + 15) / 16 * 16;   // MMA N; a multiple of 16 keeps x16 loads inside the tile
  g.nsfb = g.nb_tile <= 128 ? 4 : 8;
  g.ku = ku;
  g.tpu = tpu;
  g.img_xs_off = (uint32_t)(g.nbt * g.nb_tile) * 128u;
  g.img_bytes = (uint32_t)(g.nbt * g.nb_tile) * 144u;
  g.img_stride = (g.img_bytes + 1023) / 1024 * 1024;
  g.wbytes = (uint32_t)(tpu * ku) * kWChunk;
  pl.sf_cols = 16u * (uint32_t)(ku * tpu) + 4u * (uint32_t)(ku * g.nbt * g.nsfb);
  pl.acc_stride = (uint32_t)(tpu * g.nbt * g.nb_tile);
  pl.acc_bufs = (2 * pl.sf_cols + 2 * pl.acc_stride <= 512) ? 2 : 1;
  // One ring: a stage holds a unit's weight tile, its scales and its activation images.
  // Measured: under a saturated weight stream the L2-resident images arrive with about the
  // weights' latency, so they need the same prefetch depth.
  pl.stage_bytes = g.wbytes + (uint32_t)ku * g.img_stride;
  const size_t budget = 227 * 1024 - 1024 - kTailBytes;
  pl.stages = (int)std::min<size_t>(kMaxStages, budget / pl.stage_bytes);
  pl.smem = 1024 + (size_t)pl.stages * pl.stage_bytes + kTailBytes;
  // scale-factor buffers: one per stage when TMEM allows (the scale copy then runs ahead like TMA)
  const uint32_t acc_cols = (uint32_t)pl.acc_bufs * pl.acc_stride;
  pl.sf_bufs = (int)std::min<uint32_t>((uint32_t)std::min(pl.stages, kMaxSfBufs), (512u - acc_cols) / pl.sf_cols);
  if (pl.sf_bufs < 2) pl.sf_bufs = 2;
  pl.acc_col0 = (uint32_t)pl.sf_bufs * pl.sf_cols;
  return pl;
}

// Units of two K-chunks or two weight tiles halve the issuing thread's per-unit work (its
// waits, commit and loop bookkeeping are per unit, the MMAs per K-step and tile). Measured
// on the 27B pass: two chunks of one tile stream best while the ring keeps >= 4 stages
// (M <= 12); past that, two tiles sharing one chunk's activation images carry half the
// image bytes per weight byte, so more weight bytes fit in flight (M=17: 4 stages instead
// of 3). Either needs one B tile and a double-buffered accumulator.
// Batch-invariant passes (binv) use one unit shape for every M, so that a row's units,
// split points and summation order do not depend on how many rows share the pass.
static MxPlan mx_plan(long long M, bool k512, bool binv, int terms) {
  auto ok = [](const MxPlan& x, int min_stages) {
    return x.g.nbt == 1 && x.acc_bufs == 2 && x.stages >= min_stages;
  };
  if (binv) return mx_plan_ku(M, 1, 1, terms);
  if (k512) {
    const MxPlan two = mx_plan_ku(M, 2, 1, terms);
    if (ok(two, 4)) return two;
  }
  const MxPlan pair = mx_plan_ku(M, 1, 2, terms);
  if (ok(pair, 3) && M <= pass_max_tokens(1, 2, terms)) return pair;
  if (k512) {
    const MxPlan two = mx_plan_ku(M, 2, 1, terms);
    if (ok(two, 3)) return two;
  }
  return mx_plan_ku(M, 1, 1, terms);
}

bool mxf4_supported(long long M, long long K, int terms) {
  return M >= 1 && M * terms <= kMaxB && K % kKC == 0 && K >= kKC && K <= 32768;
}

// Activation-image bytes a wave may hold: small enough that a wave's images stay in L2
// while the weight stream passes through it.
constexpr size_t kWaveImageBudget = size_t(24) << 20;

// Workspace: counters [nwave][grid] | partials [nwave][2*grid][M][128] | (a pass) problem
// descriptors, wave starts, per-(wave, CTA) first problems, per-CTA unit counts | per
// problem: images, term scales, and (verify) the per-tile row maxima and indices.
struct WsLayout {
  int grid, nwave;
  unsigned long long units;
  std::vector<int> wave_first;              // first problem of each wave, plus n
  size_t off_part, off_desc, off_wave, off_cta, off_cunits, total;
  std::vector<size_t> off_img, off_xg, off_pv, off_pi;
};

static long long problem_groups(const MxHostProblem& h, int tpu) {
  const long long tiles = (h.N + kTileRows - 1) / kTileRows;
  return (tiles + tpu - 1) / tpu;
}

static unsigned long long problem_units(const MxHostProblem& h, int ku, int tpu) {
  return (unsigned long long)problem_groups(h, tpu) * (unsigned long long)(h.K / (kKC * ku));
}

static bool all_k512(const MxHostProblem* hp, int n) {
  for (int i = 0; i < n; ++i)
    if (hp[i].K % (2 * kKC) != 0) return false;
  return true;
}

// with_desc: a pass keeps its descriptors and wave tables in the workspace.
static WsLayout mx_layout(const MxHostProblem* hp, int n, long long M, bool with_desc, bool binv, int terms) {
  const MxPlan pl = mx_plan(M, all_k512(hp, n), binv, terms);
  // waves are cut by image bytes; a batch-invariant pass cuts them as the largest M would
  const uint32_t wave_img_stride =
      binv ? mx_plan_ku(kMaxB / terms, 1, 1, terms).g.img_stride : pl.g.img_stride;
  const int ku = pl.g.ku, tpu = pl.g.tpu;
  WsLayout L;
  L.units = 0;
  for (int i = 0; i < n; ++i) L.units += problem_units(hp[i], ku, tpu);
  const int sms = std::max(1, device_sm_count());
  L.grid = (int)std::max<unsigned long long>(1ull, std::min<unsigned long long>((unsigned long long)sms, L.units));
  // waves: greedy over the list; a wave closes when the next problem's images would pass
  // the budget and it already has >= grid units (so every CTA owns a unit of it)
  L.wave_first.push_back(0);
  size_t img = 0;
  unsigned long long wu = 0;
  for (int i = 0; i < n; ++i) {
    const size_t pimg = (size_t)(hp[i].K / kKC) * wave_img_stride;
    if (i > 0 && wu >= (unsigned long long)L.grid && img + pimg > kWaveImageBudget) {
      L.wave_first.push_back(i);
      img = 0;
      wu = 0;
    }
    img += pimg;
    wu += problem_units(hp[i], ku, tpu);
  }
  if (L.wave_first.size() > 1 && wu < (unsigned long long)L.grid) L.wave_first.pop_back();   // merge a short tail
  L.wave_first.push_back(n);
  L.nwave = (int)L.wave_first.size() - 1;
  size_t o = al256((size_t)L.nwave * L.grid * 4);
  L.off_part = o;
  o += al256((size_t)L.nwave * 2 * L.grid * tpu * kTileRows * (size_t)((M + 3) & ~3LL) * 4);
  L.off_desc = L.off_wave = L.off_cta = L.off_cunits = 0;
  if (with_desc) {
    L.off_desc = o; o += al256(sizeof(Problem) * (size_t)n);
    L.off_wave = o; o += al256(sizeof(uint32_t) * (size_t)(L.nwave + 1));
    L.off_cta = o; o += al256(sizeof(int) * (size_t)L.nwave * L.grid);
    L.off_cunits = o; o += al256(sizeof(int) * (size_t)L.grid);
  }
  for (int i = 0; i < n; ++i) {
    const long long tiles = (hp[i].N + kTileRows - 1) / kTileRows;
    L.off_img.push_back(o); o += al256((size_t)(hp[i].K / kKC) * pl.g.img_stride);
    L.off_xg.push_back(o); o += al256((size_t)pl.g.nb * 4);
    if (hp[i].verify) {
      L.off_pv.push_back(o); o += al256((size_t)tiles * M * 4);
      L.off_pi.push_back(o); o += al256((size_t)tiles * M * 4);
    } else {
      L.off_pv.push_back(0);
      L.off_pi.push_back(0);
    }
  }
  L.total = o;
  return L;
}

static int fill_problem(Problem* P, const MxHostProblem& h, const WsLayout& L, int i, unsigned long long unit0,
                        char* ws, int ku, int tpu) {
  std::memset(static_cast<void*>(P), 0, sizeof(Problem));
  if (!map_u8(&P->tm_q, h.q, h.K / 2, h.N, kKC / 2, kTileRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !map_u8(&P->tm_sf, h.sf, h.K / 16, h.N, (uint32_t)(ku * kKC / 16), kTileRows, CU_TENSOR_MAP_SWIZZLE_NONE))
    return set_error(NVFP4WS_ERR_CUDA, "cuTensorMapEncodeTiled failed (block-scaled path)");
  P->X = h.X;
  P->ximg = reinterpret_cast<uint8_t*>(ws + L.off_img[i]);
  P->xg = reinterpret_cast<float*>(ws + L.off_xg[i]);
  P->ts = h.ts;
  P->Y = h.Y;
  P->part_val = h.verify ? reinterpret_cast<float*>(ws + L.off_pv[i]) : nullptr;
  P->part_idx = h.verify ? reinterpret_cast<int*>(ws + L.off_pi[i]) : nullptr;
  P->N = h.N;
  P->unit0 = (unsigned int)unit0;
  P->K = (int)h.K;
  P->kch = (int)(h.K / (kKC * ku));
  P->groups = (int)problem_groups(h, tpu);
  P->tiles = (int)((h.N + kTileRows - 1) / kTileRows);
  P->y_bf16 = h.y_bf16;
  P->verify = h.verify;
  return NVFP4WS_OK;
}

template <int NBT, int KU, int TPU, int T>
static const void* pass_fn() { return reinterpret_cast<const void*>(&pass_kernel<NBT, KU, TPU, T>); }

// The kernel instance of a plan: B tiles, unit shape and activation terms.
template <int T>
static const void* pass_instance_t(const Geom& g) {
  return g.nbt == 2 ? pass_fn<2, 1, 1, T>() : g.tpu == 2 ? pass_fn<1, 1, 2, T>() : g.ku == 2 ? pass_fn<1, 2, 1, T>()
                                                                                          : pass_fn<1, 1, 1, T>();
}
static const void* pass_instance(const Geom& g) {
  static_assert(kGemmTerms == 5 && kVerifyTerms == 5 && kGemmTermsFast == 4,
                "pass kernel instances are built for 1, 4 and 5 terms");
  return g.T == 1 ? pass_instance_t<1>(g) : g.T == 4 ? pass_instance_t<4>(g) : pass_instance_t<5>(g);
}

static int ensure_attrs() {
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return set_error(NVFP4WS_ERR_CUDA, "cannot get the current device");
  if (!attr_set[dev]) {
    const void* fns[] = {pass_fn<1, 1, 1, 5>(), pass_fn<1, 2, 1, 5>(), pass_fn<1, 1, 2, 5>(), pass_fn<2, 1, 1, 5>(),
                         pass_fn<1, 1, 1, 4>(), pass_fn<1, 2, 1, 4>(), pass_fn<1, 1, 2, 4>(), pass_fn<2, 1, 1, 4>(),
                         pass_fn<1, 1, 1, 1>(), pass_fn<1, 2, 1, 1>(), pass_fn<1, 1, 2, 1>(), pass_fn<2, 1, 1, 1>()};
    for (const void* f : fns)
      if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
        return check_launch("cudaFuncSetAttribute(pass_kernel)");
    attr_set[dev] = true;
  }
  return NVFP4WS_OK;
}

// Enqueue prep + GEMM. `single` is used when `probs_dev` is null (one problem).
struct PassTables {           // device wave tables of a pass (all null for one GEMM)
  const uint32_t* wave_u0;
  const int* cta_prob;
  const int* cta_units;
  int nwave;
};

// CTAs per activation row in the prep of one GEMM: about 2048 elements each.
static int prep_slices(int nprob, long long K) {
  return nprob == 1 ? (int)std::max<long long>(1, std::min<long long>(16, K / 2048)) : 1;
}

// 1) Activation decomposition of the launch's problems (a programmatic dependent launch: it
//    may start while the previous kernel of the stream finishes, and waits for it before any
//    access).
static int launch_prep(const Problem& single, const Problem* probs_dev, int nprob, const MxPlan& pl, long long max_k,
                       cudaStream_t s) {
  if (int e = ensure_attrs()) return e;
  const int slices = prep_slices(nprob, max_k);
  cudaLaunchConfig_t pc = {};
  pc.gridDim = dim3((unsigned)(pl.g.M * nprob * slices));
  pc.blockDim = dim3(kPrepThreads);
  pc.stream = s;
  cudaLaunchAttribute pa[1];
  pa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pa[0].val.programmaticStreamSerializationAllowed = 1;
  pc.attrs = pa;
  pc.numAttrs = 1;
  const Geom g = pl.g;
  cudaError_t pe = g.T == 1   ? cudaLaunchKernelEx(&pc, x_prep_kernel<1>, single, probs_dev, g, slices)
                   : g.T == 4 ? cudaLaunchKernelEx(&pc, x_prep_kernel<4>, single, probs_dev, g, slices)
                              : cudaLaunchKernelEx(&pc, x_prep_kernel<5>, single, probs_dev, g, slices);
  if (pe != cudaSuccess) return set_error(NVFP4WS_ERR_CUDA, "x_prep_kernel launch: %s", cudaGetErrorString(pe));
  return check_launch("x_prep_kernel");
}

// 2) The GEMM, a programmatic dependent of the kernel before it (its prep kernel, or another
//    prep kernel that waited for that one).
static int launch_main(const Problem& single, const Problem* probs_dev, const PassTables& tb, int nprob,
                       const MxPlan& pl, int grid, unsigned long long units, size_t off_part, char* ws, cudaStream_t s) {
  if (units * (unsigned long long)grid >= (1ull << 32))
    return set_error(NVFP4WS_ERR_UNSUPPORTED, "block-scaled path: too many units for the stream-K partition");
  if (int e = ensure_attrs()) return e;
  PassParams p{};
  p.g = pl.g;
  p.probs = probs_dev;
  p.nprob = nprob;
  p.wave_u0 = tb.wave_u0;
  p.cta_prob = tb.cta_prob;
  p.cta_units = tb.cta_units;
  p.nwave = tb.nwave;
  p.units = (unsigned int)units;
  p.grid = grid;
  p.stages = pl.stages;
  p.stage_bytes = pl.stage_bytes;
  p.acc_bufs = pl.acc_bufs;
  p.sf_bufs = pl.sf_bufs;
  p.sf_cols = pl.sf_cols;
  p.acc_col0 = pl.acc_col0;
  p.acc_stride = pl.acc_stride;
  p.counters = reinterpret_cast<unsigned int*>(ws);
  p.partials = reinterpret_cast<float*>(ws + off_part);
  p.err = device_error_word();
  if (!p.err) return set_error(NVFP4WS_ERR_CUDA, "cannot resolve the device error word");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (pl.g.M > pass_max_tokens(pl.g.nbt, pl.g.tpu, pl.g.T))
    return set_error(NVFP4WS_ERR_UNSUPPORTED, "block-scaled path: M=%d exceeds the kernel's token capacity", pl.g.M);
  void* args[] = {const_cast<Problem*>(&single), &p};
  cudaError_t e = cudaLaunchKernelExC(&cfg, pass_instance(pl.g), args);
  if (e != cudaSuccess) return set_error(NVFP4WS_ERR_CUDA, "pass_kernel launch: %s", cudaGetErrorString(e));
  return check_launch("pass_kernel");
}

size_t mxf4_workspace_bytes(long long M, long long N, long long K, int terms) {
  if (!mxf4_supported(M, K, terms)) return 0;
  MxHostProblem h{nullptr, nullptr, nullptr, nullptr, N, K, nullptr, 0, 1};   // sized with the verify tail
  return mx_layout(&h, 1, M, false, false, terms).total;
}

static int launch_single(const MxHostProblem& h, long long M, void* workspace, cudaStream_t s, Problem* out,
                         int terms) {
  const MxPlan pl = mx_plan(M, all_k512(&h, 1), false, terms);
  const WsLayout L = mx_layout(&h, 1, M, false, false, terms);
  char* ws = static_cast<char*>(workspace);
  if (int e = fill_problem(out, h, L, 0, 0, ws, pl.g.ku, pl.g.tpu)) return e;
  const PassTables none{nullptr, nullptr, nullptr, 1};
  if (int e = launch_prep(*out, nullptr, 1, pl, h.K, s)) return e;
  return launch_main(*out, nullptr, none, 1, pl, L.grid, L.units, L.off_part, ws, s);
}

int launch_mxf4_gemm(const uint16_t* X, const uint8_t* q, const uint8_t* sf, const float* ts, long long M,
                     long long N, long long K, void* Y, int y_dtype, void* workspace, cudaStream_t s, int terms) {
  MxHostProblem h{X, q, sf, ts, N, K, Y, y_dtype == NVFP4WS_Y_BF16 ? 1 : 0, 0};
  Problem P;
  return launch_single(h, M, workspace, s, &P, terms);
}

int launch_mxf4_verify(const uint16_t* X, const uint8_t* q, const uint8_t* sf, const float* ts, long long M,
                       long long N, long long K, const VerifyRule& v, void* workspace, cudaStream_t s) {
  MxHostProblem h{X, q, sf, ts, N, K, nullptr, 0, 1};
  Problem P;
  if (int e = launch_single(h, M, workspace, s, &P, kVerifyTerms)) return e;
  return launch_verify_stage2(P.part_val, P.part_idx, P.tiles, (int)M, v, s);
}

// ------------------------------------------------------------------ multi-problem passes

// A pass runs as one persistent launch, or as two when it ends in a verify and its GEMMs take
// fewer activation terms than the verify (NVFP4WS_PASS_FOUR_TERMS): the GEMMs' launch, then
// the verify's. Each launch has its own plan (term count, unit shape, stages) and its own
// region of the workspace.
struct PassPart {
  int first, count, terms;
};

static int pass_parts(const MxHostProblem* hp, int n, int terms, PassPart (&parts)[2]) {
  const bool verify = hp[n - 1].verify != 0;
  if (!verify || terms == kVerifyTerms) {
    parts[0] = PassPart{0, n, verify ? kVerifyTerms : terms};
    return 1;
  }
  if (n == 1) {
    parts[0] = PassPart{0, 1, kVerifyTerms};
    return 1;
  }
  parts[0] = PassPart{0, n - 1, terms};
  parts[1] = PassPart{n - 1, 1, kVerifyTerms};
  return 2;
}

// One launch of a pass. Device addresses are offsets into the pass workspace, so two launches
// fit the caller's fixed-size handle.
struct MxLaunch {
  unsigned long long base;     // this launch's region of the workspace
  uint32_t off_part, off_desc, off_wave, off_cta, off_cunits;   // within the region
  int32_t nprob, grid, nwave, max_k, terms, k512;
  uint32_t units;
};

// Host state of a pass: plain data in caller-owned memory (no allocation).
struct MxPassState {
  uint32_t magic;
  int32_t nlaunch, verify, vtiles, binv;
  long long M;
  char* ws;
  MxLaunch L[2];
  float* pv;
  int* pi;
  VerifyRule vs;
};
static_assert(sizeof(MxPassState) <= kMxPassStateBytes, "pass state does not fit the caller's handle");
constexpr uint32_t kPassMagic = 0x4e565054u;

size_t mxf4_pass_workspace_bytes(const MxHostProblem* hp, int n, long long M, bool binv, int terms) {
  PassPart parts[2];
  const int np = pass_parts(hp, n, terms, parts);
  size_t total = 0;
  for (int k = 0; k < np; ++k)
    total = al256(total) + mx_layout(hp + parts[k].first, parts[k].count, M, true, binv, parts[k].terms).total;
  return total;
}

// Problem descriptors and wave tables of one launch, uploaded into its workspace region.
static int init_launch(MxLaunch* out, const MxHostProblem* hp, int n, long long M, bool binv, int terms, char* ws,
                       unsigned long long base, Problem* last) {
  const WsLayout L = mx_layout(hp, n, M, true, binv, terms);
  const MxPlan plan = mx_plan(M, all_k512(hp, n), binv, terms);
  const int ku = plan.g.ku, tpu = plan.g.tpu;
  char* reg = ws + base;
  std::vector<Problem> host(n);
  std::vector<unsigned long long> first(n);
  unsigned long long unit0 = 0;
  long long max_k = 0;
  for (int i = 0; i < n; ++i) {
    first[i] = unit0;
    if (int e = fill_problem(&host[i], hp[i], L, i, unit0, reg, ku, tpu)) return e;
    unit0 += (unsigned long long)host[i].groups * (unsigned long long)host[i].kch;
    max_k = std::max(max_k, hp[i].K);
  }
  if (unit0 * (unsigned long long)L.grid >= (1ull << 32))
    return set_error(NVFP4WS_ERR_UNSUPPORTED, "nvfp4_pass_init: too many units for the stream-K partition");
  // wave tables: wave starts, each CTA's first problem in each wave, each CTA's unit count
  std::vector<uint32_t> wave_u0(L.nwave + 1);
  std::vector<int> cta_prob((size_t)L.nwave * L.grid), cta_units(L.grid, 0);
  for (int w = 0; w < L.nwave; ++w) {
    const unsigned long long w0 = first[L.wave_first[w]];
    const unsigned long long w1 = (L.wave_first[w + 1] < n) ? first[L.wave_first[w + 1]] : unit0;
    wave_u0[w] = (uint32_t)w0;
    const unsigned long long Uw = w1 - w0;
    if (Uw < (unsigned long long)L.grid)
      return set_error(NVFP4WS_ERR_UNSUPPORTED, "nvfp4_pass_init: internal wave plan has a wave of %llu < %d units",
                       Uw, L.grid);
    for (int c = 0, i = L.wave_first[w]; c < L.grid; ++c) {
      const unsigned long long b = w0 + (unsigned long long)c * Uw / (unsigned long long)L.grid;
      const unsigned long long e = w0 + (unsigned long long)(c + 1) * Uw / (unsigned long long)L.grid;
      while (i + 1 < n && first[i + 1] <= b) ++i;
      cta_prob[(size_t)w * L.grid + c] = i;
      cta_units[c] += (int)(e - b);
    }
  }
  wave_u0[L.nwave] = (uint32_t)unit0;
  if (cudaMemcpy(reg + L.off_desc, host.data(), sizeof(Problem) * (size_t)n, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(reg + L.off_wave, wave_u0.data(), sizeof(uint32_t) * wave_u0.size(), cudaMemcpyHostToDevice) !=
          cudaSuccess ||
      cudaMemcpy(reg + L.off_cta, cta_prob.data(), sizeof(int) * cta_prob.size(), cudaMemcpyHostToDevice) !=
          cudaSuccess ||
      cudaMemcpy(reg + L.off_cunits, cta_units.data(), sizeof(int) * cta_units.size(), cudaMemcpyHostToDevice) !=
          cudaSuccess)
    return check_launch("nvfp4_pass_init: descriptor upload");
  out->base = base;
  out->off_part = (uint32_t)L.off_part;
  out->off_desc = (uint32_t)L.off_desc;
  out->off_wave = (uint32_t)L.off_wave;
  out->off_cta = (uint32_t)L.off_cta;
  out->off_cunits = (uint32_t)L.off_cunits;
  out->nprob = n;
  out->grid = L.grid;
  out->nwave = L.nwave;
  out->max_k = (int32_t)max_k;
  out->terms = terms;
  out->k512 = all_k512(hp, n) ? 1 : 0;
  out->units = (uint32_t)unit0;
  *last = host[n - 1];
  return NVFP4WS_OK;
}

int mxf4_pass_init(void* state, const MxHostProblem* hp, int n, long long M, const VerifyRule* vs, bool binv,
                   int terms, void* workspace, size_t workspace_bytes) {
  MxPassState* P = static_cast<MxPassState*>(state);
  std::memset(static_cast<void*>(P), 0, sizeof(MxPassState));
  const size_t need = mxf4_pass_workspace_bytes(hp, n, M, binv, terms);
  if (workspace_bytes < need)
    return set_error(NVFP4WS_ERR_WORKSPACE, "nvfp4_pass_init: workspace %zu bytes < required %zu", workspace_bytes,
                     need);
  char* ws = static_cast<char*>(workspace);
  PassPart parts[2];
  const int np = pass_parts(hp, n, terms, parts);
  unsigned long long base = 0;
  Problem last{};
  for (int k = 0; k < np; ++k) {
    base = al256(base);
    const PassPart& pt = parts[k];
    if (int e = init_launch(&P->L[k], hp + pt.first, pt.count, M, binv, pt.terms, ws, base, &last)) return e;
    // layouts keep 32-bit offsets within a launch's region
    const size_t bytes = mx_layout(hp + pt.first, pt.count, M, true, binv, pt.terms).total;
    if (bytes >= (1ull << 32))
      return set_error(NVFP4WS_ERR_UNSUPPORTED, "nvfp4_pass_init: a launch's workspace exceeds 4 GiB");
    base += bytes;
  }
  P->nlaunch = np;
  P->binv = binv ? 1 : 0;
  P->M = M;
  P->ws = ws;
  P->verify = vs != nullptr;
  if (vs) {
    P->vs = *vs;
    P->pv = last.part_val;
    P->pi = last.part_idx;
    P->vtiles = last.tiles;
  }
  P->magic = kPassMagic;
  return NVFP4WS_OK;
}

// Stream order: every launch's prep kernel, then every launch's GEMM kernel, then the verify's
// stage 2. Each kernel is a programmatic dependent of the one before it and waits for it to
// finish before reading what it wrote, so a later launch's weight loads may start while the
// earlier launch's last tiles finish.
int mxf4_pass_run(const void* state, cudaStream_t s) {
  const MxPassState* P = static_cast<const MxPassState*>(state);
  if (P->magic != kPassMagic) return set_error(NVFP4WS_ERR_INVALID_ARG, "nvfp4_pass_run: pass not initialised");
  static const Problem kNoProblem{};   // the kernels' by-value problem slot, unused by a pass
  for (int k = 0; k < P->nlaunch; ++k) {
    const MxLaunch& L = P->L[k];
    const MxPlan pl = mx_plan(P->M, L.k512 != 0, P->binv != 0, L.terms);
    char* reg = P->ws + L.base;
    if (int e = launch_prep(kNoProblem, reinterpret_cast<const Problem*>(reg + L.off_desc), L.nprob, pl, L.max_k, s))
      return e;
  }
  for (int k = 0; k < P->nlaunch; ++k) {
    const MxLaunch& L = P->L[k];
    const MxPlan pl = mx_plan(P->M, L.k512 != 0, P->binv != 0, L.terms);
    char* reg = P->ws + L.base;
    const PassTables tb{reinterpret_cast<const uint32_t*>(reg + L.off_wave), reinterpret_cast<const int*>(reg + L.off_cta),
                        reinterpret_cast<const int*>(reg + L.off_cunits), L.nwave};
    if (int e = launch_main(kNoProblem, reinterpret_cast<const Problem*>(reg + L.off_desc), tb, L.nprob, pl, L.grid,
                            L.units, L.off_part, reg, s))
      return e;
  }
  if (!P->verify) return NVFP4WS_OK;
  return launch_verify_stage2(P->pv, P->pi, P->vtiles, (int)P->M, P->vs, s);
}

}  // namespace nvfp4ws

#ifdef NVFP4WS_TRACE
// Copies the timeline of the last traced launch (16 fields x 64 units of CTA 0) to the host.
extern "C" int nvfp4ws_trace_read(unsigned long long* host, int n) {
  if (n > 16 * 64) n = 16 * 64;
  return cudaMemcpyFromSymbol(host, nvfp4ws::mxk::g_trace, sizeof(unsigned long long) * n) == cudaSuccess ? 0 : 5;
}
// Per-CTA global-timer events: [256][16] (GEMM CTAs 0..147; prep kernel rows at 200+m).
extern "C" int nvfp4ws_trace_cta_read(unsigned long long* host) {
  return cudaMemcpyFromSymbol(host, nvfp4ws::mxk::g_cta_trace, sizeof(unsigned long long) * 256 * 16) == cudaSuccess ? 0 : 5;
}
#endif
