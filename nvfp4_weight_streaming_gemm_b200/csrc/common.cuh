// Shared device helpers of libnvfp4ws: error reporting, streaming loads and the
// NVFP4 -> f16 conversions used by every kernel.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/nvfp4ws.h"

namespace nvfp4ws {

// ----------------------------------------------------------------------------
// Host-side error reporting (thread-local detail text)
// ----------------------------------------------------------------------------
int set_error(int status, const char* fmt, ...);
void clear_error();       // every entry point starts with an empty detail text
int check_launch(const char* what);

// Device error word (one per device, in api.cu). Kernels with bounded waits get
// its address as an argument and OR a code into it when a wait gives up; it is
// read and cleared by nvfp4ws_check().
unsigned int* device_error_word();
constexpr unsigned int kDevErrWaitTimeout = 1u;
constexpr unsigned int kDevErrBadTree = 2u;       // a draft tree's parent outside [0, k-1]

// ----------------------------------------------------------------------------
// Loads
// ----------------------------------------------------------------------------

// 16-byte streaming load of data that is read exactly once: read-only path, and
// no L1 allocation.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint16_t ld_stream_u16(const void* p) {
  uint16_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}

// ----------------------------------------------------------------------------
// Conversions
// ----------------------------------------------------------------------------

// Two E2M1 codes (the low byte of `v`: bits 0..3 = first element, 4..7 = second)
// -> f16x2 (first element in the low half). Exact.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t v) {
  uint32_t r;
  asm("{ .reg .b8 b; cvt.u8.u32 b, %1; cvt.rn.f16x2.e2m1x2 %0, b; }" : "=r"(r) : "r"(v));
  return r;
}

// Two E4M3 codes (low 16 bits of `v`, first in bits 0..7) -> f16x2 (first in the low half). Exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t v) {
  uint32_t r;
  asm("{ .reg .b16 b; cvt.u16.u32 b, %1; cvt.rn.f16x2.e4m3x2 %0, b; }" : "=r"(r) : "r"(v));
  return r;
}

__device__ __forceinline__ float f16lo_to_f32(uint32_t h2) {
  float f;
  asm("{ .reg .f16 l, h; mov.b32 {l, h}, %1; cvt.f32.f16 %0, l; }" : "=f"(f) : "r"(h2));
  return f;
}
__device__ __forceinline__ float f16hi_to_f32(uint32_t h2) {
  float f;
  asm("{ .reg .f16 l, h; mov.b32 {l, h}, %1; cvt.f32.f16 %0, h; }" : "=f"(f) : "r"(h2));
  return f;
}

// Two bf16 (bits 0..15 first, 16..31 second) -> f16x2, round to nearest, saturating
// at +-65504. Exact for magnitudes in [2^-14, 65504].
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_sat(uint32_t b2) {
  float lo = __uint_as_float(b2 << 16);
  float hi = __uint_as_float(b2 & 0xFFFF0000u);
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ----------------------------------------------------------------------------
// Per-row power-of-two shift of the activations (the f16 paths)
// ----------------------------------------------------------------------------
// A bf16 row is converted to f16 as x * 2^-e, with e chosen from the row's amax so that
// amax * 2^-e lies in [2^14, 2^15). Every bf16 value (8 significant bits) of the row then
// converts exactly, nothing saturates, and only values below 2^-25 of the row's amax lose
// bits (f16 subnormals). Products and fp32 sums of the shifted row are the unshifted ones
// times 2^-e exactly (barring fp32 underflow), and the epilogue multiplies by 2^e.

// floor(log2(a)) for a finite a > 0, subnormals included.
__device__ __forceinline__ int floor_log2_pos(float a) {
  const uint32_t u = __float_as_uint(a);
  const int ex = (int)((u >> 23) & 0xFFu);
  if (ex != 0) return ex - 127;
  return (31 - __clz((int)(u & 0x7FFFFFu))) - 149;          // a = m * 2^-149
}

// The shift e of a row whose largest magnitude is amax (0 for a zero or non-finite amax).
__device__ __forceinline__ int row_shift_of_amax(float amax) {
  return (amax > 0.f && amax <= 3.402823466e38f) ? floor_log2_pos(amax) - 14 : 0;
}

// v * 2^k for k in [-252, 254], by at most two multiplications by exact powers of two:
// exact unless the result leaves the normal fp32 range.
__device__ __forceinline__ float mul_pow2(float v, int k) {
  if (k > 127) { v *= __uint_as_float(254u << 23); k -= 127; }
  else if (k < -126) { v *= __uint_as_float(1u << 23); k += 126; }
  return v * __uint_as_float((uint32_t)(k + 127) << 23);
}

__device__ __forceinline__ float bf16x2_absmax(uint32_t b2) {
  return fmaxf(fabsf(__uint_as_float(b2 << 16)), fabsf(__uint_as_float(b2 & 0xFFFF0000u)));
}

// Two bf16 times 2^-e -> f16x2 (nearest); exact for a row shifted by row_shift_of_amax.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_shifted(uint32_t b2, int e) {
  const float lo = mul_pow2(__uint_as_float(b2 << 16), -e);
  const float hi = mul_pow2(__uint_as_float(b2 & 0xFFFF0000u), -e);
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// acc += a.lo * b.lo + a.hi * b.hi, f16 inputs, f32 accumulation. Each product is exact.
__device__ __forceinline__ void dot2_f16_f32(float& acc0, float& acc1, uint32_t a, uint32_t b) {
  asm("{ .reg .f16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %2;\n\t"
      "mov.b32 {bl, bh}, %3;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.f16 %1, ah, bh, %1; }"
      : "+f"(acc0), "+f"(acc1)
      : "r"(a), "r"(b));
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
  return r;
}

// Lexicographic "better" for argmax: larger value, then the smaller index.
__device__ __forceinline__ bool argmax_better(float v, int i, float bv, int bi) {
  return (v > bv) || (v == bv && i < bi);
}

inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

int device_sm_count();

}  // namespace nvfp4ws
