// nvfp4_pack: fp32 weight -> NVFP4 (E2M1 codes, E4M3 block scales, fp32 tensor scale).
//
// The format is NVFP4 group-16 ("Qwen3.8 on DGX Spark (GB10)", "The seven targets,
// and switching between them"). Quantisation is offline: it runs before the
// weight pass and is not timed inside it. The scale arithmetic is done in double
// precision and rounded once, to nearest even, so the bytes are a deterministic
// function of W:
//   ts   = fp32( amax|W| / 2688 )
//   S    = E4M3_rne_satfinite( amax_block / (6 * ts) )
//   code = E2M1_rne_satfinite( w / (S * ts) ), sign of w kept
// Three launches: an amax reduction (atomicMax on the bit pattern, exact and
// order-free), a one-thread finalisation of ts, and one thread per 16-element block.
//
// The file also holds the FP8 pack (E4M3 codes, one fp32 scale per 128 x 128 block),
// which shares the double-precision E4M3 rounding.
#include "common.cuh"
#include "fp8.h"

#include <algorithm>
#include <cmath>

namespace nvfp4ws {

// Round a non-negative double to the nearest E4M3 magnitude (ties to even), saturating at 448.
__device__ __forceinline__ double e4m3_round(double a) {
  if (!(a < 448.0)) return 448.0;
  int ex;
  frexp(a, &ex);                       // a = f * 2^ex, f in [0.5, 1)
  int e = max(ex - 1, -6);             // binade exponent; the subnormals share binade -6
  int sexp = e - 3;                    // 3 mantissa bits -> spacing 2^(e-3)
  double n = rint(ldexp(a, -sexp));
  return fmin(ldexp(n, sexp), 448.0);
}

// Bits of an exact non-negative E4M3 magnitude.
__device__ __forceinline__ uint32_t e4m3_bits(double v) {
  if (v == 0.0) return 0u;
  int ex;
  frexp(v, &ex);
  int e = ex - 1;
  if (e < -6) return (uint32_t)(v * 512.0);          // subnormal: v = m * 2^-9
  uint32_t mant = (uint32_t)((ldexp(v, -e) - 1.0) * 8.0);
  return ((uint32_t)(e + 7) << 3) | mant;
}

__device__ __forceinline__ double e4m3_value(uint32_t bits) {
  uint32_t e = (bits >> 3) & 0xF, m = bits & 0x7;
  if (e == 0) return ldexp((double)m, -9);
  return ldexp(1.0 + m / 8.0, (int)e - 7);
}

// E2M1 code of a double: nearest of {0, .5, 1, 1.5, 2, 3, 4, 6} (ties to the even
// mantissa bit), saturating at 6, with the sign bit of r kept.
__device__ __forceinline__ uint32_t e2m1_code(double r) {
  uint32_t sign = signbit(r) ? 8u : 0u;
  double a = fmin(fabs(r), 6.0);
  int ex;
  frexp(a, &ex);
  int e = max(ex - 1, 0);              // binades [1,2), [2,4), [4,8); below 1 shares spacing 0.5
  int sexp = e - 1;                    // 1 mantissa bit
  double v = fmin(ldexp(rint(ldexp(a, -sexp)), sexp), 6.0);
  uint32_t mag;
  if (v < 1.0) {
    mag = (uint32_t)(v * 2.0);         // 0 -> 0, 0.5 -> 1 (subnormal)
  } else {
    int vx;
    frexp(v, &vx);
    int ve = vx - 1;                   // 0, 1 or 2
    uint32_t m = (ldexp(v, -ve) > 1.0) ? 1u : 0u;
    mag = ((uint32_t)(ve + 1) << 1) | m;
  }
  return sign | mag;
}

__global__ void __launch_bounds__(256) amax_kernel(const float4* __restrict__ W, long long n4,
                                                   unsigned int* __restrict__ out_bits) {
  float m = 0.0f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    float4 v = W[i];
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b = fmaxf(b, red[w]);
    atomicMax(out_bits, __float_as_uint(b));   // non-negative floats order like their bit patterns
  }
}

__global__ void finalize_ts_kernel(float* ts, const float* ts_in) {
  if (ts_in != nullptr) {
    *ts = *ts_in;
  } else {
    float amax = __uint_as_float(*reinterpret_cast<const unsigned int*>(ts));
    *ts = (float)((double)amax / 2688.0);
  }
}

// One thread per 16-element block: 64 bytes of W in, 8 bytes of codes and 1 scale byte out.
__global__ void __launch_bounds__(256) pack_kernel(const float* __restrict__ W, long long N, long long K,
                                                   uint8_t* __restrict__ q, uint8_t* __restrict__ sf,
                                                   const float* __restrict__ ts_ptr) {
  const long long nblk = K / 16;
  const long long total = N * nblk;
  const double ts = (double)(*ts_ptr);
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const long long n = t / nblk, b = t - n * nblk;
    const float4* src = reinterpret_cast<const float4*>(W + n * K + b * 16);
    float w[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 v = src[i];
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(w[i]));

    uint32_t sbits = 0;
    double S = 0.0;
    if (ts > 0.0) {
      S = e4m3_round((double)amax / (6.0 * ts));
      sbits = e4m3_bits(S);
      S = e4m3_value(sbits);
    }
    uint32_t lo = 0, hi = 0;
    if (S > 0.0) {
      const double denom = S * ts;     // exact: 4 x 24 significant bits
#pragma unroll
      for (int i = 0; i < 8; ++i) lo |= e2m1_code((double)w[i] / denom) << (4 * i);
#pragma unroll
      for (int i = 0; i < 8; ++i) hi |= e2m1_code((double)w[8 + i] / denom) << (4 * i);
    }
    *reinterpret_cast<uint2*>(q + n * (K / 2) + b * 8) = make_uint2(lo, hi);
    sf[t] = (uint8_t)sbits;
  }
}

// ---------------------------------------------------------------------------- FP8 block scaling
//
// One CTA per 128 x 128 block (rows x K) of W, 256 threads, two per row, 64 elements each:
//   s    = fp32( amax_block / 448 )                     0 for an all-zero block
//   code = E4M3_rne_satfinite( w / s ), sign kept       +0 where s = 0
// The quotient is formed in double precision and rounded once, as for the NVFP4 codes.
// Blocks at the right and bottom edges hold what remains of W.

__device__ __forceinline__ uint32_t e4m3_code_signed(double r) {
  const uint32_t sign = signbit(r) ? 0x80u : 0u;
  return sign | e4m3_bits(e4m3_round(fabs(r)));
}

__global__ void __launch_bounds__(256) fp8_pack_kernel(const float* __restrict__ W, long long N, long long K,
                                                       uint8_t* __restrict__ q, float* __restrict__ scales, int kbs) {
  const long long nb = blockIdx.x;
  const int kb = blockIdx.y;
  const int r = threadIdx.x >> 1, h = threadIdx.x & 1;
  const long long n = nb * 128 + r;
  const long long k0 = (long long)kb * 128 + h * 64;
  const bool row_ok = n < N;
  float amax = 0.0f;
  if (row_ok) {
    for (int c = 0; c < 4; ++c) {
      const long long k = k0 + 16 * c;
      if (k >= K) break;
      const float4* src = reinterpret_cast<const float4*>(W + n * K + k);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = src[i];
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      }
    }
  }
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  __shared__ float red[8];
  __shared__ float s_scale;
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.0f;
    for (int w = 0; w < 8; ++w) b = fmaxf(b, red[w]);
    s_scale = (float)((double)b / 448.0);
    scales[nb * kbs + kb] = s_scale;
  }
  __syncthreads();
  const double s = (double)s_scale;
  if (!row_ok) return;
  for (int c = 0; c < 4; ++c) {
    const long long k = k0 + 16 * c;
    if (k >= K) break;
    const float4* src = reinterpret_cast<const float4*>(W + n * K + k);
    uint32_t wd[4] = {0u, 0u, 0u, 0u};
    if (s > 0.0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = src[i];
        wd[i] = e4m3_code_signed((double)v.x / s) | (e4m3_code_signed((double)v.y / s) << 8) |
                (e4m3_code_signed((double)v.z / s) << 16) | (e4m3_code_signed((double)v.w / s) << 24);
      }
    }
    *reinterpret_cast<uint4*>(q + n * K + k) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
  }
}

int launch_fp8_pack(const float* W, long long N, long long K, uint8_t* q, float* scales, cudaStream_t s) {
  const long long nbs = (N + 127) / 128, kbs = (K + 127) / 128;
  fp8_pack_kernel<<<dim3((unsigned)nbs, (unsigned)kbs), 256, 0, s>>>(W, N, K, q, scales, (int)kbs);
  return check_launch("fp8_pack_kernel");
}

int launch_pack(const float* W, long long N, long long K, uint8_t* q, uint8_t* sf, float* ts,
                const float* ts_in, cudaStream_t s) {
  const int sms = device_sm_count();
  if (sms <= 0) return set_error(NVFP4WS_ERR_CUDA, "cannot query the SM count");
  if (ts_in == nullptr) {
    if (cudaMemsetAsync(ts, 0, sizeof(float), s) != cudaSuccess) return check_launch("amax memset");
    long long n4 = N * K / 4;
    int grid = (int)std::min<long long>((n4 + 255) / 256, (long long)sms * 8);
    amax_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(W), n4,
                                      reinterpret_cast<unsigned int*>(ts));
    if (int e = check_launch("amax_kernel")) return e;
  }
  finalize_ts_kernel<<<1, 1, 0, s>>>(ts, ts_in);
  if (int e = check_launch("finalize_ts_kernel")) return e;
  long long total = N * (K / 16);
  int grid = (int)std::min<long long>((total + 255) / 256, (long long)sms * 16);
  pack_kernel<<<grid, 256, 0, s>>>(W, N, K, q, sf, ts);
  return check_launch("pack_kernel");
}

}  // namespace nvfp4ws
