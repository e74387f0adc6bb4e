// prep_kernel.cuh -- e4m3 quantisation prologue for the fp8 forward (sm_100a).
//
// The step before fp8 attention on the pages: FlashDreams PR #486
// "flashdreams.accelerated API v0", section 1.1 (FP8 E4M3 quantisation with
// tensor- or slice-granularity scales) and section 1.2 (head-scoped Q/K
// normalisation, optional FP8 SDPA), with the clamp to the e4m3fn range +-448
// that VeOmni PR #1363 describes for its quantizers.  Per (batch, head):
//   r       = 1 / sqrt(mean_d x_d^2 + eps)   per row (only with rmsnorm), fp64,
//             the squares summed over d = 0 .. 127 in ascending order
//   y_d     = (float)(x_d * r), or x_d without rmsnorm
//   descale = max |y| / 448 over the head (1 if that max is 0), fp32
//   code    = e4m3 of y / descale: fp32 quotient, round to nearest even,
//             saturating at +-448
// Every step is fixed in precision and order, so the codes and descales are a
// function of the input alone: bit for bit the same for any grid, batch or
// head split.  Three launches (after a memset of the descale array): the head
// maxima (atomicMax on the non-negative fp32 bit patterns, which order like
// integers, so the result does not depend on the order), max -> descale in
// place, and the codes.  HBM-bound: x is read twice and the codes written once.
#pragma once

#include "sm100.cuh"

namespace hattn {

constexpr int kPrepD = 128;
constexpr int kPrepThreads = 256;   // one row per thread

// Per-row normalisation factor (1 without rmsnorm): squares summed in fp64 in
// ascending d (each square is exact in fp64).  The row is streamed in 64-byte
// pieces, so few registers stay live; the second pass over the row (y) hits L1.
__device__ __forceinline__ double prep_row_factor(const uint4* __restrict__ row, int rmsnorm, double eps) {
  if (!rmsnorm) return 1.0;
  double sum = 0.0;
#pragma unroll 2
  for (int i = 0; i < 16; i += 4) {
    uint4 w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = __ldg(&row[i + k]);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t p[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const double lo = (double)__uint_as_float(p[t] << 16);
        const double hi = (double)__uint_as_float(p[t] & 0xFFFF0000u);
        sum += lo * lo;
        sum += hi * hi;
      }
    }
  }
  return 1.0 / sqrt(sum / (double)kPrepD + eps);
}

__device__ __forceinline__ float prep_y(uint32_t bits16_as_f32, double r, int rmsnorm) {
  const float v = __uint_as_float(bits16_as_f32);
  return rmsnorm ? (float)((double)v * r) : v;
}

// grid (ceil(S / 256), B*H): the largest |y| of each head into amax_bits (zeroed).
__global__ void __launch_bounds__(kPrepThreads, 4) prep_amax_kernel(const uint16_t* __restrict__ x,
                                                                      unsigned int* __restrict__ amax_bits, int S,
                                                                      int rmsnorm, double eps) {
  const int bh = blockIdx.y;
  const int s = blockIdx.x * kPrepThreads + threadIdx.x;
  float m = 0.f;
  if (s < S) {
    const uint4* row = reinterpret_cast<const uint4*>(x) + ((long long)bh * S + s) * 16;
    const double r = prep_row_factor(row, rmsnorm, eps);
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
      const uint4 w = __ldg(&row[i]);
      const uint32_t p[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        m = fmaxf(m, fabsf(prep_y(p[k] << 16, r, rmsnorm)));
        m = fmaxf(m, fabsf(prep_y(p[k] & 0xFFFF0000u, r, rmsnorm)));
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  __shared__ float wmax[kPrepThreads / 32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float bm = wmax[0];
#pragma unroll
    for (int i = 1; i < kPrepThreads / 32; ++i) bm = fmaxf(bm, wmax[i]);
    atomicMax(&amax_bits[bh], __float_as_uint(bm));
  }
}

// In place: descale = amax / 448 (1 when amax == 0).
__global__ void prep_descale_kernel(float* __restrict__ d, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float amax = d[i];
    d[i] = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  }
}

// y / ds rounded to fp32.  Fast path: y times a reciprocal, within 2 ulp of
// the quotient; that can only change the e4m3 rounding when the result lies
// within a few ulp of a midpoint between two e4m3 values (its low 20 mantissa
// bits near 0x80000) or in the small range where e4m3 steps are subnormal, and
// there the exactly rounded quotient is taken instead.
__device__ __forceinline__ float prep_quotient(float y, float ds, float rcp) {
  const float q = y * rcp;
  const uint32_t b = __float_as_uint(q) & 0x7FFFFFFFu;
  const int low = (int)(b & 0xFFFFFu) - 0x80000;
  if (b < 0x3D000000u /* 2^-5 */ || (low >= -4 && low <= 4)) return __fdiv_rn(y, ds);
  return q;
}

__device__ __forceinline__ uint16_t e4m3x2_rn_satfinite(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// grid (ceil(S / 256), B*H): the codes of each row.
__global__ void __launch_bounds__(kPrepThreads, 4) prep_quantize_kernel(const uint16_t* __restrict__ x,
                                                                          uint8_t* __restrict__ codes,
                                                                          const float* __restrict__ descale, int S,
                                                                          int rmsnorm, double eps) {
  const int bh = blockIdx.y;
  const int s = blockIdx.x * kPrepThreads + threadIdx.x;
  if (s >= S) return;
  const long long rowi = (long long)bh * S + s;
  const uint4* row = reinterpret_cast<const uint4*>(x) + rowi * 16;
  const double r = prep_row_factor(row, rmsnorm, eps);
  const float ds = __ldg(&descale[bh]);
  const float rcp = __frcp_rn(ds);
  uint4* dst = reinterpret_cast<uint4*>(codes) + rowi * 8;
#pragma unroll 2
  for (int i = 0; i < 16; i += 2) {
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 w = __ldg(&row[i + h]);
      const uint32_t p[4] = {w.x, w.y, w.z, w.w};
      uint16_t c[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        c[k] = e4m3x2_rn_satfinite(prep_quotient(prep_y(p[k] << 16, r, rmsnorm), ds, rcp),
                                   prep_quotient(prep_y(p[k] & 0xFFFF0000u, r, rmsnorm), ds, rcp));
      o[2 * h] = (uint32_t)c[0] | ((uint32_t)c[1] << 16);
      o[2 * h + 1] = (uint32_t)c[2] | ((uint32_t)c[3] << 16);
    }
    dst[i / 2] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace hattn
