// prep_kernel.cuh -- e4m3 quantisation prologue for the fp8 forward (sm_100a).
//
// The step before fp8 attention on the pages: FlashDreams PR #486
// "flashdreams.accelerated API v0", section 1.1 (FP8 E4M3 quantisation with
// tensor- or slice-granularity scales) and section 1.2 (head-scoped Q/K
// normalisation, optional FP8 SDPA), with the clamp to the e4m3fn range +-448
// that VeOmni PR #1363 describes for its quantizers.  Per (batch, head):
//   ss      = sum of x_d^2 over the row (fp32, every operation rounded to
//             nearest): lane k of the row's 16 threads adds the squares of
//             d = 8k .. 8k+7 in ascending order, then the 16 partial sums are
//             added pairwise, neighbours first (k with k^1, then pairs with
//             pairs, ...); the squares of bf16 values are exact in fp32
//   r       = 1 / sqrt(ss / 128 + eps)          per row (only with rmsnorm), fp32
//   y_d     = x_d * r (fp32), or x_d without rmsnorm
//   descale = max |y| / 448 over the head (1 if that max is 0), fp32
//   code    = e4m3 of y / descale: fp32 quotient, round to nearest even,
//             saturating at +-448
// Every step is fixed in precision and order, so the codes and descales are a
// function of the input alone: bit for bit the same for any grid, batch or
// head split.  Three launches (after a memset of the descale array): the head
// maxima (atomicMax on the non-negative fp32 bit patterns, which order like
// integers, so the result does not depend on the order), max -> descale in
// place, and the codes.  HBM-bound: x is read twice and the codes written once;
// 16 threads share a row, so a warp reads two whole rows (512 contiguous
// bytes) per load and writes two rows of codes (256 bytes) per store.
#pragma once

#include "sm100.cuh"

namespace hattn {

constexpr int kPrepD = 128;
constexpr int kPrepThreads = 256;     // 16 rows at a time: 16 threads per row, 8 values each
constexpr int kPrepRowsPerCta = 64;   // 4 rows per thread, their loads issued together

// This lane's 8 values (d = 8 (lane % 16) .. +7 of its row) as fp32.
struct PrepVals {
  float v[8];
};

__device__ __forceinline__ PrepVals prep_unpack(uint4 w) {
  PrepVals p;
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    p.v[2 * t] = __uint_as_float(u[t] << 16);
    p.v[2 * t + 1] = __uint_as_float(u[t] & 0xFFFF0000u);
  }
  return p;
}

// Row factor r = 1 / sqrt(ss / 128 + eps) (1 without rmsnorm); every lane of
// the row's 16 gets the same bits (fp32 addition is commutative).  Rounded
// operations are spelt out so that no multiply-add is contracted.
__device__ __forceinline__ float prep_row_factor(const PrepVals& p, int rmsnorm, float eps) {
  if (!rmsnorm) return 1.f;
  float s = 0.f;
#pragma unroll
  for (int t = 0; t < 8; ++t) s = __fadd_rn(s, __fmul_rn(p.v[t], p.v[t]));
#pragma unroll
  for (int off = 1; off < 16; off <<= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
  return __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fmul_rn(s, 0.0078125f), eps)));
}

// grid (ceil(S / 64), B*H): the largest |y| of each head into amax_bits (zeroed).
__global__ void __launch_bounds__(kPrepThreads) prep_amax_kernel(const uint16_t* __restrict__ x,
                                                                   unsigned int* __restrict__ amax_bits, int S,
                                                                   int rmsnorm, float eps) {
  const int bh = blockIdx.y;
  const int sub = threadIdx.x & 15;               // which 8 values of the row
  const int r0 = blockIdx.x * kPrepRowsPerCta + (threadIdx.x >> 4);
  const uint4* base = reinterpret_cast<const uint4*>(x) + (long long)bh * S * 16 + sub;
  uint4 w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int s = r0 + 16 * k;
    w[k] = s < S ? __ldg(base + (long long)s * 16) : make_uint4(0u, 0u, 0u, 0u);
  }
  float m = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const PrepVals p = prep_unpack(w[k]);
    const float r = prep_row_factor(p, rmsnorm, eps);   // rows past S are zero: y = 0
#pragma unroll
    for (int t = 0; t < 8; ++t) m = fmaxf(m, fabsf(rmsnorm ? __fmul_rn(p.v[t], r) : p.v[t]));
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

// grid (ceil(S / 64), B*H): the codes of each row.
__global__ void __launch_bounds__(kPrepThreads) prep_quantize_kernel(const uint16_t* __restrict__ x,
                                                                       uint8_t* __restrict__ codes,
                                                                       const float* __restrict__ descale, int S,
                                                                       int rmsnorm, float eps) {
  const int bh = blockIdx.y;
  const int sub = threadIdx.x & 15;
  const int r0 = blockIdx.x * kPrepRowsPerCta + (threadIdx.x >> 4);
  const uint4* base = reinterpret_cast<const uint4*>(x) + (long long)bh * S * 16 + sub;
  uint2* dst = reinterpret_cast<uint2*>(codes) + (long long)bh * S * 16 + sub;
  uint4 w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int s = r0 + 16 * k;
    w[k] = s < S ? __ldg(base + (long long)s * 16) : make_uint4(0u, 0u, 0u, 0u);
  }
  const float ds = __ldg(&descale[bh]);
  const float rcp = __frcp_rn(ds);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const PrepVals p = prep_unpack(w[k]);
    const float r = prep_row_factor(p, rmsnorm, eps);   // all 16 lanes of the row take part
    uint16_t c[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float y0 = rmsnorm ? __fmul_rn(p.v[2 * t], r) : p.v[2 * t];
      const float y1 = rmsnorm ? __fmul_rn(p.v[2 * t + 1], r) : p.v[2 * t + 1];
      c[t] = e4m3x2_rn_satfinite(prep_quotient(y0, ds, rcp), prep_quotient(y1, ds, rcp));
    }
    const int s = r0 + 16 * k;
    if (s < S)
      dst[(long long)s * 16] = make_uint2((uint32_t)c[0] | ((uint32_t)c[1] << 16), (uint32_t)c[2] | ((uint32_t)c[3] << 16));
  }
}

}  // namespace hattn
