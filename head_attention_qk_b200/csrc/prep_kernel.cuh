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
//   code    = e4m3 of the exact quotient y / descale (of the fp32 y and
//             descale), round to nearest with ties to even, saturating at
//             +-448: the fp32 quotient, moved one fp32 step towards the exact
//             one when it lands exactly on an e4m3 midpoint that the exact
//             quotient is not on
// Every step is fixed in precision and order, so the codes and descales are a
// function of the input alone: bit for bit the same for any grid, batch or
// head split.  Two launches (after a memset of the descale array): the head
// maxima (atomicMax on fp32 bit patterns, which order like integers, so the
// result does not depend on the order) and the codes, which also turn each
// head's maximum into its descale.  HBM-bound: x is read twice and the codes written once;
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

// grid (ceil(S / 64), min(B*H, 65535)); kStride: heads strided over grid y
// (more than 65535 of them), else head = blockIdx.y.  The largest |y| of each head, stored negated into
// amax_bits (zeroed): the bit patterns of non-positive floats order like
// unsigned integers by magnitude, so atomicMax keeps the largest, and the
// sign bit tells this value apart from a finished descale.
__device__ __forceinline__ void prep_amax_head(const uint16_t* __restrict__ x, unsigned int* __restrict__ amax_bits,
                                               int S, int bh, int rmsnorm, float eps, float* wmax) {
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
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float bm = wmax[0];
#pragma unroll
    for (int i = 1; i < kPrepThreads / 32; ++i) bm = fmaxf(bm, wmax[i]);
    atomicMax(&amax_bits[bh], __float_as_uint(-bm));
  }
}

template <bool kStride>
__global__ void __launch_bounds__(kPrepThreads) prep_amax_kernel(const uint16_t* __restrict__ x,
                                                                   unsigned int* __restrict__ amax_bits, int S,
                                                                   int n_bh, int rmsnorm, float eps) {
  __shared__ float wmax[kPrepThreads / 32];
  if constexpr (!kStride) {
    prep_amax_head(x, amax_bits, S, blockIdx.y, rmsnorm, eps, wmax);
  } else {
    for (int bh = blockIdx.y; bh < n_bh; bh += gridDim.y) {
      prep_amax_head(x, amax_bits, S, bh, rmsnorm, eps, wmax);
      __syncthreads();                            // wmax is rewritten for the next head
    }
  }
}

// descale of a head from its slot: either -amax (sign bit set, as the maxima
// kernel left it) or the descale already written there; both give the same.
__device__ __forceinline__ float prep_descale_of(float slot) {
  if (!signbit(slot)) return slot;
  const float amax = -slot;
  return amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

// True when the fp32 value q lies exactly on a midpoint between two
// neighbouring e4m3fn values: in the e4m3 normal range (2^-6 <= |q| < 2^9)
// the midpoints are the values whose fraction has four bits ending in 1 (the
// bit worth half an e4m3 step is bit 19 of the fp32 fraction); below it the
// e4m3 step is 2^-9 and the midpoints are the odd multiples of 2^-10 (that bit
// sits at fraction bit 13 - e for binary exponent e, and for e = -10 it is
// the leading bit, so q = 2^-10 exactly).
__device__ __forceinline__ bool e4m3_midpoint(float q) {
  const uint32_t u = __float_as_uint(q) & 0x7FFFFFFFu;
  const int e = (int)(u >> 23) - 127;
  if (e > 8 || e < -10) return false;
  if (e == -10) return u == (117u << 23);
  const uint32_t half = e >= -6 ? (1u << 19) : (1u << (13 - e));
  return (u & ((half << 1) - 1u)) == half;
}

// q = the fp32 quotient y / ds correctly rounded, res = y - q ds exactly (one
// fused multiply-add).  The e4m3 code of the exact quotient is the code of q
// unless q sits exactly on an e4m3 midpoint while the exact quotient does not
// (res != 0): then no midpoint lies strictly between q and the exact quotient
// (they are within half an fp32 step), so moving q one fp32 step towards it
// gives the code the exact quotient rounds to.  Without this the fp32 rounding
// would turn such a quotient into a tie (frequent when y and the descale come
// from bf16 values: 448 y / amax is then often an exact e4m3 midpoint).
__device__ __forceinline__ float e4m3_exact_tie(float q, float res) {
  if (res == 0.f || !e4m3_midpoint(q)) return q;
  return __uint_as_float(__float_as_uint(q) + (((res > 0.f) == (q > 0.f)) ? 1u : 0xFFFFFFFFu));
}

// Every e4m3 midpoint has the low 19 fraction bits of its fp32 value clear
// (the half-step bit is bit 19 or above), so a pair with neither value in that
// form skips the midpoint test (almost all of them).
__device__ __forceinline__ bool maybe_e4m3_midpoint2(float2 q) {
  return ((__float_as_uint(q.x) & 0x7FFFFu) == 0u) | ((__float_as_uint(q.y) & 0x7FFFFu) == 0u);
}

// y / ds for a pair, ready for the round-to-nearest e4m3 conversion (rcp =
// 1/ds correctly rounded, ds >= 2^-60 so that no residual below is
// subnormal).  q0 = y * rcp is within an ulp of the quotient; with the exact
// residual r = y - q0 ds (one fused multiply-add) the correction q0 + r * rcp
// is the correctly rounded quotient (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990), whose own residual settles an e4m3 midpoint (e4m3_exact_tie).  Below
// 2^-11 the correction is skipped: every value there, exact or not, takes the
// e4m3 code of a signed zero (the smallest e4m3 step is 2^-9, its first
// midpoint 2^-10), and the sign is the quotient's either way.
__device__ __forceinline__ float2 prep_quotient2(float2 y, float ds, float rcp) {
  const float2 r2 = make_float2(rcp, rcp), nds = make_float2(-ds, -ds);
  const float2 q0 = __fmul2_rn(y, r2);
  const float2 res = __ffma2_rn(q0, nds, y);
  const float2 q1 = __ffma2_rn(res, r2, q0);
  float2 q = make_float2(fabsf(q0.x) < 0x1p-11f ? q0.x : q1.x, fabsf(q0.y) < 0x1p-11f ? q0.y : q1.y);
  if (maybe_e4m3_midpoint2(q)) {
    const float2 res2 = __ffma2_rn(q, nds, y);
    q = make_float2(e4m3_exact_tie(q.x, res2.x), e4m3_exact_tie(q.y, res2.y));
  }
  return q;
}

// Exact division for a head of tiny values (descale < 2^-60), with the same
// midpoint rule.
__device__ __forceinline__ float prep_quotient_exact(float y, float ds) {
  const float q = __fdiv_rn(y, ds);
  return e4m3_exact_tie(q, __fmaf_rn(-q, ds, y));
}

__device__ __forceinline__ uint16_t e4m3x2_rn_satfinite(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// grid (ceil(S / 64), min(B*H, 65535)), heads strided over grid y with kStride: the codes of each row, and the descale of each
// head in place of its maximum.  CTAs walk the rows in the reverse of the
// maxima kernel's order, so the rows it read last, still in L2, come first.
__device__ __forceinline__ void prep_quantize_head(const uint16_t* __restrict__ x, uint8_t* __restrict__ codes,
                                                   float* __restrict__ descale, int S, int bh, int rmsnorm,
                                                   float eps) {
  const int tile = gridDim.x - 1 - blockIdx.x;
  const int sub = threadIdx.x & 15;
  const int r0 = tile * kPrepRowsPerCta + (threadIdx.x >> 4);
  const uint4* base = reinterpret_cast<const uint4*>(x) + (long long)bh * S * 16 + sub;
  uint2* dst = reinterpret_cast<uint2*>(codes) + (long long)bh * S * 16 + sub;
  uint4 w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int s = r0 + 16 * k;
    w[k] = s < S ? __ldg(base + (long long)s * 16) : make_uint4(0u, 0u, 0u, 0u);
  }
  const float ds = prep_descale_of(*reinterpret_cast<volatile float*>(&descale[bh]));
  if (tile == 0 && threadIdx.x == 0) descale[bh] = ds;   // the other CTAs read either form
  const float rcp = __frcp_rn(ds);
  const bool tiny_ds = ds < 0x1p-60f;    // a head of tiny values: exact division throughout
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const PrepVals p = prep_unpack(w[k]);
    const float r = prep_row_factor(p, rmsnorm, eps);   // all 16 lanes of the row take part
    uint16_t c[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float2 y = make_float2(p.v[2 * t], p.v[2 * t + 1]);
      if (rmsnorm) y = __fmul2_rn(y, make_float2(r, r));
      const float2 q = tiny_ds ? make_float2(prep_quotient_exact(y.x, ds), prep_quotient_exact(y.y, ds))
                               : prep_quotient2(y, ds, rcp);
      c[t] = e4m3x2_rn_satfinite(q.x, q.y);
    }
    const int s = r0 + 16 * k;
    if (s < S)
      dst[(long long)s * 16] = make_uint2((uint32_t)c[0] | ((uint32_t)c[1] << 16), (uint32_t)c[2] | ((uint32_t)c[3] << 16));
  }
}

template <bool kStride>
__global__ void __launch_bounds__(kPrepThreads) prep_quantize_kernel(const uint16_t* __restrict__ x,
                                                                       uint8_t* __restrict__ codes,
                                                                       float* __restrict__ descale, int S,
                                                                       int n_bh, int rmsnorm, float eps) {
  if constexpr (!kStride) {
    prep_quantize_head(x, codes, descale, S, gridDim.y - 1 - blockIdx.y, rmsnorm, eps);
  } else {
    for (int bi = blockIdx.y; bi < n_bh; bi += gridDim.y)
      prep_quantize_head(x, codes, descale, S, n_bh - 1 - bi, rmsnorm, eps);
  }
}

}  // namespace hattn
