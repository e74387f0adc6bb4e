// bwd_kernel.cuh -- deterministic attention backward for sm_100a (bf16).
//
// For dO = dL/dO, P = exp(scale * Q K^T - LSE) (LSE from the forward):
//   dV = P^T dO,   dP = dO V^T,   Delta_i = sum_d dO_id O_id,
//   dS = P * (dP - Delta),   dQ = scale * dS K,   dK = scale * dS^T Q.
// RL-Kernel PR #319 ("feat(attention): add strict bitwise ROCm path", What the
// strict contract costs) shows a deterministic mha_bwd whose workspace grows as
// O(S^2); here every output tile is owned by one CTA that sums its terms in a
// fixed order, with no atomics and no S x S buffer:
//
//   bwd_delta_kernel  Delta (fp32) from the forward's bf16 O and dO.
//   bwd_dkdv_kernel   persistent, one CTA per SM; each (b, kv head, 128-key
//                     tile) unit loops over the group's query heads
//                     (ascending) and their 128-row query tiles (ascending).
//                     Per step, four tcgen05 MMAs:
//                       S^T = K Q^T, dP^T = V dO^T, dV += P^T dO, dK += dS^T Q
//                     (S^T of the next step and dV in two query halves).
//   bwd_dq_kernel     persistent, one CTA per SM; each (b, q head, 128-row query
//                     tile) unit loops over KV tiles (ascending).  Per step,
//                     three MMAs:
//                       S = Q K^T, dP = dO V^T, dQ += dS K.
//                     Launched as a programmatic dependent of bwd_dkdv_kernel
//                     (the two read the same inputs and write different
//                     outputs): its CTAs start on the SMs whose dK/dV CTAs
//                     have finished and take units from a global counter,
//                     heaviest first, so the dK/dV kernel's last, longest
//                     units overlap dQ work instead of leaving SMs idle.
//
// Roles: warps 0-7 compute, warp 8 TMA producer, warp 9 MMA issuer and
// tensor-memory owner.  Compute warp w owns tile rows 32 (w % 4) .. +31 (its
// TMEM lane quarter) and half of the columns of S, dP: nothing in P or dS
// needs a reduction along a row (the row statistics LSE and Delta come from the
// forward), so the two warps of a lane quarter split the columns, and two
// warps per SM sub-partition keep the MUFU exponentials fed.  Each packs its
// 16-bit P or dS over the first half of the fp32 columns it read.  In dQ warp
// w holds columns 64 (w / 4) .. +63; in dK/dV it holds columns 32 (w / 4) +
// 64 c .. +31 for chunks c = 0, 1, so that all eight warps finish the P^T of
// queries 0..63 first and the MMAs of that half start while they form the
// other.  P and dS are rounded to bf16 before their MMAs; S, dP and the
// dQ/dK/dV accumulators are fp32.
#pragma once

#include "ds_layout.h"
#include "fwd_kernel.cuh"
#include "per_device.h"
#include "sm100.cuh"

namespace hattn {

constexpr int kBwdThreads = 320;
constexpr int kBwdComputeWarps = 8;
constexpr int kTile = 128;
constexpr int kTileBytesBf16 = kTile * kHeadDim * 2;     // 32 KB, two 16 KB swizzle halves

struct BwdArgs {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;
  int B, Hq, Hkv, Sq, Sk;
  int causal;
  float scale;
  float scale_log2;
  const float* lse;       // [B,Hq,Sq] natural log
  const float* delta;     // [B,Hq,Sq]
  uint16_t* dq;           // [B,Hq,Sq,D] bf16
  uint16_t* dk;           // [B,Hkv,Sk,D]
  uint16_t* dv;
  uint32_t* dq_sched;     // dQ kernel: next unit to take (zeroed by the Delta kernel)
  // attn_bwd_dsbuf: dS^T tiles written by the dK/dV kernel, [B*Hq][n_kt][nq]
  // tiles of 128 keys x 128 queries (bf16, 32 KB each, in the blocked layout
  // of ds_tile_offset); null otherwise
  uint16_t* ds_buf;
  float* dq_acc;          // one-pass backward: fp32 dQ accumulator [B,Hq,Sq,D]
  uint32_t* dq_cnt;       // one-pass backward: contributions added, per (b, q head, query tile)
};

enum : int {
  kSiteBwdKV = 20, kSiteBwdStFull, kSiteBwdStEmpty, kSiteBwdS, kSiteBwdDP, kSiteBwdP, kSiteBwdDone, kSiteBwdAlign
};

// ---------------------------------------------------------------------------- Delta
// Delta_r = sum_d dO_rd O_rd.  16 threads share a row (8 values each, one
// 16-byte load of O and of dO), so a warp reads two whole rows per load; each
// thread has four rows in flight.  The 16 partial sums meet by a xor
// butterfly in a fixed order: the result does not depend on the grid.  It
// also resets the dQ kernel's unit counter (sched, when given), which runs
// after it on the same stream.
constexpr int kDeltaRowsPerCta = 64;

__global__ void __launch_bounds__(256) bwd_delta_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                                                        float* __restrict__ delta, long long rows, uint32_t* sched) {
  griddep_wait();                                    // O comes from the grid before (the forward)
  if (threadIdx.x == 0) griddep_launch_dependents();
  if (sched && blockIdx.x == 0 && threadIdx.x == 0) *sched = 0u;
  const int sub = threadIdx.x & 15;
  const long long r0 = (long long)blockIdx.x * kDeltaRowsPerCta + (threadIdx.x >> 4);
  const uint4* o4 = reinterpret_cast<const uint4*>(o) + sub;
  const uint4* g4 = reinterpret_cast<const uint4*>(dout) + sub;
  uint4 a[4], g[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const long long r = r0 + 16 * k;
    const bool in = r < rows;
    a[k] = in ? __ldg(o4 + r * 16) : make_uint4(0u, 0u, 0u, 0u);
    g[k] = in ? __ldg(g4 + r * 16) : make_uint4(0u, 0u, 0u, 0u);
  }
  auto lo = [](uint32_t w) { return __uint_as_float(w << 16); };
  auto hi = [](uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); };
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t aw[4] = {a[k].x, a[k].y, a[k].z, a[k].w}, gw[4] = {g[k].x, g[k].y, g[k].z, g[k].w};
    float s = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) s += lo(aw[t]) * lo(gw[t]) + hi(aw[t]) * hi(gw[t]);
#pragma unroll
    for (int off = 1; off < 16; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const long long r = r0 + 16 * k;
    if (sub == 0 && r < rows) delta[r] = s;
  }
}

// Shared helpers --------------------------------------------------------------

// Load one 128 x 128 bf16 tile (two 64-column TMA boxes) of a 3-D tensor map.
__device__ __forceinline__ void tma_tile_bf16(uint8_t* dst, const CUtensorMap* m, uint64_t* bar, int row, int head) {
  tma_load_3d(dst, m, bar, 0, row, head);
  tma_load_3d(dst + 16384, m, bar, 64, row, head);
}

// D (+)= A B^T with both operands K-major bf16 tiles in shared memory (M = N = 128, K = 128).
__device__ __forceinline__ void mma_tile_ss_kmajor(uint32_t d, uint32_t sa, uint32_t sb, uint32_t acc) {
  constexpr uint32_t idesc = make_idesc(1, 1, 0, 128, 128);
  constexpr uint32_t hi = sdesc_hi(1024);
  const uint32_t a_lo = sdesc_lo(sa, 16), b_lo = sdesc_lo(sb, 16);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t off = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
    mma_f16_ss2(d, a_lo + off, hi, b_lo + off, hi, idesc, (acc || k > 0) ? 1u : 0u);
  }
}

// D (+)= A B where A (128 x 128, bf16 pairs) is in tensor memory and B is a
// shared-memory tile read MN-major: the reduction runs over the tile's rows.
// A's reduction elements 0..63 sit in columns [0, 32) and 64..127 in [64, 96)
// (each half written by the warp that owns those 64 columns of S or dP).
__device__ __forceinline__ void mma_tile_ts_mnmajor_halves(uint32_t d, uint32_t a_tmem, uint32_t sb, uint32_t acc) {
  constexpr uint32_t idesc = make_idesc(1, 1, 1, 128, 128);
  constexpr uint32_t hi = sdesc_hi(1024);
  const uint32_t b_lo = sdesc_lo(sb, 16384);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    mma_f16_ts2(d, a_tmem + k * 8 + (k >> 2) * 32, b_lo + k * (2048 >> 4), hi, idesc, (acc || k > 0) ? 1u : 0u);
}

// D = A B^T for the 64 B rows 64 h .. 64 h + 63 only (M = 128, N = 64, K = 128),
// both operands K-major bf16 tiles in shared memory.  Row 64 of a swizzled
// tile starts 8 KB into each 16 KB half, a whole number of swizzle atoms.
__device__ __forceinline__ void mma_tile_ss_kmajor_n64(uint32_t d, uint32_t sa, uint32_t sb, int h) {
  constexpr uint32_t idesc = make_idesc(1, 1, 0, 128, 64);
  constexpr uint32_t hi = sdesc_hi(1024);
  const uint32_t a_lo = sdesc_lo(sa, 16), b_lo = sdesc_lo(sb + h * 8192, 16);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t off = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
    mma_f16_ss2(d, a_lo + off, hi, b_lo + off, hi, idesc, k > 0 ? 1u : 0u);
  }
}

// TMEM column (relative to the S^T or dP^T block) of the bf16 pairs that hold
// reduction elements 16 k .. 16 k + 15 of P^T or dS^T.  Reduction element q
// (a query) is computed by the warp with column half (q / 32) % 2 in its chunk
// q / 64, which packs its 32 values over the first 16 of its 32 fp32 columns.
__device__ __forceinline__ constexpr uint32_t bwd_pair_col(int k) {
  return (uint32_t)((k >> 2) * 64 + ((k >> 1) & 1) * 32 + (k & 1) * 8);
}

// D (+)= A B over reduction groups K0 .. K1-1 (16 elements each), where A
// (128 rows of bf16 pairs, laid out by bwd_pair_col) is in tensor memory and
// B is a shared-memory tile read MN-major: the reduction runs over its rows.
template <int K0, int K1>
__device__ __forceinline__ void mma_tile_ts_mnmajor(uint32_t d, uint32_t a_tmem, uint32_t sb, uint32_t acc) {
  constexpr uint32_t idesc = make_idesc(1, 1, 1, 128, 128);
  constexpr uint32_t hi = sdesc_hi(1024);
  const uint32_t b_lo = sdesc_lo(sb, 16384);
#pragma unroll
  for (int k = K0; k < K1; ++k)
    mma_f16_ts2(d, a_tmem + bwd_pair_col(k), b_lo + k * (2048 >> 4), hi, idesc, (acc || k > K0) ? 1u : 0u);
}

// Read 64 columns of an fp32 TMEM row (from taddr), scale them and store them as
// bf16 to global memory at dst.
__device__ __forceinline__ void store_half_row_bf16(uint32_t taddr, float mul, uint16_t* dst, bool store) {
#pragma unroll 1
  for (int q = 0; q < 2; ++q) {
    uint32_t u[32];
    __syncwarp();
    tmem_ld32(taddr + q * 32, u);
    tmem_wait_ld();
    if (store) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + q * 32);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
          w[t] = pack_bf16x2(__uint_as_float(u[8 * e + 2 * t]) * mul, __uint_as_float(u[8 * e + 2 * t + 1]) * mul);
        d4[e] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

// The k-th unit of CTA c among G persistent CTAs (the dK/dV kernel and the
// one-pass backward): the heaviest-first list is dealt out in snake order (c, then
// 2G-1-c, then 2G+c, ...), which evens out the causal unit sizes.  Increasing
// in k, so the first index past the list ends the CTA's loop.
__device__ __forceinline__ int dq_unit_index(int k, int c, int G) { return k * G + ((k & 1) ? G - 1 - c : c); }

// ---------------------------------------------------------------------------- dK / dV
struct DkdvSmem {
  // Q is read by S^T_n early in a step and by dK_n at its end, so it gets a
  // third stage: Q_{n+1} can load while dK_{n-1} still reads Q_{n-1}.
  static constexpr int kQStages = 3;
  static constexpr int kDOStages = 2;
  static constexpr int kStatStages = 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTileBytesBf16;
  static constexpr int kQ = kV + kTileBytesBf16;
  static constexpr int kDO = kQ + kQStages * kTileBytesBf16;
  static constexpr int kStats = kDO + kDOStages * kTileBytesBf16;   // [stage] x (128 lse2 + 128 delta) fp32
  static constexpr int kBars = kStats + kStatStages * 2 * kTile * 4;
  static constexpr int kBytes = kBars + 26 * 8;
  // No alignment slack: this layout fills the 227 KB a CTA may hold.  The
  // dynamic shared window starts 1024-byte aligned on sm_100a (after the 1 KB
  // the driver reserves); the kernel checks that and refuses to run otherwise.
  static constexpr int kAlloc = kBytes;
  static_assert(kAlloc <= 232448, "shared memory per CTA");
};

__device__ __forceinline__ int bwd_first_q_tile(int j, int Sq, int Sk, int causal) {
  if (!causal) return 0;
  const int first_q = j * kTile - (Sk - Sq);          // smallest query that sees key j*128
  return first_q <= 0 ? 0 : first_q / kTile;
}

// One unit of dK/dV work: key tile j of (batch, KV head) bkv; its steps run
// over the group's query heads g (ascending) and their query tiles i0 ..
// nq - 1 (ascending).
struct DkdvUnit {
  int j, bkv, i0, nqi, steps;
};

// Unit t of the work list, heaviest first: key tiles are the slow index, so
// under a causal mask the tiles seen by the most query tiles (small j) come
// first.  Every key tile has at least one query tile (causal needs Sq <= Sk,
// bottom-right aligned), so steps >= 1.
__device__ __forceinline__ DkdvUnit dkdv_unit(const BwdArgs& a, int t) {
  const int BH = a.B * a.Hkv;
  DkdvUnit u;
  u.j = t / BH;
  u.bkv = t - u.j * BH;
  const int nq = (a.Sq + kTile - 1) / kTile;
  u.i0 = bwd_first_q_tile(u.j, a.Sq, a.Sk, a.causal);
  u.nqi = nq - u.i0;
  u.steps = (a.Hq / a.Hkv) * u.nqi;
  return u;
}

// Persistent: one CTA per SM walks its units (dealt out in snake order).  A
// unit's dK / dV rows are summed over its steps in the same
// order whichever CTA runs it.  Across units the Q / dO / statistics rings,
// the S^T / dP^T buffers and every barrier phase continue on one global step
// count; the next unit's K and V load as soon as the current unit's last S^T
// and dP^T have read the old ones (kv_empty), and its first S^T and dP^T run
// during the current unit's last step and epilogue.  Its first dV MMA cannot
// overwrite the accumulators early: it waits for that unit's first P^T, which
// the compute warps write only after reading dV and dK out.
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dkdv_kernel(const __grid_constant__ BwdArgs a) {
  using L = DkdvSmem;
  extern __shared__ uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {              // the layout needs a 1024-byte aligned window
    if (threadIdx.x == 0) raise_error(0x100 | kSiteBwdAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  const int warp = warp_id(), lane = lane_id();
  const int n_kt = (a.Sk + kTile - 1) / kTile, nq_t = (a.Sq + kTile - 1) / kTile;
  const int n_units = n_kt * a.B * a.Hkv;
  const int cta = blockIdx.x, n_cta = gridDim.x;
  const int G = a.Hq / a.Hkv;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;       // [3]
  uint64_t* q_empty = bars + 4;      // [3]
  uint64_t* do_full = bars + 7;      // [2]
  uint64_t* do_empty = bars + 9;     // [2]
  uint64_t* s_full = bars + 11;      // [2] S^T columns of query half 0 / 1
  uint64_t* dp_full = bars + 13;
  uint64_t* p_full = bars + 14;      // [2] P^T of query half 0 / 1 written
  uint64_t* acc_done = bars + 16;    // a unit's dK / dV MMAs have completed
  uint64_t* ds_full = bars + 17;     // dS^T written
  uint64_t* st_full = bars + 18;     // [2] LSE / Delta of a step staged (32 producer lanes)
  uint64_t* st_empty = bars + 20;    // [2] the compute warps are done with them (one arrival per warp)
  uint64_t* kv_empty = bars + 22;    // a unit's last S^T and dP^T have read K and V
  uint64_t* mma_drain = bars + 23;   // every MMA of the CTA has completed (committed once, at exit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    mbar_init(mma_drain, 1);
    for (int s = 0; s < L::kQStages; ++s) { mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1); }
    for (int s = 0; s < L::kDOStages; ++s) { mbar_init(&do_full[s], 1); mbar_init(&do_empty[s], 1); }
    for (int s = 0; s < L::kStatStages; ++s) { mbar_init(&st_full[s], 32); mbar_init(&st_empty[s], kBwdComputeWarps); }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&s_full[h], 1);
      mbar_init(&p_full[h], kBwdComputeWarps);   // one arrival per compute warp
    }
    mbar_init(dp_full, 1);
    mbar_init(ds_full, kBwdComputeWarps);
    mbar_init(acc_done, 1);
    fence_barrier_init();
  }
  if (warp == 9) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: dV [0,128), dK [128,256), S^T / P^T [256,384), dP^T / dS^T [384,512)
  // Launched as a programmatic dependent of the Delta kernel: the setup above
  // overlaps its end; Delta is read only after it has completed.  The dQ
  // kernel, launched next the same way, needs nothing this kernel writes: let
  // it start on SMs as soon as they free up.
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 8) {
    // ---------------------------------------------------------------- producer
    bool ok = true;
    int ul = 0, n0 = 0;                          // units started, global step count at the unit's start
    for (int k = 0; ok; ++k) {
      const int t = dq_unit_index(k, cta, n_cta);
      if (t >= n_units) break;
      const DkdvUnit u = dkdv_unit(a, t);
      const int b = u.bkv / a.Hkv, kvh = u.bkv - b * a.Hkv;
      if (ul > 0) ok = warp_wait(kv_empty, (ul - 1) & 1, kSiteBwdKV);   // the last unit's S^T / dP^T are done
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(kv_full, 2 * kTileBytesBf16);
        tma_tile_bf16(smem + L::kK, &a.tm_k, kv_full, u.j * kTile, u.bkv);
        tma_tile_bf16(smem + L::kV, &a.tm_v, kv_full, u.j * kTile, u.bkv);
      }
      for (int s = 0; s < u.steps && ok; ++s) {
        const int n = n0 + s;
        const int g = s / u.nqi, i = u.i0 + s % u.nqi;
        const int bh = b * a.Hq + kvh * G + g;
        const int qs = n % L::kQStages, qu = n / L::kQStages;
        if (n >= L::kQStages) ok = warp_wait(&q_empty[qs], (qu - 1) & 1, kSiteBwdStEmpty);
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&q_full[qs], kTileBytesBf16);
          tma_tile_bf16(smem + L::kQ + qs * kTileBytesBf16, &a.tm_q, &q_full[qs], i * kTile, bh);
        }
        const int ds = n % L::kDOStages, du = n / L::kDOStages;
        if (n >= L::kDOStages) ok = warp_wait(&do_empty[ds], (du - 1) & 1, kSiteBwdStEmpty);
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&do_full[ds], kTileBytesBf16);
          tma_tile_bf16(smem + L::kDO + ds * kTileBytesBf16, &a.tm_do, &do_full[ds], i * kTile, bh);
        }
        const int ss = n % L::kStatStages, su = n / L::kStatStages;
        if (n >= L::kStatStages) ok = warp_wait(&st_empty[ss], (su - 1) & 1, kSiteBwdStEmpty);
        if (!ok) break;
        float* stats = reinterpret_cast<float*>(smem + L::kStats + ss * 2 * kTile * 4);
        {
          // all eight global loads in flight before the first store
          float lv[kTile / 32], dv[kTile / 32];
#pragma unroll
          for (int kk = 0; kk < kTile / 32; ++kk) {
            const int qi = i * kTile + lane + 32 * kk;
            const bool valid = qi < a.Sq;
            const size_t idx = (size_t)bh * a.Sq + (valid ? qi : 0);
            lv[kk] = valid ? __ldg(&a.lse[idx]) * 1.4426950408889634f : INFINITY;   // P = 0 past Sq
            dv[kk] = valid ? __ldg(&a.delta[idx]) : 0.f;
          }
#pragma unroll
          for (int kk = 0; kk < kTile / 32; ++kk) {
            stats[lane + 32 * kk] = lv[kk];
            stats[kTile + lane + 32 * kk] = dv[kk];
          }
        }
        mbar_arrive(&st_full[ss]);
      }
      n0 += u.steps;
      ++ul;
    }
    // drain: every load issued must land before the CTA exits
    if (lane == 0) {
      if (ul > 0) mbar_wait_drain(kv_full, (ul - 1) & 1, kSiteBwdKV);
      for (int n = max(0, n0 - L::kQStages); n < n0; ++n)
        mbar_wait_drain(&q_full[n % L::kQStages], (n / L::kQStages) & 1, kSiteBwdStFull);
      for (int n = max(0, n0 - L::kDOStages); n < n0; ++n)
        mbar_wait_drain(&do_full[n % L::kDOStages], (n / L::kDOStages) & 1, kSiteBwdStFull);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
      auto sQ_of = [&](int n) { return smem_u32(smem + L::kQ + (n % L::kQStages) * kTileBytesBf16); };
      auto sDO_of = [&](int n) { return smem_u32(smem + L::kDO + (n % L::kDOStages) * kTileBytesBf16); };
      auto wait_q = [&](int n) { return mbar_wait(&q_full[n % L::kQStages], (n / L::kQStages) & 1, kSiteBwdStFull); };
      auto wait_do = [&](int n) {
        return mbar_wait(&do_full[n % L::kDOStages], (n / L::kDOStages) & 1, kSiteBwdStFull);
      };
      // Issue order per step n, by query halves h = 0, 1: dV_n over the
      // queries of half h (once P^T_n of that half is written), then S^T_{n+1}
      // of half h (its columns held that half of P^T_n, which dV_n has read:
      // one thread's MMAs run in order); then dK_n (once dS^T_n is written)
      // and dP^T_{n+1}.  The next step's first half of S^T thus runs while the
      // compute warps form the second half of P^T and then dS^T of this one.
      bool ok = true;
      int ul = 0, n0 = 0;
      for (int k = 0; ok; ++k) {
        const int t = dq_unit_index(k, cta, n_cta);
        if (t >= n_units) break;
        const int steps = dkdv_unit(a, t).steps;
        const int n_end = n0 + steps;
        ok = mbar_wait(kv_full, ul & 1, kSiteBwdKV);
        if (ok) ok = wait_q(n0) && wait_do(n0);
        if (!ok) break;
        tc_fence_after();
        mma_tile_ss_kmajor(tmem + 256, sK, sQ_of(n0), 0);   // S^T  = K Q^T
        mma_commit(&s_full[0]);
        mma_commit(&s_full[1]);
        mma_tile_ss_kmajor(tmem + 384, sV, sDO_of(n0), 0);  // dP^T = V dO^T
        mma_commit(dp_full);
        if (steps == 1) mma_commit(kv_empty);               // K and V read for the last time
        for (int n = n0; n < n_end && ok; ++n) {
          const bool more = n + 1 < n_end;
          ok = mbar_wait(&p_full[0], n & 1, kSiteBwdP);
          if (!ok) break;
          tc_fence_after();
          mma_tile_ts_mnmajor<0, 4>(tmem + 0, tmem + 256, sDO_of(n), n > n0);   // dV += P^T dO, queries 0..63
          if (more) {
            ok = wait_q(n + 1);
            if (!ok) break;
            tc_fence_after();
            mma_tile_ss_kmajor_n64(tmem + 256, sK, sQ_of(n + 1), 0);          // S^T of the next step, half 0
            mma_commit(&s_full[0]);
          }
          ok = mbar_wait(&p_full[1], n & 1, kSiteBwdP);
          if (!ok) break;
          tc_fence_after();
          mma_tile_ts_mnmajor<4, 8>(tmem + 0, tmem + 256, sDO_of(n), 1);       // queries 64..127
          mma_commit(&do_empty[n % L::kDOStages]);
          if (more) {
            mma_tile_ss_kmajor_n64(tmem + 320, sK, sQ_of(n + 1), 1);          // half 1
            mma_commit(&s_full[1]);
          }
          ok = mbar_wait(ds_full, n & 1, kSiteBwdP);
          if (!ok) break;
          tc_fence_after();
          mma_tile_ts_mnmajor<0, 8>(tmem + 128, tmem + 384, sQ_of(n), n > n0);  // dK += dS^T Q
          mma_commit(&q_empty[n % L::kQStages]);
          if (more) {
            ok = wait_do(n + 1);
            if (!ok) break;
            tc_fence_after();
            mma_tile_ss_kmajor(tmem + 384, sV, sDO_of(n + 1), 0);         // dP^T of the next step
            mma_commit(dp_full);
            if (n + 2 == n_end) mma_commit(kv_empty);                    // the unit's last S^T and dP^T
          }
        }
        if (!ok) break;
        mma_commit(acc_done);
        n0 = n_end;
        ++ul;
      }
      // Drain (normal and error paths): no MMA may be in flight when tensor
      // memory is freed.
      mma_commit(mma_drain);
      mbar_wait_drain(mma_drain, 0, kSiteBwdDone);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- compute (warps 0-7)
    const int r = (warp & 3) * 32 + lane;            // key row within the tile
    const int hc = warp >> 2;                        // queries 64 c + 32 hc .. +31 in chunk c = 0, 1
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + 256 + hc * 32;   // S^T (then P^T) columns of chunk 0; chunk 1 at +64
    const uint32_t tP = tmem + lane_base + 384 + hc * 32;   // dP^T (then dS^T) columns, same layout
    const float c = a.scale_log2;
    const float2 c2 = make_float2(c, c);
    bool ok = true;
    int ul = 0, n0 = 0;
    for (int k = 0; ok; ++k) {
      const int t = dq_unit_index(k, cta, n_cta);
      if (t >= n_units) break;
      const DkdvUnit u = dkdv_unit(a, t);
      const int kj = u.j * kTile + r;
      // key kj is visible to query qi iff kj <= qi + (Sk - Sq)
      const int lim = kj - (a.Sk - a.Sq);            // masked iff qi < lim
      const bool key_in = kj < a.Sk;
      for (int s = 0; s < u.steps && ok; ++s) {
        const int n = n0 + s;
        const int i = u.i0 + s % u.nqi;
        const int ss = n % L::kStatStages;
        // dS^T tile (query head of this step, key tile j, query tile i), in elements
        const size_t ds_tile =
            a.ds_buf ? ((((size_t)(u.bkv / a.Hkv) * a.Hq + (u.bkv % a.Hkv) * G + s / u.nqi) * n_kt + u.j) * nq_t + i) *
                           (size_t)(kTile * kTile)
                     : 0;
        ok = warp_wait(&st_full[ss], (n / L::kStatStages) & 1, kSiteBwdStFull);
        if (!ok) break;
        // LSE (log2 domain) then Delta of the tile's 128 queries
        const float4* stats4 = reinterpret_cast<const float4*>(smem + L::kStats + ss * 2 * kTile * 4) + hc * 8;
        // P^T as bf16 pairs, per chunk: the values dV's MMA consumes, reused for dS^T
        uint32_t pk[2][16];
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          ok = warp_wait(&s_full[ch], n & 1, kSiteBwdS);
          if (!ok) break;
          tc_fence_after();
          const int q_first = i * kTile + ch * 64 + hc * 32;   // first query of these 32 columns
          const bool need_mask = a.causal && (q_first < lim);
          uint32_t uu[32];
          tmem_ld32(tS + ch * 64, uu);
          tmem_wait_ld();
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) {
            const int e = 4 * k4;
            const float4 l4 = lds128(&stats4[ch * 16 + k4]);   // queries e .. e+3 of the chunk (broadcast)
            const float2 x0 = __ffma2_rn(make_float2(__uint_as_float(uu[e]), __uint_as_float(uu[e + 1])), c2,
                                         make_float2(-l4.x, -l4.y));
            const float2 x1 = __ffma2_rn(make_float2(__uint_as_float(uu[e + 2]), __uint_as_float(uu[e + 3])), c2,
                                         make_float2(-l4.z, -l4.w));
            float p0 = ex2_approx(x0.x), p1 = ex2_approx(x0.y), p2 = ex2_approx(x1.x), p3 = ex2_approx(x1.y);
            if (need_mask) {
              const int q0 = q_first + e;
              p0 = q0 < lim ? 0.f : p0;
              p1 = q0 + 1 < lim ? 0.f : p1;
              p2 = q0 + 2 < lim ? 0.f : p2;
              p3 = q0 + 3 < lim ? 0.f : p3;
            }
            pk[ch][e / 2] = pack_bf16x2(p0, p1);
            pk[ch][e / 2 + 1] = pack_bf16x2(p2, p3);
          }
          __syncwarp();
          tmem_st16(tS + ch * 64, pk[ch]);             // P^T over the first 16 of these columns
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[ch]);
        }
        if (!ok) break;
        ok = warp_wait(dp_full, n & 1, kSiteBwdDP);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t uu[32];
          tmem_ld32(tP + ch * 64, uu);
          tmem_wait_ld();
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) {
            const int e = 4 * k4;
            const float4 d4 = lds128(&stats4[kTile / 4 + ch * 16 + k4]);   // Delta of queries e .. e+3
            const uint32_t w0 = pk[ch][e / 2], w1 = pk[ch][e / 2 + 1];
            const float2 pa = make_float2(__uint_as_float(w0 << 16), __uint_as_float(w0 & 0xFFFF0000u));
            const float2 pb = make_float2(__uint_as_float(w1 << 16), __uint_as_float(w1 & 0xFFFF0000u));
            const float2 a0 = __fmul2_rn(pa, __fadd2_rn(make_float2(__uint_as_float(uu[e]), __uint_as_float(uu[e + 1])),
                                                        make_float2(-d4.x, -d4.y)));
            const float2 a1 = __fmul2_rn(pb, __fadd2_rn(make_float2(__uint_as_float(uu[e + 2]), __uint_as_float(uu[e + 3])),
                                                        make_float2(-d4.z, -d4.w)));
            pk[ch][e / 2] = pack_bf16x2(a0.x, a0.y);
            pk[ch][e / 2 + 1] = pack_bf16x2(a1.x, a1.y);
          }
          if (a.ds_buf) {
            // this row's 32 queries of the chunk into the step's dS^T tile,
            // 8 queries (16 bytes) per store, the warp's 32 rows contiguous;
            // rows past Sk hold zeros (the dQ product multiplies them by the
            // zero-filled K rows, and their P may not be finite)
            uint16_t* base = a.ds_buf + ds_tile + ds_tile_offset(r, ch * 64 + hc * 32);
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8)
              *reinterpret_cast<uint4*>(base + 256 * q8) =
                  key_in ? make_uint4(pk[ch][4 * q8], pk[ch][4 * q8 + 1], pk[ch][4 * q8 + 2], pk[ch][4 * q8 + 3])
                         : make_uint4(0u, 0u, 0u, 0u);
          }
          __syncwarp();
          tmem_st16(tP + ch * 64, pk[ch]);             // dS^T over the first 16 of these columns
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(ds_full);
          mbar_arrive(&st_empty[ss]);                  // done with this step's LSE / Delta
        }
      }
      if (ok) ok = warp_wait(acc_done, ul & 1, kSiteBwdDone);
      if (!ok) break;
      tc_fence_after();
      // this warp stores head dims 64 hc .. 64 hc + 63 of its rows of dV and dK
      const bool store = kj < a.Sk;
      const size_t off = ((size_t)u.bkv * a.Sk + (store ? kj : 0)) * kHeadDim + hc * 64;
      store_half_row_bf16(tmem + lane_base + 0 + hc * 64, 1.f, a.dv + off, store);
      store_half_row_bf16(tmem + lane_base + 128 + hc * 64, a.scale, a.dk + off, store);
      n0 += u.steps;
      ++ul;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// ---------------------------------------------------------------------------- dQ
struct DqSmem {
  // K is read by S_j and again by dQ_j two steps of MMAs later, so it gets a
  // third stage: K_{j+2} can load while dQ_j still reads K_j.
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kQ = 0;
  static constexpr int kDO = kQ + kTileBytesBf16;
  static constexpr int kK = kDO + kTileBytesBf16;
  static constexpr int kV = kK + kKStages * kTileBytesBf16;
  static constexpr int kBars = kV + kVStages * kTileBytesBf16;
  static constexpr int kBytes = kBars + 24 * 8;   // 22 barriers, the TMEM slot, the 2-entry unit ring
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory per CTA");
};

// One unit of dQ work: query tile i of head bh (KV head bkv), n_kv KV tiles.
struct DqUnit {
  int i, bh, bkv, n_kv;
};

// Unit t of the work list, heaviest first: query-tile rank t / (B*Hq), counted
// from the last tile under a causal mask (the last tiles see the most keys).
__device__ __forceinline__ DqUnit dq_unit(const BwdArgs& a, int t) {
  const int BH = a.B * a.Hq;
  const int nq = (a.Sq + kTile - 1) / kTile;
  const int rank = t / BH;
  DqUnit u;
  u.bh = t - rank * BH;
  u.i = a.causal ? nq - 1 - rank : rank;
  const int b = u.bh / a.Hq, h = u.bh - b * a.Hq;
  u.bkv = b * a.Hkv + h / (a.Hq / a.Hkv);
  if (!a.causal) {
    u.n_kv = (a.Sk + kTile - 1) / kTile;
  } else {
    const int last_row = min(u.i * kTile + kTile - 1, a.Sq - 1);
    u.n_kv = min(last_row + (a.Sk - a.Sq), a.Sk - 1) / kTile + 1;
  }
  return u;
}

// Persistent: one CTA per SM walks units taken from a global counter in list
// order (heaviest first); the producer warp takes them, one ahead, and hands
// each to the MMA thread and the compute warps through a two-entry ring in
// shared memory.  Every unit's dQ rows are summed over its KV tiles in
// ascending order by one CTA; only which CTA does a unit depends on timing.
// Across units the K/V ring, the S buffers and every barrier phase continue
// with a global step count, so the next unit's Q/dO load (once the last S and
// dP of a unit have read them) and its first S and dP overlap the end of the
// current unit and its dQ epilogue.  Before exiting, the CTA waits for the
// grid it was launched after (dK/dV) to complete, so the completion of this
// grid implies that of the whole backward.
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dq_kernel(const __grid_constant__ BwdArgs a) {
  using L = DqSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = warp_id(), lane = lane_id();
  const int n_units = ((a.Sq + kTile - 1) / kTile) * a.B * a.Hq;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [3]
  uint64_t* k_empty = bars + 4;   // [3]
  uint64_t* v_full = bars + 7;    // [2]
  uint64_t* v_empty = bars + 9;   // [2]
  uint64_t* s_full = bars + 11;   // [2 S buffers]
  uint64_t* dp_full = bars + 13;
  uint64_t* ds_full = bars + 14;
  uint64_t* dq_done = bars + 15;  // a unit's dQ MMAs have completed
  uint64_t* q_empty = bars + 16;  // a unit's last S and dP have read Q and dO
  uint64_t* mma_drain = bars + 17;
  uint64_t* unit_full = bars + 18;   // [2] ring entry written by the producer
  uint64_t* unit_empty = bars + 20;  // [2] read by the MMA thread and the 8 compute warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 22);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(bars + 23);   // [2]

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < L::kKStages; ++s) { mbar_init(&k_full[s], 1); mbar_init(&k_empty[s], 1); }
    for (int s = 0; s < L::kVStages; ++s) { mbar_init(&v_full[s], 1); mbar_init(&v_empty[s], 1); }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, kBwdComputeWarps);  // one arrival per compute warp
    mbar_init(dq_done, 1);
    mbar_init(q_empty, 1);
    mbar_init(mma_drain, 1);
    for (int s = 0; s < 2; ++s) { mbar_init(&unit_full[s], 1); mbar_init(&unit_empty[s], 1 + kBwdComputeWarps); }
    fence_barrier_init();
  }
  if (warp == 9) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S / dS buffer 0 [0,128), dP [128,256), dQ [256,384), S / dS buffer 1 [384,512)
  auto s_col = [](int g) { return (g & 1) ? 384u : 0u; };
  // The k-th unit of this CTA, read from the ring (MMA thread, compute warps):
  // n_units once the list is exhausted.  The entry is released after reading.
  auto take_unit = [&](int k, bool whole_warp, int& t) -> bool {
    const int slot = k & 1;
    const bool ok = whole_warp ? warp_wait(&unit_full[slot], (k >> 1) & 1, kSiteBwdKV)
                               : mbar_wait(&unit_full[slot], (k >> 1) & 1, kSiteBwdKV);
    if (!ok) return false;
    t = unit_ring[slot];
    if (whole_warp) __syncwarp();
    if (!whole_warp || lane == 0) mbar_arrive(&unit_empty[slot]);
    return true;
  };

  if (warp == 8) {
    if (lane == 0) {
      bool ok = true;
      int ul = 0, gk = 0, gv = 0;   // units started, K and V tiles requested
      for (int k = 0; ok; ++k) {
        const int slot = k & 1;
        if (k >= 2) ok = mbar_wait(&unit_empty[slot], ((k >> 1) - 1) & 1, kSiteBwdStEmpty);
        if (!ok) break;
        const uint32_t tu = atomicAdd(a.dq_sched, 1u);     // list order: heaviest first
        const int t = tu < (uint32_t)n_units ? (int)tu : n_units;
        unit_ring[slot] = t;
        mbar_arrive(&unit_full[slot]);                      // releases the ring entry
        if (t >= n_units) break;
        const DqUnit u = dq_unit(a, t);
        if (ul > 0) {   // its Q and dO into L2 while the previous unit still holds their buffers
          for (int x = 0; x < 2; ++x) {
            tma_prefetch_3d(&a.tm_q, x * 64, u.i * kTile, u.bh);
            tma_prefetch_3d(&a.tm_do, x * 64, u.i * kTile, u.bh);
          }
        }
        // K_0 and V_0 go first: their ring stages free up while the previous
        // unit still runs, before its last S and dP release Q and dO
        for (int jj = 0; jj < u.n_kv && ok; ++jj) {
          if (jj == 1 || u.n_kv == 1) {
            if (ul > 0) ok = mbar_wait(q_empty, (ul - 1) & 1, kSiteBwdStEmpty);
            if (!ok) break;
            mbar_arrive_expect_tx(q_full, 2 * kTileBytesBf16);
            tma_tile_bf16(smem + L::kQ, &a.tm_q, q_full, u.i * kTile, u.bh);
            tma_tile_bf16(smem + L::kDO, &a.tm_do, q_full, u.i * kTile, u.bh);
            ++ul;
          }
          const int ks = gk % L::kKStages, ku = gk / L::kKStages;
          if (gk >= L::kKStages) ok = mbar_wait(&k_empty[ks], (ku - 1) & 1, kSiteBwdStEmpty);
          if (!ok) break;
          mbar_arrive_expect_tx(&k_full[ks], kTileBytesBf16);
          tma_tile_bf16(smem + L::kK + ks * kTileBytesBf16, &a.tm_k, &k_full[ks], jj * kTile, u.bkv);
          ++gk;
          const int vs = gv % L::kVStages, vu = gv / L::kVStages;
          if (gv >= L::kVStages) ok = mbar_wait(&v_empty[vs], (vu - 1) & 1, kSiteBwdStEmpty);
          if (!ok) break;
          mbar_arrive_expect_tx(&v_full[vs], kTileBytesBf16);
          tma_tile_bf16(smem + L::kV + vs * kTileBytesBf16, &a.tm_v, &v_full[vs], jj * kTile, u.bkv);
          ++gv;
        }
      }
      // drain: every load issued must land before the CTA exits
      if (ul > 0) mbar_wait_drain(q_full, (ul - 1) & 1, kSiteBwdKV);
      for (int g = max(0, gk - L::kKStages); g < gk; ++g)
        mbar_wait_drain(&k_full[g % L::kKStages], (g / L::kKStages) & 1, kSiteBwdStFull);
      for (int g = max(0, gv - L::kVStages); g < gv; ++g)
        mbar_wait_drain(&v_full[g % L::kVStages], (g / L::kVStages) & 1, kSiteBwdStFull);
    }
    __syncwarp();
  } else if (warp == 9) {
    if (lane == 0) {
      const uint32_t sQ = smem_u32(smem + L::kQ), sDO = smem_u32(smem + L::kDO);
      auto sK_of = [&](int g) { return smem_u32(smem + L::kK + (g % L::kKStages) * kTileBytesBf16); };
      auto sV_of = [&](int g) { return smem_u32(smem + L::kV + (g % L::kVStages) * kTileBytesBf16); };
      // S is double-buffered in TMEM: S_{j+1} is computed while the compute
      // warps work on step j.  Issue order per unit: S_0, dP_0, S_1, then per
      // step j: dQ_j (once dS_j is written), dP_{j+1} (the compute warps have
      // read dP_j), S_{j+2} into the buffer dQ_j has just read dS_j from.  g
      // counts steps over all of this CTA's units.
      auto issue_s = [&](int g) -> bool {
        if (!mbar_wait(&k_full[g % L::kKStages], (g / L::kKStages) & 1, kSiteBwdStFull)) return false;
        tc_fence_after();
        mma_tile_ss_kmajor(tmem + s_col(g), sQ, sK_of(g), 0);           // S  = Q K^T
        mma_commit(&s_full[g & 1]);
        return true;
      };
      auto issue_dp = [&](int g) -> bool {
        if (!mbar_wait(&v_full[g % L::kVStages], (g / L::kVStages) & 1, kSiteBwdStFull)) return false;
        tc_fence_after();
        mma_tile_ss_kmajor(tmem + 128, sDO, sV_of(g), 0);               // dP = dO V^T
        mma_commit(dp_full);
        mma_commit(&v_empty[g % L::kVStages]);
        return true;
      };
      bool ok = true;
      int ul = 0, g0 = 0;
      for (int k = 0; ok; ++k) {
        int t = n_units;
        ok = take_unit(k, false, t);
        if (!ok || t >= n_units) break;
        const int n = dq_unit(a, t).n_kv;
        ok = mbar_wait(q_full, ul & 1, kSiteBwdKV);
        if (ok) ok = issue_s(g0) && issue_dp(g0);
        if (ok && n == 1) mma_commit(q_empty);                           // Q and dO read for the last time
        if (ok && n > 1) ok = issue_s(g0 + 1);
        for (int jj = 0; jj < n && ok; ++jj) {
          const int g = g0 + jj;
          ok = mbar_wait(ds_full, g & 1, kSiteBwdP);
          if (!ok) break;
          tc_fence_after();
          mma_tile_ts_mnmajor_halves(tmem + 256, tmem + s_col(g), sK_of(g), jj > 0);   // dQ += dS K
          mma_commit(&k_empty[g % L::kKStages]);
          if (jj + 1 < n) {
            ok = issue_dp(g + 1);
            if (ok && jj + 1 == n - 1) mma_commit(q_empty);
          }
          if (ok && jj + 2 < n) ok = issue_s(g + 2);
        }
        if (!ok) break;
        mma_commit(dq_done);
        g0 += n;
        ++ul;
      }
      mma_commit(mma_drain);
      mbar_wait_drain(mma_drain, 0, kSiteBwdDone);
    }
    __syncwarp();
  } else {
    const int r = (warp & 3) * 32 + lane;            // query row within the tile
    const int hc = warp >> 2;                        // column half: keys 64 hc .. 64 hc + 63
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float c = a.scale_log2;
    // This thread's row of unit t, and the loads of its LSE and Delta (issued
    // for the next unit before the current unit's dQ epilogue, which hides
    // their latency).
    auto row_of = [&](int t, bool& valid) -> size_t {
      const DqUnit u = dq_unit(a, t);
      const int qi = u.i * kTile + r;
      valid = qi < a.Sq;
      return (size_t)u.bh * a.Sq + (valid ? qi : 0);
    };
    auto load_stats = [&](int t, float& lse_raw, float& dlt) {
      lse_raw = 0.f;
      dlt = 0.f;
      if (t >= n_units) return;
      bool valid;
      const size_t ridx = row_of(t, valid);
      if (valid) {
        lse_raw = __ldg(&a.lse[ridx]);
        dlt = __ldg(&a.delta[ridx]);
      }
    };
    int ul = 0, g0 = 0;
    int t = n_units;
    bool ok = take_unit(0, true, t);
    float lse_raw, dlt;
    load_stats(t, lse_raw, dlt);
    for (int k = 0; ok && t < n_units; ++k) {
      const DqUnit u = dq_unit(a, t);
      const int qi = u.i * kTile + r;
      bool valid;
      const size_t ridx = row_of(t, valid);
      const float lse2 = valid ? lse_raw * 1.4426950408889634f : INFINITY;
      const int kv_limit = a.causal ? min(a.Sk - 1, qi + (a.Sk - a.Sq)) : a.Sk - 1;
      for (int jj = 0; jj < u.n_kv && ok; ++jj) {
        const int g = g0 + jj;
        ok = warp_wait(&s_full[g & 1], (g >> 1) & 1, kSiteBwdS);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tmem + lane_base + s_col(g) + hc * 64;   // this warp's 64 S (then dS) columns
        float p[64];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t uu[32];
          tmem_ld32(tS + q * 32, uu);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) p[q * 32 + e] = __uint_as_float(uu[e]);
        }
        const int kbase = jj * kTile + hc * 64;
        const bool need_mask = kbase + 63 > kv_limit;
        const float2 c2 = make_float2(c, c), nl2 = make_float2(-lse2, -lse2);
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const float2 t = __ffma2_rn(make_float2(p[e], p[e + 1]), c2, nl2);
          float x0 = ex2_approx(t.x), x1 = ex2_approx(t.y);
          if (need_mask) {
            x0 = kbase + e > kv_limit ? 0.f : x0;
            x1 = kbase + e + 1 > kv_limit ? 0.f : x1;
          }
          p[e] = x0;
          p[e + 1] = x1;
        }
        __syncwarp();
        ok = warp_wait(dp_full, g & 1, kSiteBwdDP);
        if (!ok) break;
        tc_fence_after();
        {
          uint32_t uu[64];
          tmem_ld32(tmem + lane_base + 128 + hc * 64, *reinterpret_cast<uint32_t(*)[32]>(&uu[0]));
          tmem_ld32(tmem + lane_base + 128 + hc * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&uu[32]));
          tmem_wait_ld();
          const float2 nd2 = make_float2(-dlt, -dlt);
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            const float2 d = __fadd2_rn(make_float2(__uint_as_float(uu[e]), __uint_as_float(uu[e + 1])), nd2);
            const float2 r = __fmul2_rn(make_float2(p[e], p[e + 1]), d);
            p[e] = r.x;
            p[e + 1] = r.y;
          }
        }
        {
          uint32_t w[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) w[e] = pack_bf16x2(p[2 * e], p[2 * e + 1]);
          tmem_st32(tS, w);                          // dS over the first 32 of these columns
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
      }
      if (!ok) break;
      // the next unit and its statistics first, then this unit's epilogue
      int tn = n_units;
      ok = take_unit(k + 1, true, tn);
      float lse_next = 0.f, dlt_next = 0.f;
      if (ok) load_stats(tn, lse_next, dlt_next);
      if (ok) ok = warp_wait(dq_done, ul & 1, kSiteBwdDone);
      if (!ok) break;
      tc_fence_after();
      // The next unit's first dQ MMA overwrites these columns only after this
      // warp's first dS of that unit, i.e. after these loads have completed.
      store_half_row_bf16(tmem + lane_base + 256 + hc * 64, a.scale, a.dq + ridx * kHeadDim + hc * 64, valid);
      g0 += u.n_kv;
      ++ul;
      t = tn;
      lse_raw = lse_next;
      dlt = dlt_next;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) { tc_fence_after(); tmem_dealloc(tmem, 512); }
  if (threadIdx.x == 0) griddep_wait();
}

// ---------------------------------------------------------------------------- host launch
bool encode_rows(CUtensorMap* m, const void* base, bool e4m3, uint64_t rows, uint64_t heads);

inline int launch_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                      const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk,
                      float scale, bool causal, float* delta, uint32_t* dq_sched, int n_sm, cudaStream_t st) {
  // the shared-memory limits, once per device
  static PerDeviceOnce setup;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -5;
  if (!setup.ensure(dev, [] {
        return cudaFuncSetAttribute(bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    DkdvSmem::kAlloc) == cudaSuccess &&
               cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DqSmem::kAlloc) ==
                   cudaSuccess;
      }))
    return -5;
  static thread_local BwdArgs a;
  memset(&a, 0, sizeof(a));
  if (!encode_rows(&a.tm_q, q, false, Sq, (uint64_t)B * Hq)) return -5;
  if (!encode_rows(&a.tm_do, dout, false, Sq, (uint64_t)B * Hq)) return -5;
  if (!encode_rows(&a.tm_k, k, false, Sk, (uint64_t)B * Hkv)) return -5;
  if (!encode_rows(&a.tm_v, v, false, Sk, (uint64_t)B * Hkv)) return -5;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Sq = Sq; a.Sk = Sk;
  a.causal = causal ? 1 : 0;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.lse = lse;
  a.delta = delta;
  a.dq = reinterpret_cast<uint16_t*>(dq);
  a.dk = reinterpret_cast<uint16_t*>(dk);
  a.dv = reinterpret_cast<uint16_t*>(dv);
  a.dq_sched = dq_sched;
  const long long rows = (long long)B * Hq * Sq;
  const long long n_kt = (Sk + kTile - 1) / kTile, nq = (Sq + kTile - 1) / kTile;
  const long long kv_units = n_kt * B * Hkv, dq_units = nq * B * Hq;
  const int kv_grid = (int)std::min<long long>(kv_units, n_sm);
  const int dq_grid = (int)std::min<long long>(dq_units, n_sm);
  // each persistent CTA counts its steps (tile pairs) in an int
  if ((kv_units + kv_grid - 1) / kv_grid * (Hq / Hkv) * nq >= (1LL << 31) ||
      (dq_units + dq_grid - 1) / dq_grid * n_kt >= (1LL << 31))
    return -2;
  // Each grid is a programmatic dependent of the one before (see the kernels):
  // Delta after the forward, dK/dV after Delta, dQ after dK/dV.
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3((unsigned)((rows + kDeltaRowsPerCta - 1) / kDeltaRowsPerCta));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  if (cudaLaunchKernelEx(&cfg, bwd_delta_kernel, reinterpret_cast<const uint16_t*>(out),
                         reinterpret_cast<const uint16_t*>(dout), delta, rows, dq_sched) != cudaSuccess)
    return -5;
  cfg.gridDim = dim3((unsigned)kv_grid);
  cfg.blockDim = dim3(kBwdThreads);
  cfg.dynamicSmemBytes = DkdvSmem::kAlloc;
  if (cudaLaunchKernelEx(&cfg, bwd_dkdv_kernel, a) != cudaSuccess) return -5;
  cfg.gridDim = dim3((unsigned)dq_grid);
  cfg.dynamicSmemBytes = DqSmem::kAlloc;
  if (cudaLaunchKernelEx(&cfg, bwd_dq_kernel, a) != cudaSuccess) return -5;
  return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

}  // namespace hattn
