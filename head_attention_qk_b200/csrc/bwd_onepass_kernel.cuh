// bwd_onepass_kernel.cuh -- one-pass deterministic attention backward for
// sm_100a (bf16): dK, dV and dQ from one kernel, 5 GEMMs per tile pair.
//
// For dO = dL/dO, P = exp(scale * Q K^T - LSE) (LSE from the forward):
//   dV = P^T dO,   dP = dO V^T,   Delta_i = sum_d dO_id O_id,
//   dS = P * (dP - Delta),   dQ = scale * dS K,   dK = scale * dS^T Q.
// RL-Kernel PR #319 ("feat(attention): add strict bitwise ROCm path", What the
// strict contract costs) measures a deterministic mha_bwd that holds an
// O(S^2) workspace.  Here the two-kernel backward of bwd_kernel.cuh recomputes
// S and dP in a separate dQ kernel (7 GEMMs per tile pair); this kernel forms
// the dQ contribution of each tile pair where dS is made and adds it into an
// fp32 accumulator in a fixed order, so dQ costs one GEMM and an ordered add:
//
//   one CTA per SM walks (key tile j, batch x KV head) units, heaviest first
//   in snake order (as the dK/dV kernel); a unit's steps visit the query tiles
//   i seen by key tile j in descending order and, inside each, the group's
//   query heads g in ascending order.  Per step, five tcgen05 MMAs:
//     S^T = K Q^T, dP^T = V dO^T, dV += P^T dO, dK += dS^T Q, dQ_ij = dS K,
//   the last two reading dS^T from shared memory (dK as a K-major A operand,
//   dQ as an MN-major one, the transposed view of the same bytes).
//
// Tensor memory (512 columns): dV [0,128), dK [128,256), S^T / P^T [256,384),
// dP^T [384,512); the step's dQ tile (queries in the lanes) takes dP^T's
// columns once the compute warps have read dP^T, and the next dP^T waits
// until they have read the dQ tile out.
//
// Ordered dQ: an fp32 accumulator per (b, query head, query tile) in the
// workspace and a counter next to it.  The key tiles that see query tile i are
// j = 0 .. jlast(i) (causal masks are bottom-right aligned, so key tile 0 sees
// every query), and tile j adds its part only after tiles 0 .. j-1 have.  Four
// writer warps take the dQ tile out of tensor memory (so the next step's MMAs
// can use the columns at once) and then each waits until the counter has
// reached 4 j (four writer warps per contributor), stores (j = 0), adds in
// memory (red.add) or, as the last contributor, adds, scales and writes the
// bf16 dQ rows, then releases one count.  Every dQ element is therefore summed over j in ascending order,
// whichever thread block adds which part: the result is bitwise the same
// from run to run and for any batch composition or head split.  Because all
// key tiles of a head visit their common (i, g) steps at the same step index,
// a tile lags its predecessor by about one step.  Progress: every wait is on a
// unit with a smaller index, each CTA takes its units in increasing index,
// and all CTAs are resident (cooperative launch, one CTA per SM), so the
// unfinished unit with the smallest index can always proceed; waits are
// bounded all the same and report through the device error word.
//
// Cost on B200 (interleaved A/B, same inputs): slower than the two-kernel
// backward, e.g. 0.372 vs 0.261 ms on B2 Hq32 Hkv8 S2048 causal.  Every tile
// pair moves a 64 KB fp32 dQ tile through L2 atomics (570 MB on that config;
// an L2 reduction of 64 KB from every SM at once takes about 1.6 us, as much as
// a step of the dQ kernel it replaces), and without any ordering at all (a
// memset, unordered red.add, a conversion pass) it still takes 0.319 ms.
#pragma once

#include "bwd_kernel.cuh"

namespace hattn {

enum : int { kSiteOpDqFull = 40, kSiteOpDqFree, kSiteOpOrder };

// 512 threads: warps 0-7 compute (P^T, dS^T, the dK / dV epilogue), warp 8 TMA
// producer, warp 9 MMA issuer, warps 10-11 no role, warps 12-15 dQ writers
// (warp 12 + q reads the dQ tile's TMEM lane quarter q, all 128 columns, into
// registers, releases the columns, then adds the rows in key-tile order).
// setmaxnreg split over the four warpgroups: compute 128 (as launched),
// producer / MMA 80, writers 176; they sum to the 128 x 512 registers the
// launch holds (checked on the host: an increase the pool cannot satisfy
// would wait forever).
constexpr int kOnePassThreads = 512;
constexpr int kOpRegsCompute = 128, kOpRegsOther = 80, kOpRegsWriter = 176;
constexpr int kOpRegsNeeded = (2 * kOpRegsCompute + kOpRegsOther + kOpRegsWriter) * 128;
static_assert(kOpRegsNeeded <= 65536, "setmaxnreg split exceeds the register file");
constexpr int kDqWriters = 4;

struct OnePassSmem {
  static constexpr int kQStages = 2;
  static constexpr int kDOStages = 2;
  static constexpr int kStatStages = 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTileBytesBf16;
  static constexpr int kQ = kV + kTileBytesBf16;
  static constexpr int kDO = kQ + kQStages * kTileBytesBf16;
  static constexpr int kDS = kDO + kDOStages * kTileBytesBf16;   // dS^T bf16: [key row][query], two 64-query atoms
  static constexpr int kStats = kDS + kTileBytesBf16;            // [stage] x (128 lse2 + 128 delta) fp32
  static constexpr int kBars = kStats + kStatStages * 2 * kTile * 4;
  static constexpr int kBytes = kBars + 28 * 8;
  // No alignment slack, as for the dK/dV kernel: the window is checked to be
  // 1024-byte aligned at run time.
  static constexpr int kAlloc = kBytes;
  static_assert(kAlloc <= 232448, "shared memory per CTA");
};

// Last key tile that query tile i sees.
__device__ __forceinline__ int onepass_last_key_tile(const BwdArgs& a, int i) {
  if (!a.causal) return (a.Sk + kTile - 1) / kTile - 1;
  const int last_row = min(i * kTile + kTile - 1, a.Sq - 1);
  return min(last_row + (a.Sk - a.Sq), a.Sk - 1) / kTile;
}

// dK += dS^T Q: A = dS^T K-major in shared memory (two 64-query atoms), B = Q
// read MN-major (the reduction runs over the tile's rows).
__device__ __forceinline__ void mma_tile_ss_kA_mnB(uint32_t d, uint32_t sa, uint32_t sb, uint32_t acc) {
  constexpr uint32_t idesc = make_idesc(1, 1, 1, 128, 128);
  constexpr uint32_t hi = sdesc_hi(1024);
  const uint32_t a_lo = sdesc_lo(sa, 16), b_lo = sdesc_lo(sb, 16384);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t a_off = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
    mma_f16_ss2(d, a_lo + a_off, hi, b_lo + k * (2048 >> 4), hi, idesc, (acc || k > 0) ? 1u : 0u);
  }
}

// dQ_ij = dS K: A = dS, held as dS^T in shared memory, i.e. MN-major (queries
// contiguous, two 64-query blocks 16 KB apart); B = K read MN-major.
__device__ __forceinline__ void mma_tile_ss_mnA_mnB(uint32_t d, uint32_t sa, uint32_t sb) {
  constexpr uint32_t idesc = make_idesc_ab(1, 1, 1, 1, 128, 128);
  constexpr uint32_t hi = sdesc_hi(1024);
  const uint32_t a_lo = sdesc_lo(sa, 16384), b_lo = sdesc_lo(sb, 16384);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    mma_f16_ss2(d, a_lo + k * (2048 >> 4), hi, b_lo + k * (2048 >> 4), hi, idesc, k > 0 ? 1u : 0u);
}

__global__ void __launch_bounds__(kOnePassThreads, 1) bwd_onepass_kernel(const __grid_constant__ BwdArgs a) {
  using L = OnePassSmem;
  extern __shared__ uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {              // the layout needs a 1024-byte aligned window
    if (threadIdx.x == 0) raise_error(0x100 | kSiteBwdAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  const int warp = warp_id(), lane = lane_id();
  const int n_kt = (a.Sk + kTile - 1) / kTile;
  const int nq = (a.Sq + kTile - 1) / kTile;
  const int n_units = n_kt * a.B * a.Hkv;
  const int cta = blockIdx.x, n_cta = gridDim.x;
  const int G = a.Hq / a.Hkv;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;     // a unit's last MMA reading K and V has completed
  uint64_t* q_full = bars + 2;       // [2]
  uint64_t* q_empty = bars + 4;      // [2]
  uint64_t* do_full = bars + 6;      // [2]
  uint64_t* do_empty = bars + 8;     // [2]
  uint64_t* s_full = bars + 10;      // [2] S^T columns of query half 0 / 1
  uint64_t* dp_full = bars + 12;
  uint64_t* p_full = bars + 13;      // [2] P^T of query half 0 / 1 written
  uint64_t* acc_done = bars + 15;    // a unit's dK / dV MMAs have completed
  uint64_t* ds_full = bars + 16;     // dS^T written to shared memory
  uint64_t* st_full = bars + 17;     // [2] LSE / Delta of a step staged (32 producer lanes)
  uint64_t* st_empty = bars + 19;    // [2] the compute warps are done with them
  uint64_t* dq_full = bars + 21;     // the step's dQ tile is in tensor memory
  uint64_t* dq_free = bars + 22;     // the writers have read it out (one arrival per writer warp)
  uint64_t* mma_drain = bars + 23;
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
      mbar_init(&p_full[h], kBwdComputeWarps);
    }
    mbar_init(dp_full, 1);
    mbar_init(ds_full, kBwdComputeWarps);
    mbar_init(acc_done, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, kDqWriters);
    fence_barrier_init();
  }
  if (warp == 9) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8 && warp < 12) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kOpRegsOther) : "memory");
  if (warp == 8) {
    // ---------------------------------------------------------------- producer
    bool ok = true;
    int ul = 0, n0 = 0;
    for (int k = 0; ok; ++k) {
      const int t = dq_unit_index(k, cta, n_cta);
      if (t >= n_units) break;
      const DkdvUnit u = dkdv_unit(a, t);
      const int b = u.bkv / a.Hkv, kvh = u.bkv - b * a.Hkv;
      if (ul > 0) ok = warp_wait(kv_empty, (ul - 1) & 1, kSiteBwdKV);
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(kv_full, 2 * kTileBytesBf16);
        tma_tile_bf16(smem + L::kK, &a.tm_k, kv_full, u.j * kTile, u.bkv);
        tma_tile_bf16(smem + L::kV, &a.tm_v, kv_full, u.j * kTile, u.bkv);
      }
      for (int s = 0; s < u.steps && ok; ++s) {
        const int n = n0 + s;
        const int i = nq - 1 - s / G, g = s % G;      // query tiles descending, heads ascending
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
      const uint32_t sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV), sDS = smem_u32(smem + L::kDS);
      auto sQ_of = [&](int n) { return smem_u32(smem + L::kQ + (n % L::kQStages) * kTileBytesBf16); };
      auto sDO_of = [&](int n) { return smem_u32(smem + L::kDO + (n % L::kDOStages) * kTileBytesBf16); };
      auto wait_q = [&](int n) { return mbar_wait(&q_full[n % L::kQStages], (n / L::kQStages) & 1, kSiteBwdStFull); };
      auto wait_do = [&](int n) {
        return mbar_wait(&do_full[n % L::kDOStages], (n / L::kDOStages) & 1, kSiteBwdStFull);
      };
      // Per step n: dV_n by query halves (each once its P^T half is written)
      // with S^T_{n+1} of that half after it; then dK_n and dQ_n (once dS^T_n
      // is in shared memory); then dP^T_{n+1}, once the compute warps have
      // read dQ_n out of the columns it takes.
      bool ok = true;
      int ul = 0, n0 = 0;
      for (int k = 0; ok; ++k) {
        const int t = dq_unit_index(k, cta, n_cta);
        if (t >= n_units) break;
        const int steps = dkdv_unit(a, t).steps;
        const int n_end = n0 + steps;
        ok = mbar_wait(kv_full, ul & 1, kSiteBwdKV);
        if (ok) ok = wait_q(n0) && wait_do(n0);
        if (ok && n0 > 0) ok = mbar_wait(dq_free, (n0 - 1) & 1, kSiteOpDqFree);
        if (!ok) break;
        tc_fence_after();
        mma_tile_ss_kmajor(tmem + 256, sK, sQ_of(n0), 0);   // S^T  = K Q^T
        mma_commit(&s_full[0]);
        mma_commit(&s_full[1]);
        mma_tile_ss_kmajor(tmem + 384, sV, sDO_of(n0), 0);  // dP^T = V dO^T
        mma_commit(dp_full);
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
          mma_tile_ss_kA_mnB(tmem + 128, sDS, sQ_of(n), n > n0);              // dK += dS^T Q
          mma_commit(&q_empty[n % L::kQStages]);
          mma_tile_ss_mnA_mnB(tmem + 384, sDS, sK);                            // dQ_n = dS K
          mma_commit(dq_full);
          if (more) {
            ok = wait_do(n + 1) && mbar_wait(dq_free, n & 1, kSiteOpDqFree);
            if (!ok) break;
            tc_fence_after();
            mma_tile_ss_kmajor(tmem + 384, sV, sDO_of(n + 1), 0);         // dP^T of the next step
            mma_commit(dp_full);
          }
        }
        if (!ok) break;
        mma_commit(acc_done);
        mma_commit(kv_empty);                                                 // the unit's last dQ read K
        n0 = n_end;
        ++ul;
      }
      mma_commit(mma_drain);
      mbar_wait_drain(mma_drain, 0, kSiteBwdDone);
    }
    __syncwarp();
  }
  } else if (warp >= 12) {
    // ---------------------------------------------------------------- dQ writers (warps 12-15)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kOpRegsWriter) : "memory");
    const int r = (warp & 3) * 32 + lane;            // query row of the dQ tile (TMEM lane)
    const uint32_t tQ = tmem + ((uint32_t)((warp & 3) * 32) << 16) + 384;
    bool ok = true;
    int n0 = 0;
    for (int k = 0; ok; ++k) {
      const int t = dq_unit_index(k, cta, n_cta);
      if (t >= n_units) break;
      const DkdvUnit u = dkdv_unit(a, t);
      const int b = u.bkv / a.Hkv, kvh = u.bkv - b * a.Hkv;
      for (int s = 0; s < u.steps && ok; ++s) {
        const int n = n0 + s;
        const int i = nq - 1 - s / G, g = s % G;
        ok = warp_wait(dq_full, n & 1, kSiteOpDqFull);
        if (!ok) break;
        tc_fence_after();
        uint32_t dq[128];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tQ + 32 * c4, *reinterpret_cast<uint32_t(*)[32]>(&dq[32 * c4]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_free);          // the MMAs may take these columns again
        const int bh = b * a.Hq + kvh * G + g;
        const int jl = onepass_last_key_tile(a, i);
        uint32_t* cnt = a.dq_cnt + (size_t)bh * nq + i;
        if (u.j > 0) {
          bool w = true;
          if (lane == 0) w = wait_counter_geq(cnt, (uint32_t)kDqWriters * (uint32_t)u.j, kSiteOpOrder);
          ok = __shfl_sync(0xffffffffu, w, 0);
          if (!ok) break;
        }
        const int qi = i * kTile + r;
        if (qi < a.Sq) {
          const size_t row = (size_t)bh * a.Sq + qi;
          float* acc = a.dq_acc + row * kHeadDim;
          if (u.j == jl) {
            // last contributor: dQ = scale * (sum of the earlier tiles + this one), bf16
            uint4* dst = reinterpret_cast<uint4*>(a.dq + row * kHeadDim);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float v[8];
#pragma unroll
              for (int t2 = 0; t2 < 8; ++t2) v[t2] = __uint_as_float(dq[8 * e + t2]);
              if (u.j > 0) {
                const float4 p0 = __ldcg(reinterpret_cast<const float4*>(acc + 8 * e));
                const float4 p1 = __ldcg(reinterpret_cast<const float4*>(acc + 8 * e + 4));
                v[0] = p0.x + v[0]; v[1] = p0.y + v[1]; v[2] = p0.z + v[2]; v[3] = p0.w + v[3];
                v[4] = p1.x + v[4]; v[5] = p1.y + v[5]; v[6] = p1.z + v[6]; v[7] = p1.w + v[7];
              }
              dst[e] = make_uint4(pack_bf16x2(v[0] * a.scale, v[1] * a.scale), pack_bf16x2(v[2] * a.scale, v[3] * a.scale),
                                  pack_bf16x2(v[4] * a.scale, v[5] * a.scale), pack_bf16x2(v[6] * a.scale, v[7] * a.scale));
            }
          } else if (u.j == 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              __stcg(reinterpret_cast<float4*>(acc + 4 * e),
                     make_float4(__uint_as_float(dq[4 * e]), __uint_as_float(dq[4 * e + 1]),
                                 __uint_as_float(dq[4 * e + 2]), __uint_as_float(dq[4 * e + 3])));
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              red_add_v4(acc + 4 * e, make_float4(__uint_as_float(dq[4 * e]), __uint_as_float(dq[4 * e + 1]),
                                                  __uint_as_float(dq[4 * e + 2]), __uint_as_float(dq[4 * e + 3])));
          }
        }
        if (u.j < jl) {
          __syncwarp();
          if (lane == 0) red_release_gpu_add(cnt, 1u);
        }
      }
      n0 += u.steps;
    }
  } else if (warp < 8) {
    // ---------------------------------------------------------------- compute (warps 0-7)
    const int r = (warp & 3) * 32 + lane;            // key row of S^T / P^T / dS^T
    const int hc = warp >> 2;                        // queries 64 c + 32 hc .. +31 in chunk c
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + 256 + hc * 32;   // S^T (then P^T) columns of chunk 0; chunk 1 at +64
    const uint32_t tP = tmem + lane_base + 384 + hc * 32;   // dP^T columns, same layout
    uint8_t* sds_row = smem + L::kDS + r * 128;             // row r of each 64-query atom of dS^T
    const float c = a.scale_log2;
    const float2 c2 = make_float2(c, c);
    bool ok = true;
    int ul = 0, n0 = 0;
    for (int k = 0; ok; ++k) {
      const int t = dq_unit_index(k, cta, n_cta);
      if (t >= n_units) break;
      const DkdvUnit u = dkdv_unit(a, t);
      const int kj = u.j * kTile + r;
      const int lim = kj - (a.Sk - a.Sq);            // key kj is masked for query qi iff qi < lim
      for (int s = 0; s < u.steps && ok; ++s) {
        const int n = n0 + s;
        const int i = nq - 1 - s / G;
        const int ss = n % L::kStatStages;
        ok = warp_wait(&st_full[ss], (n / L::kStatStages) & 1, kSiteBwdStFull);
        if (!ok) break;
        const float4* stats4 = reinterpret_cast<const float4*>(smem + L::kStats + ss * 2 * kTile * 4) + hc * 8;
        uint32_t pk[2][16];
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          ok = warp_wait(&s_full[ch], n & 1, kSiteBwdS);
          if (!ok) break;
          tc_fence_after();
          const int q_first = i * kTile + ch * 64 + hc * 32;
          const bool need_mask = a.causal && (q_first < lim);
          uint32_t uu[32];
          tmem_ld32(tS + ch * 64, uu);
          tmem_wait_ld();
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) {
            const int e = 4 * k4;
            const float4 l4 = lds128(&stats4[ch * 16 + k4]);
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
            const float4 d4 = lds128(&stats4[kTile / 4 + ch * 16 + k4]);
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
          // dS^T row r, queries 64 ch + 32 hc .. +31: 16-byte chunks 4 hc .. 4 hc + 3
          // of atom ch, at chunk position c ^ (r & 7) (128-byte swizzle)
          uint8_t* atom = sds_row + ch * 16384;
#pragma unroll
          for (int m = 0; m < 4; ++m)
            *reinterpret_cast<uint4*>(atom + ((((hc << 2) + m) ^ (r & 7)) << 4)) =
                make_uint4(pk[ch][4 * m], pk[ch][4 * m + 1], pk[ch][4 * m + 2], pk[ch][4 * m + 3]);
        }
        // the MMAs read dS^T through the async proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(ds_full);
          mbar_arrive(&st_empty[ss]);
        }
      }
      if (ok) ok = warp_wait(acc_done, ul & 1, kSiteBwdDone);
      if (!ok) break;
      tc_fence_after();
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

// Bytes of workspace of the one-pass backward: Delta (fp32 per row), the dQ
// accumulator (fp32 per row and head dim) and one counter per query tile,
// each part 256-byte aligned.
inline size_t onepass_workspace_parts(long long B, long long Hq, long long Sq, size_t* off_acc, size_t* off_cnt) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t rows = (size_t)(B * Hq * Sq);
  const size_t nq = (size_t)((Sq + kTile - 1) / kTile);
  *off_acc = up(rows * sizeof(float));
  *off_cnt = *off_acc + up(rows * kHeadDim * sizeof(float));
  return *off_cnt + up((size_t)(B * Hq) * nq * sizeof(uint32_t));
}

inline int launch_bwd_onepass(const void* q, const void* k, const void* v, const void* out, const float* lse,
                              const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk,
                              float scale, bool causal, void* workspace, int n_sm, cudaStream_t st) {
  static PerDeviceOnce setup;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -5;
  if (!setup.ensure(dev, [dev] {
        int coop = 0;
        cudaFuncAttributes fa;
        return cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) == cudaSuccess && coop &&
               cudaFuncSetAttribute(bwd_onepass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    OnePassSmem::kAlloc) == cudaSuccess &&
               cudaFuncGetAttributes(&fa, bwd_onepass_kernel) == cudaSuccess &&
               fa.numRegs * kOnePassThreads >= kOpRegsNeeded;   // the setmaxnreg split must fit the launch
      }))
    return -5;
  size_t off_acc = 0, off_cnt = 0;
  const size_t ws_bytes = onepass_workspace_parts(B, Hq, Sq, &off_acc, &off_cnt);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
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
  float* delta = reinterpret_cast<float*>(ws);
  a.lse = lse;
  a.delta = delta;
  a.dq_acc = reinterpret_cast<float*>(ws + off_acc);
  a.dq_cnt = reinterpret_cast<uint32_t*>(ws + off_cnt);
  a.dq = reinterpret_cast<uint16_t*>(dq);
  a.dk = reinterpret_cast<uint16_t*>(dk);
  a.dv = reinterpret_cast<uint16_t*>(dv);
  const long long rows = (long long)B * Hq * Sq;
  const long long n_kt = (Sk + kTile - 1) / kTile, nq = (Sq + kTile - 1) / kTile;
  const long long units = n_kt * B * Hkv;
  const int grid = (int)std::min<long long>(units, n_sm);
  if ((units + grid - 1) / grid * (Hq / Hkv) * nq >= (1LL << 31) || n_kt * 8 >= (1LL << 32)) return -2;
  if (cudaMemsetAsync(a.dq_cnt, 0, ws_bytes - off_cnt, st) != cudaSuccess) return -5;
  bwd_delta_kernel<<<(unsigned)((rows + kDeltaRowsPerCta - 1) / kDeltaRowsPerCta), 256, 0, st>>>(
      reinterpret_cast<const uint16_t*>(out), reinterpret_cast<const uint16_t*>(dout), delta, rows, nullptr);
  if (cudaGetLastError() != cudaSuccess) return -5;
  // cooperative: every CTA is resident, which the ordered dQ adds rely on
  void* params[] = {&a};
  if (cudaLaunchCooperativeKernel((const void*)bwd_onepass_kernel, dim3(grid), dim3(kOnePassThreads), params,
                                  OnePassSmem::kAlloc, st) != cudaSuccess)
    return -5;
  return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

}  // namespace hattn
