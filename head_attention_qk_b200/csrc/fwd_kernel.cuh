// fwd_kernel.cuh -- fused attention forward for sm_100a (bf16 and e4m3 inputs).
//
// Computes, for one (batch, query head) and 256 query rows per CTA,
//   O = softmax(scale * Q K^T [+ causal mask]) V   and   LSE = ln sum_j exp(s_j),
// the operation of fmha_v3_fwd with return_softmax_lse and q/k/v descales
// (AITER PR #2911 "F8 fmha ASM gfx950", Test Result), at head dim 128 with
// grouped KV heads (RL-Kernel PR #319, ROCm Validation table: Hq=32, Hkv=8).
//
// CTA layout (384 threads, one CTA per SM):
//   warps 0-3  softmax group 0: query tile 0 (rows q0 .. q0+127), one row per thread
//   warps 4-7  softmax group 1: query tile 1 (rows q0+128 .. q0+255)
//   warp 8     TMA producer: Q once, then K_j / V_j into stage rings
//   warp 9     MMA issuer (one thread) and tensor-memory owner
//   warps 10-11  fp8 only: widen each e4m3 V tile to fp16 in shared memory
//
// Tensor memory (512 columns x 128 lanes, fp32):
//   [  0,128) S0 = Q0 K_j^T   (P0 = softmax numerators, 16-bit, aliases its first 64 columns)
//   [128,256) S1 = Q1 K_j^T   (P1 likewise)
//   [256,384) O0 accumulator, [384,512) O1 accumulator
//
// MMA issue order per KV tile j (one thread):
//   PV0_j, S0_{j+1}, PV1_j, S1_{j+1}
// S0_{j+1} overwrites the columns PV0_j reads its A operand (P0) from; the MMAs
// of one thread execute in issue order, so PV0_j has consumed P0 first.  A
// commit after S_i(j) also covers PV_i(j-1), so when softmax i sees S_i(j) it
// may rescale O_i and overwrite P_i.
//
// Online softmax in base 2: x = s * c with c = scale * log2(e) (fp8: times the
// q and k descales), p = 2^(x - m), l = sum p.  The running max m is raised
// only when a row's new max exceeds it by more than kRescaleThreshold; until
// then p <= 2^8 and O, l keep the stale m, which cancels in O / l.
#pragma once

#include "sm100.cuh"

namespace hattn {

constexpr int kBlockM = 128;      // rows per query tile (TMEM lanes)
constexpr int kBlockN = 128;      // keys per KV tile
constexpr int kHeadDim = 128;
constexpr int kQTilesPerCta = 2;
constexpr int kFwdThreads = 384;
constexpr int kMaxKvBlocks = 32;  // KV-cache blocks per launch of the block-KV forward
constexpr float kRescaleThreshold = 8.0f;

struct FwdArgs {
  CUtensorMap tm_q;
  CUtensorMap tm_k[kMaxKvBlocks];
  CUtensorMap tm_v[kMaxKvBlocks];
  int sk[kMaxKvBlocks];          // key length of each KV block (one block for attn_fwd)
  int B, Hq, Hkv, Sq;
  int causal;
  int n_qpairs;                  // number of 256-row query tiles per (b, h)
  float scale_log2;              // scale * log2(e)
  void* out;                     // bf16 [B,Hq,Sq,D]  or  fp32 partials [blk][B,Hq,Sq,D]
  float* lse;                    // fp32 [B,Hq,Sq]    or  fp32 partials [blk][B,Hq,Sq]
  const float* q_descale;        // fp8 only: [B*Hq], [B*Hkv], [B*Hkv]
  const float* k_descale;
  const float* v_descale;
  int block_offset;              // index of this launch's first block among all blocks
};

template <bool kFp8>
struct FwdSmemLayout {
  static constexpr int kElt = kFp8 ? 1 : 2;
  static constexpr int kTileBytes = kBlockM * kHeadDim * kElt;      // Q or K tile
  static constexpr int kStagesK = kFp8 ? 3 : 2;
  static constexpr int kStagesV = 2;                                 // V as loaded (bf16 / e4m3)
  static constexpr int kStagesV16 = kFp8 ? 2 : 0;                    // fp8: V widened to fp16
  static constexpr int kV16Bytes = kBlockN * kHeadDim * 2;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQTilesPerCta * kTileBytes;
  static constexpr int kVOff = kKOff + kStagesK * kTileBytes;
  static constexpr int kV16Off = kVOff + kStagesV * kTileBytes;
  static constexpr int kBarOff = kV16Off + kStagesV16 * kV16Bytes;
  static constexpr int kNumBars = 1 + 2 * kStagesK + 2 * kStagesV + 2 * kStagesV16 + 6;
  static constexpr int kBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;                       // slack for 1024-byte alignment
};

struct FwdBars {
  uint64_t* q_full;
  uint64_t* k_full;
  uint64_t* k_empty;
  uint64_t* v_full;
  uint64_t* v_empty;
  uint64_t* v16_full;
  uint64_t* v16_empty;
  uint64_t* s_full;   // [2]
  uint64_t* p_full;   // [2]
  uint64_t* o_done;   // [2]
  uint32_t* tmem_slot;
};

// Barrier sites recorded in the error word when a wait times out.
enum : int {
  kSiteQFull = 1, kSiteKFull, kSiteKEmpty, kSiteVFull, kSiteVEmpty, kSiteV16Full, kSiteV16Empty,
  kSiteSFull, kSitePFull, kSiteODone
};

__device__ __forceinline__ int fwd_num_kv_tiles(int sk, int Sq, int causal, int q_row0) {
  if (!causal) return (sk + kBlockN - 1) / kBlockN;
  int last_row = min(q_row0 + kQTilesPerCta * kBlockM - 1, Sq - 1);
  int max_key = min(last_row + (sk - Sq), sk - 1);
  return max_key / kBlockN + 1;
}

template <bool kFp8, bool kPartial>
__global__ void __launch_bounds__(kFwdThreads, 1) attn_fwd_kernel(const __grid_constant__ FwdArgs args) {
  using L = FwdSmemLayout<kFp8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = warp_id();
  const int lane = lane_id();

  const int blk_local = blockIdx.z;
  const int bh = blockIdx.y;
  const int b = bh / args.Hq;
  const int h = bh - b * args.Hq;
  const int G = args.Hq / args.Hkv;
  const int kvh = b * args.Hkv + h / G;
  // heaviest tiles first under a causal mask
  const int qpair = args.causal ? (args.n_qpairs - 1 - (int)blockIdx.x) : (int)blockIdx.x;
  const int q_row0 = qpair * (kQTilesPerCta * kBlockM);
  const int sk = args.sk[blk_local];
  const int n_kv = fwd_num_kv_tiles(sk, args.Sq, args.causal, q_row0);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  FwdBars bb;
  {
    uint64_t* p = bars;
    bb.q_full = p; p += 1;
    bb.k_full = p; p += L::kStagesK;
    bb.k_empty = p; p += L::kStagesK;
    bb.v_full = p; p += L::kStagesV;
    bb.v_empty = p; p += L::kStagesV;
    bb.v16_full = p; p += L::kStagesV16;
    bb.v16_empty = p; p += L::kStagesV16;
    bb.s_full = p; p += 2;
    bb.p_full = p; p += 2;
    bb.o_done = p; p += 2;
    bb.tmem_slot = reinterpret_cast<uint32_t*>(p);
  }

  if (threadIdx.x == 0) {
    mbar_init(bb.q_full, 1);
    for (int s = 0; s < L::kStagesK; ++s) { mbar_init(&bb.k_full[s], 1); mbar_init(&bb.k_empty[s], 1); }
    for (int s = 0; s < L::kStagesV; ++s) {
      mbar_init(&bb.v_full[s], 1);
      mbar_init(&bb.v_empty[s], kFp8 ? 64 : 1);    // fp8: released by the 64 widening threads
    }
    for (int s = 0; s < L::kStagesV16; ++s) { mbar_init(&bb.v16_full[s], 64); mbar_init(&bb.v16_empty[s], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bb.s_full[i], 1);
      mbar_init(&bb.p_full[i], kBlockM);
      mbar_init(&bb.o_done[i], 1);
    }
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(bb.tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&args.tm_q);
    prefetch_tmap(&args.tm_k[blk_local]);
    prefetch_tmap(&args.tm_v[blk_local]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *bb.tmem_slot;

  uint8_t* sQ = smem + L::kQOff;
  uint8_t* sK = smem + L::kKOff;
  uint8_t* sV = smem + L::kVOff;
  uint8_t* sV16 = smem + L::kV16Off;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const CUtensorMap* tq = &args.tm_q;
      const CUtensorMap* tk = &args.tm_k[blk_local];
      const CUtensorMap* tv = &args.tm_v[blk_local];
      constexpr int kBoxes = kFp8 ? 1 : 2;                 // 128-byte-wide boxes per 128-column row
      constexpr int kBoxBytes = L::kTileBytes / kBoxes;
      constexpr int kBoxCols = 128 / L::kElt;
      mbar_arrive_expect_tx(bb.q_full, kQTilesPerCta * L::kTileBytes);
      for (int t = 0; t < kQTilesPerCta; ++t)
        for (int x = 0; x < kBoxes; ++x)
          tma_load_3d(sQ + t * L::kTileBytes + x * kBoxBytes, tq, bb.q_full, x * kBoxCols, q_row0 + t * kBlockM, bh);
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        const int sk_ = j % L::kStagesK, uk = j / L::kStagesK;
        if (j >= L::kStagesK) ok = mbar_wait(&bb.k_empty[sk_], (uk - 1) & 1, kSiteKEmpty);
        if (!ok) break;
        mbar_arrive_expect_tx(&bb.k_full[sk_], L::kTileBytes);
        for (int x = 0; x < kBoxes; ++x)
          tma_load_3d(sK + sk_ * L::kTileBytes + x * kBoxBytes, tk, &bb.k_full[sk_], x * kBoxCols, j * kBlockN, kvh);
        const int sv = j % L::kStagesV, uv = j / L::kStagesV;
        if (j >= L::kStagesV) ok = mbar_wait(&bb.v_empty[sv], (uv - 1) & 1, kSiteVEmpty);
        if (!ok) break;
        mbar_arrive_expect_tx(&bb.v_full[sv], L::kTileBytes);
        for (int x = 0; x < kBoxes; ++x)
          tma_load_3d(sV + sv * L::kTileBytes + x * kBoxBytes, tv, &bb.v_full[sv], x * kBoxCols, j * kBlockN, kvh);
      }
      // Drain: every load issued must land before the CTA may exit.
      const int last = n_kv - 1;
      if (n_kv > 0) {
        for (int j = max(0, last - L::kStagesK + 1); j <= last; ++j)
          mbar_wait(&bb.k_full[j % L::kStagesK], (j / L::kStagesK) & 1, kSiteKFull);
        for (int j = max(0, last - L::kStagesV + 1); j <= last; ++j)
          mbar_wait(&bb.v_full[j % L::kStagesV], (j / L::kStagesV) & 1, kSiteVFull);
      }
      mbar_wait(bb.q_full, 0, kSiteQFull);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // S = Q K^T: A = Q tile (K-major), B = K tile (K-major), M = N = 128.
      // O += P V:  A = P in TMEM, B = V tile (MN-major along the head dim), M = N = 128.
      constexpr uint32_t kIdescQK = kFp8 ? make_idesc(0, 0, 0, 128, 128) : make_idesc(1, 1, 0, 128, 128);
      constexpr uint32_t kIdescPV = kFp8 ? make_idesc(0, 0, 1, 128, 128) : make_idesc(1, 1, 1, 128, 128);
      constexpr int kQKSteps = kFp8 ? 4 : 8;               // K = 32 (e4m3) or 16 (bf16) per MMA
      constexpr int kQKStepBytes = 32;
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK);
      const uint32_t sVa = kFp8 ? smem_u32(sV16) : smem_u32(sV);
      constexpr int kVStageBytes = kFp8 ? L::kV16Bytes : L::kTileBytes;
      constexpr int kVStages = kFp8 ? L::kStagesV16 : L::kStagesV;

      auto issue_qk = [&](int t, int kstage) {
        const uint32_t d = tmem + t * 128;
        for (int k = 0; k < kQKSteps; ++k) {
          // bf16: two 64-column swizzle atoms of 16 KB; step k in atom k/4 at byte (k%4)*32.
          const uint32_t off = kFp8 ? k * kQKStepBytes : (k >> 2) * 16384 + (k & 3) * kQKStepBytes;
          const uint64_t da = make_sdesc(sQa + t * L::kTileBytes + off, 16, 1024);
          const uint64_t db = make_sdesc(sKa + kstage * L::kTileBytes + off, 16, 1024);
          if (kFp8) mma_f8_ss(d, da, db, kIdescQK, k > 0);
          else mma_f16_ss(d, da, db, kIdescQK, k > 0);
        }
      };
      auto issue_pv = [&](int t, int vstage, uint32_t acc) {
        const uint32_t d = tmem + 256 + t * 128;
        const uint32_t a = tmem + t * 128;                 // P_t: 64 columns of packed 16-bit pairs
        for (int k = 0; k < kBlockN / 16; ++k) {
          // 16 keys per MMA: rows 16k..16k+15 of the V tile = 2048 bytes; the two
          // 64-column halves of the head dim are 16 KB apart (LBO).
          const uint64_t db = make_sdesc(sVa + vstage * kVStageBytes + k * 2048, 16384, 1024);
          mma_f16_ts(d, a + k * 8, db, kIdescPV, (acc || k > 0) ? 1u : 0u);
        }
      };

      bool ok = mbar_wait(bb.q_full, 0, kSiteQFull);
      if (ok && n_kv > 0) ok = mbar_wait(&bb.k_full[0], 0, kSiteKFull);
      if (ok && n_kv > 0) {
        tc_fence_after();
        issue_qk(0, 0);
        mma_commit(&bb.s_full[0]);
        issue_qk(1, 0);
        mma_commit(&bb.s_full[1]);
        mma_commit(&bb.k_empty[0]);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int vs = j % kVStages, uv = j / kVStages;
        if (kFp8) ok = mbar_wait(&bb.v16_full[vs], uv & 1, kSiteV16Full);
        else ok = mbar_wait(&bb.v_full[vs], uv & 1, kSiteVFull);
        if (ok) ok = mbar_wait(&bb.p_full[0], j & 1, kSitePFull);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, vs, j > 0);
        if (j == n_kv - 1) mma_commit(&bb.o_done[0]);
        const int jn = j + 1;
        const int ks = jn % L::kStagesK;
        if (jn < n_kv) {
          ok = mbar_wait(&bb.k_full[ks], (jn / L::kStagesK) & 1, kSiteKFull);
          if (!ok) break;
          tc_fence_after();
          issue_qk(0, ks);
          mma_commit(&bb.s_full[0]);
        }
        ok = mbar_wait(&bb.p_full[1], j & 1, kSitePFull);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, vs, j > 0);
        if (kFp8) mma_commit(&bb.v16_empty[vs]);
        else mma_commit(&bb.v_empty[vs]);
        if (j == n_kv - 1) mma_commit(&bb.o_done[1]);
        if (jn < n_kv) {
          issue_qk(1, ks);
          mma_commit(&bb.s_full[1]);
          mma_commit(&bb.k_empty[ks]);
        }
      }
      if (!ok) {
        // Error path: make sure no MMA is still in flight before TMEM is freed.
        mma_commit(&bb.o_done[0]);
        mma_commit(&bb.o_done[1]);
      }
      // Drain: wait for the final commits so no tcgen05 op outlives the CTA.
      mbar_wait(&bb.o_done[0], 0, kSiteODone);
      mbar_wait(&bb.o_done[1], 0, kSiteODone);
    }
    __syncwarp();
  } else if (warp >= 10) {
    // ------------------------------------------------------------ fp8: widen V to fp16
    if (kFp8) {
      const int t = threadIdx.x - 320;                       // 0..63
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        const int sv = j % L::kStagesV, uv = j / L::kStagesV;
        const int s16 = j % max(L::kStagesV16, 1), u16 = j / max(L::kStagesV16, 1);
        ok = warp_wait(&bb.v_full[sv], uv & 1, kSiteVFull);
        if (ok && j >= L::kStagesV16) ok = warp_wait(&bb.v16_empty[s16], (u16 - 1) & 1, kSiteV16Empty);
        if (!ok) break;
        const uint8_t* src = sV + sv * L::kTileBytes;
        uint8_t* dst = sV16 + s16 * L::kV16Bytes;
        // e4m3 tile: row r (key) = 128 bytes, 16-byte chunk c holds head dims [16c, 16c+16),
        // stored at chunk c ^ (r & 7).  fp16 tile: two 64-dim halves of 16 KB; row r of a
        // half = 128 bytes, chunk c8 holds dims [8 c8, 8 c8 + 8) of the half at c8 ^ (r & 7).
#pragma unroll 4
        for (int it = 0; it < 16; ++it) {
          const int idx = t + 64 * it;
          const int r = idx >> 3, c = idx & 7;
          const uint4 in = *reinterpret_cast<const uint4*>(src + r * 128 + ((c ^ (r & 7)) << 4));
          const uint32_t w[4] = {in.x, in.y, in.z, in.w};
          uint32_t o[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            o[2 * q] = e4m3x2_to_f16x2((uint16_t)(w[q] & 0xFFFFu));
            o[2 * q + 1] = e4m3x2_to_f16x2((uint16_t)(w[q] >> 16));
          }
          const int half = c >> 2;
          const int c8 = (c & 3) * 2;
          uint8_t* rowp = dst + half * 16384 + r * 128;
          *reinterpret_cast<uint4*>(rowp + ((c8 ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(rowp + (((c8 + 1) ^ (r & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&bb.v16_full[s16]);
        mbar_arrive(&bb.v_empty[sv]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax groups 0 and 1
    const int tile = warp >> 2;                       // 0 or 1
    const int r = threadIdx.x & 127;                  // row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + tile * 128;
    const uint32_t tO = tmem + lane_base + 256 + tile * 128;
    const int row = q_row0 + tile * kBlockM + r;
    const int kv_limit = args.causal ? min(sk - 1, row + (sk - args.Sq)) : sk - 1;

    float c = args.scale_log2;
    float v_scale = 1.f;
    if (kFp8) {
      c *= __ldg(&args.q_descale[bh]) * __ldg(&args.k_descale[kvh]);
      v_scale = __ldg(&args.v_descale[kvh]);
    }

    float m = -INFINITY;     // running max of x = s * c (base-2 units)
    float l = 0.f;           // running sum of 2^(x - m)
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      ok = warp_wait(&bb.s_full[tile], j & 1, kSiteSFull);
      if (!ok) break;
      tc_fence_after();
      float s[128];
      {
        uint32_t u[32];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          tmem_ld32(tS + q * 32, u);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) s[q * 32 + e] = __uint_as_float(u[e]);
        }
      }
      const int kbase = j * kBlockN;
      if (kbase + kBlockN - 1 > kv_limit) {
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (kbase + e > kv_limit) s[e] = -INFINITY;
      }
      __syncwarp();
      float mx = s[0];
#pragma unroll
      for (int e = 1; e < 128; ++e) mx = fmaxf(mx, s[e]);
      const float m_tile = mx * c;                     // -inf if every key of the tile is masked
      const bool need = m_tile > m + kRescaleThreshold || (m == -INFINITY && m_tile > -INFINITY);
      float f = 1.f;
      if (need) {
        f = ex2_approx(m - m_tile);                    // 0 when m = -inf
        m = m_tile;
        l *= f;
      }
      __syncwarp();
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // Rescale this warp's 32 rows of O (PV_{j-1} completed before S_j).
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          uint32_t u[32];
          tmem_ld32(tO + q * 32, u);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * f);
          tmem_st32(tO + q * 32, u);
        }
        tmem_wait_st();
      }
      const float mneg = (m == -INFINITY) ? 0.f : -m;
      float sum0 = 0.f, sum1 = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int e = 0; e < 128; e += 2) {
        const float p0 = ex2_approx(fmaf(s[e], c, mneg));
        const float p1 = ex2_approx(fmaf(s[e + 1], c, mneg));
        sum0 += p0;
        sum1 += p1;
        pk[e >> 1] = kFp8 ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1);
      }
      l += sum0 + sum1;
      {
        uint32_t u[32];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
#pragma unroll
          for (int e = 0; e < 32; ++e) u[e] = pk[q * 32 + e];
          tmem_st32(tS + q * 32, u);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bb.p_full[tile]);
    }
    if (ok) ok = warp_wait(&bb.o_done[tile], 0, kSiteODone);
    if (ok) {
      tc_fence_after();
      const float inv_l = (l > 0.f) ? (v_scale / l) : 0.f;
      const bool store = row < args.Sq;
      const size_t orow = ((size_t)bh * args.Sq + (size_t)max(row, 0)) * kHeadDim;
      const size_t part = (size_t)(args.block_offset + blk_local);
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t u[32];
        __syncwarp();
        tmem_ld32(tO + q * 32, u);
        tmem_wait_ld();
        if (store) {
          if (kPartial) {
            float* dst = reinterpret_cast<float*>(args.out) +
                         part * ((size_t)args.B * args.Hq * args.Sq * kHeadDim) + orow + q * 32;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dst + e) =
                  make_float4(__uint_as_float(u[e]) * inv_l, __uint_as_float(u[e + 1]) * inv_l,
                              __uint_as_float(u[e + 2]) * inv_l, __uint_as_float(u[e + 3]) * inv_l);
          } else {
            uint32_t pkd[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pkd[e] = pack_bf16x2(__uint_as_float(u[2 * e]) * inv_l, __uint_as_float(u[2 * e + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(args.out) + orow + q * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pkd[4 * e], pkd[4 * e + 1], pkd[4 * e + 2], pkd[4 * e + 3]);
          }
        }
      }
      if (store) {
        const float lse2 = (l > 0.f) ? (m + __log2f(l)) : -INFINITY;
        float* lse = args.lse + (kPartial ? part * ((size_t)args.B * args.Hq * args.Sq) : 0);
        lse[(size_t)bh * args.Sq + row] = lse2 * 0.69314718055994530942f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Fixed-order merge of per-block partial results (RL-Kernel PR #319, Summary
// table: one attention-domain LSE, fixed global_block_index merge order).
// One warp per query row; blocks are folded in ascending order:
//   M = max(L, L_b), w = e^(L-M), w_b = e^(L_b-M), L = M + ln(w + w_b),
//   O = (w O + w_b O_b) / (w + w_b),  starting from (O, L) = (0, -inf).
__global__ void __launch_bounds__(256) lse_merge_kernel(const float* __restrict__ o_parts,
                                                        const float* __restrict__ lse_parts, int n_blocks,
                                                        long long rows, uint16_t* __restrict__ out,
                                                        float* __restrict__ lse_out) {
  const long long rowi = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (rowi >= rows) return;
  const int lane = threadIdx.x & 31;
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = -INFINITY;
  for (int bl = 0; bl < n_blocks; ++bl) {
    const float Lb = __ldg(&lse_parts[(long long)bl * rows + rowi]);
    if (Lb == -INFINITY) continue;
    const float4 ob = __ldg(reinterpret_cast<const float4*>(o_parts + ((long long)bl * rows + rowi) * kHeadDim) + lane);
    const float M = fmaxf(L, Lb);
    const float w = __expf(L - M);
    const float wb = __expf(Lb - M);
    const float inv = 1.f / (w + wb);
    o.x = (w * o.x + wb * ob.x) * inv;
    o.y = (w * o.y + wb * ob.y) * inv;
    o.z = (w * o.z + wb * ob.z) * inv;
    o.w = (w * o.w + wb * ob.w) * inv;
    L = M + __logf(w + wb);
  }
  uint2 pk;
  pk.x = pack_bf16x2(o.x, o.y);
  pk.y = pack_bf16x2(o.z, o.w);
  reinterpret_cast<uint2*>(out + rowi * kHeadDim)[lane] = pk;
  if (lane == 0) lse_out[rowi] = L;
}

}  // namespace hattn
