// fwd_kernel.cuh -- fused attention forward for sm_100a (bf16 and e4m3 inputs).
//
// Computes, for one (batch, query head) and 256 query rows per work unit,
//   O = softmax(scale * Q K^T [+ causal mask]) V   and   LSE = ln sum_j exp(s_j),
// the operation of fmha_v3_fwd with return_softmax_lse and q/k/v descales
// (AITER PR #2911 "F8 fmha ASM gfx950", Test Result), at head dim 128 with
// grouped KV heads (RL-Kernel PR #319, ROCm Validation table: Hq=32, Hkv=8).
//
// Persistent: one CTA per SM loops over work units (256 query rows of one
// (b, h) against one KV block); barrier phases and ring positions carry over
// from unit to unit, tensor memory is allocated once, and the next unit's Q is
// loaded as soon as the current unit's last S = Q K^T has been issued.
//
// CTA layout (384 threads, one CTA per SM):
//   warps 0-3  softmax group 0: query tile 0 (rows q0 .. q0+127), one row per thread
//   warps 4-7  softmax group 1: query tile 1 (rows q0+128 .. q0+255)
//   warp 8     TMA producer: Q once, then K_j / V_j into one ring
//   warp 9     MMA issuer (one thread) and tensor-memory owner
//   warps 10-11  e4m3 V widened here (kWidenV): e4m3 V tile -> fp16 in shared
//              memory; otherwise no role (they hold the registers the softmax
//              groups give up)
//
// e4m3 inputs: Q and K stay e4m3 (S = Q K^T runs as an 8-bit MMA) and P V is an
// fp16 MMA with P in fp16.  V reaches it as fp16 (exact) in one of two ways:
// already widened in global memory by a separate pass (the fast form, for
// callers that give scratch memory), or loaded as e4m3 and widened in shared
// memory by warps 10-11 (kWidenV: no scratch; the conversion competes with the
// softmax for issue slots and shared-memory bandwidth, about 2 % slower).
//
// Descales (e4m3): per (b, head) and, for the block-KV forward, per block.  The
// K descale scales block b's scores (c = scale log2(e) q_ds k_ds[b]); the V
// descale of block b enters as the factor vd_b / vd_max <= 1 on that block's
// probabilities before they are rounded to fp16 for P V (added to the exponent
// as log2(vd_b / vd_max), so no multiply per element), with the row sum l
// corrected once per tile; the epilogue multiplies by vd_max / l.
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
// may rescale O_i and overwrite P_i.  P is written and released in two halves of
// 64 keys so the P V of the first half can start while the second is computed.
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
// setmaxnreg split: 2 softmax warpgroups at kRegsSoftmax, 1 warpgroup at
// kRegsOther.  The sum must not exceed the registers the launch holds
// (registers per thread x 384); the host checks this before every launch, since
// an increase that cannot be satisfied would wait forever.
constexpr int kRegsSoftmax = 208;
constexpr int kRegsOther = 88;
constexpr int kRegsNeeded = (2 * kRegsSoftmax + kRegsOther) * 128;
static_assert(kRegsNeeded <= (65536 / 384) / 8 * 8 * 384, "setmaxnreg split exceeds a 384-thread launch");

struct FwdArgs {
  CUtensorMap tm_q;
  CUtensorMap tm_o;              // bf16 O (boxes of 64 columns x 32 rows), stored by TMA from the persistent kernel
  CUtensorMap tm_k[kMaxKvBlocks];
  CUtensorMap tm_v[kMaxKvBlocks];
  int sk[kMaxKvBlocks];          // key length of each KV block (one block for attn_fwd)
  int B, Hq, Hkv, Sq;
  int causal;
  int n_qpairs;                  // number of 256-row query tiles per (b, h)
  float scale_log2;              // scale * log2(e)
  void* out;                     // bf16 [B,Hq,Sq,D]  or  fp32 partials [blk][B,Hq,Sq,D]
  float* lse;                    // fp32 [B,Hq,Sq]    or  fp32 partials [blk][B,Hq,Sq]
  const float* q_descale;        // fp8 only: [B*Hq]
  const float* k_descale;        // fp8 only: [n_blocks][B*Hkv] (one block for attn_fwd)
  const float* v_descale;
  int block_offset;              // index of this launch's first block among all blocks
  int total_units;               // work units of this launch; CTAs loop over them
  int fused_blocks;              // > 1: one unit runs over all these blocks in order (no partials)
  int fused_tiles;               // KV tiles over all fused blocks
};

template <bool kFp8, bool kWidenV = false, bool kEpiStage = false>
struct FwdSmemLayout {
  static_assert(!kWidenV || kFp8, "only e4m3 V is widened in shared memory");
  static constexpr int kElt = kFp8 ? 1 : 2;                            // Q and K element bytes
  static constexpr int kTileBytes = kBlockM * kHeadDim * kElt;         // Q or K tile as loaded
  static constexpr int kVTileBytes = kBlockN * kHeadDim * 2;           // V tile as P V reads it: bf16 or fp16
  static constexpr int kVLoadBytes = kWidenV ? kTileBytes : kVTileBytes;   // V tile as loaded
  static constexpr int kSlotBytes = kVLoadBytes;
  // One ring holds the K and V tiles in load order K_0, V_0, K_1, V_1, ...; they
  // are also released in that order (K_j when S1_j completes, V_j when PV1_j
  // completes, or when it is widened), so the producer can run kRing tiles
  // ahead of the MMAs.  With kWidenV the ring has an even number of slots, so
  // every slot keeps one role (K in even slots, V in odd ones), and the widened
  // V tiles go through kStagesV16 fp16 buffers.
  // kEpiStage (the persistent kernel, bf16 O): one 32 KB slot's worth of the
  // ring (two for the 16 KB e4m3 slots) becomes the O staging area.
  static constexpr int kRing = kWidenV ? (kEpiStage ? 6 : 8) : (kFp8 ? (kEpiStage ? 5 : 6) : (kEpiStage ? 4 : 5));
  static_assert(!kWidenV || kRing % 2 == 0, "widening needs slots of one role");
  static constexpr int kStagesV16 = kWidenV ? 2 : 0;
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = kQOff + kQTilesPerCta * kTileBytes;
  static constexpr int kV16Off = kRingOff + kRing * kSlotBytes;
  // O staging: per query tile, 128 rows x 64 columns of bf16 (16 KB, the
  // layout of one 128-byte-swizzled TMA box); the epilogue stores each tile
  // in two passes of 64 columns
  static constexpr int kEpiTileBytes = kBlockM * 64 * 2;
  static constexpr int kEpiOff = kV16Off + kStagesV16 * kVTileBytes;
  static constexpr int kBarOff = kEpiOff + (kEpiStage ? kQTilesPerCta * kEpiTileBytes : 0);
  static constexpr int kNumBars = 3 + 2 * kRing + 2 * kStagesV16 + 8;
  static constexpr int kBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;                       // slack for 1024-byte alignment
  static_assert(kAlloc <= 232448, "shared memory per CTA");
};

struct FwdBars {
  uint64_t* q_full;
  uint64_t* q_empty;  // the unit's last S MMA has been issued (Q may be reloaded)
  uint64_t* mma_drain;  // every MMA of the CTA has completed (committed once, at exit)
  uint64_t* ring_full;   // [kRing]
  uint64_t* ring_empty;  // [kRing]
  uint64_t* v16_full;    // [kStagesV16]: widened V tile written (one arrival per widening warp)
  uint64_t* v16_empty;   // [kStagesV16]: the P V MMAs of that tile have completed
  uint64_t* s_full;   // [2]: S_t ready
  uint64_t* p_full;   // [2 tiles][2 halves of 64 keys]: P_t,h written (128 arrivals)
  uint64_t* o_done;   // [2]: last P V of the tile completed
  uint32_t* tmem_slot;
};

// Barrier sites recorded in the error word when a wait times out.
enum : int {
  kSiteQFull = 1, kSiteKFull, kSiteKEmpty, kSiteVFull, kSiteVEmpty,
  kSiteSFull, kSitePFull, kSiteODone, kSiteDrain, kSiteV16Full, kSiteV16Empty
};

__device__ __forceinline__ int fwd_num_kv_tiles(int sk, int Sq, int causal, int q_row0) {
  if (!causal) return (sk + kBlockN - 1) / kBlockN;
  int last_row = min(q_row0 + kQTilesPerCta * kBlockM - 1, Sq - 1);
  int max_key = min(last_row + (sk - Sq), sk - 1);
  return max_key / kBlockN + 1;
}

// One work unit: 256 query rows of one (b, h) against one KV block, or against
// all the launch's blocks in ascending order when they are fused.
struct FwdUnit {
  int bh, kvh, q_row0, blk, sk, n_kv;
};

// KV tiles of a block of sk keys.
__device__ __forceinline__ int fwd_block_tiles(int sk) { return (sk + kBlockN - 1) / kBlockN; }

// Units are numbered block-major.  Without a mask, consecutive units share a
// head (its K/V stays hot in L2); under a causal mask the order is rank-major
// over heads, heaviest query tiles first, so the persistent CTAs pick up the
// long units before the short ones.
__device__ __forceinline__ FwdUnit fwd_unit(const FwdArgs& a, int u) {
  FwdUnit w;
  const int nbh = a.B * a.Hq;
  const int per_blk = a.n_qpairs * nbh;
  w.blk = a.fused_blocks > 1 ? 0 : u / per_blk;
  const int r = u - w.blk * per_blk;
  int qpair;
  if (a.causal) {
    const int rank = r / nbh;
    w.bh = r - rank * nbh;
    qpair = a.n_qpairs - 1 - rank;
  } else {
    w.bh = r / a.n_qpairs;
    qpair = r - w.bh * a.n_qpairs;
  }
  const int b = w.bh / a.Hq, h = w.bh - b * a.Hq;
  w.kvh = b * a.Hkv + h / (a.Hq / a.Hkv);
  w.q_row0 = qpair * (kQTilesPerCta * kBlockM);
  w.sk = a.sk[w.blk];
  w.n_kv = a.fused_blocks > 1 ? a.fused_tiles : fwd_num_kv_tiles(w.sk, a.Sq, a.causal, w.q_row0);
  return w;
}

// The units of one CTA.  Persistent: the (heaviest-first) unit list is dealt
// out in snake order, unit k of CTA c being k G + c for even k and
// k G + G - 1 - c for odd k (G = gridDim.x), which evens out unequal causal
// units; increasing in k, so the loop ends at the first index past the list.
// One unit per CTA: blockIdx.x, then past it.
template <bool kPersist>
__device__ __forceinline__ int fwd_unit_index(int k) {
  if (!kPersist) return (int)blockIdx.x + k;
  const int G = (int)gridDim.x, c = (int)blockIdx.x;
  return k * G + ((k & 1) ? G - 1 - c : c);
}

// Unit loop condition.  Persistent launches loop while units remain; a
// one-unit-per-CTA launch runs the body exactly once (the compiler sees a single
// iteration, so the per-tile code is the same as a kernel without the loop).
template <bool kPersist>
__device__ __forceinline__ bool fwd_more_units(int u, int u_first, int u_end, bool ok) {
  return kPersist ? (u < u_end && ok) : (u == u_first);
}

template <bool kFp8, bool kPartial, bool kPersist, bool kWidenV = false>
__global__ void __launch_bounds__(kFwdThreads, 1) attn_fwd_kernel(const __grid_constant__ FwdArgs args) {
  constexpr bool kEpiStage = kPersist && !kPartial;   // bf16 O staged in shared memory, stored by TMA
  using L = FwdSmemLayout<kFp8, kWidenV, kEpiStage>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = warp_id();
  const int lane = lane_id();
  // Persistent: this CTA takes units fwd_unit_index(0), (1), ...; otherwise
  // the grid holds one CTA per unit.
  const int u_first = blockIdx.x, u_end = args.total_units;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  FwdBars bb;
  {
    uint64_t* p = bars;
    bb.q_full = p; p += 1;
    bb.q_empty = p; p += 1;
    bb.mma_drain = p; p += 1;
    bb.ring_full = p; p += L::kRing;
    bb.ring_empty = p; p += L::kRing;
    bb.v16_full = p; p += L::kStagesV16;
    bb.v16_empty = p; p += L::kStagesV16;
    bb.s_full = p; p += 2;
    bb.p_full = p; p += 4;
    bb.o_done = p; p += 2;
    bb.tmem_slot = reinterpret_cast<uint32_t*>(p);
  }

  if (threadIdx.x == 0) {
    mbar_init(bb.q_full, 1);
    mbar_init(bb.q_empty, 1);
    mbar_init(bb.mma_drain, 1);
    for (int s = 0; s < L::kRing; ++s) {
      mbar_init(&bb.ring_full[s], 1);
      // widened V (odd slots) is released by the two widening warps, every
      // other slot by one MMA commit
      mbar_init(&bb.ring_empty[s], (kWidenV && (s & 1)) ? 2 : 1);
    }
    for (int s = 0; s < L::kStagesV16; ++s) {
      mbar_init(&bb.v16_full[s], 2);
      mbar_init(&bb.v16_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bb.s_full[i], 1);
      // one arrival per softmax warp (elected after __syncwarp), not per thread:
      // 128 atomic updates of one shared-memory word per half tile would contend
      // with the MMA thread polling it
      mbar_init(&bb.p_full[2 * i], kBlockM / 32);
      mbar_init(&bb.p_full[2 * i + 1], kBlockM / 32);
      mbar_init(&bb.o_done[i], 1);
    }
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(bb.tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) prefetch_tmap(&args.tm_q);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *bb.tmem_slot;
  // Launched as a programmatic dependent of whatever precedes it on the
  // stream: the setup above overlaps that grid's end, and nothing in global
  // memory is touched before it has completed.  The grid after this one may
  // then launch (it waits for this one the same way).
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();

  uint8_t* sQ = smem + L::kQOff;
  uint8_t* sRing = smem + L::kRingOff;
  uint8_t* sV16 = smem + L::kV16Off;

  // Register split (see kRegsSoftmax): the producer / MMA warpgroup gives
  // registers up, the two softmax warpgroups take them.
  if (warp >= 8) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsOther) : "memory");
  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      constexpr int kBoxes = kFp8 ? 1 : 2;                 // 128-byte-wide boxes per 128-column Q/K row
      constexpr int kBoxBytes = L::kTileBytes / kBoxes;
      constexpr int kBoxCols = 128 / L::kElt;
      constexpr int kVBoxes = kWidenV ? 1 : 2;             // V: one e4m3 box, or two of 64 16-bit columns
      constexpr int kVBoxBytes = L::kVLoadBytes / kVBoxes;
      constexpr int kVBoxCols = kWidenV ? 128 : 64;
      bool ok = true;
      int slot = 0, units = 0;
      uint32_t ph = 0;
      long long nseq = 0;                                  // K/V tiles loaded by this CTA
      for (int u = u_first; fwd_more_units<kPersist>(u, u_first, u_end, ok); u = fwd_unit_index<kPersist>(++units)) {
        const FwdUnit w = fwd_unit(args, u);
        // K/V tile j of the unit: tile lt of block b (fused blocks run in order)
        int b = w.blk, lt = 0, nt = fwd_block_tiles(args.sk[b]);
        // the previous unit's last S has been issued before Q is overwritten
        if (units > 0) ok = mbar_wait(bb.q_empty, (units - 1) & 1, kSiteQFull);
        if (!ok) break;
        mbar_arrive_expect_tx(bb.q_full, kQTilesPerCta * L::kTileBytes);
        for (int t = 0; t < kQTilesPerCta; ++t)
          for (int x = 0; x < kBoxes; ++x)
            tma_load_3d(sQ + t * L::kTileBytes + x * kBoxBytes, &args.tm_q, bb.q_full, x * kBoxCols,
                        w.q_row0 + t * kBlockM, w.bh);
        // sequence n: K_{n/2} for even n, V_{n/2} for odd n
        for (int n = 0; n < 2 * w.n_kv && ok; ++n, ++nseq) {
          if (nseq >= L::kRing) ok = mbar_wait(&bb.ring_empty[slot], ph ^ 1u, kSiteKEmpty);
          if (!ok) break;
          uint8_t* dst = sRing + slot * L::kSlotBytes;
          if (n & 1) {
            mbar_arrive_expect_tx(&bb.ring_full[slot], L::kVLoadBytes);
            for (int x = 0; x < kVBoxes; ++x)
              tma_load_3d(dst + x * kVBoxBytes, &args.tm_v[b], &bb.ring_full[slot], x * kVBoxCols, lt * kBlockN,
                          w.kvh);
            if (++lt == nt && n + 1 < 2 * w.n_kv) {         // next block
              ++b;
              lt = 0;
              nt = fwd_block_tiles(args.sk[b]);
            }
          } else {
            mbar_arrive_expect_tx(&bb.ring_full[slot], L::kTileBytes);
            for (int x = 0; x < kBoxes; ++x)
              tma_load_3d(dst + x * kBoxBytes, &args.tm_k[b], &bb.ring_full[slot], x * kBoxCols, lt * kBlockN,
                          w.kvh);
          }
          if (++slot == L::kRing) { slot = 0; ph ^= 1u; }
        }
      }
      // Drain: every load issued must land before the CTA may exit.
      for (long long pos = nseq - L::kRing < 0 ? 0 : nseq - L::kRing; pos < nseq; ++pos)
        mbar_wait_drain(&bb.ring_full[pos % L::kRing], (uint32_t)((pos / L::kRing) & 1), kSiteDrain);
      if (units > 0) mbar_wait_drain(bb.q_full, (units - 1) & 1, kSiteDrain);
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
      const uint32_t sQa = smem_u32(sQ), sRa = smem_u32(sRing), sV16a = smem_u32(sV16);
      // Descriptor halves: Q / K tiles K-major (SBO 1024 B), V MN-major (LBO 16 KB
      // between the two 64-column halves of the head dim, SBO 1024 B).
      constexpr uint32_t kHi = sdesc_hi(1024);
      const uint32_t q_lo0 = sdesc_lo(sQa, 16);
      const uint32_t ring_lo0 = sdesc_lo(sRa, 16);
      auto issue_qk = [&](int t, int kslot) {
        const uint32_t d = tmem + t * 128;
        const uint32_t a_lo = q_lo0 + t * (L::kTileBytes >> 4);
        const uint32_t b_lo = ring_lo0 + kslot * (L::kSlotBytes >> 4);
#pragma unroll
        for (int k = 0; k < kQKSteps; ++k) {
          // bf16: two 64-column swizzle atoms of 16 KB; step k in atom k/4 at byte (k%4)*32.
          const uint32_t off = (kFp8 ? k * kQKStepBytes : (k >> 2) * 16384 + (k & 3) * kQKStepBytes) >> 4;
          if (kFp8) mma_f8_ss2(d, a_lo + off, kHi, b_lo + off, kHi, kIdescQK, k > 0);
          else mma_f16_ss2(d, a_lo + off, kHi, b_lo + off, kHi, kIdescQK, k > 0);
        }
      };
      // O_t (+)= P_t V for keys [64 half, 64 half + 64): 4 MMAs of 16 keys.
      auto issue_pv_half = [&](int t, uint32_t vbase, int half, uint32_t acc) {
        const uint32_t d = tmem + 256 + t * 128;
        const uint32_t a = tmem + t * 128;                 // P_t: 64 columns of packed 16-bit pairs
        const uint32_t b_lo = sdesc_lo(vbase, 16384);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int k = half * 4 + kk;
          // 16 keys per MMA: rows 16k..16k+15 of the V tile = 2048 bytes.
          mma_f16_ts2(d, a + k * 8, b_lo + k * (2048 >> 4), kHi, kIdescPV, (acc || k > 0) ? 1u : 0u);
        }
      };
      // Wait for each half of P_t and issue its MMAs (jg: this CTA's tile count).
      auto pv = [&](int t, uint32_t vbase, uint32_t jg, int j) -> bool {
        for (int half = 0; half < 2; ++half) {
          if (!mbar_wait(&bb.p_full[t * 2 + half], jg & 1, kSitePFull)) return false;
          tc_fence_after();
          issue_pv_half(t, vbase, half, j > 0);
        }
        return true;
      };
      auto next_pos = [](int& slot, uint32_t& ph) {
        if (++slot == L::kRing) { slot = 0; ph ^= 1u; }
      };

      bool ok = true;
      int kslot = 0, units = 0, vs16 = 0;
      uint32_t kph = 0, jg = 0, vph16 = 0;
      for (int u = u_first; fwd_more_units<kPersist>(u, u_first, u_end, ok); u = fwd_unit_index<kPersist>(++units)) {
        const FwdUnit w = fwd_unit(args, u);
        const int n_kv = w.n_kv;
        ok = mbar_wait(bb.q_full, units & 1, kSiteQFull);
        if (ok) ok = mbar_wait(&bb.ring_full[kslot], kph, kSiteKFull);
        if (!ok) break;
        tc_fence_after();
        issue_qk(0, kslot);
        mma_commit(&bb.s_full[0]);
        issue_qk(1, kslot);
        mma_commit(&bb.s_full[1]);
        mma_commit(&bb.ring_empty[kslot]);
        if (n_kv == 1) mma_commit(bb.q_empty);             // last S of the unit issued
        for (int j = 0; j < n_kv && ok; ++j, ++jg) {
          int vslot = kslot;
          uint32_t vph = kph;
          next_pos(vslot, vph);                            // V_j follows K_j
          uint32_t vbase;
          if (kWidenV) {
            ok = mbar_wait(&bb.v16_full[vs16], vph16, kSiteV16Full);
            vbase = sV16a + vs16 * L::kVTileBytes;
          } else {
            ok = mbar_wait(&bb.ring_full[vslot], vph, kSiteVFull);
            vbase = sRa + vslot * L::kSlotBytes;
          }
          if (ok) ok = pv(0, vbase, jg, j);
          if (!ok) break;
          if (j == n_kv - 1) mma_commit(&bb.o_done[0]);
          kslot = vslot;
          kph = vph;
          next_pos(kslot, kph);                            // K_{j+1} (or the next unit's K_0)
          const bool more = j + 1 < n_kv;
          if (more) {
            ok = mbar_wait(&bb.ring_full[kslot], kph, kSiteKFull);
            if (!ok) break;
            tc_fence_after();
            issue_qk(0, kslot);
            mma_commit(&bb.s_full[0]);
          }
          ok = pv(1, vbase, jg, j);
          if (!ok) break;
          if (kWidenV) {
            mma_commit(&bb.v16_empty[vs16]);
            if (++vs16 == L::kStagesV16) { vs16 = 0; vph16 ^= 1u; }
          } else {
            mma_commit(&bb.ring_empty[vslot]);
          }
          if (j == n_kv - 1) mma_commit(&bb.o_done[1]);
          if (more) {
            issue_qk(1, kslot);
            mma_commit(&bb.s_full[1]);
            mma_commit(&bb.ring_empty[kslot]);
            if (j + 1 == n_kv - 1) mma_commit(bb.q_empty);  // last S of the unit issued
          }
        }
      }
      // Drain (normal and error paths): the commit tracks every MMA this thread
      // issued, so none is in flight when tensor memory is freed.
      mma_commit(bb.mma_drain);
      mbar_wait_drain(bb.mma_drain, 0, kSiteDrain);
    }
    __syncwarp();
  } else if constexpr (kWidenV) {
    // ------------------------------------------------------------ warps 10-11: widen e4m3 V to fp16
    const int t = threadIdx.x - 320;                     // 0..63
    bool ok = true;
    uint32_t jg = 0;                                     // this CTA's tile count
    int units = 0;
    for (int u = u_first; fwd_more_units<kPersist>(u, u_first, u_end, ok); u = fwd_unit_index<kPersist>(++units)) {
      const int n_kv = fwd_unit(args, u).n_kv;
      for (int j = 0; j < n_kv && ok; ++j, ++jg) {
        // V of tile jg sits at ring position 2 jg + 1 (an odd slot: the ring is even)
        const int vslot = (int)((2u * jg + 1u) % L::kRing);
        const uint32_t vph = ((2u * jg + 1u) / L::kRing) & 1u;
        const int s16 = (int)(jg % L::kStagesV16);
        const uint32_t u16 = jg / L::kStagesV16;
        ok = warp_wait(&bb.ring_full[vslot], vph, kSiteVFull);
        if (ok && jg >= (uint32_t)L::kStagesV16) ok = warp_wait(&bb.v16_empty[s16], (u16 - 1) & 1, kSiteV16Empty);
        if (!ok) break;
        const uint8_t* src = sRing + vslot * L::kSlotBytes;
        uint8_t* dst = sV16 + s16 * L::kVTileBytes;
        // e4m3 tile (128-byte swizzle): key row r is 128 bytes, 16-byte chunk c
        // holds head dims [16 c, 16 c + 16) and sits at chunk c ^ (r & 7).  fp16
        // tile: two 16 KB halves of 64 head dims; row r of a half is 128 bytes,
        // chunk c8 holds dims [8 c8, 8 c8 + 8) of the half at chunk c8 ^ (r & 7).
#pragma unroll 4
        for (int it = 0; it < 16; ++it) {
          const int idx = t + 64 * it;
          const int r = idx >> 3, c = idx & 7;
          const uint4 in = *reinterpret_cast<const uint4*>(src + r * 128 + ((c ^ (r & 7)) << 4));
          const uint32_t wv[4] = {in.x, in.y, in.z, in.w};
          uint32_t o[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            o[2 * q] = e4m3x2_to_f16x2((uint16_t)(wv[q] & 0xFFFFu));
            o[2 * q + 1] = e4m3x2_to_f16x2((uint16_t)(wv[q] >> 16));
          }
          const int half = c >> 2;
          const int c8 = (c & 3) * 2;
          uint8_t* rowp = dst + half * 16384 + r * 128;
          *reinterpret_cast<uint4*>(rowp + ((c8 ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(rowp + (((c8 + 1) ^ (r & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
        }
        // the MMAs read the fp16 tile through the async proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bb.v16_full[s16]);
          mbar_arrive(&bb.ring_empty[vslot]);             // this warp is done reading the e4m3 slot
        }
      }
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsSoftmax) : "memory");
    // ------------------------------------------------------------ softmax groups 0 and 1
    const int tile = warp >> 2;                       // 0 or 1
    const int r = threadIdx.x & 127;                  // row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + tile * 128;
    const uint32_t tO = tmem + lane_base + 256 + tile * 128;

    bool ok = true;
    uint32_t jg = 0;                                  // this CTA's tile count
    int units = 0;
    for (int u = u_first; fwd_more_units<kPersist>(u, u_first, u_end, ok); u = fwd_unit_index<kPersist>(++units)) {
      const FwdUnit w = fwd_unit(args, u);
      const int n_kv = w.n_kv, sk = w.sk, bh = w.bh;
      const int row = w.q_row0 + tile * kBlockM + r;
      const int kv_limit = args.causal ? min(sk - 1, row + (sk - args.Sq)) : sk - 1;
      const bool fused = args.fused_blocks > 1;
      // Score factor c (base 2) and, for e4m3, the V descale v_scale the
      // epilogue applies; with fused e4m3 blocks both change per block: c_b
      // per tile, and block b's probabilities enter P V scaled by
      // vd_b / v_scale (v_scale = the largest of the unit's V descales) through
      // the exponent offset lg_pv = log2(vd_b / v_scale) <= 0, its row sum by
      // inv_pv = v_scale / vd_b.
      const size_t bhkv = (size_t)args.B * args.Hkv;
      float cq = args.scale_log2, c = cq;
      float v_scale = 1.f, lg_pv = 0.f, inv_pv = 1.f;
      if (kFp8) {
        cq *= __ldg(&args.q_descale[bh]);
        const size_t d0 = (size_t)(args.block_offset + w.blk) * bhkv + w.kvh;
        c = cq * __ldg(&args.k_descale[d0]);
        v_scale = __ldg(&args.v_descale[d0]);
        if (fused) {
          for (int b = 1; b < args.fused_blocks; ++b)
            v_scale = fmaxf(v_scale, __ldg(&args.v_descale[(size_t)b * bhkv + w.kvh]));
          const float vd0 = __ldg(&args.v_descale[d0]);
          lg_pv = __log2f(vd0 / v_scale);
          inv_pv = v_scale / vd0;
        }
      }

      float m = -INFINITY;     // running max of x = s * c (base-2 units)
      float l = 0.f;           // running sum of 2^(x - m)
      int fb = 0, flt = 0, fsk = args.sk[0], fnt = fwd_block_tiles(fsk);   // fused: block / tile walk
      for (int j = 0; j < n_kv; ++j, ++jg) {
        // last unmasked key column of this tile (>= 127: none masked)
        int lim;
        float c_t = c, lg_t = lg_pv, inv_t = inv_pv;    // this tile's block factors
        if (fused) {
          lim = fsk - flt * kBlockN - 1;
          if (++flt == fnt && j + 1 < n_kv) {
            ++fb;
            flt = 0;
            fsk = args.sk[fb];
            fnt = fwd_block_tiles(fsk);
            if (kFp8) {                                  // the next tile starts block fb
              const size_t db = (size_t)fb * bhkv + w.kvh;
              c = cq * __ldg(&args.k_descale[db]);
              const float vdb = __ldg(&args.v_descale[db]);
              lg_pv = __log2f(vdb / v_scale);
              inv_pv = v_scale / vdb;
            }
          }
        } else {
          lim = kv_limit - j * kBlockN;
        }
        ok = warp_wait(&bb.s_full[tile], jg & 1, kSiteSFull);
        if (!ok) break;
        tc_fence_after();
        float s[128];
        {
          uint32_t uu[128];
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, *reinterpret_cast<uint32_t(*)[32]>(&uu[q * 32]));
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 128; ++e) s[e] = __uint_as_float(uu[e]);
        }
        const bool masked = lim < kBlockN - 1;
        if (masked) {
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e > lim) s[e] = -INFINITY;
        }
        // row max: eight independent three-input chains
        float mx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = fmax3(s[i], s[8 + i], s[16 + i]);
#pragma unroll
        for (int e = 24; e < 120; e += 16) {
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = fmax3(mx[i], s[e + i], s[e + 8 + i]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], s[120 + i]);
        const float m_tile = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * c_t;
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
            uint32_t uq[32];
            tmem_ld32(tO + q * 32, uq);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) uq[e] = __float_as_uint(__uint_as_float(uq[e]) * f);
            tmem_st32(tO + q * 32, uq);
          }
          tmem_wait_st();
        }
        const float mneg = ((m == -INFINITY) ? 0.f : -m) + lg_t;
        const float2 c2 = make_float2(c_t, c_t), mneg2 = make_float2(mneg, mneg);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        // Two halves of 64 keys: each half is written to TMEM and released to the
        // MMA warp as soon as it is ready, so P V can start on keys 0..63.
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) {
            const int e = half * 64 + 2 * e2;
            const float2 x = __ffma2_rn(make_float2(s[e], s[e + 1]), c2, mneg2);
            const float2 p = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            pk[e2] = kFp8 ? pack_f16x2(p.x, p.y) : pack_bf16x2(p.x, p.y);
            acc[e2 & 3] = __fadd2_rn(acc[e2 & 3], p);
          }
          __syncwarp();
          tmem_st32(tS + half * 32, pk);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bb.p_full[tile * 2 + half]);
        }
        const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
        const float2 a2 = __fadd2_rn(a01, a23);
        l += (a2.x + a2.y) * inv_t;
      }
      if (ok) ok = warp_wait(&bb.o_done[tile], units & 1, kSiteODone);
      if (!ok) break;
      // Epilogue.  The next unit's first P V (which overwrites O) waits for this
      // group's first P of that unit, so these O reads complete first.
      tc_fence_after();
      const float inv_l = (l > 0.f) ? (v_scale / l) : 0.f;
      const bool store = row < args.Sq;
      const size_t orow = ((size_t)bh * args.Sq + (size_t)row) * kHeadDim;
      const size_t part = (size_t)(args.block_offset + w.blk);
      if constexpr (kEpiStage) {
        // O through shared memory, stored by TMA in two passes of 64 columns:
        // each thread writes its row (128 bytes a pass, 16-byte chunks at
        // chunk ^ (row & 7), the 128-byte swizzle of the tensor map), and each
        // warp's lane 0 stores the warp's 32 x 64 box as soon as the warp has
        // written it; before the warp writes again, lane 0 waits until its
        // previous store has read the rows.  Rows past Sq are clipped.
        uint8_t* srow = smem + L::kEpiOff + tile * L::kEpiTileBytes + r * 128;
        const uint8_t* wbox = smem + L::kEpiOff + tile * L::kEpiTileBytes + (warp & 3) * 32 * 128;
        const int wrow0 = w.q_row0 + tile * kBlockM + (warp & 3) * 32;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          uint32_t uq[64];
          __syncwarp();
          tmem_ld32(tO + h * 64, *reinterpret_cast<uint32_t(*)[32]>(&uq[0]));
          tmem_ld32(tO + h * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&uq[32]));
          tmem_wait_ld();
          if (lane == 0) bulk_wait_read();             // this warp's last store has read its rows
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(srow + ((c ^ (r & 7)) << 4)) = make_uint4(
                pack_bf16x2(__uint_as_float(uq[8 * c]) * inv_l, __uint_as_float(uq[8 * c + 1]) * inv_l),
                pack_bf16x2(__uint_as_float(uq[8 * c + 2]) * inv_l, __uint_as_float(uq[8 * c + 3]) * inv_l),
                pack_bf16x2(__uint_as_float(uq[8 * c + 4]) * inv_l, __uint_as_float(uq[8 * c + 5]) * inv_l),
                pack_bf16x2(__uint_as_float(uq[8 * c + 6]) * inv_l, __uint_as_float(uq[8 * c + 7]) * inv_l));
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the TMA store reads it
          __syncwarp();
          if (lane == 0 && wrow0 < args.Sq) {
            tma_store_3d(&args.tm_o, wbox, h * 64, wrow0, bh);
            bulk_commit();
          }
        }
      } else {
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t uq[32];
        __syncwarp();
        tmem_ld32(tO + q * 32, uq);
        tmem_wait_ld();
        if (store) {
          if (kPartial) {
            float* dst = reinterpret_cast<float*>(args.out) +
                         part * ((size_t)args.B * args.Hq * args.Sq * kHeadDim) + orow + q * 32;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dst + e) =
                  make_float4(__uint_as_float(uq[e]) * inv_l, __uint_as_float(uq[e + 1]) * inv_l,
                              __uint_as_float(uq[e + 2]) * inv_l, __uint_as_float(uq[e + 3]) * inv_l);
          } else {
            uint32_t pkd[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pkd[e] = pack_bf16x2(__uint_as_float(uq[2 * e]) * inv_l, __uint_as_float(uq[2 * e + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(args.out) + orow + q * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pkd[4 * e], pkd[4 * e + 1], pkd[4 * e + 2], pkd[4 * e + 3]);
          }
        }
      }
      }
      if (store) {
        const float lse2 = (l > 0.f) ? (m + __log2f(l)) : -INFINITY;
        float* lse = args.lse + (kPartial ? part * ((size_t)args.B * args.Hq * args.Sq) : 0);
        lse[(size_t)bh * args.Sq + row] = lse2 * 0.69314718055994530942f;
      }
    }
    if (kEpiStage && lane == 0) bulk_wait_all();    // O stores complete before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// e4m3 -> fp16 widening of the V operand of the e4m3 forward (exact: every
// e4m3 value is an fp16 value).  One 16-byte group of codes per thread and
// step, grid-stride; HBM-bound.
__global__ void __launch_bounds__(256) widen_e4m3_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                         long long n16) {
  for (long long i = (long long)blockIdx.x * 256 + threadIdx.x; i < n16; i += (long long)gridDim.x * 256) {
    const uint4 in = __ldg(&src[i]);
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    uint32_t o[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      o[2 * q] = e4m3x2_to_f16x2((uint16_t)(w[q] & 0xFFFFu));
      o[2 * q + 1] = e4m3x2_to_f16x2((uint16_t)(w[q] >> 16));
    }
    dst[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
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
