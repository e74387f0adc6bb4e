// bwd_dq_gemm_kernel.cuh -- dQ of the backward from stored dS tiles (sm_100a, bf16).
//
// attn_bwd_dsbuf: the dK/dV kernel of bwd_kernel.cuh, which forms
// dS^T = P^T * (dP^T - Delta) for every (key tile, query tile) pair anyway,
// also writes those bf16 tiles to the workspace.  dQ is then a plain product
//     dQ_i = scale * sum_j dS_ij K_j      (j ascending, one CTA per row block)
// read back from memory, instead of the dQ kernel's recomputation of S, P and
// dP (3 MMAs per tile pair become 1, for an O(Sq x Sk) workspace: RL-Kernel
// PR #319, "What the strict contract costs", shows a deterministic mha_bwd
// that holds such an O(S^2) workspace).  The dS values are the ones the dQ
// kernel would form (bf16 P and dS, fp32 S and dP), summed in the same
// ascending key-tile order: results stay bitwise reproducible and independent
// of batch composition and head split.
//
// Roles: warps 0-3 read the dQ accumulator out (TMEM lane quarter = warp),
// warp 4 producer (per stage a dS^T tile by bulk copy, a K tile by TMA), warp 5 MMA issuer
// and tensor-memory owner.  Persistent, one CTA per SM over (b, q head,
// 128-row query tile) units dealt heaviest first in snake order; the dQ
// accumulator is double-buffered in TMEM, so a unit's read-out overlaps the
// next unit's MMAs.
#pragma once

#include "bwd_kernel.cuh"

namespace hattn {

enum : int { kSiteDsFull = 60, kSiteDsEmpty, kSiteDsAcc, kSiteDsAccFree, kSiteDsDrain };

constexpr int kDsThreads = 192;

struct DsSmem {
  static constexpr int kStages = 3;
  static constexpr int kStageBytes = 2 * kTileBytesBf16;   // dS^T tile, then K tile
  static constexpr int kBars = kStages * kStageBytes;
  static constexpr int kBytes = kBars + 12 * 8;            // 11 barriers and the TMEM slot
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory per CTA");
};

// D (+)= dS K for one key tile (M = 128 queries, N = 128 head dims, K = 128
// keys): A = dS, held as the stored dS^T tile (ds_tile_offset: no-swizzle
// MN-major core blocks of 8 keys x 8 queries, 128 bytes apart along keys and
// 512 along queries; keys 16 k .. 16 k + 15 start at byte 8192 (k / 2) +
// 256 (k % 2)).  For this no-swizzle MN-major operand the descriptor's leading
// byte offset is the step between core blocks along K and the stride byte
// offset the step along MN -- the reverse of the 128-byte-swizzle MN-major
// convention; the parity tests of attn_bwd_dsbuf fail with them swapped.
// B = the K tile, 128-byte swizzle, read MN-major (head dims contiguous,
// 2048 bytes per 16 keys).
__device__ __forceinline__ void mma_tile_ds_k(uint32_t d, uint32_t sa, uint32_t sb, uint32_t acc) {
  constexpr uint32_t idesc = make_idesc_ab(1, 1, 1, 1, 128, 128);
  constexpr uint32_t a_hi = sdesc_hi_noswizzle(512), b_hi = sdesc_hi(1024);
  const uint32_t a_lo = sdesc_lo(sa, 128), b_lo = sdesc_lo(sb, 16384);
#pragma unroll
  for (int k = 0; k < 8; ++k)
    mma_f16_ss2(d, a_lo + (((k >> 1) * 8192 + (k & 1) * 256) >> 4), a_hi, b_lo + k * (2048 >> 4), b_hi, idesc,
                (acc || k > 0) ? 1u : 0u);
}

__global__ void __launch_bounds__(kDsThreads, 1) bwd_dq_gemm_kernel(const __grid_constant__ BwdArgs a) {
  using L = DsSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = warp_id(), lane = lane_id();
  const int nq = (a.Sq + kTile - 1) / kTile, n_kt = (a.Sk + kTile - 1) / kTile;
  const int n_units = nq * a.B * a.Hq;
  const int cta = blockIdx.x, n_cta = gridDim.x;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* full = bars + 0;        // [3] dS^T and K tiles of a step landed
  uint64_t* empty = bars + 3;       // [3] the step's MMAs have read them
  uint64_t* acc_full = bars + 6;    // [2] a unit's dQ is complete in accumulator b
  uint64_t* acc_free = bars + 8;    // [2] the read-out warps are done with accumulator b
  uint64_t* drain = bars + 10;      // every MMA of the CTA has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_free[b], 4); }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 5) { tmem_alloc(tmem_slot, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;     // dQ accumulators: columns [0,128) and [128,256)
  // Launched as a programmatic dependent of the dK/dV kernel, whose dS tiles
  // it reads: nothing in global memory is touched before that grid completes.
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      bool ok = true;
      int gs = 0;                                   // steps loaded by this CTA
      for (int k = 0; ok; ++k) {
        const int t = dq_unit_index(k, cta, n_cta);
        if (t >= n_units) break;
        const DqUnit u = dq_unit(a, t);
        for (int j = 0; j < u.n_kv && ok; ++j, ++gs) {
          const int st = gs % L::kStages;
          if (gs >= L::kStages) ok = mbar_wait(&empty[st], (gs / L::kStages - 1) & 1, kSiteDsEmpty);
          if (!ok) break;
          uint8_t* dst = smem + st * L::kStageBytes;
          mbar_arrive_expect_tx(&full[st], L::kStageBytes);
          bulk_load(dst, a.ds_buf + (((size_t)u.bh * n_kt + j) * nq + u.i) * (kTile * kTile), kTileBytesBf16,
                    &full[st]);                                                          // dS^T tile (j, i)
          tma_tile_bf16(dst + kTileBytesBf16, &a.tm_k, &full[st], j * kTile, u.bkv);     // K tile j
        }
      }
      // every load issued must land before the CTA exits
      for (int g = gs - L::kStages < 0 ? 0 : gs - L::kStages; g < gs; ++g)
        mbar_wait_drain(&full[g % L::kStages], (g / L::kStages) & 1, kSiteDsDrain);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      bool ok = true;
      int gs = 0, ul = 0;
      for (int k = 0; ok; ++k) {
        const int t = dq_unit_index(k, cta, n_cta);
        if (t >= n_units) break;
        const int n = dq_unit(a, t).n_kv;
        const int b = ul & 1;
        if (ul >= 2) ok = mbar_wait(&acc_free[b], ((ul >> 1) - 1) & 1, kSiteDsAccFree);
        if (!ok) break;
        tc_fence_after();
        for (int j = 0; j < n && ok; ++j, ++gs) {
          const int st = gs % L::kStages;
          ok = mbar_wait(&full[st], (gs / L::kStages) & 1, kSiteDsFull);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + st * L::kStageBytes);
          mma_tile_ds_k(tmem + b * 128, sa, sa + kTileBytesBf16, j > 0 ? 1u : 0u);   // dQ += dS K
          mma_commit(&empty[st]);
        }
        if (!ok) break;
        mma_commit(&acc_full[b]);
        ++ul;
      }
      mma_commit(drain);
      mbar_wait_drain(drain, 0, kSiteDsDrain);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- read-out (warps 0-3)
    const int r = warp * 32 + lane;                 // query row within the tile (TMEM lane)
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    bool ok = true;
    int ul = 0;
    for (int k = 0; ok; ++k) {
      const int t = dq_unit_index(k, cta, n_cta);
      if (t >= n_units) break;
      const DqUnit u = dq_unit(a, t);
      const int b = ul & 1;
      ok = warp_wait(&acc_full[b], (ul >> 1) & 1, kSiteDsAcc);
      if (!ok) break;
      tc_fence_after();
      const int qi = u.i * kTile + r;
      const bool valid = qi < a.Sq;
      const size_t ridx = (size_t)u.bh * a.Sq + (valid ? qi : 0);
      store_half_row_bf16(tmem + lane_base + b * 128, a.scale, a.dq + ridx * kHeadDim, valid);
      store_half_row_bf16(tmem + lane_base + b * 128 + 64, a.scale, a.dq + ridx * kHeadDim + 64, valid);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_free[b]);
      ++ul;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) { tc_fence_after(); tmem_dealloc(tmem, 256); }
}

// Workspace of attn_bwd_dsbuf: Delta (256-byte aligned), then the dS^T tiles
// (1024-byte aligned), B*Hq*ceil(Sk/128)*ceil(Sq/128) tiles of 32 KB.
inline size_t dsbuf_workspace_parts(int B, int Hq, int Sq, int Sk, size_t* off_ds) {
  const size_t rows = (size_t)B * Hq * Sq;
  const size_t tiles = (size_t)B * Hq * ((Sk + kTile - 1) / kTile) * ((Sq + kTile - 1) / kTile);
  *off_ds = (rows * sizeof(float) + 1023) & ~(size_t)1023;
  return *off_ds + tiles * (size_t)kTileBytesBf16;
}

inline int launch_bwd_dsbuf(const void* q, const void* k, const void* v, const void* out, const float* lse,
                            const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk,
                            float scale, bool causal, void* workspace, int n_sm, cudaStream_t st) {
  static PerDeviceOnce setup;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -5;
  if (!setup.ensure(dev, [] {
        return cudaFuncSetAttribute(bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    DkdvSmem::kAlloc) == cudaSuccess &&
               cudaFuncSetAttribute(bwd_dq_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    DsSmem::kAlloc) == cudaSuccess;
      }))
    return -5;
  size_t off_ds = 0;
  dsbuf_workspace_parts(B, Hq, Sq, Sk, &off_ds);
  static thread_local BwdArgs a;
  memset(&a, 0, sizeof(a));
  const long long n_kt = (Sk + kTile - 1) / kTile, nq = (Sq + kTile - 1) / kTile;
  if (!encode_rows(&a.tm_q, q, false, Sq, (uint64_t)B * Hq)) return -5;
  if (!encode_rows(&a.tm_do, dout, false, Sq, (uint64_t)B * Hq)) return -5;
  if (!encode_rows(&a.tm_k, k, false, Sk, (uint64_t)B * Hkv)) return -5;
  if (!encode_rows(&a.tm_v, v, false, Sk, (uint64_t)B * Hkv)) return -5;
  a.ds_buf = reinterpret_cast<uint16_t*>(static_cast<char*>(workspace) + off_ds);
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Sq = Sq; a.Sk = Sk;
  a.causal = causal ? 1 : 0;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.lse = lse;
  float* delta = reinterpret_cast<float*>(workspace);
  a.delta = delta;
  a.dq = reinterpret_cast<uint16_t*>(dq);
  a.dk = reinterpret_cast<uint16_t*>(dk);
  a.dv = reinterpret_cast<uint16_t*>(dv);
  const long long rows = (long long)B * Hq * Sq;
  const long long kv_units = n_kt * B * Hkv, dq_units = nq * B * Hq;
  const int kv_grid = (int)std::min<long long>(kv_units, n_sm);
  const int dq_grid = (int)std::min<long long>(dq_units, n_sm);
  // each persistent CTA counts its steps (tile pairs) in an int
  if ((kv_units + kv_grid - 1) / kv_grid * (Hq / Hkv) * nq >= (1LL << 31) ||
      (dq_units + dq_grid - 1) / dq_grid * n_kt >= (1LL << 31))
    return -2;
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
                         reinterpret_cast<const uint16_t*>(dout), delta, rows, static_cast<uint32_t*>(nullptr)) !=
      cudaSuccess)
    return -5;
  cfg.gridDim = dim3((unsigned)kv_grid);
  cfg.blockDim = dim3(kBwdThreads);
  cfg.dynamicSmemBytes = DkdvSmem::kAlloc;
  if (cudaLaunchKernelEx(&cfg, bwd_dkdv_kernel, a) != cudaSuccess) return -5;
  cfg.gridDim = dim3((unsigned)dq_grid);
  cfg.blockDim = dim3(kDsThreads);
  cfg.dynamicSmemBytes = DsSmem::kAlloc;
  if (cudaLaunchKernelEx(&cfg, bwd_dq_gemm_kernel, a) != cudaSuccess) return -5;
  return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

}  // namespace hattn
