// hattn.cu -- host side of libhattn.so: argument checks, TMA descriptor
// encoding, launch configuration and the extern "C" entry points of hattn.h.
//
// The library allocates no device memory (its one static array serves
// attn_bwd_noalloc) and never synchronises the host except in
// attn_get_device_error().  cuTensorMapEncodeTiled is resolved
// through cudaGetDriverEntryPoint so the library links only the static CUDA
// runtime and loads on machines without a GPU driver (calls then fail with
// HATTN_ELAUNCH).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <cfloat>
#include <climits>
#include <mutex>

#include "../../include/hattn.h"
#include "bwd_kernel.cuh"
#include "bwd_dq_gemm_kernel.cuh"
#include "bwd_onepass_kernel.cuh"
#include "fwd_kernel.cuh"
#include "per_device.h"
#include "prep_kernel.cuh"

namespace hattn {

// Failure-detection self-test: one warp waits on a barrier that nothing ever
// arrives on; the bounded wait must give up after limit_ns, record the site in
// the error word and let the kernel return normally.
constexpr int kSiteSelfTest = 0x7F;
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_for(&bar, 0, kSiteSelfTest, limit_ns);
  __syncwarp();
}

// Self-test of the bounded counter wait the one-pass backward orders its dQ
// additions with: one thread waits for a counter that nothing increments.
__global__ void selftest_counter_kernel(const uint32_t* counter, unsigned long long limit_ns) {
  if (threadIdx.x == 0) wait_counter_geq(counter, 1u, kSiteOpOrder, limit_ns);
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename K>
bool set_smem_attr(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

// Number of SMs of the current device, looked up once per device.
int device_sm_count() {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return -1;
  if (dev < kMaxDevices) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev < kMaxDevices) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

int current_device() {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

template <bool kFp8, bool kPartial, bool kPersist, bool kWidenV>
int launch_fwd_grid(const FwdArgs& a, int grid, cudaStream_t st) {
  using L = FwdSmemLayout<kFp8, kWidenV, kPersist && !kPartial>;
  auto kernel = attn_fwd_kernel<kFp8, kPartial, kPersist, kWidenV>;
  // once per device: the shared-memory limit, and the check that the
  // setmaxnreg split fits the registers the launch holds
  static PerDeviceOnce setup;
  if (!setup.ensure(current_device(), [&] {
        cudaFuncAttributes fa;
        return set_smem_attr(kernel, L::kAlloc) && cudaFuncGetAttributes(&fa, kernel) == cudaSuccess &&
               fa.numRegs * kFwdThreads >= kRegsNeeded;
      }))
    return HATTN_ELAUNCH;
  // a programmatic dependent of the grid before it on the stream (the kernel
  // waits for that grid before touching global memory)
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kFwdThreads);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = st;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, a) != cudaSuccess) return HATTN_ELAUNCH;
  return cudaGetLastError() == cudaSuccess ? HATTN_OK : HATTN_ELAUNCH;
}

// Units of 256 query rows x one KV block.  Short units (on average at most 8
// KV tiles: up to 8 without a mask, up to 16 under a causal mask, whose units
// average half the longest) go to the persistent kernel, one CTA per SM, which
// overlaps each unit's epilogue and the next unit's Q load with the running
// MMAs and deals the heaviest-first unit list out in snake order; long units
// go one CTA per unit, ordered heaviest first, and the hardware scheduler
// balances them.
constexpr int kPersistMaxKvTiles = 8;

template <bool kFp8, bool kPartial, bool kWidenV = false>
int launch_fwd(const FwdArgs& a, int n_blocks_in_launch, long long max_tiles, cudaStream_t st) {
  const long long units = (long long)a.n_qpairs * a.B * a.Hq * n_blocks_in_launch;
  if (units <= 0 || units > INT_MAX) return HATTN_EUNSUPPORTED;
  const int sms = device_sm_count();
  if (sms <= 0) return HATTN_ELAUNCH;
  FwdArgs args = a;
  args.total_units = (int)units;
  const bool persist = max_tiles <= (a.causal ? 2 : 1) * kPersistMaxKvTiles && units > sms;
  if (persist) return launch_fwd_grid<kFp8, kPartial, true, kWidenV>(args, sms, st);
  return launch_fwd_grid<kFp8, kPartial, false, kWidenV>(args, (int)units, st);
}

int check_common(int B, int Hq, int Hkv, int Sq, int D, float scale) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || D <= 0) return HATTN_EINVAL;
  if (Hq % Hkv != 0) return HATTN_EINVAL;
  if (!(scale > 0.f && scale <= FLT_MAX)) return HATTN_EINVAL;   // also refuses NaN and +inf
  if (D != kHeadDim) return HATTN_EUNSUPPORTED;
  return HATTN_OK;
}

int check_descales(int dtype, const float* qd, const float* kd, const float* vd) {
  if (dtype == HATTN_BF16) return (qd || kd || vd) ? HATTN_EINVAL : HATTN_OK;
  if (dtype == HATTN_E4M3) {
    return (qd && kd && vd) ? HATTN_OK : HATTN_EINVAL;   // read as 4-byte scalars
  }
  return HATTN_EINVAL;
}

// Guard against 32-bit overflow of grid dimensions and row counts.
bool sizes_fit(long long B, long long H, long long S) {
  return B * H <= 65535LL * 1024 && B * H * S < (1LL << 40) && S < (1LL << 30);
}

// The backward's launch sizes: the persistent dQ and dK/dV kernels count
// their units (B*Hq*ceil(Sq/128), B*Hkv*ceil(Sk/128)) in an int, and the Delta
// kernel takes one CTA per 64 rows in grid x.  (launch_bwd also bounds the
// steps one persistent CTA counts.)
bool bwd_sizes_ok(int B, int Hq, int Hkv, int Sq, int Sk) {
  if (!sizes_fit(B, Hq, Sq) || !sizes_fit(B, Hkv, Sk)) return false;
  const long long rows = (long long)B * Hq * Sq;
  if ((long long)B * Hq * ((Sq + kTile - 1) / kTile) > INT_MAX) return false;
  if ((long long)B * Hkv * ((Sk + kTile - 1) / kTile) > INT_MAX) return false;
  return (rows + kDeltaRowsPerCta - 1) / kDeltaRowsPerCta <= INT_MAX;
}

}  // namespace

// 3-D view (D, S, heads) of a [.., heads, S, D] tensor, box (box_x, box_rows, 1 head),
// 128-byte swizzle.  box_x * elt_bytes == 128.
bool encode_rows_typed(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t rows, uint64_t heads,
                       uint32_t box_rows = kBlockM) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const uint64_t eb = dt == CU_TENSOR_MAP_DATA_TYPE_UINT8 ? 1 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)(kHeadDim * eb), (cuuint64_t)(rows * kHeadDim * eb)};
  cuuint32_t box[3] = {(cuuint32_t)(128 / eb), (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_rows(CUtensorMap* m, const void* base, bool e4m3, uint64_t rows, uint64_t heads) {
  return encode_rows_typed(m, base, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rows,
                           heads);
}

}  // namespace hattn

using namespace hattn;

extern "C" {

size_t attn_fwd_workspace_size(int B, int Hkv, int Sk, int D, int dtype) {
  if (B <= 0 || Hkv <= 0 || Sk <= 0 || D <= 0 || dtype != HATTN_E4M3) return 0;
  return (size_t)B * Hkv * Sk * D * 2;
}

}  // extern "C"

namespace {

// Forward.  e4m3 with `v16` (B*Hkv*Sk*D*2 bytes): V is widened to fp16 there by
// a separate pass first; e4m3 without it: V is widened in shared memory inside
// the attention kernel (nothing allocated).  v16 is unused for bf16.
int attn_fwd_core(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                  int Sq, int Sk, float scale, int causal, int dtype, const float* q_descale,
                  const float* k_descale, const float* v_descale, void* v16, cudaStream_t st) {
  const bool fp8 = dtype == HATTN_E4M3;
  static thread_local FwdArgs a;   // ~8 KB: kept off the stack
  memset(&a, 0, sizeof(a));
  if (!encode_rows(&a.tm_q, q, fp8, Sq, (uint64_t)B * Hq)) return HATTN_ELAUNCH;
  if (!encode_rows_typed(&a.tm_o, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Sq, (uint64_t)B * Hq, 32))
    return HATTN_ELAUNCH;
  if (!encode_rows(&a.tm_k[0], k, fp8, Sk, (uint64_t)B * Hkv)) return HATTN_ELAUNCH;
  if (fp8 && !v16) {
    if (!encode_rows(&a.tm_v[0], v, true, Sk, (uint64_t)B * Hkv)) return HATTN_ELAUNCH;
  } else if (fp8) {
    // V widened to fp16 once (exact), read by the attention kernel's P V MMAs
    const long long n16 = (long long)B * Hkv * Sk * kHeadDim / 16;
    const int sms = device_sm_count();
    if (sms <= 0) return HATTN_ELAUNCH;
    const long long want = (n16 + 255) / 256;
    const int grid = (int)(want < 8LL * sms ? want : 8LL * sms);
    widen_e4m3_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(v), reinterpret_cast<uint4*>(v16), n16);
    if (cudaGetLastError() != cudaSuccess) return HATTN_ELAUNCH;
    if (!encode_rows_typed(&a.tm_v[0], v16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Sk, (uint64_t)B * Hkv))
      return HATTN_ELAUNCH;
  } else if (!encode_rows(&a.tm_v[0], v, false, Sk, (uint64_t)B * Hkv)) {
    return HATTN_ELAUNCH;
  }
  a.sk[0] = Sk;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Sq = Sq;
  a.causal = causal ? 1 : 0;
  a.n_qpairs = (Sq + kQTilesPerCta * kBlockM - 1) / (kQTilesPerCta * kBlockM);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.out = out;
  a.lse = lse;
  a.q_descale = q_descale; a.k_descale = k_descale; a.v_descale = v_descale;
  a.block_offset = 0;
  const long long kv_tiles = (Sk + kBlockN - 1) / kBlockN;
  if (!fp8) return launch_fwd<false, false>(a, 1, kv_tiles, st);
  return v16 ? launch_fwd<true, false>(a, 1, kv_tiles, st) : launch_fwd<true, false, true>(a, 1, kv_tiles, st);
}

int check_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv, int Sq,
              int Sk, int D, float scale, int causal, int dtype, const float* q_descale, const float* k_descale,
              const float* v_descale) {
  if (!q || !k || !v || !out || !lse) return HATTN_EINVAL;
  int rc = check_common(B, Hq, Hkv, Sq, D, scale);
  if (rc) return rc;
  if (Sk <= 0) return HATTN_EINVAL;
  if ((rc = check_descales(dtype, q_descale, k_descale, v_descale))) return rc;
  if (causal && Sq > Sk) return HATTN_EUNSUPPORTED;
  if (!sizes_fit(B, Hq, Sq) || !sizes_fit(B, Hkv, Sk)) return HATTN_EUNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse)) return HATTN_EALIGN;
  return HATTN_OK;
}

}  // namespace

extern "C" {

int attn_fwd_ws(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv, int Sq,
                int Sk, int D, float scale, int causal, int dtype, const float* q_descale, const float* k_descale,
                const float* v_descale, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_fwd(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, dtype, q_descale, k_descale, v_descale);
  if (rc) return rc;
  const size_t need = attn_fwd_workspace_size(B, Hkv, Sk, D, dtype);
  if (need) {
    if (!workspace) return HATTN_EINVAL;
    if (!aligned16(workspace)) return HATTN_EALIGN;
    if (workspace_bytes < need) return HATTN_EWORKSPACE;
  }
  return attn_fwd_core(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, scale, causal, dtype, q_descale, k_descale, v_descale,
                       workspace, reinterpret_cast<cudaStream_t>(stream));
}

int attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv, int Sq,
             int Sk, int D, float scale, int causal, int dtype, const float* q_descale, const float* k_descale,
             const float* v_descale, void* stream) {
  int rc = check_fwd(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, dtype, q_descale, k_descale, v_descale);
  if (rc) return rc;
  // e4m3 without a caller workspace: V is widened inside the attention kernel
  return attn_fwd_core(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, scale, causal, dtype, q_descale, k_descale, v_descale,
                       nullptr, reinterpret_cast<cudaStream_t>(stream));
}

int attn_quantize_e4m3(const void* x, void* codes, float* descale, int B, int H, int S, int D, int rmsnorm,
                       double eps, void* stream) {
  if (!x || !codes || !descale) return HATTN_EINVAL;
  if (B <= 0 || H <= 0 || S <= 0 || D <= 0) return HATTN_EINVAL;
  const float eps32 = (float)eps;                  // the normalisation runs in fp32
  if (rmsnorm && !(eps32 > 0.f && eps32 < 3.0e38f)) return HATTN_EINVAL;
  if (D != kPrepD) return HATTN_EUNSUPPORTED;
  if (!sizes_fit(B, H, S) || (S + kPrepRowsPerCta - 1) / kPrepRowsPerCta > INT_MAX) return HATTN_EUNSUPPORTED;
  if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(descale) & 3u)) return HATTN_EALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int bh = B * H;
  const dim3 grid((S + kPrepRowsPerCta - 1) / kPrepRowsPerCta, bh < 65535 ? bh : 65535);   // heads strided over y
  if (cudaMemsetAsync(descale, 0, (size_t)bh * sizeof(float), st) != cudaSuccess) return HATTN_ELAUNCH;
  const uint16_t* xs = reinterpret_cast<const uint16_t*>(x);
  unsigned int* amax = reinterpret_cast<unsigned int*>(descale);
  uint8_t* cs = reinterpret_cast<uint8_t*>(codes);
  const int rms = rmsnorm ? 1 : 0;
  if (bh <= 65535) {
    prep_amax_kernel<false><<<grid, kPrepThreads, 0, st>>>(xs, amax, S, bh, rms, eps32);
    prep_quantize_kernel<false><<<grid, kPrepThreads, 0, st>>>(xs, cs, descale, S, bh, rms, eps32);
  } else {
    prep_amax_kernel<true><<<grid, kPrepThreads, 0, st>>>(xs, amax, S, bh, rms, eps32);
    prep_quantize_kernel<true><<<grid, kPrepThreads, 0, st>>>(xs, cs, descale, S, bh, rms, eps32);
  }
  return cudaGetLastError() == cudaSuccess ? HATTN_OK : HATTN_ELAUNCH;
}

size_t attn_fwd_kvblocks_workspace_size(int B, int Hq, int Sq, int D, int n_blocks) {
  if (B <= 0 || Hq <= 0 || Sq <= 0 || D <= 0 || n_blocks <= 0) return 0;
  if (n_blocks <= kMaxKvBlocks) return 0;   // one launch folds the blocks in order: no partials
  return (size_t)n_blocks * (size_t)B * Hq * Sq * ((size_t)D + 1) * sizeof(float);
}

int attn_fwd_kvblocks(const void* q, const void* const* k_blocks, const void* const* v_blocks, const int* blk_len,
                      int n_blocks, void* out, float* lse, int B, int Hq, int Hkv, int Sq, int D, float scale,
                      int dtype, const float* q_descale, const float* k_descale, const float* v_descale,
                      void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k_blocks || !v_blocks || !blk_len || !out || !lse) return HATTN_EINVAL;
  if (n_blocks <= 0) return HATTN_EINVAL;
  int rc = check_common(B, Hq, Hkv, Sq, D, scale);
  if (rc) return rc;
  if ((rc = check_descales(dtype, q_descale, k_descale, v_descale))) return rc;
  if (!sizes_fit(B, Hq, Sq)) return HATTN_EUNSUPPORTED;
  const bool fp8 = dtype == HATTN_E4M3;
  for (int i = 0; i < n_blocks; ++i) {
    if (!k_blocks[i] || !v_blocks[i]) return HATTN_EINVAL;
    if (blk_len[i] <= 0) return HATTN_EUNSUPPORTED;
    if (!sizes_fit(B, Hkv, blk_len[i])) return HATTN_EUNSUPPORTED;
    if (!aligned16(k_blocks[i]) || !aligned16(v_blocks[i])) return HATTN_EALIGN;
  }
  const size_t need = attn_fwd_kvblocks_workspace_size(B, Hq, Sq, D, n_blocks);
  if (need && !workspace) return HATTN_EINVAL;
  if (!aligned16(q) || !aligned16(out) || !aligned16(lse) || (need && !aligned16(workspace))) return HATTN_EALIGN;
  if (workspace_bytes < need) return HATTN_EWORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  static thread_local FwdArgs a;

  if (n_blocks <= kMaxKvBlocks) {
    // One unit per (256 query rows, b, h) runs over all blocks in ascending
    // order: its online softmax folds block after block, so no per-block
    // partials are written and no merge pass is needed.
    memset(&a, 0, sizeof(a));
    if (!encode_rows(&a.tm_q, q, fp8, Sq, (uint64_t)B * Hq)) return HATTN_ELAUNCH;
    if (!encode_rows_typed(&a.tm_o, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Sq, (uint64_t)B * Hq, 32))
      return HATTN_ELAUNCH;
    long long tiles = 0;
    for (int i = 0; i < n_blocks; ++i) {
      if (!encode_rows(&a.tm_k[i], k_blocks[i], fp8, blk_len[i], (uint64_t)B * Hkv)) return HATTN_ELAUNCH;
      if (!encode_rows(&a.tm_v[i], v_blocks[i], fp8, blk_len[i], (uint64_t)B * Hkv)) return HATTN_ELAUNCH;
      a.sk[i] = blk_len[i];
      tiles += (blk_len[i] + kBlockN - 1) / kBlockN;
    }
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Sq = Sq;
    a.causal = 0;
    a.n_qpairs = (Sq + kQTilesPerCta * kBlockM - 1) / (kQTilesPerCta * kBlockM);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.out = out;
    a.lse = lse;
    a.q_descale = q_descale; a.k_descale = k_descale; a.v_descale = v_descale;
    a.fused_blocks = n_blocks;
    a.fused_tiles = (int)tiles;   // < 32 * 2^23
    if (n_blocks == 1) a.fused_blocks = 0;   // a single block is a plain forward
    return fp8 ? launch_fwd<true, false, true>(a, 1, tiles, st) : launch_fwd<false, false>(a, 1, tiles, st);
  }

  const long long rows = (long long)B * Hq * Sq;
  if ((rows + 7) / 8 > INT_MAX) return HATTN_EUNSUPPORTED;   // the merge takes 8 rows per CTA in grid x
  float* o_parts = reinterpret_cast<float*>(workspace);
  float* lse_parts = o_parts + (size_t)n_blocks * rows * kHeadDim;
  for (int first = 0; first < n_blocks; first += kMaxKvBlocks) {
    const int cnt = n_blocks - first < kMaxKvBlocks ? n_blocks - first : kMaxKvBlocks;
    memset(&a, 0, sizeof(a));
    if (!encode_rows(&a.tm_q, q, fp8, Sq, (uint64_t)B * Hq)) return HATTN_ELAUNCH;
    int max_len = 0;
    for (int i = 0; i < cnt; ++i) {
      max_len = blk_len[first + i] > max_len ? blk_len[first + i] : max_len;
      if (!encode_rows(&a.tm_k[i], k_blocks[first + i], fp8, blk_len[first + i], (uint64_t)B * Hkv))
        return HATTN_ELAUNCH;
      if (!encode_rows(&a.tm_v[i], v_blocks[first + i], fp8, blk_len[first + i], (uint64_t)B * Hkv))
        return HATTN_ELAUNCH;
      a.sk[i] = blk_len[first + i];
    }
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Sq = Sq;
    a.causal = 0;
    a.n_qpairs = (Sq + kQTilesPerCta * kBlockM - 1) / (kQTilesPerCta * kBlockM);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.out = o_parts;
    a.lse = lse_parts;
    a.q_descale = q_descale; a.k_descale = k_descale; a.v_descale = v_descale;
    a.block_offset = first;
    const long long max_tiles = (max_len + kBlockN - 1) / kBlockN;
    rc = fp8 ? launch_fwd<true, true, true>(a, cnt, max_tiles, st) : launch_fwd<false, true>(a, cnt, max_tiles, st);
    if (rc) return rc;
  }
  const unsigned grid = (unsigned)((rows + 7) / 8);
  lse_merge_kernel<<<grid, 256, 0, st>>>(o_parts, lse_parts, n_blocks, rows, reinterpret_cast<uint16_t*>(out), lse);
  return cudaGetLastError() == cudaSuccess ? HATTN_OK : HATTN_ELAUNCH;
}

namespace {
// attn_bwd's workspace: Delta (one fp32 per query row), then at the next
// 256-byte boundary the dQ kernel's unit counter.
size_t bwd_sched_offset(int B, int Hq, int Sq) { return ((size_t)B * Hq * Sq * sizeof(float) + 255) & ~(size_t)255; }
}  // namespace

size_t attn_bwd_workspace_size(int B, int Hq, int Sq) {
  if (B <= 0 || Hq <= 0 || Sq <= 0) return 0;
  return bwd_sched_offset(B, Hq, Sq) + 256;
}

int attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
             void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
             void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || !workspace) return HATTN_EINVAL;
  int rc = check_common(B, Hq, Hkv, Sq, D, scale);
  if (rc) return rc;
  if (Sk <= 0) return HATTN_EINVAL;
  if (causal && Sq > Sk) return HATTN_EUNSUPPORTED;
  if (!bwd_sizes_ok(B, Hq, Hkv, Sq, Sk)) return HATTN_EUNSUPPORTED;
  const void* ptrs[] = {q, k, v, out, lse, dout, dq, dk, dv, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return HATTN_EALIGN;
  if (workspace_bytes < attn_bwd_workspace_size(B, Hq, Sq)) return HATTN_EWORKSPACE;
  const int sms = device_sm_count();
  if (sms <= 0) return HATTN_ELAUNCH;
  uint32_t* sched = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + bwd_sched_offset(B, Hq, Sq));
  return launch_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, Sq, Sk, scale, causal != 0,
                    reinterpret_cast<float*>(workspace), sched, sms, reinterpret_cast<cudaStream_t>(stream));
}

size_t attn_bwd_dsbuf_workspace_size(int B, int Hq, int Sq, int Sk) {
  if (B <= 0 || Hq <= 0 || Sq <= 0 || Sk <= 0) return 0;
  size_t off_ds = 0;
  return dsbuf_workspace_parts(B, Hq, Sq, Sk, &off_ds);
}

int attn_bwd_dsbuf(const void* q, const void* k, const void* v, const void* out, const float* lse,
                   const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                   float scale, int causal, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || !workspace) return HATTN_EINVAL;
  int rc = check_common(B, Hq, Hkv, Sq, D, scale);
  if (rc) return rc;
  if (Sk <= 0) return HATTN_EINVAL;
  if (causal && Sq > Sk) return HATTN_EUNSUPPORTED;
  if (!bwd_sizes_ok(B, Hq, Hkv, Sq, Sk)) return HATTN_EUNSUPPORTED;
  const void* ptrs[] = {q, k, v, out, lse, dout, dq, dk, dv, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return HATTN_EALIGN;
  if (workspace_bytes < attn_bwd_dsbuf_workspace_size(B, Hq, Sq, Sk)) return HATTN_EWORKSPACE;
  const int sms = device_sm_count();
  if (sms <= 0) return HATTN_ELAUNCH;
  const int r = launch_bwd_dsbuf(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, Sq, Sk, scale, causal != 0,
                                 workspace, sms, reinterpret_cast<cudaStream_t>(stream));
  return r == -2 ? HATTN_EUNSUPPORTED : (r ? HATTN_ELAUNCH : HATTN_OK);
}

size_t attn_bwd_onepass_workspace_size(int B, int Hq, int Sq) {
  if (B <= 0 || Hq <= 0 || Sq <= 0) return 0;
  size_t off_acc = 0, off_cnt = 0;
  return onepass_workspace_parts(B, Hq, Sq, &off_acc, &off_cnt);
}

int attn_bwd_onepass(const void* q, const void* k, const void* v, const void* out, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                     float scale, int causal, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || !workspace) return HATTN_EINVAL;
  int rc = check_common(B, Hq, Hkv, Sq, D, scale);
  if (rc) return rc;
  if (Sk <= 0) return HATTN_EINVAL;
  if (causal && Sq > Sk) return HATTN_EUNSUPPORTED;
  if (!bwd_sizes_ok(B, Hq, Hkv, Sq, Sk)) return HATTN_EUNSUPPORTED;
  const void* ptrs[] = {q, k, v, out, lse, dout, dq, dk, dv, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return HATTN_EALIGN;
  if (workspace_bytes < attn_bwd_onepass_workspace_size(B, Hq, Sq)) return HATTN_EWORKSPACE;
  const int sms = device_sm_count();
  if (sms <= 0) return HATTN_ELAUNCH;
  return launch_bwd_onepass(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, Sq, Sk, scale, causal != 0, workspace,
                            sms, reinterpret_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------- allocation-free backward
// Scratch for attn_bwd_noalloc: the Delta vector (one fp32 per query row),
// followed by the dQ kernel's unit counter (in the last 256 bytes), lives in
// this file-scope device array instead of a caller-provided workspace.
// Every GPU that loads the library holds it until the process exits.  In host
// code the name g_noalloc_delta is only a host-side stand-in; the device
// address comes from cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) float g_noalloc_delta[HATTN_NOALLOC_MAX_ROWS + 64];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_delta on the current device, or nullptr.
float* noalloc_scratch() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_delta) != cudaSuccess || !p) return nullptr;
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  return g_noalloc_ptr[dev];
}
}  // namespace

int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* out, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk, int D,
                     float scale, int causal, void* stream) {
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv) return HATTN_EINVAL;
  int rc = check_common(B, Hq, Hkv, Sq, D, scale);
  if (rc) return rc;
  if (Sk <= 0) return HATTN_EINVAL;
  if (causal && Sq > Sk) return HATTN_EUNSUPPORTED;
  if (!bwd_sizes_ok(B, Hq, Hkv, Sq, Sk)) return HATTN_EUNSUPPORTED;
  if ((long long)B * Hq * Sq > (long long)HATTN_NOALLOC_MAX_ROWS) return HATTN_EWORKSPACE;
  const void* ptrs[] = {q, k, v, out, lse, dout, dq, dk, dv};
  for (const void* p : ptrs)
    if (!aligned16(p)) return HATTN_EALIGN;
  float* delta = noalloc_scratch();
  if (!delta) return HATTN_ELAUNCH;
  // Delta is fully rewritten for every row this call reads, so the array needs
  // no clearing between calls.
  const int sms = device_sm_count();
  if (sms <= 0) return HATTN_ELAUNCH;
  uint32_t* sched = reinterpret_cast<uint32_t*>(delta + HATTN_NOALLOC_MAX_ROWS);
  return launch_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, Hq, Hkv, Sq, Sk, scale, causal != 0, delta, sched, sms,
                    reinterpret_cast<cudaStream_t>(stream));
}

int attn_selftest_bounded_wait(void* stream, unsigned int timeout_us) {
  if (timeout_us == 0 || timeout_us > 10000000u) return HATTN_EINVAL;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(1000ull * timeout_us);
  return cudaGetLastError() == cudaSuccess ? HATTN_OK : HATTN_ELAUNCH;
}

int attn_selftest_counter_wait(const void* counter, void* stream, unsigned int timeout_us) {
  if (!counter || timeout_us == 0 || timeout_us > 10000000u) return HATTN_EINVAL;
  if (reinterpret_cast<uintptr_t>(counter) & 3u) return HATTN_EALIGN;
  selftest_counter_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(counter), 1000ull * timeout_us);
  return cudaGetLastError() == cudaSuccess ? HATTN_OK : HATTN_ELAUNCH;
}

int attn_get_device_error(void* stream, int* code_out) {
  if (!code_out) return HATTN_EINVAL;
  *code_out = 0;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return HATTN_ELAUNCH;
  int code = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&code, g_device_error, sizeof(int)) != cudaSuccess) return HATTN_ELAUNCH;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return HATTN_ELAUNCH;
  *code_out = code;
  return HATTN_OK;
}

const char* attn_error_string(int code) {
  switch (code) {
    case HATTN_OK: return "ok";
    case HATTN_EINVAL: return "invalid argument";
    case HATTN_EUNSUPPORTED: return "unsupported request (refused, not approximated)";
    case HATTN_EALIGN: return "device pointer not 16-byte aligned";
    case HATTN_EWORKSPACE: return "workspace too small";
    case HATTN_ELAUNCH: return "CUDA error while encoding or launching";
    case HATTN_EDEVICE: return "a kernel gave up on a bounded wait";
    default: return "unknown error code";
  }
}

}  // extern "C"
