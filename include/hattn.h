/*
 * hattn.h -- C ABI of the B200 (sm_100a) fused attention library libhattn.so.
 *
 * The library computes scaled-dot-product multi-head attention
 *     O = softmax(scale * Q K^T [+ causal mask]) V
 * together with the per-row log-sum-exp LSE_i = ln sum_j exp(scale * q_i . k_j),
 * the operation AITER's fmha_v3_fwd performs with return_softmax_lse and
 * q/k/v descales (AITER PR #2911 "F8 fmha ASM gfx950", Test Result), the
 * "(out, lse)" attention core with an attention-domain LSE, a fixed block
 * merge order and a deterministic backward (RL-Kernel PR #319 "feat(attention):
 * add strict bitwise ROCm path", Summary table), and the block-KV-cache
 * streaming self-attention of FlashDreams PR #486 "flashdreams.accelerated
 * API v0", section 1.2 Optimized MHA.
 *
 * Conventions shared by every entry point:
 *  - Tensors are dense, contiguous, row-major [B, H, S, D] in device memory;
 *    D (head dim) must be 128.  LSE arrays are fp32 [B, Hq, Sq] in natural log.
 *  - Grouped KV heads: Hq % Hkv == 0, and query head h reads KV head
 *    h / (Hq / Hkv).
 *  - causal != 0 masks key j for query i unless j <= i + (Sk - Sq)
 *    (bottom-right aligned); it requires Sq <= Sk so every row sees a key.
 *  - All device pointers must be 16-byte aligned.
 *  - The caller owns every buffer.  Calls allocate nothing, never synchronise
 *    the host, and enqueue their kernels on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream), so they may be captured into a CUDA graph.
 *    The attention kernels are launched as programmatic dependents of the
 *    kernel before them on the stream: their setup may overlap its end, but
 *    they touch no global memory until it has completed, and the last kernel
 *    of each call completes only after the call's other kernels, so stream
 *    order holds for everything the caller enqueues around a call.
 *  - Results are bitwise reproducible: every output element is written by one
 *    thread block, reductions run in a fixed order, and tile sizes do not depend
 *    on B, H or the number of SMs, so a row's result does not change with the
 *    batch it is submitted in or with how many heads are launched.
 *  - Return value: 0 on success or a negative HATTN_E* code; arguments are
 *    checked before anything is launched, and unsupported requests are refused,
 *    never approximated.
 */
#ifndef HATTN_H_
#define HATTN_H_

#include <stddef.h>

#if defined(__GNUC__)
#define HATTN_API __attribute__((visibility("default")))
#else
#define HATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { HATTN_BF16 = 0, HATTN_E4M3 = 1 } hattn_dtype;

enum {
  HATTN_OK = 0,
  HATTN_EINVAL = -1,        /* null pointer, size <= 0, Hq % Hkv != 0, scale not a
                               finite positive number, descales given for bf16 or
                               missing for e4m3 */
  HATTN_EUNSUPPORTED = -2,  /* D != 128, causal with Sq > Sk, fp8 backward, a zero-length block */
  HATTN_EALIGN = -3,        /* a device pointer is not 16-byte aligned */
  HATTN_EWORKSPACE = -4,    /* workspace smaller than the matching *_workspace_size() */
  HATTN_ELAUNCH = -5,       /* CUDA reported an error: no usable device, scratch
                               allocation, descriptor encoding or kernel launch */
  HATTN_EDEVICE = -6        /* a kernel gave up on a bounded wait (see attn_get_device_error) */
};

/*
 * Forward attention (fmha_v3_fwd semantics, AITER PR #2911 Test Result).
 *   q    [B, Hq,  Sq, D]  bf16, or e4m3fn codes when dtype == HATTN_E4M3
 *   k, v [B, Hkv, Sk, D]  same element type as q
 *   out  [B, Hq,  Sq, D]  bf16, written
 *   lse  [B, Hq,  Sq]     fp32, written
 *   scale: softmax scale (finite, > 0), e.g. 1/sqrt(D).
 *   q_descale [B*Hq], k_descale [B*Hkv], v_descale [B*Hkv]: fp32 device arrays
 *     for e4m3 (the real value of a code x of head (b, h) is x * descale[b*H + h];
 *     one value per tensor is the case where all entries are equal); all three
 *     must be NULL for bf16.  Descales must be positive.
 * Softmax statistics and both matrix products accumulate in fp32.  For e4m3
 * inputs S = Q K^T is an 8-bit product; V is widened to fp16 (exactly) and the
 * probabilities are rounded to fp16 before the P V product.  attn_fwd widens
 * each V tile in shared memory inside the attention kernel and allocates
 * nothing; attn_fwd_ws, given scratch memory, widens V there first in one
 * pass and runs about 2 % faster.  Both give the same bits.
 */
HATTN_API int attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
             int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal, int dtype,
             const float* q_descale, const float* k_descale, const float* v_descale,
             void* stream);

/*
 * attn_fwd with caller-provided scratch for the fp16 copy of an e4m3 V:
 * workspace must hold at least attn_fwd_workspace_size(B, Hkv, Sk, D, dtype)
 * bytes (B*Hkv*Sk*D*2 for e4m3, 0 for bf16, where workspace may be NULL); its
 * contents on entry do not matter.  Too small a workspace returns
 * HATTN_EWORKSPACE.  Same results as attn_fwd, bit for bit.
 */
HATTN_API int attn_fwd_ws(const void* q, const void* k, const void* v, void* out, float* lse,
             int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal, int dtype,
             const float* q_descale, const float* k_descale, const float* v_descale,
             void* workspace, size_t workspace_bytes, void* stream);

HATTN_API size_t attn_fwd_workspace_size(int B, int Hkv, int Sk, int D, int dtype);

/*
 * e4m3 quantisation prologue for the fp8 forward (FlashDreams PR #486 section
 * 1.1 Quantization toolkit: FP8 E4M3 with per-slice scales, and section 1.2:
 * head-scoped Q/K normalisation; e4m3fn range +-448 as in VeOmni PR #1363).
 *   x       [B, H, S, D] bf16 in (D must be 128)
 *   codes   [B, H, S, D] e4m3fn codes out
 *   descale [B*H] fp32 out: the real value of code c of head (b, h) is
 *           decode(c) * descale[b*H + h], ready for attn_fwd's descales.
 * Per head: with rmsnorm != 0 each row is first multiplied by
 * r = 1 / sqrt(ss / 128 + eps), giving y; without it y = x.  The norm runs in
 * fp32 with every operation rounded to nearest (eps > 0 is taken as fp32; ss,
 * the sum of the row's squares, adds the squares of d = 8k .. 8k+7 in
 * ascending d for k = 0 .. 15, then those 16 partial sums pairwise, neighbours
 * first), so y has a relative error below 68 * 2^-24 (a sum of 128
 * non-negative terms in any order is within 127 * 2^-24 of the exact sum).
 * descale = max |y| / 448 (fp32; 1 if the head is all zero); code = the
 * e4m3fn value nearest to the exact quotient y / descale of those fp32 values,
 * ties to even, saturating at +-448 (the fp32 quotient is correctly rounded,
 * and when it lands exactly on an e4m3 midpoint the exact residual decides).
 * Without the norm the codes and descales are exactly those of the definition.
 * The result is bitwise the same for any batch or head split.  Enqueues a
 * memset of descale and two kernels (head maxima; codes, which also turn each
 * maximum into its descale); x is read twice (the second pass starts with the
 * rows read last, which L2 may still hold) and the codes are written once: at
 * most 5 bytes of HBM traffic * per element.
 */
HATTN_API int attn_quantize_e4m3(const void* x, void* codes, float* descale, int B, int H, int S, int D,
                                 int rmsnorm, double eps, void* stream);

/*
 * Streaming forward over a block KV cache (FlashDreams PR #486 section 1.2;
 * merge rule from RL-Kernel PR #319 Summary table).  Queries attend, without a
 * mask, to the concatenation of n_blocks caller-managed KV blocks, folded in
 * ascending block order.  Up to 32 blocks are folded inside one launch: each
 * unit of 256 query rows runs its online softmax over block 0, then block 1,
 * and so on (no workspace: attn_fwd_kvblocks_workspace_size() returns 0).
 * With more blocks, each is computed separately into the workspace as
 * (O_b, LSE_b), then the blocks are folded in ascending order:
 *     M = max(L, L_b); w = e^(L - M); w_b = e^(L_b - M);
 *     L = M + ln(w + w_b); O = (w O + w_b O_b) / (w + w_b),  from (O, L) = (0, -inf).
 *   q          [B, Hq, Sq, D] bf16, or e4m3fn codes when dtype == HATTN_E4M3
 *   k_blocks, v_blocks: HOST arrays of n_blocks device pointers; block i is
 *              [B, Hkv, blk_len[i], D] of q's element type
 *   blk_len    HOST array of n_blocks lengths, each > 0
 *   out, lse   as for attn_fwd
 *   q_descale  e4m3 only: [B*Hq] fp32, as for attn_fwd
 *   k_descale, v_descale  e4m3 only: [n_blocks * B*Hkv] fp32, block-major: the
 *              value of code x of block i, head (b, h) is
 *              x * descale[i*B*Hkv + b*Hkv + h] (an FP8 KV cache whose blocks
 *              were each quantised with their own scales, e.g. by
 *              attn_quantize_e4m3 writing a block's codes and its B*Hkv
 *              descales in place).  NULL for bf16.
 * e4m3 arithmetic as for attn_fwd (V widened in shared memory); within one
 * launch block i's probabilities enter P V scaled by vd_i / max_i vd_i, and
 * the output by max_i vd_i.
 *   workspace  device buffer of at least attn_fwd_kvblocks_workspace_size() bytes
 *              (may be NULL when that is 0); its contents on entry do not matter.
 */
HATTN_API int attn_fwd_kvblocks(const void* q, const void* const* k_blocks, const void* const* v_blocks,
                      const int* blk_len, int n_blocks, void* out, float* lse,
                      int B, int Hq, int Hkv, int Sq, int D, float scale, int dtype,
                      const float* q_descale, const float* k_descale, const float* v_descale,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace attn_fwd_kvblocks needs: 0 for up to 32 blocks (folded
 * in one launch), else n_blocks * B*Hq*Sq * (D + 1) * 4 (per-block partials). */
HATTN_API size_t attn_fwd_kvblocks_workspace_size(int B, int Hq, int Sq, int D, int n_blocks);

/*
 * Deterministic backward (RL-Kernel PR #319: mha_bwd with deterministic
 * reduction, dQ/dK/dV bitwise stable across repeats and batch composition).
 * For dO = dL/dO and P = exp(scale Q K^T - LSE):
 *     dV = P^T dO;  dP = dO V^T;  Delta_i = sum_d dO_id O_id;
 *     dS = P * (dP - Delta);  dQ = scale dS K;  dK = scale dS^T Q,
 * with dK, dV of a KV head summed over its Hq/Hkv query heads in ascending
 * order.  bf16 only.
 *   q, out, dout [B, Hq, Sq, D] bf16;  k, v [B, Hkv, Sk, D] bf16;
 *   lse [B, Hq, Sq] fp32 from attn_fwd on the same inputs;
 *   dq [B, Hq, Sq, D], dk, dv [B, Hkv, Sk, D] bf16, written;
 *   workspace: at least attn_bwd_workspace_size() bytes.
 * Memory is O(S): no Sq x Sk buffer and no atomics.
 */
HATTN_API int attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
             const void* dout, void* dq, void* dk, void* dv,
             int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
             void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace attn_bwd needs: B*Hq*Sq * 4 (the Delta vector) rounded
 * up to a multiple of 256, plus 256 (a work counter of the dQ kernel).  Its
 * contents on entry do not matter. */
HATTN_API size_t attn_bwd_workspace_size(int B, int Hq, int Sq);

/*
 * Backward with dS stored (RL-Kernel PR #319, "What the strict contract
 * costs": a deterministic mha_bwd holding an O(S^2) workspace).  The same
 * arguments, layouts and checks as attn_bwd, bf16 only.  The dK/dV pass also
 * writes every bf16 dS tile it forms into the workspace; dQ is then the
 * product scale * dS K read back from there (one matrix product per pair of
 * 128-row tiles instead of attn_bwd's recomputation of S, P and dP: 5 in all
 * instead of 7), summed over key tiles in ascending order by one thread block
 * per query tile.  Results are bitwise reproducible and independent of batch
 * composition and head split; they agree with attn_bwd within the gradient
 * tolerance, not bitwise (dS is formed from the transposed S).
 *   workspace: at least attn_bwd_dsbuf_workspace_size(B, Hq, Sq, Sk) bytes:
 *   Delta, then B*Hq*ceil(Sk/128)*ceil(Sq/128) tiles of 32 KB -- memory that
 *   grows as Sq x Sk (about 537 MB at B2 Hq32 S2048); its contents on entry do
 *   not matter.
 */
HATTN_API int attn_bwd_dsbuf(const void* q, const void* k, const void* v, const void* out, const float* lse,
             const void* dout, void* dq, void* dk, void* dv,
             int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
             void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace attn_bwd_dsbuf needs (for D = 128); 0 for a size <= 0. */
HATTN_API size_t attn_bwd_dsbuf_workspace_size(int B, int Hq, int Sq, int Sk);

/*
 * One-pass deterministic backward (RL-Kernel PR #319: deterministic mha_bwd,
 * "What the strict contract costs"): the same dQ, dK, dV as attn_bwd (same
 * arguments and layouts, bf16 only), computed by one kernel that forms each
 * tile pair's dQ contribution where dS is made (5 matrix products per pair of
 * 128-row tiles instead of attn_bwd's 7) and adds it into an fp32 dQ
 * accumulator in ascending key-tile order, ordered by counters in the
 * workspace (bounded waits; a wait that gives up sets the device error word).
 * Results are bitwise reproducible and independent of batch composition and
 * head split; they are not bitwise those of attn_bwd (dK and dV sum the
 * query tiles in another fixed order).  The kernel is launched cooperatively
 * (all its thread blocks resident at once), which the ordering relies on.
 *   workspace: at least attn_bwd_onepass_workspace_size(B, Hq, Sq) bytes:
 *   Delta, the fp32 dQ accumulator (B*Hq*Sq*D*4 bytes) and the counters; its
 *   contents on entry do not matter (the counters are cleared by a memset
 *   enqueued on `stream`).
 */
HATTN_API int attn_bwd_onepass(const void* q, const void* k, const void* v, const void* out, const float* lse,
             const void* dout, void* dq, void* dk, void* dv,
             int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
             void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace attn_bwd_onepass needs (for D = 128). */
HATTN_API size_t attn_bwd_onepass_workspace_size(int B, int Hq, int Sq);

/*
 * Backward without a workspace argument, for callers that cannot allocate
 * device memory at call time -- for example a plug-in running inside a host
 * framework that owns the GPU allocator and its memory budget, or an engine
 * whose device memory is planned once up front.  (The pages have no
 * counterpart; this is an interface convenience of this library.)
 * Same arguments, results and bitwise reproducibility as attn_bwd, minus the
 * workspace.  The Delta scratch lives in a static device array of
 * HATTN_NOALLOC_MAX_ROWS floats (16 MiB), followed by 256 bytes for a work
 * counter, that every GPU loading the library holds until the process
 * exits; this call allocates nothing.
 *  - B*Hq*Sq must be <= HATTN_NOALLOC_MAX_ROWS, else HATTN_EWORKSPACE and
 *    nothing is launched.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.  The graph-capture remark at the top of this
 *    file does not cover this entry point.  The address is kept for the
 *    process: after a cudaDeviceReset (or anything else that destroys the
 *    device's primary context) it is stale, and this entry point must not be
 *    called again in that process.
 *  - All calls share the one array: calls that overlap on the GPU (different
 *    streams, or several host threads) race on it and must be serialised by
 *    the caller.  Every call rewrites all the rows it reads, so no clearing is
 *    needed between calls.
 */
#define HATTN_NOALLOC_MAX_ROWS (1 << 22)
HATTN_API int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* out, const float* lse,
             const void* dout, void* dq, void* dk, void* dv,
             int B, int Hq, int Hkv, int Sq, int Sk, int D, float scale, int causal,
             void* stream);

/*
 * Synchronises `stream`, then reads and clears the device error word that
 * kernels set when a bounded wait gives up (0 = none; 0x100 | site otherwise).
 * Returns 0, or HATTN_ELAUNCH if CUDA reports an error.  For tests and
 * diagnostics; it is the one call that blocks the host.
 */
HATTN_API int attn_get_device_error(void* stream, int* code_out);

/*
 * Failure-detection self-test (no counterpart on the pages): enqueues one small
 * kernel whose only wait can never be satisfied, with a limit of timeout_us
 * microseconds (1 .. 10^7).  The wait gives up, sets the device error word to
 * 0x17F (0x100 | site 0x7F) and the kernel returns normally; the context stays
 * usable.  Read the word with attn_get_device_error.  Returns 0, HATTN_EINVAL
 * or HATTN_ELAUNCH.
 */
HATTN_API int attn_selftest_bounded_wait(void* stream, unsigned int timeout_us);

/*
 * Failure-detection self-test of the bounded wait on a global counter that
 * attn_bwd_onepass orders its dQ additions with (no counterpart on the
 * pages): one thread waits for the 32-bit device word `counter` (4-byte
 * aligned; the caller keeps it below 1 while the kernel runs) to reach 1,
 * with a limit of timeout_us microseconds (1 .. 10^7).  The wait gives up,
 * sets the device error word to 0x12A (0x100 | site 0x2A) and the kernel
 * returns normally.  Returns 0, HATTN_EINVAL, HATTN_EALIGN or HATTN_ELAUNCH.
 */
HATTN_API int attn_selftest_counter_wait(const void* counter, void* stream, unsigned int timeout_us);

/* Static text for a return code. */
HATTN_API const char* attn_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* HATTN_H_ */
