/*
 * attn_oracle.c -- CPU fp64 oracle for fused scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously-correct
 * statement of what the GPU library computes.  Only the test suite, the smoke
 * check and the CPU-baseline leg of the benchmark may load it.  It shares no
 * code, header, table or constant with the CUDA library under
 * head_attention_qk_b200/csrc, and it never includes or links it.
 *
 * Everything is computed in double precision with plain loops: no blocking,
 * no fusion, no reordering beyond the definition.  OpenMP splits independent
 * (batch, head, query-row) units across host threads; each unit is summed in
 * a fixed ascending order, so results do not depend on the thread count.
 *
 * Sources (web pages of the subject, cited by title and section):
 *  - AITER PR #2911 "F8 fmha ASM gfx950", Test Result: the operation is
 *    fmha_v3_fwd(q, k, v, softmax_scale, is_causal, return_softmax_lse,
 *    q/k/v_descale): O = softmax(Q K^T * scale [+ causal mask]) V plus the
 *    per-row log-sum-exp, with fp8 inputs scaled by per-tensor descales.
 *  - RL-Kernel PR #319 "feat(attention): add strict bitwise ROCm path",
 *    Summary table: the attention core returns (out, lse) in the
 *    "attention-domain LSE", partial results are merged by LSE in a fixed
 *    block order, and the backward (dQ, dK, dV) is deterministic; GQA with
 *    Qwen3-8B heads Hq=32, Hkv=8, D=128 (ROCm Validation table).
 *  - FlashDreams PR #486 "flashdreams.accelerated API v0", section 1.2
 *    Optimized MHA: streaming self-attention over a block KV cache and static
 *    cross-attention; sections 1.1-1.2 for the e4m3 prologue.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - layout is [B, H, S, D] contiguous; LSE is [B, Hq, Sq] in natural log;
 *  - query head h reads KV head floor(h / (Hq / Hkv));
 *  - causal is bottom-right aligned: key j is visible to query i iff
 *    j <= i + (Sk - Sq);
 *  - a row that sees no key has O = 0 and LSE = -inf;
 *  - fp8 inputs are OCP e4m3fn codes; the dequantized value is
 *    decode(code) * descale[b, h], with one descale per (batch, head).
 *
 * The pin suite checks this file against closed forms, brute force, library
 * routines and invariants, and checks that the pins catch plausible mistakes
 * by applying text patches to a copy of this source (tests/oracle_mutants.py);
 * nothing of that machinery lives here.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Storage kinds of the input arrays.  The oracle reads the same bytes the GPU
 * reads and widens them exactly to double. */
enum { ORACLE_F64 = 0, ORACLE_BF16 = 1, ORACLE_E4M3 = 2 };

/* bfloat16: the upper 16 bits of an IEEE-754 binary32.  Widening is exact. */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP 8-bit floating point, E4M3 "fn" variant: 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN.  Written
 * from the format definition: normal (1 + m/8) * 2^(e-7), subnormal
 * (m/8) * 2^-6. */
double oracle_e4m3_to_double(uint8_t code) {
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Read element idx of an input array of the given storage kind, scaled by
 * its descale (1.0 for non-fp8 kinds). */
static double load_elem(int kind, const void* p, int64_t idx, double descale) {
    switch (kind) {
    case ORACLE_F64:  return ((const double*)p)[idx];
    case ORACLE_BF16: return bf16_to_double(((const uint16_t*)p)[idx]);
    case ORACLE_E4M3: return oracle_e4m3_to_double(((const uint8_t*)p)[idx]) * descale;
    default:          return NAN;
    }
}

static int check_shape(int B, int Hq, int Hkv, int Sq, int Sk, int D) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Sk <= 0 || D <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    return 0;
}

/* Last key index visible to query row i (inclusive); Sk - 1 without a mask. */
static int64_t last_visible_key(int64_t i, int Sq, int Sk, int causal) {
    if (!causal) return (int64_t)Sk - 1;
    int64_t last = i + ((int64_t)Sk - (int64_t)Sq);
    if (last > (int64_t)Sk - 1) last = (int64_t)Sk - 1;
    return last;   /* may be negative: no key visible */
}

/*
 * Forward.  For each query row i of head h (KV head kh = h / G):
 *   s_j   = scale * sum_d q_id k_jd           for visible keys j
 *   LSE_i = ln sum_j exp(s_j)                 (computed as m + ln sum exp(s_j - m))
 *   O_i   = sum_j exp(s_j - LSE_i) v_j
 *
 * q, k, v: [B,Hq,Sq,D], [B,Hkv,Sk,D], [B,Hkv,Sk,D] of storage kind `kind`.
 * q/k/v_descale: [B*Hq], [B*Hkv], [B*Hkv] doubles for E4M3, else NULL.
 * rows: n_rows query indices evaluated for every (b, h); NULL = all Sq rows
 *       (then n_rows must equal Sq).
 * o: [B,Hq,n_rows,D] doubles; lse: [B,Hq,n_rows] doubles.
 * Returns 0, or -1 on a bad argument, -2 if scratch allocation failed.
 */
int oracle_attn_fwd(int kind, const void* q, const void* k, const void* v,
                    const double* q_descale, const double* k_descale,
                    const double* v_descale,
                    int B, int Hq, int Hkv, int Sq, int Sk, int D,
                    double scale, int causal,
                    const int64_t* rows, int n_rows,
                    double* o, double* lse) {
    if (check_shape(B, Hq, Hkv, Sq, Sk, D)) return -1;
    if (!q || !k || !v || !o || !lse || n_rows <= 0) return -1;
    if (!rows && n_rows != Sq) return -1;
    if (kind == ORACLE_E4M3 && (!q_descale || !k_descale || !v_descale)) return -1;
    if (kind < 0 || kind > 2) return -1;
    const int G = Hq / Hkv;
    const int64_t units = (int64_t)B * Hq * n_rows;
    int failed = 0;

#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)Sk);
        double* qrow = (double*)malloc(sizeof(double) * (size_t)D);
        if (!s || !qrow) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t u = 0; u < units; ++u) {
                const int r = (int)(u % n_rows);
                const int h = (int)((u / n_rows) % Hq);
                const int b = (int)(u / ((int64_t)n_rows * Hq));
                const int kh = h / G;
                const int64_t i = rows ? rows[r] : r;
                const double dq = kind == ORACLE_E4M3 ? q_descale[(int64_t)b * Hq + h] : 1.0;
                const double dk = kind == ORACLE_E4M3 ? k_descale[(int64_t)b * Hkv + kh] : 1.0;
                const double dv = kind == ORACLE_E4M3 ? v_descale[(int64_t)b * Hkv + kh] : 1.0;
                const int64_t qbase = (((int64_t)b * Hq + h) * Sq + i) * D;
                const int64_t kvbase = ((int64_t)b * Hkv + kh) * (int64_t)Sk * D;
                double* orow = o + u * D;
                for (int d = 0; d < D; ++d) qrow[d] = load_elem(kind, q, qbase + d, dq);

                const int64_t last = last_visible_key(i, Sq, Sk, causal);
                double m = -INFINITY;
                for (int64_t j = 0; j <= last; ++j) {
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d)
                        acc += qrow[d] * load_elem(kind, k, kvbase + j * D + d, dk);
                    s[j] = scale * acc;
                    if (s[j] > m) m = s[j];
                }
                for (int d = 0; d < D; ++d) orow[d] = 0.0;
                if (last < 0) {           /* no visible key */
                    lse[u] = -INFINITY;
                    continue;
                }
                double sum = 0.0;
                for (int64_t j = 0; j <= last; ++j) sum += exp(s[j] - m);
                const double L = m + log(sum);
                lse[u] = L;
                for (int64_t j = 0; j <= last; ++j) {
                    const double p = exp(s[j] - L);
                    for (int d = 0; d < D; ++d)
                        orow[d] += p * load_elem(kind, v, kvbase + j * D + d, dv);
                }
            }
        }
        free(s);
        free(qrow);
    }
    return failed ? -2 : 0;
}

/*
 * Fixed-order merge of per-block partial results by their log-sum-exp
 * (RL-Kernel PR #319, Summary table: "same attention-domain LSE, same fixed
 * global_block_index merge order").  Blocks are folded in ascending index:
 *   start (O, L) = (0, -inf)
 *   M   = max(L, L_b);  w = exp(L - M);  w_b = exp(L_b - M)
 *   L  <- M + ln(w + w_b)
 *   O  <- (w O + w_b O_b) / (w + w_b)
 * A block with L_b = -inf (no visible key) leaves (O, L) unchanged.
 *
 * o_parts: [n_blocks][rows][D], lse_parts: [n_blocks][rows];
 * o: [rows][D], lse: [rows].
 */
int oracle_lse_merge(const double* o_parts, const double* lse_parts,
                     int n_blocks, int64_t rows, int D,
                     double* o, double* lse) {
    if (!o_parts || !lse_parts || !o || !lse || n_blocks <= 0 || rows <= 0 || D <= 0)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double L = -INFINITY;
        double* orow = o + r * D;
        for (int d = 0; d < D; ++d) orow[d] = 0.0;
        for (int bl = 0; bl < n_blocks; ++bl) {
            const double Lb = lse_parts[(int64_t)bl * rows + r];
            if (Lb == -INFINITY) continue;
            const double* ob = o_parts + ((int64_t)bl * rows + r) * D;
            const double M = L > Lb ? L : Lb;
            const double w = exp(L - M);      /* 0 when L = -inf */
            const double wb = exp(Lb - M);
            const double den = w + wb;
            for (int d = 0; d < D; ++d) orow[d] = (w * orow[d] + wb * ob[d]) / den;
            L = M + log(den);
        }
        lse[r] = L;
    }
    return 0;
}

/*
 * Backward of O = softmax(scale Q K^T [+ mask]) V for a scalar loss with
 * upstream gradient dO (RL-Kernel PR #319: deterministic mha_bwd producing
 * dQ, dK, dV).  From the chain rule, for each query row i:
 *   P_ij   = exp(s_ij - LSE_i)
 *   dV_j  += P_ij dO_i
 *   dP_ij  = dO_i . v_j
 *   Delta_i = sum_j P_ij dP_ij = dO_i . O_i
 *   dS_ij  = P_ij (dP_ij - Delta_i)
 *   dQ_i   = scale sum_j dS_ij k_j
 *   dK_j  += scale dS_ij q_i
 * dK and dV of a KV head sum the contributions of its G query heads.  The
 * oracle uses its own fp64 O (and returns it with LSE for inspection).
 *
 * Inputs q,k,v,dout of storage kind F64 or BF16 (the backward is not defined
 * for fp8 inputs).  Outputs (doubles): dq [B,Hq,Sq,D], dk/dv [B,Hkv,Sk,D],
 * o [B,Hq,Sq,D], lse [B,Hq,Sq].
 * Work is split over (b, kv-head) so each dK/dV element has one writer.
 */
int oracle_attn_bwd(int kind, const void* q, const void* k, const void* v,
                    const void* dout,
                    int B, int Hq, int Hkv, int Sq, int Sk, int D,
                    double scale, int causal,
                    double* dq, double* dk, double* dv,
                    double* o, double* lse) {
    if (check_shape(B, Hq, Hkv, Sq, Sk, D)) return -1;
    if (kind != ORACLE_F64 && kind != ORACLE_BF16) return -1;
    if (!q || !k || !v || !dout || !dq || !dk || !dv || !o || !lse) return -1;
    const int G = Hq / Hkv;
    const int64_t units = (int64_t)B * Hkv;
    int failed = 0;

#pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)Sk);
        double* qrow = (double*)malloc(sizeof(double) * (size_t)D);
        double* dorow = (double*)malloc(sizeof(double) * (size_t)D);
        if (!p || !qrow || !dorow) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t u = 0; u < units; ++u) {
                const int b = (int)(u / Hkv);
                const int kh = (int)(u % Hkv);
                const int64_t kvbase = ((int64_t)b * Hkv + kh) * (int64_t)Sk * D;
                double* dkh = dk + kvbase;
                double* dvh = dv + kvbase;
                for (int64_t e = 0; e < (int64_t)Sk * D; ++e) { dkh[e] = 0.0; dvh[e] = 0.0; }
                for (int g = 0; g < G; ++g) {
                    const int h = kh * G + g;
                    for (int64_t i = 0; i < Sq; ++i) {
                        const int64_t qoff = (((int64_t)b * Hq + h) * Sq + i) * D;
                        const int64_t lidx = ((int64_t)b * Hq + h) * Sq + i;
                        double* orow = o + qoff;
                        double* dqrow = dq + qoff;
                        for (int d = 0; d < D; ++d) {
                            qrow[d] = load_elem(kind, q, qoff + d, 1.0);
                            dorow[d] = load_elem(kind, dout, qoff + d, 1.0);
                            orow[d] = 0.0;
                            dqrow[d] = 0.0;
                        }
                        const int64_t last = last_visible_key(i, Sq, Sk, causal);
                        if (last < 0) { lse[lidx] = -INFINITY; continue; }
                        /* scores, then LSE with the row maximum */
                        double m = -INFINITY;
                        for (int64_t j = 0; j <= last; ++j) {
                            double sij = 0.0;
                            for (int d = 0; d < D; ++d)
                                sij += qrow[d] * load_elem(kind, k, kvbase + j * D + d, 1.0);
                            p[j] = scale * sij;
                            if (p[j] > m) m = p[j];
                        }
                        double z = 0.0;
                        for (int64_t j = 0; j <= last; ++j) z += exp(p[j] - m);
                        const double Lrow = m + log(z);
                        lse[lidx] = Lrow;
                        /* P_ij overwrites s_ij; O_i = sum_j P_ij v_j */
                        for (int64_t j = 0; j <= last; ++j) {
                            p[j] = exp(p[j] - Lrow);
                            for (int d = 0; d < D; ++d)
                                orow[d] += p[j] * load_elem(kind, v, kvbase + j * D + d, 1.0);
                        }
                        double delta = 0.0;
                        for (int d = 0; d < D; ++d) delta += dorow[d] * orow[d];
                        for (int64_t j = 0; j <= last; ++j) {
                            double dp = 0.0;
                            for (int d = 0; d < D; ++d)
                                dp += dorow[d] * load_elem(kind, v, kvbase + j * D + d, 1.0);
                            const double ds = p[j] * (dp - delta);
                            for (int d = 0; d < D; ++d) {
                                dqrow[d] += scale * ds * load_elem(kind, k, kvbase + j * D + d, 1.0);
                                dkh[j * D + d] += scale * ds * qrow[d];
                                dvh[j * D + d] += p[j] * dorow[d];
                            }
                        }
                    }
                }
            }
        }
        free(p);
        free(qrow);
        free(dorow);
    }
    return failed ? -2 : 0;
}

/*
 * e4m3 quantisation prologue: the step before fp8 attention.
 * FlashDreams PR #486 "flashdreams.accelerated API v0": section 1.1
 * Quantization toolkit (FP8 E4M3 with tensor- or slice-granularity scales)
 * and section 1.2 (head-scoped Q/K normalization, optional FP8 SDPA); the
 * clamp to the e4m3fn range +-448 as VeOmni PR #1363 describes its quantizers.
 * The pages give no formula; the readings (listed in the design notes) are:
 * the scale slice is one (batch, head); the optional normalisation is a plain
 * RMS over the head dimension with eps and no weight.  In exact arithmetic
 * (here fp64), per head:
 *   r_s     = 1 / sqrt( (1/D) sum_d x_sd^2 + eps )   for each row s (1 without
 *             the normalisation)
 *   y_sd    = x_sd * r_s
 *   amax    = max |y| over the head's S x D values
 *   descale = amax / 448, as the nearest fp32 (the descales travel as fp32),
 *             or 1 when amax == 0
 *   code    = e4m3 of y_sd / descale, rounded to nearest with ties to the
 *             even code, saturating at +-448; the sign bit is the quotient's.
 */

/* The non-negative finite e4m3fn values in code order (codes 0x00..0x7E),
 * from the format definition; ascending. */
static double e4m3_pos_value(int code) { return oracle_e4m3_to_double((uint8_t)code); }

uint8_t oracle_e4m3_rne(double v) {
    if (isnan(v)) return 0x7F;
    const int neg = signbit(v) ? 1 : 0;
    const double a = fabs(v);
    int code;
    if (a >= 448.0) {
        code = 0x7E;                           /* saturate */
    } else {
        /* largest code whose value is <= a (binary search over ascending values) */
        int lo = 0, hi = 0x7E;
        while (lo < hi) {
            int mid = (lo + hi + 1) / 2;
            if (e4m3_pos_value(mid) <= a) lo = mid; else hi = mid - 1;
        }
        code = lo;
        if (e4m3_pos_value(code) < a) {        /* between code and code + 1 */
            const double dl = a - e4m3_pos_value(code), dh = e4m3_pos_value(code + 1) - a;
            if (dh < dl || (dh == dl && ((code + 1) & 1) == 0)) code = code + 1;
        }
    }
    return (uint8_t)(code | (neg << 7));
}

/* x: [B,H,S,D] bf16 bit patterns.  codes: [B,H,S,D]; descale: [B*H] fp32.
 * quotient (optional, may be NULL): [B,H,S,D] doubles, y / descale before
 * rounding, for tests that need the distance to a rounding boundary. */
int oracle_quantize_e4m3(const uint16_t* x, uint8_t* codes, float* descale, double* quotient,
                         int B, int H, int S, int D, int rmsnorm, double eps) {
    if (B <= 0 || H <= 0 || S <= 0 || D <= 0 || !x || !codes || !descale) return -1;
    const int64_t heads = (int64_t)B * H;
    const int64_t n = (int64_t)S * D;
    int failed = 0;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < heads; ++bh) {
        double* y = (double*)malloc(sizeof(double) * (size_t)n);
        if (!y) { failed = 1; continue; }
        const uint16_t* xh = x + bh * n;
        double amax = 0.0;
        for (int64_t s = 0; s < S; ++s) {
            double r = 1.0;
            if (rmsnorm) {
                double ss = 0.0;
                for (int d = 0; d < D; ++d) {
                    const double xv = bf16_to_double(xh[s * D + d]);
                    ss += xv * xv;
                }
                r = 1.0 / sqrt(ss / D + eps);
            }
            for (int d = 0; d < D; ++d) {
                const double yv = bf16_to_double(xh[s * D + d]) * r;
                y[s * D + d] = yv;
                if (fabs(yv) > amax) amax = fabs(yv);
            }
        }
        const float ds = amax > 0.0 ? (float)(amax / 448.0) : 1.0f;
        descale[bh] = ds;
        uint8_t* ch = codes + bh * n;
        for (int64_t i = 0; i < n; ++i) {
            const double qv = y[i] / (double)ds;
            ch[i] = oracle_e4m3_rne(qv);
            if (quotient) quotient[bh * n + i] = qv;
        }
        free(y);
    }
    return failed ? -2 : 0;
}

/* Number of OpenMP threads a parallel region will use (for reporting). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
