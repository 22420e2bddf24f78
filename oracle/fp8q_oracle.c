/*
 * fp8q_oracle.c -- plain, slow CPU oracle for the blockwise FP8 (E4M3) W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this file:
 * only the test-suite, the smoke check and the benchmark's CPU-baseline leg use it.  It shares
 * no code, header, table or constant generator with the CUDA library; it is written from the
 * definitions the source pages give (or, where they are silent, from the stated readings).
 *
 * Sources (by page title and section):
 *   [FP8-RL]      "FP8-RL: A Practical and Stable Low-Precision Stack for LLM Reinforcement
 *                 Learning", abstract, item (i): W8A8 linear layers with blockwise FP8
 *                 quantization; policy weights change every step, so they are requantized
 *                 every step.
 *   [DSv4-WOA]    "DeepSeek V4 performance: FP8 WO_A output projection (vLLM PR 54894
 *                 analysis)", section 1 (E8M0 scale normalisation: unsigned exponent, bias
 *                 127, lossless only for exact powers of two), section 2 (128-divisibility
 *                 check; scale grid viewed as [groups, out/128, in/128]), section 3 (group-128
 *                 activation quant feeding a batched FP8 GEMM with per-group weights).
 *   [SGL-RMSQ]    "SGLang AMD GPU optimisation: fusing RMSNorm with FP8 per-token quantization
 *                 (SGLang PR 21403 analysis)", section 1 (RMSNorm with weight and epsilon fused
 *                 with FP8 quant), section 3 (the GEMM takes a pre-quantized (codes, scale)
 *                 tuple).
 *   [OCP-FP8]     the OCP 8-bit floating point formats linked from [DSv4-WOA]'s references
 *                 (OCP Microscaling spec v1.0, element type E4M3): sign, 4 exponent bits with
 *                 bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN, max 448.
 *   [torch-RMS]   torch.nn.RMSNorm documentation linked from [SGL-RMSQ]:
 *                 y = x / sqrt(mean(x^2) + eps) * weight.
 *
 * Readings taken where the pages are silent (each is repeated in the design notes):
 *   R1  scale s = amax / 448 in fp32 (IEEE round-to-nearest division); an all-zero block takes
 *       s = 1.  Codes are q = RNEsat(x / s), fp32 IEEE division then round-to-nearest-even to
 *       E4M3 with saturation to +-448.
 *   R2  E8M0 scales: s = 2^e with e the smallest integer such that 2^e >= fp32(amax / 448),
 *       clamped to [-127, 127]; byte = e + 127; all-zero block -> byte 127.
 *   R3  the sign of zero is kept: a negative value that rounds to zero gives code 0x80.
 *   R4  RMSNorm: per 128-block fp64 sum of squares in ascending k, then the fp64 sum of the
 *       block sums in ascending block order; v = S / K + eps (eps widened from fp32);
 *       r = fp32(1 / sqrt(v)) (fp64 sqrt and division, one final rounding to fp32);
 *       y_k = bf16_RNE( fp32( fp32(x_k * r) * gamma_k ) ), which is what an unfused bf16
 *       RMSNorm writes; then the 1x128 token quant runs on y.
 *   R5  activation scales sa are fp32, stored K-block-major: sa[kb * lds + m].
 *   R6  GEMM reference: out[m,n] = sum_kb (sa[m,kb] * sw[nb,kb]) * P_kb[m,n], P_kb the exact
 *       dot product of the decoded codes over K-block kb; all in fp64.
 *   R7  per-token / per-channel ("PTPC") variant [SGL-RMSQ sections 1-3: group_size 0 means
 *       per token; CHANNEL weight strategy; the GEMM takes (codes, x_scale) and weight_scale]:
 *       one scale per full row of K, s = amax / 448 as in R1 (0 -> 1), codes as in R1; the
 *       same rule quantizes a weight per output channel (one row of W).  With gamma, the row
 *       is first normalised as in R4.  GEMM reference: out[m,n] = sa[m] * sw[n] * P[m,n], P the
 *       exact dot product of the decoded codes over all of K, in fp64.
 *   R8  SiLU-and-mul front end of the MoE down projection [FP8-RL abstract (i): MoE models; the
 *       gate/up GEMM output feeds the down GEMM]: h = [gate | up] (bf16 [R, 2I]), y_k =
 *       bf16_RNE( fp32( silu(g_k) * u_k ) ) with silu(g) = g / (1 + e^-g) in fp32 (IEEE division)
 *       and e^x in fp32 by Cody-Waite range reduction and a degree-7 Taylor polynomial (below);
 *       then the 1x128 token quant of R1 on y.
 *   R9  inverse RoPE + group-128 quant [DSv4-WOA section 3: inverse_rope_group_quant(o [T,
 *       heads, head_dim], positions, cos cache, sin cache, num_groups, quant_group_size=128)
 *       feeding a batched per-group GEMM]: the rotary part is the last R dims of each head,
 *       rotated by -theta_i in pairs (a, b) = (2i, 2i+1) (interleaved) or (i, i+R/2) (halves):
 *       with c = cos[p][i], s = sin[p][i] (fp32 caches [max_pos][R/2]), y_a = bf16(fp32(x_a c)
 *       + fp32(x_b s)) and y_b = bf16(fp32(x_b c) - fp32(x_a s)), each product and sum one fp32
 *       rounding; the other dims pass through.  Then 1x128 groups along the flattened
 *       heads x head_dim row of each token, scales K-block-major as R5 (each head group's
 *       K-blocks are then contiguous).  The scale is R1's fp32 amax/448, or, since the GEMM that
 *       follows on the page takes MX (E8M0) scales, R2's power of two, stored as its fp32 value.
 *   R10 FP8 KV cache with per-step QKV scale recalibration [FP8-RL abstract, item (ii)]: each
 *       step, one fp32 scale per tensor (Q, K, V of a layer) is recomputed from the step's QKV
 *       activations with R1's rule, s = amax / 448 over the whole tensor (0 -> 1); K and V
 *       are then stored in the cache as E4M3 codes RNEsat(x / s) (R1's element rule) at the
 *       slots given per token (a negative slot: the token is not cached), and Q is quantized
 *       the same way for the attention that reads the cache.  The QKV row of a token holds
 *       Hq heads of Q, then Hkv of K, then Hkv of V, each of D values.
 *   R11 residual add ahead of the RMSNorm front end [SGL-RMSQ section 1: the fused kernel the
 *       page calls is the AMD library's add_rmsnorm_quant; the call it prints passes no
 *       residual]: h_k = bf16_RNE( fp32(x_k) + fp32(res_k) ), the value an unfused bf16 add
 *       writes; h replaces res (the updated residual stream, as a pre-norm block carries it),
 *       and the RMSNorm and quant of R4 (1x128 groups) or R7 (one scale per row) run on h.
 *   R12 E8M0 activation scales for the 1x128 front ends (plain token quant, RMSNorm + quant,
 *       SiLU-and-mul + quant, residual add + RMSNorm + quant) [DSv4-WOA sections 1 and 3: the
 *       MX-scaled GEMM takes E8M0 scales on both operands]: the group's scale is R2's power of
 *       two 2^e (the smallest with 2^e >= fp32(amax / 448), clamped to [-127, 127]), stored as
 *       its fp32 value, as R9 stores it; codes are RNEsat(y / 2^e), a division that is exact.
 *   R13 decode attention over the FP8 KV cache of R10 [FP8-RL abstract, item (ii): the cache
 *       exists for the attention that reads it; the page gives no attention arithmetic]: plain
 *       scaled dot-product attention on the dequantized tensors.  For sequence b (one query
 *       token) and query head h, with kv head g = h / (Hq / Hkv) (grouped-query attention) and
 *       the sequence's L positions j at cache slot block_table[b][j / bs] * bs + j % bs:
 *       z_j = sm_scale * s_q * s_k * sum_d dec(q[h][d]) dec(k_j[g][d]), p = softmax(z),
 *       o[h][d] = s_v * sum_j p_j dec(v_j[g][d]); the kernel writes bf16_RNE(o).  L = 0 gives
 *       o = 0.  The reference is fp64 (exp from the C library).
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fno-fast-math -fopenmp.
 * fp32 arithmetic below relies on FLT_EVAL_METHOD == 0 (SSE on x86-64), so every float
 * operation rounds once to nearest-even, as IEEE 754 single precision.
 */
#include <math.h>
#include <stdlib.h>
#include <stdint.h>
#include <string.h>
#include <float.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#if FLT_EVAL_METHOD != 0
#error "the oracle needs float arithmetic evaluated in single precision"
#endif

/* ------------------------------------------------------------------------------------------ */
/* bf16 and fp32 bit-level conversions                                                         */
/* ------------------------------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE fp32; widening is exact. */
static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even (finite inputs).  Drop the low 16 bits and round
 * up when the dropped part is above half, or exactly half with an odd kept part. */
static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xFFFFu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1u;
    return (uint16_t)kept;
}

/* ------------------------------------------------------------------------------------------ */
/* E4M3 codec [OCP-FP8]                                                                       */
/* ------------------------------------------------------------------------------------------ */

/* Decode one E4M3 code.  Bits: s eeee mmm, exponent bias 7.
 *   e == 0          : subnormal, (-1)^s * (m / 8) * 2^-6
 *   e == 15, m == 7 : NaN
 *   otherwise       : (-1)^s * (1 + m / 8) * 2^(e - 7)                                       */
double oracle_e4m3_decode(uint8_t code) {
    int s = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);            /* m/8 * 2^-6 */
    else        v = ldexp((double)(8 + m), e - 10);  /* (8+m)/8 * 2^(e-7) */
    return s ? -v : v;
}

/* Round a non-negative double that holds an exact value to the nearest integer, ties to even. */
static double rne_integer(double q) {
    double fl = floor(q);
    double frac = q - fl;                 /* exact: q has at most 53 significant bits */
    if (frac > 0.5) return fl + 1.0;
    if (frac < 0.5) return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* RNEsat: finite fp32 -> E4M3 code, round to nearest (ties to the even code) with saturation to
 * +-448 (the largest finite E4M3 magnitude, code 0x7E).  Reading R3 keeps the sign of zero. */
uint8_t oracle_e4m3_encode(float v) {
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: the grid is k * 2^-9, k = 0..8 (k = 8 is the smallest normal,
         * code 0x08, whose bit pattern is exactly 8) */
        double k = rne_integer(a * 512.0);  /* scaling by a power of two is exact */
        return sign | (uint8_t)k;
    }
    int ex;
    (void)frexp(a, &ex);                    /* a = f * 2^ex, f in [0.5, 1) */
    int E = ex - 1;                         /* floor(log2 a), in [-6, 8] */
    double n = rne_integer(ldexp(a, 3 - E));/* significand in eighths: 8..16 */
    if (n == 16.0) { E += 1; n = 8.0; }
    return sign | (uint8_t)(((E + 7) << 3) | ((int)n - 8));
}

/* ------------------------------------------------------------------------------------------ */
/* Scales                                                                                     */
/* ------------------------------------------------------------------------------------------ */

/* Reading R1: fp32 scale from the block's absolute maximum. */
static float scale_f32_from_amax(float amax) {
    if (amax == 0.0f) return 1.0f;
    return amax / 448.0f;                   /* one IEEE fp32 division */
}

/* Reading R2: E8M0 exponent byte from the block's absolute maximum.  r = fp32(amax / 448);
 * e = the smallest integer with 2^e >= r (r's unbiased exponent, plus one when r is not an
 * exact power of two); clamp to [-127, 127]; byte = e + 127 [DSv4-WOA section 1: bias 127]. */
static uint8_t e8m0_from_amax(float amax) {
    if (amax == 0.0f) return 127;
    float r = amax / 448.0f;
    int ex;
    double f = frexp((double)r, &ex);       /* r = f * 2^ex, f in [0.5, 1) */
    int e = (f == 0.5) ? ex - 1 : ex;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return (uint8_t)(e + 127);
}

/* Value of an E8M0 byte as fp32: 2^(byte - 127); byte 255 is NaN and never produced here. */
static float e8m0_value(uint8_t byte) {
    return ldexpf(1.0f, (int)byte - 127);
}

/* [DSv4-WOA section 1]: an fp32 scale converts to E8M0 only when it is an exact power of two;
 * e = round(log2 s), accepted iff 2^e == s, byte = e + 127.  Returns the byte, or -1 when the
 * conversion would lose information (the page's "None"). */
int oracle_e8m0_lossless_from_f32(float s) {
    if (!(s > 0.0f) || isinf(s)) return -1;
    double e = nearbyint(log2((double)s));
    if (ldexp(1.0, (int)e) != (double)s) return -1;
    if (e < -127 || e > 127) return -1;
    return (int)e + 127;
}

double oracle_e8m0_decode(uint8_t byte) {
    if (byte == 255) return NAN;
    return ldexp(1.0, (int)byte - 127);
}

/* ------------------------------------------------------------------------------------------ */
/* a1 / a2: weight requantization in 128x128 blocks [FP8-RL (i)], [DSv4-WOA section 2]         */
/* ------------------------------------------------------------------------------------------ */

/* W is bf16 [N, K] row-major with leading dimension ldw (elements).  Produces codes q [N, K]
 * (leading dimension ldq) and one scale per 128x128 block in a row-major [N/128, K/128] grid:
 * fp32 when fmt == 0, E8M0 bytes when fmt == 1.  N and K are multiples of 128. */
void oracle_quant_weight_block(const uint16_t *w, int64_t N, int64_t K, int64_t ldw,
                               uint8_t *q, int64_t ldq, void *sw, int fmt) {
    int64_t NB = N / 128, KB = K / 128;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t blk = 0; blk < NB * KB; ++blk) {
        int64_t nb = blk / KB, kb = blk % KB;
        float amax = 0.0f;
        for (int64_t i = 0; i < 128; ++i)
            for (int64_t j = 0; j < 128; ++j) {
                float a = fabsf(bf16_to_f32(w[(nb * 128 + i) * ldw + kb * 128 + j]));
                if (a > amax) amax = a;
            }
        float s;
        if (fmt == 0) {
            s = scale_f32_from_amax(amax);
            ((float *)sw)[nb * KB + kb] = s;
        } else {
            uint8_t byte = e8m0_from_amax(amax);
            s = e8m0_value(byte);
            ((uint8_t *)sw)[nb * KB + kb] = byte;
        }
        for (int64_t i = 0; i < 128; ++i)
            for (int64_t j = 0; j < 128; ++j) {
                float x = bf16_to_f32(w[(nb * 128 + i) * ldw + kb * 128 + j]);
                q[(nb * 128 + i) * ldq + kb * 128 + j] = oracle_e4m3_encode(x / s);
            }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* a3: per-token 1x128 activation quantization [DSv4-WOA section 3: quant_group_size=128]      */
/* ------------------------------------------------------------------------------------------ */

/* Quantize one 128-wide group of fp32 values (already bf16-representable).  Writes 128 codes
 * and returns the scale as fp32: amax/448 (fmt 0, reading R1) or the E8M0 power of two of
 * reading R2 (fmt 1, reading R12). */
static float quant_group_1x128_fmt(const float *y, uint8_t *q, int fmt) {
    float amax = 0.0f;
    for (int j = 0; j < 128; ++j) {
        float a = fabsf(y[j]);
        if (a > amax) amax = a;
    }
    float s = (fmt == 0) ? scale_f32_from_amax(amax) : e8m0_value(e8m0_from_amax(amax));
    for (int j = 0; j < 128; ++j) q[j] = oracle_e4m3_encode(y[j] / s);
    return s;
}

/* X bf16 [M, K] (leading dimension ldx) -> codes [M, K] (ldq) and scales sa[kb*lds + m]
 * (fmt 0: fp32 amax/448; fmt 1: E8M0 powers of two stored as fp32, reading R12). */
void oracle_quant_token_1x128(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                              uint8_t *q, int64_t ldq, float *sa, int64_t lds, int fmt) {
    int64_t KB = K / 128;
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t m = 0; m < M; ++m) {
        float y[128];
        for (int64_t kb = 0; kb < KB; ++kb) {
            for (int j = 0; j < 128; ++j) y[j] = bf16_to_f32(x[m * ldx + kb * 128 + j]);
            sa[kb * lds + m] = quant_group_1x128_fmt(y, q + m * ldq + kb * 128, fmt);
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* a4: RMSNorm followed by the 1x128 token quant [SGL-RMSQ section 1], [torch-RMS], reading R4  */
/* ------------------------------------------------------------------------------------------ */

/* The per-row inverse RMS of reading R4.  x is one bf16 row of length K. */
static float rms_inverse(const uint16_t *x, int64_t K, float eps) {
    int64_t KB = K / 128;
    double S = 0.0;
    for (int64_t b = 0; b < KB; ++b) {
        double P = 0.0;
        for (int j = 0; j < 128; ++j) {
            double v = (double)bf16_to_f32(x[b * 128 + j]);
            P = P + v * v;                  /* v*v is exact in fp64 (<= 16 significant bits) */
        }
        S = S + P;
    }
    double var = S / (double)K + (double)eps;
    return (float)(1.0 / sqrt(var));
}

/* Unfused RMSNorm as a bf16 layer writes it: y bf16 [M, K] (leading dimension ldy). */
void oracle_rmsnorm_bf16(const uint16_t *x, const uint16_t *gamma, float eps, int64_t M,
                         int64_t K, int64_t ldx, uint16_t *y, int64_t ldy) {
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t m = 0; m < M; ++m) {
        float r = rms_inverse(x + m * ldx, K, eps);
        for (int64_t k = 0; k < K; ++k) {
            float t = bf16_to_f32(x[m * ldx + k]) * r;   /* fp32, rounded once */
            float u = t * bf16_to_f32(gamma[k]);         /* fp32, rounded once */
            y[m * ldy + k] = f32_to_bf16_rne(u);
        }
    }
}

/* Fused front end: RMSNorm (gamma != NULL) then 1x128 token quant; gamma == NULL is the plain
 * token quant of a3.  The normalised row is never stored.  fmt as oracle_quant_token_1x128. */
void oracle_rmsnorm_quant_token(const uint16_t *x, const uint16_t *gamma, float eps, int64_t M,
                                int64_t K, int64_t ldx, uint8_t *q, int64_t ldq, float *sa,
                                int64_t lds, int fmt) {
    if (gamma == NULL) {
        oracle_quant_token_1x128(x, M, K, ldx, q, ldq, sa, lds, fmt);
        return;
    }
    int64_t KB = K / 128;
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t m = 0; m < M; ++m) {
        float r = rms_inverse(x + m * ldx, K, eps);
        float y[128];
        for (int64_t kb = 0; kb < KB; ++kb) {
            for (int j = 0; j < 128; ++j) {
                int64_t k = kb * 128 + j;
                float t = bf16_to_f32(x[m * ldx + k]) * r;
                float u = t * bf16_to_f32(gamma[k]);
                y[j] = bf16_to_f32(f32_to_bf16_rne(u));
            }
            sa[kb * lds + m] = quant_group_1x128_fmt(y, q + m * ldq + kb * 128, fmt);
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* SiLU-and-mul + 1x128 quant, reading R8                                                      */
/* ------------------------------------------------------------------------------------------ */

/* Constants of the fp32 exponential below: 1/ln 2 rounded to fp32; ln 2 = c1 + c2 with c1 holding
 * few enough significant bits that k c1 is exact for |k| <= 150 and c2 = RN_fp32(ln 2 - c1);
 * then the Taylor coefficients 1/n! rounded to fp32, n = 7 down to 0. */
static const float EXP_CONST[11] = {
    0x1.715476p+0f,                                    /* 1/ln 2 */
    0x1.62e400p-1f,                                    /* c1 */
    0x1.7f7d1cp-20f,                                   /* c2 */
    0x1.a01a02p-13f,                                   /* 1/7! */
    0x1.6c16c2p-10f,                                   /* 1/6! */
    0x1.111112p-7f,                                    /* 1/5! */
    0x1.555556p-5f,                                    /* 1/4! */
    0x1.555556p-3f,                                    /* 1/3! */
    0x1.000000p-1f,                                    /* 1/2! */
    1.0f,                                              /* 1/1! */
    1.0f,                                              /* 1/0! */
};

/* The constants above, for the oracle's own pins (n <= 11 values). */
void oracle_exp_constants(float *out, int n) {
    for (int i = 0; i < n && i < 11; ++i) out[i] = EXP_CONST[i];
}

/* e^x in fp32 by the method of Cody and Waite (1980): k = rint(x / ln 2); r = (x - k c1) - k c2
 * with ln 2 = c1 + c2 split so that k c1 is exact for |k| <= 150; e^r from its Taylor series to
 * degree 7 by Horner's rule (|r| <= ln2 / 2, truncation below 2^-27 relative); then the exact
 * scaling by 2^k (in two steps where 2^k alone is not a normal fp32).  Each operation below is
 * one IEEE fp32 rounding. */
float oracle_exp_f32(float x) {
    if (x > 0x1.62e430p+6f) return INFINITY;          /* above ln(FLT_MAX) */
    if (x < -104.0f) return 0.0f;                      /* below half the smallest subnormal */
    const float inv_ln2 = EXP_CONST[0], c1 = EXP_CONST[1], c2 = EXP_CONST[2];
    float kf = rintf(x * inv_ln2);
    float r = (x - kf * c1) - kf * c2;
    float p = EXP_CONST[3];
    for (int n = 4; n < 11; ++n) p = p * r + EXP_CONST[n];
    int k = (int)kf;
    if (k > 127) { p = p * 0x1p127f; k -= 127; }
    if (k < -126) { p = p * 0x1p-126f; k += 126; }
    union { uint32_t u; float f; } two_k = { (uint32_t)(k + 127) << 23 };
    return p * two_k.f;
}

/* silu(g) = g / (1 + e^-g), fp32 (IEEE division). */
float oracle_silu_f32(float g) {
    return g / (1.0f + oracle_exp_f32(-g));
}

/* h bf16 [R, 2I] (leading dimension ldh): gate = h[:, 0:I], up = h[:, I:2I].  Writes the codes
 * of y = bf16(silu(gate) * up) [R, I] (ldq) and scales sa[kb * lds + m] (1x128 groups; fmt as
 * oracle_quant_token_1x128). */
void oracle_silu_mul_quant(const uint16_t *h, int64_t R, int64_t I, int64_t ldh, uint8_t *q,
                           int64_t ldq, float *sa, int64_t lds, int fmt) {
    int64_t IB = I / 128;
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t m = 0; m < R; ++m) {
        float y[128];
        for (int64_t kb = 0; kb < IB; ++kb) {
            for (int j = 0; j < 128; ++j) {
                int64_t k = kb * 128 + j;
                float g = bf16_to_f32(h[m * ldh + k]), u = bf16_to_f32(h[m * ldh + I + k]);
                y[j] = bf16_to_f32(f32_to_bf16_rne(oracle_silu_f32(g) * u));
            }
            sa[kb * lds + m] = quant_group_1x128_fmt(y, q + m * ldq + kb * 128, fmt);
        }
    }
}

/* The bf16 y of reading R8 alone (for the oracle's own pins). */
void oracle_silu_mul_bf16(const uint16_t *h, int64_t R, int64_t I, int64_t ldh, uint16_t *y) {
    for (int64_t m = 0; m < R; ++m)
        for (int64_t k = 0; k < I; ++k) {
            float g = bf16_to_f32(h[m * ldh + k]), u = bf16_to_f32(h[m * ldh + I + k]);
            y[m * I + k] = f32_to_bf16_rne(oracle_silu_f32(g) * u);
        }
}

/* ------------------------------------------------------------------------------------------ */
/* Inverse RoPE + group-128 quant [DSv4-WOA section 3], reading R9                              */
/* ------------------------------------------------------------------------------------------ */

/* The inverse rotation of one rotary element of a head.  x is the head (D bf16 values), j the
 * index inside the rotary part (0 <= j < R), cs/sn the cache rows of the token's position.
 * Pairs are (2i, 2i+1) when interleaved, else (i, i + R/2); both rotate by -theta_i:
 * first = x_a cos + x_b sin, second = x_b cos - x_a sin, every product and sum rounded once
 * in fp32, the result rounded to bf16. */
static float inverse_rope_element(const uint16_t *x, int64_t D, int64_t R, int64_t j,
                                  const float *cs, const float *sn, int interleaved) {
    int64_t half = R / 2, i, ia, ib;
    int second;
    if (interleaved) {
        i = j / 2;
        second = (int)(j % 2);
        ia = 2 * i;
        ib = 2 * i + 1;
    } else {
        i = j % half;
        second = j >= half;
        ia = i;
        ib = i + half;
    }
    float xa = bf16_to_f32(x[D - R + ia]), xb = bf16_to_f32(x[D - R + ib]);
    float c = cs[i], s = sn[i];
    float v;
    if (!second) {
        float p = xa * c, r = xb * s;
        v = p + r;
    } else {
        float p = xb * c, r = xa * s;
        v = p - r;
    }
    return bf16_to_f32(f32_to_bf16_rne(v));
}

/* o bf16 [T][H][D] (contiguous), positions [T], cos/sin fp32 [max_pos][R/2].  Writes the
 * rotated bf16 values y [T][H*D] (what an unfused inverse RoPE would write to memory). */
void oracle_inverse_rope_bf16(const uint16_t *o, const int64_t *pos, const float *cosc,
                              const float *sinc, int64_t T, int64_t H, int64_t D, int64_t R,
                              int interleaved, uint16_t *y) {
    int64_t half = R / 2;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t h = 0; h < H; ++h) {
            const uint16_t *x = o + (t * H + h) * D;
            const float *cs = cosc + pos[t] * half, *sn = sinc + pos[t] * half;
            for (int64_t d = 0; d < D; ++d)
                y[(t * H + h) * D + d] =
                    d < D - R ? x[d]
                              : f32_to_bf16_rne(inverse_rope_element(x, D, R, d - (D - R), cs,
                                                                     sn, interleaved));
        }
}

/* The fused front end: inverse RoPE, then 1x128 quant along each token's flattened H*D row.
 * Codes q [T][H*D]; scales sa[kb * lds + t], fp32 amax/448 when fmt == 0 (reading R1), the
 * E8M0 power of two of reading R2 stored as its fp32 value when fmt == 1. */
void oracle_inverse_rope_quant(const uint16_t *o, const int64_t *pos, const float *cosc,
                               const float *sinc, int64_t T, int64_t H, int64_t D, int64_t R,
                               int interleaved, int fmt, uint8_t *q, float *sa, int64_t lds) {
    int64_t K = H * D, KB = K / 128, half = R / 2;
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t t = 0; t < T; ++t) {
        const float *cs = cosc + pos[t] * half, *sn = sinc + pos[t] * half;
        for (int64_t kb = 0; kb < KB; ++kb) {
            float y[128];
            for (int j = 0; j < 128; ++j) {
                int64_t k = kb * 128 + j, h = k / D, d = k % D;
                const uint16_t *x = o + (t * H + h) * D;
                y[j] = d < D - R ? bf16_to_f32(x[d])
                                 : inverse_rope_element(x, D, R, d - (D - R), cs, sn,
                                                        interleaved);
            }
            sa[kb * lds + t] = quant_group_1x128_fmt(y, q + t * K + kb * 128, fmt);
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* FP8 KV cache: per-step QKV scale recalibration and cache write [FP8-RL (ii)], reading R10    */
/* ------------------------------------------------------------------------------------------ */

/* Absolute maxima of the Q, K and V parts of qkv bf16 [T][ld] (row = Hq*D of Q, Hkv*D of K,
 * Hkv*D of V) into amax3[0..2]. */
void oracle_qkv_amax(const uint16_t *qkv, int64_t T, int64_t ld, int64_t Hq, int64_t Hkv,
                     int64_t D, float *amax3) {
    int64_t width[3] = {Hq * D, Hkv * D, Hkv * D};
    int64_t start = 0;
    for (int part = 0; part < 3; ++part) {
        float amax = 0.0f;
        for (int64_t t = 0; t < T; ++t)
            for (int64_t c = 0; c < width[part]; ++c) {
                float a = fabsf(bf16_to_f32(qkv[t * ld + start + c]));
                if (a > amax) amax = a;
            }
        amax3[part] = amax;
        start += width[part];
    }
}

/* The per-tensor scales of reading R10 from the maxima. */
void oracle_qkv_scales(const float *amax3, float *scale3) {
    for (int part = 0; part < 3; ++part) scale3[part] = scale_f32_from_amax(amax3[part]);
}

/* Quantize every token's Q into q_out [T][ldq] and write its K and V codes into row slots[t] of
 * k_cache / v_cache ([num_slots][Hkv*D] each); slots[t] < 0 leaves the caches untouched. */
void oracle_kv_cache_write(const uint16_t *qkv, int64_t T, int64_t ld, int64_t Hq, int64_t Hkv,
                           int64_t D, const int64_t *slots, const float *scale3, uint8_t *q_out,
                           int64_t ldq, uint8_t *k_cache, uint8_t *v_cache) {
    int64_t wq = Hq * D, wkv = Hkv * D;
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t *row = qkv + t * ld;
        for (int64_t c = 0; c < wq; ++c)
            q_out[t * ldq + c] = oracle_e4m3_encode(bf16_to_f32(row[c]) / scale3[0]);
        if (slots[t] < 0) continue;
        for (int64_t c = 0; c < wkv; ++c) {
            k_cache[slots[t] * wkv + c] = oracle_e4m3_encode(bf16_to_f32(row[wq + c]) / scale3[1]);
            v_cache[slots[t] * wkv + c] =
                oracle_e4m3_encode(bf16_to_f32(row[wq + wkv + c]) / scale3[2]);
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Decode attention over the FP8 KV cache [FP8-RL (ii)], reading R13                            */
/* ------------------------------------------------------------------------------------------ */

/* q [B][ldq] codes (Hq heads of D), caches [slots][Hkv * D] codes, scale3 = (s_q, s_k, s_v),
 * block_table [B][max_blocks] block ids, seq_lens [B].  Writes, per (b, h, d), out = o in fp64,
 * absref = s_v * sum_j p_j |dec(v_j[g][d])|, and per (b, h) zabs = the largest
 * |sm_scale * s_q * s_k| * sum_d |dec(q) dec(k_j)| over j (0 when L = 0). */
void oracle_attention_decode(const uint8_t *q, int64_t ldq, const uint8_t *k_cache,
                             const uint8_t *v_cache, const float *scale3,
                             const int32_t *block_table, int64_t max_blocks,
                             const int32_t *seq_lens, int64_t B, int64_t Hq, int64_t Hkv,
                             int64_t D, int64_t block_size, float sm_scale, double *out,
                             double *absref, double *zabs) {
    const int64_t G = Hq / Hkv, row = Hkv * D;
    const double c = (double)sm_scale * (double)scale3[0] * (double)scale3[1];
    const double sv = (double)scale3[2];
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < B * Hq; ++bh) {
        const int64_t b = bh / Hq, h = bh % Hq, g = h / G;
        const int64_t L = seq_lens[b];
        double *o = out + bh * D, *a = absref + bh * D;
        for (int64_t d = 0; d < D; ++d) o[d] = a[d] = 0.0;
        zabs[bh] = 0.0;
        if (L <= 0) continue;
        double *z = (double *)malloc((size_t)L * sizeof(double));
        int64_t *slot = (int64_t *)malloc((size_t)L * sizeof(int64_t));
        double zmax = -INFINITY;
        for (int64_t j = 0; j < L; ++j) {
            slot[j] = (int64_t)block_table[b * max_blocks + j / block_size] * block_size +
                      j % block_size;
            const uint8_t *kr = k_cache + slot[j] * row + g * D;
            const uint8_t *qr = q + b * ldq + h * D;
            double dot = 0.0, dabs = 0.0;
            for (int64_t d = 0; d < D; ++d) {
                const double t = oracle_e4m3_decode(qr[d]) * oracle_e4m3_decode(kr[d]);
                dot += t;
                dabs += fabs(t);
            }
            z[j] = c * dot;
            if (z[j] > zmax) zmax = z[j];
            if (fabs(c) * dabs > zabs[bh]) zabs[bh] = fabs(c) * dabs;
        }
        double S = 0.0;
        for (int64_t j = 0; j < L; ++j) {
            z[j] = exp(z[j] - zmax);
            S += z[j];
        }
        for (int64_t j = 0; j < L; ++j) {
            const double p = z[j] / S;
            const uint8_t *vr = v_cache + slot[j] * row + g * D;
            for (int64_t d = 0; d < D; ++d) {
                const double v = oracle_e4m3_decode(vr[d]);
                o[d] += p * v;
                a[d] += p * fabs(v);
            }
        }
        for (int64_t d = 0; d < D; ++d) {
            o[d] *= sv;
            a[d] *= fabs(sv);
        }
        free(z);
        free(slot);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Per-token / per-channel quantization [SGL-RMSQ section 1, group_size 0], reading R7          */
/* ------------------------------------------------------------------------------------------ */

/* Rows of bf16 x [R, K] (leading dimension ldx) -> codes [R, K] (ldq) and one fp32 scale per row
 * in s[R].  gamma == NULL: plain; otherwise each row is the bf16 RMSNorm of reading R4 first. */
void oracle_quant_rowwise(const uint16_t *x, const uint16_t *gamma, float eps, int64_t R,
                          int64_t K, int64_t ldx, uint8_t *q, int64_t ldq, float *s) {
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t m = 0; m < R; ++m) {
        const uint16_t *xr = x + m * ldx;
        float r = (gamma != NULL) ? rms_inverse(xr, K, eps) : 1.0f;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float y = bf16_to_f32(xr[k]);
            if (gamma != NULL) y = bf16_to_f32(f32_to_bf16_rne((y * r) * bf16_to_f32(gamma[k])));
            float a = fabsf(y);
            if (a > amax) amax = a;
        }
        float sc = scale_f32_from_amax(amax);
        for (int64_t k = 0; k < K; ++k) {
            float y = bf16_to_f32(xr[k]);
            if (gamma != NULL) y = bf16_to_f32(f32_to_bf16_rne((y * r) * bf16_to_f32(gamma[k])));
            q[m * ldq + k] = oracle_e4m3_encode(y / sc);
        }
        s[m] = sc;
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Residual add + RMSNorm + quant, reading R11                                                  */
/* ------------------------------------------------------------------------------------------ */

/* res[m, k] <- bf16_RNE(fp32(x[m, k]) + fp32(res[m, k])) for every row, then the RMSNorm front
 * end on the updated res: 1x128 groups with K-block-major scales sa[kb * lds + m]
 * (per_token == 0, reading R4; fmt as oracle_quant_token_1x128) or one fp32 scale per row in
 * sa[m] (per_token != 0, reading R7; fmt must be 0). */
void oracle_add_rmsnorm_quant(const uint16_t *x, int64_t ldx, uint16_t *res, int64_t ldr,
                              const uint16_t *gamma, float eps, int64_t M, int64_t K,
                              int per_token, int fmt, uint8_t *q, int64_t ldq, float *sa,
                              int64_t lds) {
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            float sum = bf16_to_f32(x[m * ldx + k]) + bf16_to_f32(res[m * ldr + k]);
            res[m * ldr + k] = f32_to_bf16_rne(sum);
        }
    if (per_token)
        oracle_quant_rowwise(res, gamma, eps, M, K, ldr, q, ldq, sa);
    else
        oracle_rmsnorm_quant_token(res, gamma, eps, M, K, ldr, q, ldq, sa, lds, fmt);
}

/* ------------------------------------------------------------------------------------------ */
/* Per-channel GEMM [SGL-RMSQ section 3], reading R7                                           */
/* ------------------------------------------------------------------------------------------ */

/* Per-channel GEMM reference on a subset of rows, reading R7: ref = sa[m] * sw[n] * P and
 * absref = sa[m] * sw[n] * sum_k |dec(a) * dec(w)|, in fp64 (P is exact: 8-bit products). */
void oracle_gemm_w8a8_rowwise_rows(const uint8_t *aq, int64_t lda, const float *sa,
                                   const uint8_t *wq, int64_t ldw, const float *sw, int64_t N,
                                   int64_t K, const int64_t *rows, int64_t nrows, double *ref,
                                   double *absref) {
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < nrows; ++i)
        for (int64_t n = 0; n < N; ++n) {
            int64_t m = rows[i];
            double P = 0.0, PA = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double prod = oracle_e4m3_decode(aq[m * lda + k]) * oracle_e4m3_decode(wq[n * ldw + k]);
                P += prod;
                PA += fabs(prod);
            }
            double sc = (double)sa[m] * (double)sw[n];
            ref[i * N + n] = sc * P;
            absref[i * N + n] = fabs(sc) * PA;
        }
}

/* ------------------------------------------------------------------------------------------ */
/* a5 / a6: block-scaled W8A8 GEMM reference, reading R6                                       */
/* ------------------------------------------------------------------------------------------ */

/* One output element in fp64: ref = sum_kb (sa*sw) * P_kb, P_kb = sum_{k in kb} dec(a)*dec(w)
 * (exact in fp64), and absref = sum_k |dec(a) * sa * dec(w) * sw|, the magnitude the error
 * bound is relative to. */
static void gemm_element(const uint8_t *arow, const uint8_t *wrow, int64_t K, const float *sa,
                         int64_t lds, int64_t m, const void *sw_row, int sw_fmt, double *ref,
                         double *absref) {
    int64_t KB = K / 128;
    double acc = 0.0, aacc = 0.0;
    for (int64_t kb = 0; kb < KB; ++kb) {
        double P = 0.0, PA = 0.0;
        for (int j = 0; j < 128; ++j) {
            double prod = oracle_e4m3_decode(arow[kb * 128 + j]) *
                          oracle_e4m3_decode(wrow[kb * 128 + j]);
            P += prod;
            PA += fabs(prod);
        }
        double swv = (sw_fmt == 0) ? (double)((const float *)sw_row)[kb]
                                   : oracle_e8m0_decode(((const uint8_t *)sw_row)[kb]);
        double sc = (double)sa[kb * lds + m] * swv;
        acc += sc * P;
        aacc += fabs(sc) * PA;
    }
    *ref = acc;
    *absref = aacc;
}

/* Dense GEMM reference on a subset of rows.  aq [M, K] (lda), wq [N, K] (ldw), sa as R5,
 * sw [N/128, K/128] (fp32 or E8M0).  rows[i] selects the output row; ref/absref are
 * [nrows, N] fp64. */
void oracle_gemm_w8a8_block_rows(const uint8_t *aq, int64_t lda, const float *sa, int64_t lds,
                                 const uint8_t *wq, int64_t ldw, const void *sw, int sw_fmt,
                                 int64_t N, int64_t K, const int64_t *rows, int64_t nrows,
                                 double *ref, double *absref) {
    int64_t KB = K / 128;
    size_t sw_elem = (sw_fmt == 0) ? sizeof(float) : 1;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < nrows; ++i)
        for (int64_t n = 0; n < N; ++n) {
            int64_t m = rows[i];
            const char *sw_row = (const char *)sw + (size_t)((n / 128) * KB) * sw_elem;
            gemm_element(aq + m * lda, wq + n * ldw, K, sa, lds, m, sw_row, sw_fmt,
                         &ref[i * N + n], &absref[i * N + n]);
        }
}

/* Grouped GEMM reference [DSv4-WOA section 3: batched per-group GEMM].  Expert e owns the rows
 * [off[e], off[e+1]) of aq and uses wq[e] ([N, K], stride N*ldw per expert) and
 * sw[e] ([N/128, K/128]).  Computes the selected rows only. */
void oracle_grouped_gemm_w8a8_block_rows(const uint8_t *aq, int64_t lda, const float *sa,
                                         int64_t lds, const uint8_t *wq, int64_t ldw,
                                         const void *sw, int sw_fmt, const int32_t *off,
                                         int64_t E, int64_t N, int64_t K, const int64_t *rows,
                                         int64_t nrows, double *ref, double *absref) {
    int64_t KB = K / 128, NB = N / 128;
    size_t sw_elem = (sw_fmt == 0) ? sizeof(float) : 1;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows[i];
        int64_t e = 0;
        while (e < E && !(m >= off[e] && m < off[e + 1])) ++e;
        for (int64_t n = 0; n < N; ++n) {
            if (e == E) {                      /* row owned by no expert: no output */
                ref[i * N + n] = 0.0;
                absref[i * N + n] = 0.0;
                continue;
            }
            const uint8_t *we = wq + e * N * ldw;
            const char *sw_row = (const char *)sw + (size_t)((e * NB + n / 128) * KB) * sw_elem;
            gemm_element(aq + m * lda, we + n * ldw, K, sa, lds, m, sw_row, sw_fmt,
                         &ref[i * N + n], &absref[i * N + n]);
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Helpers exposed for the oracle's own pin tests                                              */
/* ------------------------------------------------------------------------------------------ */

void oracle_e4m3_encode_array(const float *v, int64_t n, uint8_t *out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

void oracle_f32_to_bf16_array(const float *v, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(v[i]);
}

float oracle_rms_inverse(const uint16_t *x, int64_t K, float eps) {
    return rms_inverse(x, K, eps);
}

/* Exhaustive check of the encoder over every fp32 bit pattern whose value is finite, against
 * an independent formulation: a search of the sorted table of the 127 non-negative finite E4M3
 * values for the nearest one, ties to the even code, saturating above 448.  Returns the number
 * of disagreements and stores the first one's bit pattern in *first_bad. */
int64_t oracle_e4m3_encode_exhaustive_check(uint32_t *first_bad) {
    double table[127];
    for (int c = 0; c < 127; ++c) table[c] = oracle_e4m3_decode((uint8_t)c);
    int64_t bad = 0;
    uint32_t first = 0;
    #pragma omp parallel for schedule(static) reduction(+ : bad)
    for (int64_t u = 0; u < (1LL << 32); ++u) {
        uint32_t bits = (uint32_t)u;
        if (((bits >> 23) & 0xFF) == 0xFF) continue;      /* inf / NaN: out of scope */
        float f;
        memcpy(&f, &bits, sizeof f);
        double a = fabs((double)f);
        int code;
        if (a >= 448.0) code = 126;
        else {
            /* binary search: largest index lo with table[lo] <= a */
            int lo = 0, hi = 126;
            while (lo < hi) {
                int mid = (lo + hi + 1) / 2;
                if (table[mid] <= a) lo = mid; else hi = mid - 1;
            }
            code = lo;
            if (lo < 126) {
                double dlo = a - table[lo], dhi = table[lo + 1] - a;
                if (dhi < dlo || (dhi == dlo && (lo & 1))) code = lo + 1;
            }
        }
        uint8_t expect = (uint8_t)(code | ((bits >> 24) & 0x80));
        if (oracle_e4m3_encode(f) != expect) {
            bad += 1;
            #pragma omp critical
            { if (first == 0 || bits < first) first = bits; }
        }
    }
    *first_bad = first;
    return bad;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
