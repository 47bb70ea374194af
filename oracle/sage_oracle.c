/*
 * sage_oracle.c -- plain, slow CPU oracle for SageAttention-style quantized
 * attention.  TEST INFRASTRUCTURE ONLY: it exists so that tests/, the smoke
 * check and the benchmark's CPU-baseline leg can check the CUDA library
 * against an independent statement of the method.  Nothing in the product
 * path may call it, and it shares no code with the CUDA sources.
 *
 * Every routine follows the method in the order the pages give it:
 *
 *   [SA2]  "SageAttention2" paper summary (sgqg.cn/news/89714),
 *          sections 相关工作 (SageAttention bullet) and SageAttention2方法
 *          (smooth Q; per-thread quantization; FP8 quantization of P~V;
 *          FP32 buffer for the FP22 accumulator).
 *   [KAI]  "Kairos的注意力加速利器SageAttention INT8/FP8量化内核..." (mhpq.cn),
 *          section 二, 2.1 (kernel table: fp32 / fp32+fp32 accumulation,
 *          per_warp granularity) and 2.2 (block INT8 quantization, smoothing,
 *          two-level accumulation).
 *   [GUIDE] "SageAttention量化加速框架完整指南" (mhpq.cn), sections 五分钟跑通
 *          (sageattn(q,k,v,tensor_layout,is_causal)) and 性能调优实战
 *          (pv_accum_dtype).
 *
 * The pages give no formulas, block sizes or rounding rules.  The readings
 * taken where they are silent are stated at each routine; the main ones:
 * round-to-nearest-even everywhere, symmetric INT8 codes in
 * [-127, 127], the group shapes of orc_q_group/orc_k_group, 128-key tiles in
 * increasing order for the online softmax, the row sum taken over the
 * unquantized P~, a static FP8 scale of 448 (the E4M3 maximum) for P~.
 *
 * Precision: floating point in fp64 except where the method itself fixes a
 * float32 value that decides an integer code (the smoothed K/Q fed to the
 * INT8 quantizer, the scale products, the P~*448 fed to the E4M3 encoder);
 * those steps are written in float32 so that both sides decide each code in
 * the same precision.  Build with -ffp-contract=off: no fused multiply-adds.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* OCP 8-bit floating point, E4M3 ("FN": no infinities).                     */
/* Bias 7, 3 mantissa bits, largest finite 448 = 1.75 * 2^8 (code 0x7E),     */
/* smallest subnormal 2^-9 (code 0x01), S.1111.111 is NaN.                   */
/* The pages name only the E4M3 flavour [SA2, FP8 quantization of P~V]; the   */
/* format is the OCP one that tensor cores implement.  Conversion: round to  */
/* nearest, ties to even, then saturate to +-448 ("satfinite"); NaN stays    */
/* NaN, +-Inf saturates.                                                     */
/* ------------------------------------------------------------------------ */
ORC_EXPORT float orc_e4m3_to_float(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);               /* subnormal: m/8 * 2^-6 */
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

ORC_EXPORT uint8_t orc_e4m3_from_float(float x) {
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (isnan(x)) return sign | 0x7F;
    if (a >= 448.0) return sign | 0x7E;                  /* saturate (incl. Inf) */
    if (a < ldexp(1.0, -6)) {                            /* subnormal range */
        double q = nearbyint(a * 512.0);                 /* units of 2^-9, RNE */
        /* q == 8 is exactly the smallest normal 2^-6, whose code is 0x08. */
        return sign | (uint8_t)q;
    }
    int e;
    double f = frexp(a, &e);                             /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;                                              /* a = (2f) * 2^e, 2f in [1, 2) */
    double mant = nearbyint((2.0 * f - 1.0) * 8.0);      /* 3 fraction bits, RNE */
    if (mant == 8.0) { mant = 0.0; e += 1; }
    if (e > 8 || (e == 8 && mant > 6.0)) return sign | 0x7E;   /* rounds past 448 */
    return sign | (uint8_t)(((e + 7) << 3) | (int)mant);
}

ORC_EXPORT void orc_e4m3_from_float_array(const float* x, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_from_float(x[i]);
}
ORC_EXPORT void orc_e4m3_to_float_array(const uint8_t* c, float* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_to_float(c[i]);
}

/* IEEE binary16 / bfloat16 rounding of a double (RNE), used for the 16-bit
 * P~ of the FP16-PV mode [KAI 2.1, sm80 row: INT8 QK^T, FP16 PV].            */
static double round_to_f16(double x) {
    if (x == 0.0 || isnan(x)) return x;
    double a = fabs(x);
    int e;
    frexp(a, &e);                                        /* a in [2^(e-1), 2^e) */
    int ulp_exp = (e - 1) - 10;                          /* 10 fraction bits */
    if (ulp_exp < -24) ulp_exp = -24;                    /* subnormal spacing 2^-24 */
    double r = ldexp(nearbyint(ldexp(a, -ulp_exp)), ulp_exp);
    if (r > 65504.0) r = INFINITY;
    return x < 0 ? -r : r;
}
static double round_to_bf16(double x) {
    float f = (float)x;                                  /* the P~ value is an fp32 */
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return x;
    uint32_t lsb = (u >> 16) & 1u;
    u = (u + 0x7FFFu + lsb) & 0xFFFF0000u;
    memcpy(&f, &u, 4);
    return (double)f;
}

ORC_EXPORT double orc_round_f16(double x) { return round_to_f16(x); }
ORC_EXPORT double orc_round_bf16(double x) { return round_to_bf16(x); }

/* ------------------------------------------------------------------------ */
/* Quantization groups (reading; the pages name the granularities --        */
/* per-block, per-warp [KAI 2.1/2.2], per-thread [SA2, per-thread           */
/* quantization] -- but define none of them).  Tokens are counted from the  */
/* start of their sequence.  Q is split in 128-token blocks, K in 128-token */
/* blocks (two 64-token halves).  Within one block:                         */
/*   per_block : Q one group of 128 rows;      K two groups of 64 rows.     */
/*   per_warp  : Q four groups of 32 rows;     K two groups of 64 rows.     */
/*   per_thread: Q rows of a 32-row slice with equal (row mod 8) -> 8 groups */
/*               per slice, 32 per block;                                   */
/*               K rows of a 64-row half with equal (row mod 8) -> 8 groups  */
/*               per half, 16 per block.                                    */
/*   per_token : Q one group per row [REPO, Tinh nang chinh: per-token      */
/*               granularity];                K two groups of 64 rows.     */
/* (per_thread mirrors the thread-to-row map of the m16n8k32 MMA fragments  */
/* the pages' kernels were written for: a thread owns rows r and r+8 of     */
/* each 16-row slab, hence one scale per residue mod 8.)                    */
/* ------------------------------------------------------------------------ */
enum { ORC_PER_BLOCK = 0, ORC_PER_WARP = 1, ORC_PER_THREAD = 2, ORC_PER_TOKEN = 3 };

ORC_EXPORT int orc_q_groups_per_block(int gran) {
    return gran == ORC_PER_BLOCK ? 1 : gran == ORC_PER_WARP ? 4 : gran == ORC_PER_TOKEN ? 128 : 32;
}
ORC_EXPORT int orc_k_groups_per_block(int gran) {
    return gran == ORC_PER_THREAD ? 16 : 2;
}
ORC_EXPORT int orc_q_group(int gran, int r) {           /* r: row within its 128-block */
    if (gran == ORC_PER_BLOCK) return 0;
    if (gran == ORC_PER_WARP) return r / 32;
    if (gran == ORC_PER_TOKEN) return r;
    return (r / 32) * 8 + (r % 8);
}
ORC_EXPORT int orc_k_group(int gran, int r) {
    if (gran == ORC_PER_THREAD) return (r / 64) * 8 + (r % 8);
    return r / 64;
}

/* ------------------------------------------------------------------------ */
/* Smooth K [SA2, 相关工作/SageAttention: K is preprocessed to protect the   */
/* accuracy; KAI 2.2, smoothing]: subtract the per-channel mean of K over   */
/* the tokens of its sequence (reading: all tokens, also under a causal     */
/* mask).  Softmax rows are invariant to it: q.(k_j - mu) = q.k_j - q.mu,   */
/* a constant shift of the whole score row.                                 */
/*                                                                          */
/* The mean is fixed to the last bit: the sum is exact (fp16 inputs are     */
/* integers times 2^-24 and are summed in int64; bf16 inputs are summed in  */
/* fp64, which is exact unless the values span more than ~45 binary orders) */
/* then mean = float( double(sum) / L ).                                    */
/*   x: [L][D] values (exactly the fp16/bf16 inputs), mu: [D] float out.    */
/* ------------------------------------------------------------------------ */
ORC_EXPORT void orc_channel_mean(const double* x, int64_t L, int D, int is_fp16, float* mu) {
    for (int c = 0; c < D; ++c) {
        double mean;
        if (is_fp16) {
            int64_t acc = 0;
            for (int64_t t = 0; t < L; ++t) acc += (int64_t)ldexp(x[t * D + c], 24);
            mean = ldexp((double)acc, -24) / (double)L;
        } else {
            double acc = 0.0;
            for (int64_t t = 0; t < L; ++t) acc += x[t * D + c];
            mean = acc / (double)L;
        }
        mu[c] = L > 0 ? (float)mean : 0.0f;
    }
}

/* xs[t][c] = float(x[t][c] - mu[c]): one float32 subtraction (x is exactly a
 * float32 value).  mu == NULL means no smoothing.                           */
ORC_EXPORT void orc_subtract_channel(const double* x, int64_t L, int D, const float* mu, float* xs) {
    for (int64_t t = 0; t < L; ++t)
        for (int c = 0; c < D; ++c) {
            float v = (float)x[t * D + c];
            xs[t * D + c] = mu ? v - mu[c] : v;
        }
}

/* Smooth Q [SA2, 平滑Q]: subtract the mean of each 128-token Q block.       *
 * QK^T = (Q - mu_Q) K^T + mu_Q K^T: the first product runs on the INT8     *
 * tensor cores, the second is a per-block row vector added to the scores   *
 * (orc_smooth_q_bias).  Block means: exact fp64 sum of the block's tokens  *
 * (at most 128 fp16/bf16 values), mean = float(sum / n).                   *
 *   mu_blk: [ceil(L/128)][D] float out; xs: [L][D] float out.               */
ORC_EXPORT void orc_smooth_q_blocks(const double* x, int64_t L, int D, float* mu_blk, float* xs) {
    int64_t nblk = (L + 127) / 128;
    for (int64_t b = 0; b < nblk; ++b) {
        int64_t t0 = b * 128, t1 = t0 + 128 < L ? t0 + 128 : L;
        for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int64_t t = t0; t < t1; ++t) acc += x[t * D + c];
            float m = (float)(acc / (double)(t1 - t0));
            mu_blk[b * D + c] = m;
            for (int64_t t = t0; t < t1; ++t) xs[t * D + c] = (float)x[t * D + c] - m;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Symmetric INT8 quantization per group [KAI 2.2 block INT8 quantization;  */
/* SA2 per-thread quantization].  For a group G:                            */
/*   amax  = max |x| over G  (valid tokens only)                            */
/*   delta = amax / 127                      (float32 IEEE division)        */
/*   code  = clamp(rne(x * (127 / amax)), -127, 127)                        */
/* with 127/amax one float32 division per group and the product rounded to  */
/* float32 before the round-to-nearest-even to an integer (reading: the     */
/* pages give neither rounding nor range; x/delta is taken as x times the   */
/* reciprocal of delta expressed as 127/amax).  amax == 0 gives delta = 0   */
/* and all codes 0.                                                         */
/*   xs: [L][D] float (already smoothed), is_q selects the Q or K groups.   */
/*   codes: [L][D]; scales: [nblk][groups_per_block].                       */
/* ------------------------------------------------------------------------ */
ORC_EXPORT void orc_quant_int8(const float* xs, int64_t L, int D, int is_q, int gran,
                               int8_t* codes, float* scales) {
    int ng = is_q ? orc_q_groups_per_block(gran) : orc_k_groups_per_block(gran);
    int64_t nblk = (L + 127) / 128;
    float* amax = (float*)malloc(sizeof(float) * ng);
    for (int64_t b = 0; b < nblk; ++b) {
        for (int g = 0; g < ng; ++g) amax[g] = 0.0f;
        for (int r = 0; r < 128 && b * 128 + r < L; ++r) {
            int g = is_q ? orc_q_group(gran, r) : orc_k_group(gran, r);
            const float* row = xs + (b * 128 + r) * D;
            for (int c = 0; c < D; ++c) {
                float a = fabsf(row[c]);
                if (a > amax[g]) amax[g] = a;
            }
        }
        for (int g = 0; g < ng; ++g) scales[b * ng + g] = amax[g] / 127.0f;
        for (int r = 0; r < 128 && b * 128 + r < L; ++r) {
            int g = is_q ? orc_q_group(gran, r) : orc_k_group(gran, r);
            float inv = amax[g] > 0.0f ? 127.0f / amax[g] : 0.0f;
            const float* row = xs + (b * 128 + r) * D;
            int8_t* out = codes + (b * 128 + r) * D;
            for (int c = 0; c < D; ++c) {
                float y = row[c] * inv;                    /* float32 product */
                double q = nearbyint((double)y);           /* ties to even */
                if (q > 127.0) q = 127.0;
                if (q < -127.0) q = -127.0;
                out[c] = (int8_t)q;
            }
        }
    }
    free(amax);
}

/* Per-row view of the group scales: rs[t] = scale of the group of token t. */
ORC_EXPORT void orc_row_scales(const float* scales, int64_t L, int is_q, int gran, float* rs) {
    int ng = is_q ? orc_q_groups_per_block(gran) : orc_k_groups_per_block(gran);
    for (int64_t t = 0; t < L; ++t) {
        int r = (int)(t % 128);
        int g = is_q ? orc_q_group(gran, r) : orc_k_group(gran, r);
        rs[t] = scales[(t / 128) * ng + g];
    }
}

/* ------------------------------------------------------------------------ */
/* V to FP8 E4M3 per channel [SA2, FP8 quantization of P~V: per channel]:   */
/*   amax_c = max_t |V[t][c]|; delta_c = amax_c / 448; code = E4M3(V * (448 */
/*   / amax_c)) with the product rounded to float32 (same reading of x /    */
/*   delta as for INT8; 448 is the largest finite E4M3 value).              */
/*   v: [L][D] values; codes [L][D]; dv [D].                                 */
/* ------------------------------------------------------------------------ */
ORC_EXPORT void orc_quant_v_fp8(const double* v, int64_t L, int D, uint8_t* codes, float* dv) {
    for (int c = 0; c < D; ++c) {
        float amax = 0.0f;
        for (int64_t t = 0; t < L; ++t) {
            float a = fabsf((float)v[t * D + c]);
            if (a > amax) amax = a;
        }
        dv[c] = amax / 448.0f;
        float inv = amax > 0.0f ? 448.0f / amax : 0.0f;
        for (int64_t t = 0; t < L; ++t) {
            float y = (float)v[t * D + c] * inv;
            codes[t * D + c] = orc_e4m3_from_float(y);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* INT8 QK^T with int32 accumulation [SA2 / KAI 2.2]: exact integer dot     */
/* products, |S| <= D * 127^2 < 2^22.  out: [Lq][Lk].                        */
/* ------------------------------------------------------------------------ */
ORC_EXPORT void orc_scores_int32(const int8_t* qc, const int8_t* kc, int64_t Lq, int64_t Lk,
                                 int D, int32_t* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < Lq; ++i)
        for (int64_t j = 0; j < Lk; ++j) {
            int32_t acc = 0;
            for (int c = 0; c < D; ++c) acc += (int32_t)qc[i * D + c] * (int32_t)kc[j * D + c];
            out[i * Lk + j] = acc;
        }
}

/* Smooth-Q score correction [SA2, 平滑Q]: bias[b][j] = sum_c mu_Q[b][c] *   *
 * Khat[j][c] with Khat = delta_K(j) * K_code the dequantized smoothed K     *
 * (reading: the only choice that needs no second pass over full-precision  *
 * K).  Evaluated in fp64.  bias: [nqblk][Lk].                               */
ORC_EXPORT void orc_smooth_q_bias(const float* mu_blk, int64_t nqblk, const int8_t* kc,
                                  const float* k_rs, int64_t Lk, int D, double* bias) {
    for (int64_t b = 0; b < nqblk; ++b)
        for (int64_t j = 0; j < Lk; ++j) {
            double acc = 0.0;
            for (int c = 0; c < D; ++c) acc += (double)mu_blk[b * D + c] * (double)kc[j * D + c];
            bias[b * Lk + j] = acc * (double)k_rs[j];
        }
}

/* ------------------------------------------------------------------------ */
/* Ambiguous roundings of P~.                                               */
/*                                                                          */
/* The oracle evaluates 2^x exactly (fp64).  An implementation reaches P~   */
/* through float32 steps and an approximate exp2, so its P~ is off by a     */
/* small relative amount; where the exact P~ (times its static scale) lies  */
/* that close to the midpoint between two neighbouring E4M3 (or 16-bit)     */
/* values, either neighbour is a correct rounding.  orc_p_band derives that */
/* relative distance per score from the arithmetic of a kernel that         */
/*   - keeps S*c exact inside one fused multiply-add, where the oracle      */
/*     rounds s = float(S*c): half an ulp of s;                              */
/*   - folds the FP8 static scale into the subtracted maximum in float32,   */
/*     nb = -float(float(m - float(log2 448)) + tau): the error of           */
/*     float(log2 448) and half an ulp per rounding;                        */
/*   - rounds the exponent S*c + nb once: half an ulp of it;                */
/*   - evaluates 2^x with a relative error of at most ORC_EXP2_REL, two     */
/*     units in the last place of a float32 result (the documented bound of */
/*     the GPU's approximate base-2 exponential);                           */
/* plus the oracle's own rounding of the scaled P~ to float32 before it is  */
/* encoded (2^-24).  With the smooth-Q correction the score and the running */
/* maximum carry further roundings, passed in as `extra` (log2 units).      */
/* orc_e4m3_alt_step / orc_h16_alt_step return |other - chosen| for a value */
/* within `rel` of a midpoint, else 0; orc_attn_quant_head turns these into */
/* a per-output allowance.                                                  */
/* ------------------------------------------------------------------------ */
#define ORC_EXP2_REL 0x1p-22

/* Half an ulp of a float32 of magnitude |x| (rounded up to the next binade
 * when |x| is within 2^-20 of its top, so that a rounding that carries into
 * the next binade is covered). */
static double hulp32(double x) {
    double a = fabs(x) * (1.0 + 0x1p-20);
    if (!(a >= 0x1p-126)) return 0x1p-150;               /* subnormal spacing / 2; also 0 */
    int e;
    frexp(a, &e);                                        /* a in [2^(e-1), 2^e) */
    return ldexp(1.0, e - 25);                           /* ulp 2^(e-24), halved */
}

static double log2_448(void) { return 6.0 + log2(7.0); }  /* 448 = 7 * 2^6 */

ORC_EXPORT double orc_p_band(double s, double m, int fold, int tau, double extra) {
    const double L = log2_448(), Lf = (double)(float)L;
    double arg = s - m + (fold ? L - tau : 0.0);
    double bl = hulp32(s) + hulp32(arg) + extra;
    if (fold) {
        bl += fabs(Lf - L) + hulp32(m - Lf);
        if (tau) bl += hulp32(m - Lf + tau);
    }
    return (1.0 + ORC_EXP2_REL) * exp2(bl) - 1.0 + 0x1p-24;
}

static double e4m3_alt_step(double y, double rel) {
    uint8_t c = orc_e4m3_from_float((float)y);
    double v0 = (double)orc_e4m3_to_float(c);
    double v1;
    if (y >= v0) { if ((c & 0x7F) >= 0x7E) return 0.0; v1 = (double)orc_e4m3_to_float((uint8_t)(c + 1)); }
    else { if ((c & 0x7F) == 0) return 0.0; v1 = (double)orc_e4m3_to_float((uint8_t)(c - 1)); }
    double mid = 0.5 * (v0 + v1);
    return fabs(y - mid) <= rel * y ? fabs(v1 - v0) : 0.0;
}
static double h16_alt_step(double p, int bf16, double rel) {
    double h0 = bf16 ? round_to_bf16(p) : round_to_f16((double)(float)p);
    if (h0 <= 0.0) {                                     /* below half the smallest step */
        double tiny = bf16 ? 0x1p-133 : 0x1p-24;
        return fabs(p - 0.5 * tiny) <= rel * p ? tiny : 0.0;
    }
    int e;
    frexp(h0, &e);                                       /* h0 in [2^(e-1), 2^e) */
    int fb = bf16 ? 7 : 10;
    double up = ldexp(1.0, (e - 1) - fb);
    double down = (h0 == ldexp(1.0, e - 1)) ? up / 2 : up;
    if (!bf16 && (e - 1) - fb < -24) up = down = ldexp(1.0, -24);
    double h1 = p >= h0 ? h0 + up : h0 - down;
    double mid = 0.5 * (h0 + h1);
    return fabs(p - mid) <= rel * p ? fabs(h1 - h0) : 0.0;
}

ORC_EXPORT double orc_e4m3_alt_step(double y, double rel) { return e4m3_alt_step(y, rel); }
ORC_EXPORT double orc_h16_alt_step(double p, int bf16, double rel) { return h16_alt_step(p, bf16, rel); }

/* One unit in the last place of an IEEE binary16 value of magnitude |x|.   */
static double ulp16(double x) {
    double a = fabs(x);
    if (a < 0x1p-14) return 0x1p-24;
    int e;
    frexp(a, &e);
    return ldexp(1.0, e - 11);
}

/* ------------------------------------------------------------------------ */
/* Quantized attention for one (sequence, head), following the FlashAttention */
/* tiling the method is built on [SA2, 相关工作: SageAttention reuses the    */
/* FlashAttention block decomposition]:                                     */
/*                                                                          */
/*  for each query row i, for each 128-key tile in increasing order          */
/*  (reading: the tile size is the kernel's; the online-softmax state then   */
/*  matches the kernel's, which matters because P~ is rounded relative to   */
/*  the running maximum), skipping tiles with no visible key:               */
/*    c_ij   = float(float(dQ_i * dK_j) * float(sm_scale * log2 e))          */
/*    s_ij   = float(S_ij * c_ij)          (+ smooth-Q bias, see below)      */
/*    m_new  = max(m, max_j s_ij);  alpha = 2^(m - m_new)                    */
/*    p_ij   = 2^(s_ij - m_new)            (P~ <= 1)                         */
/*    l      = alpha * l + sum_j p_ij      (unquantized P~; reading)        */
/*    FP8 mode  [SA2, FP8 quantization of P~V: static scale for P~,         */
/*               per-channel for V]:                                        */
/*       P8_ij = E4M3(float(p_ij * 448))   (static scale 1/448; reading)     */
/*       Opart = sum_j P8_ij * V8_j        (exact products, fp64 sum)        */
/*    16-bit mode [KAI 2.1, sm80 row]: Ph = rne16(p), Opart = sum Ph * V_j   */
/*    O = alpha * O + Opart               (two-level: per-tile partial sums  */
/*                                         added into an outer accumulator   */
/*                                         [SA2, FP32 MMA buffer]; in exact  */
/*                                         arithmetic the one-level "fp32"   */
/*                                         mode computes the same value)     */
/*  out_i = O * dV / (448 * l)  (FP8)      or  O / l  (16-bit)               */
/*                                                                          */
/* Causal (reading): top-left aligned, key j visible to query i iff j <= i.  */
/* Smooth Q: s_ij = float(s_ij + bias[i/128][j] * float(sm_scale * log2 e)). */
/* Conditional (lazy) rescaling, lazy_tau > 0 [reading of the NEXT item     */
/* "skip the alpha update unless the maximum grows by more than tau"]: the  */
/* reference r that P~ and O are kept relative to moves to the running      */
/* maximum only when a tile's maximum exceeds float(r + tau); otherwise     */
/* alpha = 1.  P~ = 2^(s - r) <= 2^tau, so the FP8 static scale becomes      */
/* 448 * 2^-tau (P8 <= 448); the output divides it out again.  lazy_tau = 0 */
/* is the plain online softmax above.                                       */
/*                                                                          */
/* FP16 inner accumulation, acc_mode 1 ("fp32+fp16") [KAI 2.1, sm89 row:    */
/* fp32fp16 two-level accumulation; GUIDE, 性能调优实战: pv_accum_dtype]: the */
/* partial sum of each 128-key tile is held in binary16 and added into the  */
/* fp32 outer accumulator.  Readings: (1) the partial is rounded to binary16 */
/* after every 32 keys of the tile (one tensor-core instruction's depth),   */
/* the 32 products themselves summed exactly; (2) one tile's partial must   */
/* not overflow binary16 (max 65504), and with V codes up to 448 a P~ scale */
/* of 448 would overflow on a single product; the largest static scale that */
/* keeps 128 * scale * 448 <= 65504 is 1, so P8 = E4M3(p) and out = O*dV/l.  */
/* FP8 only, plain online softmax (lazy_tau = 0).                           */
/*                                                                          */
/* Identity quantizers, pv_mode 2 (a debug reading that pins the           */
/* bookkeeping above): scores q_i . k_j * sm_scale * log2 e in fp64 from the */
/* unquantized qf, kf; P~ and V (v16) unrounded; no float32 step anywhere.  */
/* The loop is the same one, so with the tiling removed it must equal       */
/* orc_attn_exact_head to fp64 round-off.                                   */
/*                                                                          */
/*   qc [Lq][D] int8, q_rs [Lq] row scales; kc [Lk][D], k_rs [Lk];           */
/*   pv_mode 0: v8 [Lk][D] E4M3 codes, dv [D];                               */
/*   pv_mode 1: v16 [Lk][D] 16-bit V values (exact), v_is_bf16 picks the    */
/*              16-bit type P~ is rounded to;                               */
/*   pv_mode 2: qf [Lq][D], kf [Lk][D], v16 [Lk][D] fp64 (qc..dv unused);    */
/*   bias [ceil(Lq/128)][Lk] or NULL; rows [row0, row1) are computed.        */
/*   out [Lq][D] (only the computed rows are written).                       */
/*   allow [Lq][D] or NULL: the largest change of each output that ambiguous */
/*   roundings of P~ (orc_p_band) and, with acc_mode 1, the binary16        */
/*   roundings of the partial sums (one ulp per rounding: covers rounding to */
/*   nearest and toward zero) can cause, carried through the same alpha    */
/*   rescaling and normalization as O.                                       */
/* ------------------------------------------------------------------------ */
enum { ORC_PV_FP8 = 0, ORC_PV_16 = 1, ORC_PV_IDENTITY = 2 };

ORC_EXPORT void orc_attn_quant_head(const int8_t* qc, const float* q_rs, const int8_t* kc,
                                    const float* k_rs, const uint8_t* v8, const float* dv,
                                    const double* v16, const double* qf, const double* kf,
                                    int pv_mode, int acc_mode, int v_is_bf16,
                                    const double* bias, int64_t Lq, int64_t Lk, int D,
                                    int causal, float sm_scale, int64_t row0, int64_t row1,
                                    double* out, double* allow, int lazy_tau) {
    const int ident = pv_mode == ORC_PV_IDENTITY;
    const int acc16 = pv_mode == ORC_PV_FP8 && acc_mode == 1;
    const float sl2 = sm_scale * 1.44269504f;             /* float(log2 e) */
    const double sl2d = (double)sm_scale * 1.4426950408889634;
    const int fold = pv_mode == ORC_PV_FP8 && !acc16;     /* 448 folded into the maximum */
    const double pscale = !fold ? 1.0 : 448.0 * ldexp(1.0, -lazy_tau);   /* FP8 static P~ scale */
    const double taud = (double)lazy_tau;
    int64_t ntile = (Lk + 127) / 128;
    #pragma omp parallel
    {
        double* O = (double*)malloc(sizeof(double) * D);
        double* Op = (double*)malloc(sizeof(double) * D);
        double* Cp = (double*)malloc(sizeof(double) * D);
        double* A = (double*)malloc(sizeof(double) * D);
        double* Ap = (double*)malloc(sizeof(double) * D);
        double* s = (double*)malloc(sizeof(double) * 128);
        double* ds = (double*)malloc(sizeof(double) * 128);
        double* v8f = NULL;
        if (pv_mode == ORC_PV_FP8) v8f = (double*)malloc(sizeof(double) * 256);
        if (v8f) for (int c = 0; c < 256; ++c) v8f[c] = (double)orc_e4m3_to_float((uint8_t)c);
        #pragma omp for schedule(dynamic, 4)
        for (int64_t i = row0; i < row1; ++i) {
            double m = -INFINITY, l = 0.0;
            double dm = 0.0;                               /* smooth Q: bound on the kernel's maximum's offset */
            for (int c = 0; c < D; ++c) O[c] = A[c] = 0.0;
            for (int64_t t = 0; t < ntile; ++t) {
                int64_t j0 = t * 128, j1 = j0 + 128 < Lk ? j0 + 128 : Lk;
                if (causal && j1 > i + 1) j1 = i + 1;
                if (j1 <= j0) continue;                    /* fully masked tile */
                double mt = -INFINITY;
                for (int64_t j = j0; j < j1; ++j) {
                    double sc, e = 0.0;
                    if (ident) {
                        double d = 0.0;
                        for (int c = 0; c < D; ++c) d += qf[i * D + c] * kf[j * D + c];
                        sc = d * sl2d;
                    } else {
                        int32_t S = 0;
                        for (int c = 0; c < D; ++c) S += (int32_t)qc[i * D + c] * (int32_t)kc[j * D + c];
                        float cij = (q_rs[i] * k_rs[j]) * sl2;
                        float sf = (float)S * cij;
                        sc = sf;
                        if (bias) {
                            double b64 = bias[(i / 128) * Lk + j];
                            float b32 = (float)b64;
                            sc = (double)(float)((double)sf + b64 * (double)sl2);
                            /* a kernel holding the correction as float32 b32 and
                             * adding float(b32 * sl2) to the exact S*c in one
                             * fused multiply-add differs from sc by at most: */
                            e = 2.0 * hulp32(sc) + hulp32(b64) * (double)sl2
                              + hulp32((double)b32 * (double)sl2) + hulp32(sf);
                        }
                    }
                    s[j - j0] = sc;
                    ds[j - j0] = e;
                    if (sc > mt) mt = sc;
                    if (e > dm) dm = e;                    /* the running maximum's score may be off by e */
                }
                const double lim = ident ? m + taud : (double)(float)(m + taud);
                const int move = (m == -INFINITY) || (mt > lim);
                double mn = move ? (m > mt ? m : mt) : m;
                double alpha = (m == -INFINITY) ? 0.0 : exp2(m - mn);
                double lt = 0.0;
                for (int c = 0; c < D; ++c) Op[c] = Ap[c] = 0.0;
                for (int64_t c0 = j0; c0 < j0 + 128; c0 += 32) {          /* 32-key chunks */
                    int64_t c1 = c0 + 32 < j1 ? c0 + 32 : j1;
                    for (int c = 0; c < D; ++c) Cp[c] = 0.0;
                    for (int64_t j = c0; j < c1; ++j) {
                        double p = exp2(s[j - j0] - mn);
                        lt += p;
                        if (ident) {
                            const double* vr = v16 + j * D;
                            for (int c = 0; c < D; ++c) Cp[c] += p * vr[c];
                        } else if (pv_mode == ORC_PV_FP8) {
                            double y = p * pscale;
                            double p8 = v8f[orc_e4m3_from_float((float)y)];
                            const uint8_t* vr = v8 + j * D;
                            for (int c = 0; c < D; ++c) Cp[c] += p8 * v8f[vr[c]];
                            double st = allow ? e4m3_alt_step(y, orc_p_band(s[j - j0], mn, fold, fold ? lazy_tau : 0,
                                                                            ds[j - j0] + dm)) : 0.0;
                            if (st > 0.0)
                                for (int c = 0; c < D; ++c) Ap[c] += st * fabs(v8f[vr[c]]);
                        } else {
                            double ph = v_is_bf16 ? round_to_bf16(p) : round_to_f16((double)(float)p);
                            const double* vr = v16 + j * D;
                            for (int c = 0; c < D; ++c) Cp[c] += ph * vr[c];
                            double st = allow ? h16_alt_step(p, v_is_bf16, orc_p_band(s[j - j0], mn, 0, 0,
                                                                                      ds[j - j0] + dm)) : 0.0;
                            if (st > 0.0)
                                for (int c = 0; c < D; ++c) Ap[c] += st * fabs(vr[c]);
                        }
                    }
                    for (int c = 0; c < D; ++c) {
                        if (acc16) {
                            Op[c] = round_to_f16(Op[c] + Cp[c]);
                            if (c1 > c0) Ap[c] += ulp16(Op[c]);   /* a chunk of masked keys adds 0 exactly */
                        } else {
                            Op[c] += Cp[c];
                        }
                    }
                }
                l = alpha * l + lt;
                for (int c = 0; c < D; ++c) {
                    O[c] = alpha * O[c] + Op[c];
                    A[c] = alpha * A[c] + Ap[c];
                }
                m = mn;
            }
            for (int c = 0; c < D; ++c) {
                double o, a;
                if (l <= 0.0) o = a = 0.0;                 /* no visible key at all */
                else if (pv_mode == ORC_PV_FP8) {
                    o = O[c] * (double)dv[c] / (pscale * l);
                    a = A[c] * (double)dv[c] / (pscale * l);
                } else {
                    o = O[c] / l;
                    a = A[c] / l;
                }
                out[i * D + c] = o;
                if (allow) allow[i * D + c] = a;
            }
        }
        free(O); free(Op); free(Cp); free(A); free(Ap); free(s); free(ds); free(v8f);
    }
}
/* ------------------------------------------------------------------------ */
/* Exact attention, the quantity the method approximates: softmax(q k^T *    */
/* sm_scale [+ causal mask]) v, in fp64, one pass with the true row maximum. */
/* sm_scale defaults to 1/sqrt(D) at the API (reading: the pages use the    */
/* scaled_dot_product_attention convention they replace [GUIDE, 换进真实模型]). */
/* ------------------------------------------------------------------------ */
ORC_EXPORT void orc_attn_exact_head(const double* q, const double* k, const double* v,
                                    int64_t Lq, int64_t Lk, int D, int causal, double sm_scale,
                                    int64_t row_offset, double* out) {
    /* q holds rows row_offset .. row_offset+Lq-1 of the sequence (causal
     * masking uses the sequence row index). */
    #pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (Lk > 0 ? Lk : 1));
        #pragma omp for schedule(dynamic, 4)
        for (int64_t i = 0; i < Lq; ++i) {
            int64_t n = causal ? (row_offset + i + 1 < Lk ? row_offset + i + 1 : Lk) : Lk;
            double mx = -INFINITY;
            for (int64_t j = 0; j < n; ++j) {
                double d = 0.0;
                for (int c = 0; c < D; ++c) d += q[i * D + c] * k[j * D + c];
                s[j] = d * sm_scale;
                if (s[j] > mx) mx = s[j];
            }
            double den = 0.0;
            for (int64_t j = 0; j < n; ++j) { s[j] = exp(s[j] - mx); den += s[j]; }
            for (int c = 0; c < D; ++c) {
                double acc = 0.0;
                for (int64_t j = 0; j < n; ++j) acc += s[j] * v[j * D + c];
                out[i * D + c] = n > 0 ? acc / den : 0.0;
            }
        }
        free(s);
    }
}
